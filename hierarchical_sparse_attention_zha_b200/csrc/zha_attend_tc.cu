// zha_attend_tc.cu -- sparse attention over the routed leaf tokens on the
// sm_100a tensor cores (bf16 caches, head_dim 128).
//
// Citations: [Attention: "Scaled dot-product attention 의 식"] o = softmax(q K^T /
// sqrt(d)) V; [Attention: "FlashAttention 계열"] online softmax (running max m,
// sum l, output rescaled by exp(m_old - m_new)) and Flash-Decoding's split of
// the cache along its length with a max-and-sum combine; [ZHA: 전제와 한계]
// (page "ZHA는 KV 캐시를 트리로 요약해 어텐션 비용을 준(sub)이차로 낮춘다") token 0
// and the in-progress chunk are always attended.
//
// Three launches:
//  1. union_prep_kernel, one CTA per unit (group = KV head g with a block of up
//     to 32 of its query heads; unit = the group inside one block of chunks):
//     folds the heads' ascending chunk lists into one ascending union list with
//     a 32-bit head mask per chunk (chunk 0 always present, for the sink), and
//     validates the lists. Warp q marks head q's chunks in its own bitmap row;
//     a 32 x 32 bit transpose by shuffles turns rows into per-chunk masks.
//  2. attend_split_kernel, one CTA per SM: each unit's list is cut into tiles of
//     128 rows (floor(128 / C) chunks; a group's last unit also carries the tail
//     [N_b, N)); the tiles of all units form one sequence that is split evenly
//     over the CTAs. Each CTA streams its span with warp-specialised roles:
//       producers (2 warps)  cp.async of K and V rows into a 3-stage ring of
//                            128-byte-swizzled tiles, per-tile row metadata
//                            (prefetched one tile ahead)
//       MMA issuer (1 lane)  S^T = K_tile . Q^T (M = 128 rows, N = 32 heads,
//                            Q in two bf16 terms) into one of two TMEM buffers;
//                            O^T += V_tile^T . P (M = d, N = 32, P in two bf16
//                            terms) into a TMEM accumulator kept across tiles;
//                            it polls both "tile landed" and "P ready" so that
//                            neither kind of MMA waits behind the other
//       softmax (4 warps)    thread = tile row: masked scores in log2 units, a
//                            running maximum per head that is raised only when
//                            a score exceeds it by more than 2^8 (then O and the
//                            row sums are rescaled), P written into the K half of
//                            the stage (K is consumed once S is done)
//     When its span leaves a group the CTA writes one state [m, l, o] per head.
//  3. combine_split_kernel, one warp per query head: merges the states of the
//     CTAs whose span met the head's group.
// Every wait on an mbarrier is bounded; a time-out sets ZHA_DEV_TIMEOUT and the
// roles leave their loops, release TMEM and return.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "zha_host.cuh"
#include "zha_internal.cuh"
#include "zha_tc.cuh"

namespace zha {

namespace {

constexpr int kTok = 128;                 // rows per tile
constexpr int kQ = 32;                    // query heads per group
constexpr int kD = 128;
constexpr int kStages = 3;
constexpr int kStageBytes = 65536;        // K [2][128][128 B] then V [2][128][128 B]
constexpr int kOffQ = kStages * kStageBytes;          // [2 halves][64 rows: 32 hi, 32 lo][128 B]
constexpr int kOffMisc = kOffQ + 16384;
constexpr uint32_t kTmemCols = 256;      // S: 2 x 64 columns, O: 64 columns at 128
constexpr uint32_t kTmemO = 128;
constexpr int kThreads = 384;             // warps 0-1 producers, 2 MMA, 3 idle, 4-11 softmax
constexpr int kHalfQ = 16;                // heads per softmax warpgroup
constexpr int kProducers = 64;
constexpr int kMaxEntries = 64;           // chunks per tile (C >= 2)
constexpr uint32_t kWaitTries = tc::kWaitPolls;
constexpr uint32_t kPollLimit = 1u << 27; // polls of the MMA issuer without progress
constexpr float kRescaleSlack = 8.f;      // log2 units: p may reach 2^8 before a rescale
constexpr int kWinChunks = 16384;         // chunks per pass of the union fold
constexpr int kWinWords = kWinChunks / 32;
constexpr int kRowWords = kWinWords + 1;  // padded bitmap row (bank-conflict-free columns)

struct Misc {
  uint64_t full[kStages], empty[kStages], s_full[2], p_full[2], o_done, q_ready, drain;
  uint32_t tmem_base, err;
  float red[2][2][4][16];
  float mrun[2][kQ];                      // running maxima per head, by group parity
  float scl[kQ];                          // rescale factors of the current tile
  int32_t tok0[kStages][kMaxEntries];
  int32_t page[kStages][kMaxEntries];     // paged caches: pool page of the entry's chunk
  int32_t nvalid[kStages][kMaxEntries];
  uint32_t emask[kStages][kMaxEntries];
  uint16_t rowj[kTok];                    // (entry << 8) | row in chunk, 0xffff = unused row
};

__host__ inline size_t split_smem_bytes(int64_t units) {
  return size_t(kOffMisc) + sizeof(Misc) + 4 * size_t(units + 1) + 1024;
}

// Chunks per tile for chunk size C.
__host__ __device__ inline int chunks_per_tile(int C) { return C >= kTok ? 1 : kTok / C; }

template <bool kMax>
__device__ __forceinline__ float transpose_reduce32(float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 16, half = 16; o > 0; o >>= 1, half >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? v[i] : v[i + half];
      const float keep = upper ? v[i + half] : v[i];
      const float got = __shfl_xor_sync(0xffffffffu, send, o);
      v[i] = kMax ? fmaxf(keep, got) : keep + got;
    }
  }
  return v[0];   // lane L holds the reduction of value L
}

// Reduction of 16 values over the 32 lanes of a warp: lane L ends with the
// reduction of value L % 16.
template <bool kMax>
__device__ __forceinline__ float transpose_reduce16(float (&v)[16]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 8, half = 8; o > 0; o >>= 1, half >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? v[i] : v[i + half];
      const float keep = upper ? v[i + half] : v[i];
      const float got = __shfl_xor_sync(0xffffffffu, send, o);
      v[i] = kMax ? fmaxf(keep, got) : keep + got;
    }
  }
  const float other = __shfl_xor_sync(0xffffffffu, v[0], 16);
  return kMax ? fmaxf(v[0], other) : v[0] + other;
}

// 32 x 32 bit transpose across a warp: lane i holds row i (bit j = column j);
// afterwards lane j holds column j (bit i = row i). Five block swaps.
__device__ __forceinline__ uint32_t transpose_bits32(uint32_t x) {
  const int lane = threadIdx.x & 31;
  constexpr uint32_t kMask[5] = {0x0000FFFFu, 0x00FF00FFu, 0x0F0F0F0Fu, 0x33333333u, 0x55555555u};
#pragma unroll
  for (int i = 0, s = 16; i < 5; ++i, s >>= 1) {
    const uint32_t y = __shfl_xor_sync(0xffffffffu, x, s);
    const uint32_t m = kMask[i];
    x = (lane & s) == 0 ? ((x & m) | ((y & m) << s)) : ((x & ~m) | ((y & ~m) >> s));
  }
  return x;
}

// Query head (flattened b * hq + h) of query q of group v.
__device__ __forceinline__ int64_t head_of(const Geom& G, int q_blocks, int v, int q) {
  const int g = v / q_blocks, qi = (v % q_blocks) * kQ + q;
  return int64_t(qi / G.group) * G.hq + g * G.group + qi % G.group;
}

__device__ __forceinline__ int group_width(const Geom& G, int batch, int q_blocks, int v) {
  return min(kQ, batch * G.group - (v % q_blocks) * kQ);
}

// First index of the ascending list a[0..n) with a[i] >= x (warp-cooperative:
// each round probes 32 evenly spaced entries of the remaining range).
__device__ __forceinline__ int warp_lower_bound(const int32_t* a, int n, int64_t x) {
  const int lane = threadIdx.x & 31;
  int lo = 0, hi = n;                      // answer in [lo, hi]
  while (hi - lo > 32) {
    const int step = (hi - lo + 31) / 32;
    const int idx = lo + lane * step;
    const bool below = idx < hi && int64_t(a[idx]) < x;
    const uint32_t ball = __ballot_sync(0xffffffffu, below);
    const int k = __popc(ball);            // probes below x (a prefix when ascending)
    const int nlo = k == 0 ? lo : lo + (k - 1) * step + 1;
    const int nhi = min(hi, lo + k * step);
    lo = nlo;
    hi = max(nlo, nhi);
  }
  const int idx = lo + lane;
  const bool below = idx < hi && int64_t(a[idx]) < x;
  return lo + __popc(__ballot_sync(0xffffffffu, below));
}

}  // namespace

// ---------------------------------------------------------------------------
// 1. Union of a group's chunk lists inside one block of chunks. A list entry is
// valid when it lies in [0, N_b / C) and is above the entry before it; anything
// else (and a count outside [0, max_sel]) sets ZHA_DEV_BAD_SELECTION, and which
// in-range entries of such a list are attended is then unspecified. Each unit
// validates its share of every list's indices, so each entry is checked once.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024)
union_prep_kernel(Geom G, int32_t batch, int32_t q_blocks, int32_t n_blocks, int64_t block_chunks,
                  int64_t nb, int64_t n_chunks, const int32_t* __restrict__ chunk_ids,
                  const int32_t* __restrict__ n_sel, int32_t max_sel, int32_t* __restrict__ ids,
                  uint32_t* __restrict__ masks, int64_t cap, int32_t* __restrict__ counts,
                  int32_t* status) {
  extern __shared__ uint32_t s_bits[];                 // [32][kRowWords]
  __shared__ uint32_t s_scan[33];
  pdl_trigger();
  pdl_wait();
  const int u = blockIdx.x, v = u / n_blocks, blk = u % n_blocks;
  const int tid = threadIdx.x, lane = tid & 31, q = tid >> 5;
  const int nq = group_width(G, batch, q_blocks, v);
  const int64_t c_lo = int64_t(blk) * block_chunks;
  const int64_t c_hi = min64(n_chunks, c_lo + block_chunks);
  const int32_t* list = nullptr;
  int n = 0, cursor = 0;
  bool bad = false;
  if (q < nq) {
    const int64_t bh = head_of(G, q_blocks, v, q);
    list = chunk_ids + bh * max_sel;
    const int raw = n_sel[bh];
    bad = raw < 0 || raw > max_sel;
    n = max(0, min(raw, max_sel));
    const int i0 = int(int64_t(n) * blk / n_blocks), i1 = int(int64_t(n) * (blk + 1) / n_blocks);
    for (int i = i0 + lane; i < i1; i += 32) {
      const int32_t id = list[i], prev = i > 0 ? list[i - 1] : -1;
      if (!(id >= 0 && int64_t(id) < n_chunks && id > prev)) bad = true;
    }
    if (n > 0 && c_lo < c_hi) cursor = warp_lower_bound(list, n, c_lo);
  }
  uint32_t* row = s_bits + q * kRowWords;
  int64_t total = 0;
  int32_t* out_ids = ids + int64_t(v) * cap + c_lo;
  uint32_t* out_masks = masks + int64_t(v) * cap + c_lo;

  for (int64_t win0 = c_lo; win0 < c_hi; win0 += kWinChunks) {
    const int wlen = int(min64(kWinChunks, c_hi - win0));
    const int words = (wlen + 31) / 32;
    const int64_t win_end = win0 + wlen;
    for (int w = lane; w < words; w += 32) row[w] = 0u;
    __syncwarp();
    while (cursor < n) {
      int stop = 0x7fffffff;
      int32_t id[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int idx = cursor + 32 * k + lane;
        id[k] = idx < n ? list[idx] : 0x7fffffff;
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int idx = cursor + 32 * k + lane;
        if (idx >= n) break;
        if (int64_t(id[k]) >= win_end) stop = min(stop, idx);
        else if (int64_t(id[k]) >= win0) {
          const int off = int(id[k] - win0);
          atomicOr(&row[off >> 5], 1u << (off & 31));
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) stop = min(stop, __shfl_xor_sync(0xffffffffu, stop, o));
      if (stop != 0x7fffffff) { cursor = stop; break; }
      cursor += 256;
    }
    __syncthreads();
    // Warp wq owns words [wq * per, wq * per + per): transpose each word's 32
    // rows into per-chunk masks, then compact in chunk order.
    const int per = (words + 31) / 32;            // <= 16
    uint32_t msk[16], ball[16];
    uint32_t warp_cnt = 0;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      msk[k] = 0u;
      ball[k] = 0u;
      const int w = q * per + k;
      if (k < per && w < words) {                  // uniform over the warp
        const uint32_t x = s_bits[lane * kRowWords + w];
        const uint32_t m = transpose_bits32(x);
        const int off = 32 * w + lane;
        const bool present = off < wlen && (m != 0u || (win0 + off == 0 && nb > 0));
        msk[k] = m;
        ball[k] = __ballot_sync(0xffffffffu, present);
        warp_cnt += __popc(ball[k]);
      }
    }
    if (lane == 0) s_scan[q] = warp_cnt;
    __syncthreads();
    if (q == 0) {                                  // exclusive scan of the 32 warp counts
      const uint32_t c = s_scan[lane];
      uint32_t incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      s_scan[lane] = incl - c;
      if (lane == 31) s_scan[32] = incl;
    }
    __syncthreads();
    int64_t pos = total + s_scan[q];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      if ((ball[k] >> lane) & 1u) {
        const int64_t at = pos + __popc(ball[k] & ((1u << lane) - 1u));
        const int off = 32 * (q * per + k) + lane;
        out_ids[at] = int32_t(win0 + off);
        out_masks[at] = msk[k];
      }
      pos += __popc(ball[k]);
    }
    total += s_scan[32];
    __syncthreads();                                   // s_bits and s_scan are reused
  }
  const int any_bad = __syncthreads_or(bad ? 1 : 0);
  if (tid == 0) {
    counts[u] = int32_t(total);
    if (any_bad && status != nullptr) atomicOr(status, ZHA_DEV_BAD_SELECTION);
  }
}

// ---------------------------------------------------------------------------
// 2. Split attention over the units' tiles. Each role walks the CTA's span
// [t0, t1) of the tile sequence the same way; li is the CTA-local tile index
// that drives every barrier's phase.
// ---------------------------------------------------------------------------
struct SpanWalk {
  const int32_t* toff;       // tile offsets of the units (shared memory)
  int n_blocks;
  int u;                     // current unit
  int g = -1;                // its group, and the group's first and end tile
  int32_t g_lo = 0, g_hi = 0;
  // Advance to the unit holding tile t (t is non-decreasing between calls).
  __device__ __forceinline__ void seek(int64_t t) {
    while (t >= toff[u + 1]) ++u;
    const int gu = u / n_blocks;
    if (gu != g) {
      g = gu;
      g_lo = toff[gu * n_blocks];
      g_hi = toff[(gu + 1) * n_blocks];
    }
  }
  __device__ __forceinline__ int group() const { return g; }
  __device__ __forceinline__ bool group_start(int64_t t, int64_t t0) const {
    return t == t0 || t == g_lo;
  }
  __device__ __forceinline__ bool group_end(int64_t t, int64_t t1) const {
    return t + 1 == t1 || t + 1 == g_hi;
  }
};

// kTma: K and V rows arrive by tiled tensor copies (one box of C rows per chunk
// and 64-column half, issued by one thread); needs C % 8 == 0 so that every box
// starts on a 1024-byte swizzle atom. Otherwise two warps stage rows with
// cp.async (zero-filling rows without a token).
// 2^x by the hardware approximation (a few ulp; results below 2^-126 are 0).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two fp32 values -> their bf16x2 rounding and the bf16x2 rounding of the
// remainders (x0 in the low halves).
__device__ __forceinline__ void split_bf16x2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float2 f = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - f.x, x1 - f.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

template <bool kTma>
__global__ void __launch_bounds__(kThreads, 1)
attend_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    Geom G, int32_t batch, int32_t q_blocks, int32_t n_blocks, int64_t block_chunks,
                    int32_t units, int64_t n_tokens, int64_t nb, const float* __restrict__ Q,
                    KvView kv, const int32_t* __restrict__ ids, const uint32_t* __restrict__ masks,
                    int64_t cap, const int32_t* __restrict__ counts, int32_t* __restrict__ split,
                    float* __restrict__ slots, int32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Misc& ms = *reinterpret_cast<Misc*>(smem + kOffMisc);
  int32_t* s_toff = reinterpret_cast<int32_t*>(smem + kOffMisc + sizeof(Misc));   // [units + 1]
  pdl_trigger();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int C = G.chunk;
  const int cpt = chunks_per_tile(C);
  const bool paged = kv.table != nullptr;
  const __nv_bfloat16* __restrict__ K = static_cast<const __nv_bfloat16*>(kv.k);
  const __nv_bfloat16* __restrict__ V = static_cast<const __nv_bfloat16*>(kv.v);
  const int64_t n_tail = n_tokens - nb;
  const int has_tail = n_tail > 0 ? 1 : 0;
  // Tiles of unit u: its entries, plus the tail in a group's last block.
  auto unit_tiles = [&](int uu) -> int {
    const int e = counts[uu] + ((uu % n_blocks == n_blocks - 1) ? has_tail : 0);
    return (e + cpt - 1) / cpt;
  };

  // Setup that reads nothing the previous kernel writes runs before the
  // dependency wait (programmatic dependent launch).
  if (tid < kTok) {
    const int j = C >= kTok ? 0 : tid / C, rr = C >= kTok ? tid : tid % C;
    ms.rowj[tid] = (j < cpt && rr < C) ? uint16_t((j << 8) | rr) : uint16_t(0xffff);
  }
  if (tid < kQ) ms.mrun[0][tid] = -INFINITY;
  if (tid == 0) {
    ms.err = 0u;
    for (int st = 0; st < kStages; ++st) {
      tc::mbar_init(&ms.full[st], kTma ? 1 : kProducers + 1);
      tc::mbar_init(&ms.empty[st], 1);
    }
    for (int bb = 0; bb < 2; ++bb) {
      tc::mbar_init(&ms.s_full[bb], 1);
      tc::mbar_init(&ms.p_full[bb], 8);           // one arrival per softmax warp
    }
    tc::mbar_init(&ms.o_done, 1);
    tc::mbar_init(&ms.q_ready, 8);
    tc::mbar_init(&ms.drain, 1);
  }
  if (kTma) {
    // Rows of a tile that no chunk fills keep what the stage held before; the
    // V rows must at least be finite (P is 0 there), so clear them once.
    for (int i = tid; i < kStages * 2048; i += kThreads) {
      const int st = i / 2048, k = i % 2048;
      *reinterpret_cast<uint4*>(smem + st * kStageBytes + 32768 + k * 16) = make_uint4(0u, 0u, 0u, 0u);
    }
    tc::fence_async_smem();
  }
  if (warp == 2) tc::tmem_alloc(&ms.tmem_base, kTmemCols);
  pdl_wait();                                    // counts of the union prep from here on
  // Tile offsets of the units: warp 0, a blocked scan.
  if (warp == 0) {
    const int per = (units + 31) / 32;
    const int b0 = min(units, lane * per), b1 = min(units, b0 + per);
    int sum = 0;
    for (int uu = b0; uu < b1; ++uu) sum += unit_tiles(uu);
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int run = incl - sum;
    for (int uu = b0; uu < b1; ++uu) {
      s_toff[uu] = run;
      run += unit_tiles(uu);
    }
    if (lane == 31) s_toff[units] = incl;
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = ms.tmem_base;

  const int64_t T = s_toff[units];
  const int nct = int(gridDim.x), cta = int(blockIdx.x);
  const int64_t t0 = int64_t(cta) * T / nct, t1 = int64_t(cta + 1) * T / nct;
  if (cta == 0) {
    for (int uu = tid; uu <= units; uu += blockDim.x) split[uu] = s_toff[uu];
    if (tid == 0) split[units + 1] = nct;
  }
  int u0 = 0;
  if (t0 < t1) {            // last unit whose first tile is <= t0 (it holds t0)
    int lo = 0, hi = units - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (int64_t(s_toff[mid]) <= t0) lo = mid; else hi = mid - 1;
    }
    u0 = lo;
  }

  if (warp < 2) {
    // ---------------- producers: K and V rows of each tile ----------------
    // Warp 0 lanes read the entries of the next tile into registers while the
    // current tile's copies are issued; they land in shared memory once the
    // stage is free.
    const int ptid = tid, piece = ptid & 15, rs = ptid >> 4;
    SpanWalk wk{s_toff, n_blocks, u0};
    int32_t pf_tok0[2] = {-1, -1}, pf_nv[2] = {0, 0}, pf_pg[2] = {0, 0};
    uint32_t pf_m[2] = {0u, 0u};
    bool bad_page = false;
    int e_unit = -1, e_count = 0;                  // the unit whose entry count is held
    auto prefetch = [&](int64_t t) {
      wk.seek(t);
      const int uu = wk.u, v = uu / n_blocks, blk = uu % n_blocks;
      const int gkv = v / q_blocks;
      if (uu != e_unit) {                          // a load only when the unit changes
        e_unit = uu;
        e_count = counts[uu];
      }
      const int E = e_count;
      const bool tail_here = has_tail && blk == n_blocks - 1;
      const int nq = group_width(G, batch, q_blocks, v);
      const uint32_t allq = nq == 32 ? 0xffffffffu : ((1u << nq) - 1u);
      const int64_t tu = t - s_toff[uu];
      const int64_t base = int64_t(v) * cap + int64_t(blk) * block_chunks;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int j = lane + 32 * h;
        const int64_t e = tu * cpt + j;
        pf_tok0[h] = -1; pf_nv[h] = 0; pf_m[h] = 0u;
        if (j < cpt) {
          if (e < E) {
            pf_tok0[h] = ids[base + e] * C;
            pf_nv[h] = C;
            pf_m[h] = masks[base + e];
          } else if (e == E && tail_here) {
            pf_tok0[h] = int32_t(nb);
            pf_nv[h] = int32_t(n_tail);
            pf_m[h] = allq;
          }
          // Paged cache: the entry's page; one outside the pool drops the entry.
          if (paged && pf_tok0[h] >= 0) {
            const int64_t row = kv_row(kv, gkv, pf_tok0[h], C);
            if (row < 0) {
              pf_tok0[h] = -1; pf_nv[h] = 0; pf_m[h] = 0u;
              bad_page = true;
            } else {
              pf_pg[h] = int32_t(row / C);
            }
          }
        }
      }
    };
    bool failed = false;
    if (warp == 0 && t0 < t1) prefetch(t0);
    SpanWalk wc{s_toff, n_blocks, u0};
    int64_t li = 0;
    if (kTma) {
      if (warp == 0) {
        for (int64_t t = t0; t < t1; ++t, ++li) {
          wc.seek(t);
          const int32_t g = wc.group() / q_blocks;
          const int st = int(li % kStages);
          const int64_t use = li / kStages;
          bool bad = false;
          if (use > 0) bad = !tc::mbar_wait(&ms.empty[st], uint32_t((use - 1) & 1), kWaitTries);
          if (__any_sync(0xffffffffu, bad)) { failed = true; break; }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int j = lane + 32 * h;
            if (j < cpt) {
              ms.tok0[st][j] = pf_tok0[h];
              ms.page[st][j] = pf_pg[h];
              ms.nvalid[st][j] = pf_nv[h];
              ms.emask[st][j] = pf_m[h];
            }
          }
          const uint32_t n_ok = __popc(__ballot_sync(0xffffffffu, pf_tok0[0] >= 0 && lane < cpt)) +
                                __popc(__ballot_sync(0xffffffffu, pf_tok0[1] >= 0 && lane + 32 < cpt));
          __syncwarp();
          // The stage's byte count first (after the entries above), then each
          // lane issues the copies of its own entries.
          if (lane == 0) tc::mbar_arrive_expect_tx(&ms.full[st], n_ok * 512u * uint32_t(C));
          __syncwarp();
          {
            const uint32_t sK = tc::smem_u32(smem + st * kStageBytes), sV = sK + 32768;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int j = lane + 32 * h;
              if (j < cpt && pf_tok0[h] >= 0) {
                const uint32_t roff = uint32_t(j * C * 128);
                // contiguous: {d, tokens, KV head}; paged: {d, row in page, page}
                const int32_t y = paged ? 0 : pf_tok0[h], z = paged ? pf_pg[h] : g;
                tc::tma_load_3d(sK + roff, &tmK, 0, y, z, &ms.full[st]);
                tc::tma_load_3d(sK + 16384 + roff, &tmK, 64, y, z, &ms.full[st]);
                tc::tma_load_3d(sV + roff, &tmV, 0, y, z, &ms.full[st]);
                tc::tma_load_3d(sV + 16384 + roff, &tmV, 64, y, z, &ms.full[st]);
              }
            }
          }
          __syncwarp();
          if (t + 1 < t1) prefetch(t + 1);
        }
        // Every tensor copy issued into the stages lands before the CTA may exit.
        if (lane == 0)
          for (int64_t j = li > kStages ? li - kStages : 0; j < li; ++j)
            if (!tc::mbar_wait(&ms.full[j % kStages], uint32_t((j / kStages) & 1), kWaitTries)) failed = true;
        if (failed && lane == 0) atomicOr(&ms.err, 1u);
        if (__any_sync(0xffffffffu, bad_page) && lane == 0 && status != nullptr)
          atomicOr(status, ZHA_DEV_BAD_PAGE);
      }
    } else {
    for (int64_t t = t0; t < t1; ++t, ++li) {
      wc.seek(t);
      const int64_t g = wc.group() / q_blocks;
      const int st = int(li % kStages);
      const int64_t use = li / kStages;
      bool bad = false;
      if (use > 0) bad = !tc::mbar_wait(&ms.empty[st], uint32_t((use - 1) & 1), kWaitTries);
      if (warp == 0 && !bad) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int j = lane + 32 * h;
          if (j < cpt) {
            ms.tok0[st][j] = pf_tok0[h];
            ms.page[st][j] = pf_pg[h];
            ms.nvalid[st][j] = pf_nv[h];
            ms.emask[st][j] = pf_m[h];
          }
        }
      }
      if (tc::named_sync_or(2, kProducers, bad)) { failed = true; break; }
      if (warp == 0 && t + 1 < t1) prefetch(t + 1);
      const uint32_t sK = tc::smem_u32(smem + st * kStageBytes), sV = sK + 32768;
#pragma unroll 4
      for (int k = 0; k < kTok / 4; ++k) {
        const int r = rs + 4 * k;
        const uint32_t jr = ms.rowj[r];
        bool valid = false;
        int64_t row = 0;
        if (jr != 0xffffu) {
          const int j = int(jr >> 8), rr = int(jr & 255u);
          const int32_t tok0 = ms.tok0[st][j];
          if (tok0 >= 0 && rr < ms.nvalid[st][j]) {
            // contiguous: row of KV head g; paged: row rr of the entry's page
            row = paged ? int64_t(ms.page[st][j]) * C + rr : g * kv.ld + int64_t(tok0) + rr;
            valid = true;
          }
        }
        const uint32_t off = tc::sw128_offset(r, 8 * piece, kTok);
        tc::cp_async16(sK + off, K + row * kD + 8 * piece, valid ? 16u : 0u);
        tc::cp_async16(sV + off, V + row * kD + 8 * piece, valid ? 16u : 0u);
      }
      tc::cp_async_arrive_noinc(&ms.full[st]);
      if (ptid == 0) tc::mbar_arrive(&ms.full[st]);
    }
    tc::cp_async_wait_pending0();
    if (failed && ptid == 0) atomicOr(&ms.err, 1u);
    if (warp == 0 && __any_sync(0xffffffffu, bad_page) && lane == 0 && status != nullptr)
      atomicOr(status, ZHA_DEV_BAD_PAGE);
    }
  } else if (warp == 2) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      // The two bf16 terms of Q (and of P) are stacked along N: one MMA gives
      // both partial products, summed when TMEM is read.
      constexpr uint32_t idesc_s = tc::idesc_bf16(kTok, 2 * kQ, 0, 0);
      constexpr uint32_t idesc_pv = tc::idesc_bf16(kD, 2 * kQ, 1, 1);
      const uint32_t sQ = tc::smem_u32(smem + kOffQ);
      const int64_t n = t1 - t0;
      SpanWalk ws_{s_toff, n_blocks, u0}, wp_{s_toff, n_blocks, u0};
      int64_t ns = 0, np = 0;        // next tile to score (S), next tile to apply (PV)
      int seg = 0;                   // groups whose Q has been taken
      uint32_t idle = 0;
      bool failed = false;
      while (np < n) {
        bool progress = false;
        // PV first: it frees a stage for the producers.
        if (np < ns && tc::mbar_test(&ms.p_full[np & 1], uint32_t((np >> 1) & 1))) {
          const int64_t t = t0 + np;
          wp_.seek(t);
          const bool first = wp_.group_start(t, t0);
          tc::fence_after_sync();
          const uint32_t sP = tc::smem_u32(smem + (np % kStages) * kStageBytes), sV = sP + 32768;
#pragma unroll
          for (int ks = 0; ks < kTok / 16; ++ks) {
            const uint64_t a = tc::desc_sw128(sV + ks * 2048, 16384, 1024);
            const uint64_t b = tc::desc_sw128(sP + ks * 2048, 8192, 1024);
            tc::mma_bf16(tbase + kTmemO, a, b, idesc_pv, (first && ks == 0) ? 0u : 1u);
          }
          tc::mma_commit(&ms.o_done);
          tc::mma_commit(&ms.empty[np % kStages]);
          ++np;
          progress = true;
        }
        // S of the next tile once it has landed, its S buffer is free (the
        // softmax has taken S of tile ns - 2, i.e. PV of it was issued) and,
        // at a group start, the group's Q is in place.
        if (ns < n && ns <= np + 1 &&
            tc::mbar_test(&ms.full[ns % kStages], uint32_t((ns / kStages) & 1))) {
          const int64_t t = t0 + ns;
          ws_.seek(t);
          const bool start = ws_.group_start(t, t0);
          if (!start || tc::mbar_test(&ms.q_ready, uint32_t(seg & 1))) {
            if (start) ++seg;
            tc::fence_after_sync();
            const uint32_t sK = tc::smem_u32(smem + (ns % kStages) * kStageBytes);
            const uint32_t d_s = tbase + uint32_t(ns & 1) * 64;
#pragma unroll
            for (int ks = 0; ks < kD / 16; ++ks) {
              const uint64_t a = tc::desc_sw128(sK + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
              const uint64_t b = tc::desc_sw128(sQ + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024);
              tc::mma_bf16(d_s, a, b, idesc_s, ks != 0 ? 1u : 0u);
            }
            tc::mma_commit(&ms.s_full[ns & 1]);
            ++ns;
            progress = true;
          }
        }
        if (progress) {
          idle = 0;
        } else if (++idle > kPollLimit) {
          failed = true;
          break;
        }
      }
      tc::mma_commit(&ms.drain);
      if (!tc::mbar_wait(&ms.drain, 0u, kWaitTries)) failed = true;
      if (failed) atomicOr(&ms.err, 1u);
    }
  } else if (warp >= 4) {
    // ---------------- softmax: two warpgroups, thread = tile row / TMEM lane ----------------
    // Warpgroup wg (warps 4 + 4 wg .. 7 + 4 wg) owns heads [16 wg, 16 wg + 16):
    // its S and O columns, its part of P, its running maxima and row sums.
    const int wg = (warp - 4) >> 2;
    const int sw = warp & 3;                       // TMEM lane quadrant
    const int stid = tid - 128;                    // 0..255 over both warpgroups
    const int r = sw * 32 + lane;                  // tile row / output dim
    const int q0 = kHalfQ * wg;
    const int bar_id = 1 + 2 * wg;                 // named barrier of the warpgroup
    const uint32_t t_lane = uint32_t(sw * 32) << 16;
    const float scale2 = G.scale * 1.4426950408889634f;     // 1/sqrt(d) * log2(e)
    float lrow[kHalfQ];
#pragma unroll
    for (int i = 0; i < kHalfQ; ++i) lrow[i] = 0.f;
    int gp = 0;                                    // group parity: ms.mrun[gp] is live
    float mr[kHalfQ];                              // this warpgroup's running maxima (= ms.mrun[gp])
#pragma unroll
    for (int i = 0; i < kHalfQ; ++i) mr[i] = -INFINITY;

    // Q of group vq -> two bf16 terms, K-major 128-byte-swizzled rows: row q the
    // high term of head q, row 32 + q its low term (both warpgroups share it).
    auto write_q = [&](int vq) {
      const int nq = group_width(G, batch, q_blocks, vq);
      const int q = stid >> 3, part = stid & 7;
#pragma unroll
      for (int c8 = 0; c8 < 2; ++c8) {
        const int col = part * 16 + c8 * 8;
        float x[8];
        if (q < nq) {
          const float* src = Q + head_of(G, q_blocks, vq, q) * kD + col;
          const float4 a = *reinterpret_cast<const float4*>(src);
          const float4 b = *reinterpret_cast<const float4*>(src + 4);
          x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) x[i] = 0.f;
        }
        __align__(16) __nv_bfloat16 hi[8], lo[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          hi[i] = __float2bfloat16_rn(x[i]);
          lo[i] = __float2bfloat16_rn(x[i] - __bfloat162float(hi[i]));
        }
        *reinterpret_cast<uint4*>(smem + kOffQ + tc::sw128_offset(q, col, 2 * kQ)) =
            *reinterpret_cast<const uint4*>(hi);
        *reinterpret_cast<uint4*>(smem + kOffQ + tc::sw128_offset(kQ + q, col, 2 * kQ)) =
            *reinterpret_cast<const uint4*>(lo);
      }
      tc::fence_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&ms.q_ready);
    };

    SpanWalk wk{s_toff, n_blocks, u0};
    int64_t od = 0;                // PV completions of o_done known to this thread
    bool failed = false, pending_bad = false;
    // Wait for the PV of tile k (k = li - 1 before this thread's P of tile li
    // is signalled, or k = li after it at a group's last tile, once PV of
    // li - 1 is known complete). Once s_full of tile li is observed, the PVs of
    // tiles < li - 1 are complete: S of tile li was issued after them, and its
    // commit tracks every earlier MMA. So before P of tile li, o_done has
    // completed li - 1 or li times; after it, with PV of li - 1 waited for, li
    // or li + 1 times (PV of li + 1 needs this thread's next P). Each phase
    // waited for (in order, from od) is therefore unambiguous.
    auto wait_pv = [&](int64_t k) -> bool {
      bool ok = true;
      while (od <= k) {
        ok &= tc::mbar_wait(&ms.o_done, uint32_t(od & 1), kWaitTries);
        ++od;
      }
      return ok;
    };
    uint32_t allq = 0u;
    const uint32_t jr = ms.rowj[r];                // this row's (chunk entry, row in chunk)
    if (t0 < t1) write_q(u0 / n_blocks);
    int64_t li = 0;
    int st = 0;                                    // li % kStages
    uint32_t st_ph = 0u;                           // (li / kStages) & 1
    for (int64_t t = t0; t < t1; ++t, ++li) {
      if (li > 0 && ++st == kStages) {
        st = 0;
        st_ph ^= 1u;
      }
      wk.seek(t);
      const int v = wk.group();
      const bool start = wk.group_start(t, t0);
      const bool end = wk.group_end(t, t1);
      if (start) {
        const int nq = group_width(G, batch, q_blocks, v);
        allq = nq == 32 ? 0xffffffffu : ((1u << nq) - 1u);
      }
      bool bad = !tc::mbar_wait(&ms.full[st], st_ph, kWaitTries);
      bad |= !tc::mbar_wait(&ms.s_full[li & 1], uint32_t((li >> 1) & 1), kWaitTries);
      bad |= pending_bad;
      pending_bad = false;
      if (od < li - 1) od = li - 1;                // PVs before tile li - 1 are complete
      tc::fence_after_sync();
      float s[kHalfQ];
      {
        const uint32_t col = tbase + t_lane + uint32_t(li & 1) * 64 + q0;
        float s_lo[kHalfQ];
        tc::tmem_ld16(col, s);
        tc::tmem_ld16(col + 32, s_lo);
#pragma unroll
        for (int i = 0; i < kHalfQ; ++i) s[i] += s_lo[i];
      }
      uint32_t rmask = 0u;
      {
        if (jr != 0xffffu) {
          const int j = int(jr >> 8), rr = int(jr & 255u);
          const int32_t tok0 = ms.tok0[st][j];
          if (tok0 >= 0 && rr < ms.nvalid[st][j]) {
            rmask = (tok0 + rr == 0) ? allq : ms.emask[st][j];
          } else if (kTma && paged && wg == 0 && tok0 >= 0) {
            // A tensor copy brings whole pages: this row of the in-progress
            // chunk's page holds no token yet, and its V must not carry
            // non-finite bytes into the P.V product (P is 0 there).
            uint8_t* vrow = smem + st * kStageBytes + 32768 + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int c16 = 0; c16 < 8; ++c16)
                *reinterpret_cast<uint4*>(vrow + h * 16384 + c16 * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        rmask >>= q0;
      }
      bool fire = false;
#pragma unroll
      for (int i = 0; i < kHalfQ; ++i) {
        s[i] = ((rmask >> i) & 1u) ? s[i] * scale2 : -INFINITY;
        fire |= s[i] > mr[i] + kRescaleSlack;
      }
      // One barrier tells the warpgroup whether any thread saw a score past its
      // running maximum plus the slack, or a failed wait; only then a second
      // one tells the two apart.
      bool rescale = false;
      if (tc::named_sync_or(bar_id, 128, fire || bad)) {
        if (tc::named_sync_or(bar_id, 128, bad)) { failed = true; break; }
        rescale = true;
      }
      // S of this tile is complete, so Q may be replaced for the next group now.
      if (end && t + 1 < t1) write_q(v + 1);
      if (rescale) {
        // Raise this warpgroup's running maxima to the tile's, rescale l and O.
        float tmp[kHalfQ];
#pragma unroll
        for (int i = 0; i < kHalfQ; ++i) tmp[i] = s[i];
        const float wmax = transpose_reduce16<true>(tmp);
        if (lane < kHalfQ) ms.red[0][wg][sw][lane] = wmax;
        tc::named_sync(bar_id, 128);
        if (sw == 0 && lane < kHalfQ) {  // lane = head q0 + lane
          const float mt = fmaxf(fmaxf(ms.red[0][wg][0][lane], ms.red[0][wg][1][lane]),
                                 fmaxf(ms.red[0][wg][2][lane], ms.red[0][wg][3][lane]));
          const float mo = ms.mrun[gp][q0 + lane];
          const float mn = fmaxf(mo, mt);
          ms.scl[q0 + lane] = mn == -INFINITY ? 1.f : exp2f(mo - mn);
          ms.mrun[gp][q0 + lane] = mn;
        }
        tc::named_sync(bar_id, 128);
        const float* scl = ms.scl + q0;
#pragma unroll
        for (int i = 0; i < kHalfQ; ++i) {
          lrow[i] *= scl[i];
          mr[i] = ms.mrun[gp][q0 + i];
        }
        if (!start) {                    // O holds earlier tiles of this group
          pending_bad |= !wait_pv(li - 1);
          tc::fence_after_sync();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            float o[kHalfQ];
            tc::tmem_ld16(tbase + t_lane + kTmemO + 32 * h + q0, o);
#pragma unroll
            for (int i = 0; i < kHalfQ; ++i) o[i] *= scl[i];
            tc::tmem_st16(tbase + t_lane + kTmemO + 32 * h + q0, o);
          }
        }
      }
      // p = 2^(s - m), stored MN-major over the stage's consumed K rows: row =
      // token, 64 bf16 (the high terms of the 32 heads, then the low terms),
      // 128-byte swizzled; this warpgroup writes its 16 heads of each half.
      // The exponent is at most kRescaleSlack; ex2.approx (flushing results
      // below 2^-126 to zero) is accurate to a few ulp there. Pairs of heads
      // are rounded to bf16x2 in one conversion.
      uint8_t* sP = smem + st * kStageBytes;
#pragma unroll
      for (int c = 0; c < kHalfQ / 8; ++c) {
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int jp = 0; jp < 4; ++jp) {
          const int i = 8 * c + 2 * jp;
          const float p0 = mr[i] == -INFINITY ? 0.f : fast_exp2(s[i] - mr[i]);
          const float p1 = mr[i + 1] == -INFINITY ? 0.f : fast_exp2(s[i + 1] - mr[i + 1]);
          lrow[i] += p0;
          lrow[i + 1] += p1;
          split_bf16x2(p0, p1, hi[jp], lo[jp]);
        }
        *reinterpret_cast<uint4*>(sP + tc::sw128_offset(r, q0 + 8 * c, kTok)) =
            make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(sP + tc::sw128_offset(r, kQ + q0 + 8 * c, kTok)) =
            make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      // At a group's last tile PV of the previous tile completes first, so that
      // the wait for this tile's PV below starts from a known phase.
      if (end && li > 0) pending_bad |= !wait_pv(li - 1);
      tc::fence_async_smem();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&ms.p_full[li & 1]);   // for the warp's 32 rows
      if (end) {
        // The group's piece of this span is done: write one state per head.
        const bool bad2 = !wait_pv(li) || pending_bad;
        pending_bad = false;
        tc::fence_after_sync();
        float o[kHalfQ];
        {
          float o_lo[kHalfQ];
          tc::tmem_ld16(tbase + t_lane + kTmemO + q0, o);
          tc::tmem_ld16(tbase + t_lane + kTmemO + 32 + q0, o_lo);
#pragma unroll
          for (int i = 0; i < kHalfQ; ++i) o[i] += o_lo[i];
        }
        float tmp[kHalfQ];
#pragma unroll
        for (int i = 0; i < kHalfQ; ++i) tmp[i] = lrow[i];
        const float wsum = transpose_reduce16<false>(tmp);
        if (lane < kHalfQ) ms.red[1][wg][sw][lane] = wsum;
        if (sw == 0 && lane < kHalfQ) ms.mrun[gp ^ 1][q0 + lane] = -INFINITY;   // next group
        if (tc::named_sync_or(bar_id, 128, bad2)) { failed = true; break; }
        const int nq = group_width(G, batch, q_blocks, v);
        float* base = slots + int64_t(cta + v) * kQ * (kD + 4);
#pragma unroll
        for (int i = 0; i < kHalfQ; ++i)
          if (q0 + i < nq) base[(q0 + i) * (kD + 4) + 4 + r] = o[i];
        if (sw == 0 && lane < kHalfQ && q0 + lane < nq) {
          const float mq = ms.mrun[gp][q0 + lane];
          const float L = ms.red[1][wg][0][lane] + ms.red[1][wg][1][lane] + ms.red[1][wg][2][lane] +
                          ms.red[1][wg][3][lane];
          // maximum back to natural-log units
          *reinterpret_cast<float4*>(base + (q0 + lane) * (kD + 4)) =
              make_float4(mq * 0.6931471805599453f, L, 0.f, 0.f);
        }
#pragma unroll
        for (int i = 0; i < kHalfQ; ++i) {
          lrow[i] = 0.f;
          mr[i] = -INFINITY;             // the next group's maxima (set above)
        }
        gp ^= 1;
      }
    }
    if (failed && (stid & 127) == 0) atomicOr(&ms.err, 1u);
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 2) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, kTmemCols);
  }
  if (tid == 0 && ms.err != 0u && status != nullptr) atomicOr(status, ZHA_DEV_TIMEOUT);
}

// ---------------------------------------------------------------------------
// 3. Combine: one CTA of 4 warps per query head over the states of the CTAs
// whose span met the head's group. CTA c covers tiles [c T / n, (c + 1) T / n),
// so the CTA holding tile t is ((t + 1) n - 1) / T. Warp w merges states
// i = w, w + 4, ... (lane = 4 output dims); the four partial merges are then
// combined through shared memory.
// ---------------------------------------------------------------------------
constexpr int kCombineWarps = 4;

__global__ void __launch_bounds__(32 * kCombineWarps)
combine_split_kernel(Geom G, int32_t batch, int32_t q_blocks, int32_t n_blocks, int32_t units,
                     const int32_t* __restrict__ split, const float* __restrict__ slots,
                     float* __restrict__ O, float* __restrict__ lse) {
  __shared__ float4 s_acc[kCombineWarps][32];
  __shared__ float s_m[kCombineWarps], s_l[kCombineWarps];
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t bh = blockIdx.x;
  const int b = int(bh / G.hq), h = int(bh % G.hq);
  const int qi = b * G.group + h % G.group;
  const int v = (h / G.group) * q_blocks + qi / kQ, q = qi % kQ;
  const int64_t lo = split[v * n_blocks], hi = split[(v + 1) * n_blocks], T = split[units];
  const int64_t nct = split[units + 1];
  const int c_lo = int(((lo + 1) * nct - 1) / T), c_hi = int((hi * nct - 1) / T);
  const int n_st = c_hi - c_lo + 1;                     // >= 1: every group has a tile
  // A CTA between c_lo and c_hi meets the group unless its span is empty (more
  // CTAs than tiles); only states that were written are read.
  auto written = [&](int i) -> bool {
    const int64_t c = c_lo + i;
    return (c + 1) * T / nct > c * T / nct;
  };
  auto state = [&](int i) -> const float* {
    return slots + (int64_t(c_lo + i + v) * kQ + q) * (kD + 4);
  };
  // This warp's states: i = warp + 4 (32 r + j); in round r lane j holds
  // state (r, j)'s (m, l). Rounds are merged with the usual rescaling.
  float M = -INFINITY, L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int r0 = 0; warp + kCombineWarps * r0 < n_st; r0 += 32) {
    float m_j = -INFINITY, l_j = 0.f;
    const int i_lane = warp + kCombineWarps * (r0 + lane);
    if (i_lane < n_st && written(i_lane)) {
      const float2 ml = *reinterpret_cast<const float2*>(state(i_lane));
      if (ml.y > 0.f) { m_j = ml.x; l_j = ml.y; }
    }
    const float Mr = warp_max(m_j);
    if (Mr == -INFINITY) continue;
    const float Mn = fmaxf(M, Mr);
    const float sc = M == -INFINITY ? 0.f : expf(M - Mn);
    L *= sc;
    acc.x *= sc; acc.y *= sc; acc.z *= sc; acc.w *= sc;
    M = Mn;
    const float w_j = l_j > 0.f ? expf(m_j - M) : 0.f;
    L += warp_sum(w_j * l_j);
    uint32_t ball = __ballot_sync(0xffffffffu, w_j > 0.f);
    while (ball) {                 // up to four states per step, loads in flight together
      int src[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        src[k] = ball ? __ffs(ball) - 1 : -1;
        if (ball) ball &= ball - 1u;
      }
      float4 o[4];
      float wk[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        wk[k] = __shfl_sync(0xffffffffu, w_j, src[k] < 0 ? 0 : src[k]);
        o[k] = src[k] < 0 ? make_float4(0.f, 0.f, 0.f, 0.f)
                          : *reinterpret_cast<const float4*>(
                                state(warp + kCombineWarps * (r0 + src[k])) + 4 + 4 * lane);
        if (src[k] < 0) wk[k] = 0.f;
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        acc.x += wk[k] * o[k].x; acc.y += wk[k] * o[k].y;
        acc.z += wk[k] * o[k].z; acc.w += wk[k] * o[k].w;
      }
    }
  }
  s_acc[warp][lane] = acc;
  if (lane == 0) { s_m[warp] = M; s_l[warp] = L; }
  __syncthreads();
  if (warp == 0) {
    float Mt = -INFINITY;
#pragma unroll
    for (int w = 0; w < kCombineWarps; ++w)
      if (s_l[w] > 0.f) Mt = fmaxf(Mt, s_m[w]);
    float Lt = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < kCombineWarps; ++w) {
      if (!(s_l[w] > 0.f)) continue;
      const float r = expf(s_m[w] - Mt);
      Lt += r * s_l[w];
      const float4 a = s_acc[w][lane];
      o.x += r * a.x; o.y += r * a.y; o.z += r * a.z; o.w += r * a.w;
    }
    const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
    *reinterpret_cast<float4*>(O + bh * kD + 4 * lane) = make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
    if (lse != nullptr && lane == 0) lse[bh] = Lt > 0.f ? Mt + logf(Lt) : -INFINITY;
  }
}

namespace {

// [Hkv][ld][d] bf16 cache as a 3-D tensor {d, n_tokens, Hkv}: rows at or past
// n_tokens read as zeros. Box = 64 columns (128 B, the swizzle span) x box_rows.
bool kv_tensor_map(CUtensorMap* m, const void* base, int64_t n_tokens, int64_t ld, int hkv,
                   int box_rows) {
  const PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {cuuint64_t(kD), cuuint64_t(n_tokens), cuuint64_t(hkv)};
  const cuuint64_t strides[2] = {cuuint64_t(kD) * 2, cuuint64_t(ld) * kD * 2};
  const cuuint32_t box[3] = {64u, cuuint32_t(box_rows), 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A bf16 page pool [n_pages][C][d] as a 3-D tensor {d, C, n_pages}: box = 64
// columns x the C rows of one page; a page id outside the pool reads as zeros.
bool page_tensor_map(CUtensorMap* m, const void* base, int64_t n_pages, int chunk) {
  const PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {cuuint64_t(kD), cuuint64_t(chunk), cuuint64_t(n_pages)};
  const cuuint64_t strides[2] = {cuuint64_t(kD) * 2, cuuint64_t(chunk) * kD * 2};
  const cuuint32_t box[3] = {64u, cuuint32_t(chunk), 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_attend_tc(const Geom& G, const float* Q, const KvView& kv, int64_t n_tokens,
                             int32_t batch, const int32_t* chunk_ids, const int32_t* n_chunks,
                             int32_t max_sel, float* O, float* lse, void* ws, const TcAttendLayout& lay,
                             int32_t* status, cudaStream_t s) {
  char* base = static_cast<char*>(ws);
  int32_t* ids = reinterpret_cast<int32_t*>(base + lay.ids_off);
  uint32_t* masks = reinterpret_cast<uint32_t*>(base + lay.masks_off);
  int32_t* counts = reinterpret_cast<int32_t*>(base + lay.counts_off);
  int32_t* split = reinterpret_cast<int32_t*>(base + lay.split_off);
  float* slots = reinterpret_cast<float*>(base + lay.slots_off);
  const int64_t nb = int64_t(G.chunk) * (n_tokens / G.chunk);
  const int units = int(lay.units);

  const size_t prep_smem = sizeof(uint32_t) * 32 * kRowWords;
  cudaError_t e = ensure_dynamic_smem(union_prep_kernel, prep_smem);
  if (e != cudaSuccess) return e;
  {
    TraceScope ts("union_prep_kernel", 0, s);
    e = launch_pdl(union_prep_kernel, dim3(unsigned(units)), dim3(1024), prep_smem, s, G, batch,
                   lay.q_blocks, lay.n_blocks, lay.block_chunks, nb, lay.n_chunks, chunk_ids, n_chunks,
                   max_sel, ids, masks, lay.cap, counts, status);
  }
  if (e != cudaSuccess) return e;
  zha_count_launch();

  // Tensor copies when every chunk box starts on a swizzle atom (C % 8 == 0).
  CUtensorMap mk{}, mv{};
  const bool tma = G.chunk % 8 == 0 &&
                   (kv.table == nullptr
                        ? kv_tensor_map(&mk, kv.k, n_tokens, kv.ld, G.hkv, G.chunk) &&
                              kv_tensor_map(&mv, kv.v, n_tokens, kv.ld, G.hkv, G.chunk)
                        : page_tensor_map(&mk, kv.k, kv.ld, G.chunk) &&
                              page_tensor_map(&mv, kv.v, kv.ld, G.chunk));
  auto kern = tma ? attend_split_kernel<true> : attend_split_kernel<false>;
  const size_t smem = split_smem_bytes(units);
  if ((e = ensure_dynamic_smem(kern, smem)) != cudaSuccess) return e;
  int sms = 148;
  if ((e = device_sm_count(&sms)) != cudaSuccess) return e;
  const unsigned ctas = unsigned(sms < kTcMaxCtas ? sms : kTcMaxCtas);
  {
    TraceScope ts("attend_split_kernel", 0, s);
    e = launch_pdl(kern, dim3(ctas), dim3(kThreads), smem, s, mk, mv, G, batch, lay.q_blocks,
                   lay.n_blocks, lay.block_chunks, units, n_tokens, nb, Q, kv, ids, masks, lay.cap,
                   counts, split, slots, status);
  }
  if (e != cudaSuccess) return e;
  zha_count_launch();

  const int64_t heads = int64_t(batch) * G.hq;
  if ((e = ensure_dynamic_smem(combine_split_kernel, 0)) != cudaSuccess) return e;
  TraceScope ts("combine_split_kernel", 0, s);
  e = launch_pdl(combine_split_kernel, dim3(unsigned(heads)), dim3(32 * kCombineWarps), 0, s, G, batch,
                 lay.q_blocks, lay.n_blocks, units, split, slots, O, lse);
  zha_count_launch();
  return e;
}

}  // namespace zha
