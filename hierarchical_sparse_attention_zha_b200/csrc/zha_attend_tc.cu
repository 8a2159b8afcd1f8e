// zha_attend_tc.cu -- sparse attention over the routed leaf tokens on the
// sm_100a tensor cores (bf16 caches, head_dim 128), and the combine of the
// per-range states used by both attention kernels.
//
// Citations: [Attention: "Scaled dot-product attention 의 식"] o = softmax(q K^T /
// sqrt(d)) V; [Attention: "FlashAttention 계열"] online softmax (running max m,
// sum l, output rescaled by exp(m_old - m_new)) and Flash-Decoding's split of
// the cache along its length with a max-and-sum combine; [ZHA: 전제와 한계]
// (page "ZHA는 KV 캐시를 트리로 요약해 어텐션 비용을 준(sub)이차로 낮춘다") token 0
// and the in-progress chunk are always attended.
//
// Work item = (range of W chunks, KV head, block of 32 query heads of that KV
// head), built by attend_items_kernel; attend_tc_kernel is persistent (two
// CTAs of 128 threads per SM take items from a queue). The selected chunks of
// an item are streamed in tiles of 128 tokens. Per tile:
//   S^T[tok][q] = K_tile . Q^T          tcgen05.mma, M=128 tokens, N=32 heads, K=d,
//                                       Q split in three bf16 terms (fp32 accuracy),
//                                       accumulator in TMEM columns [0, 32)
//   masked online softmax per head      thread = token row (tcgen05.ld), per-head
//                                       max / sum by warp transpose-reductions
//   O^T[d][q] = V_tile^T . P            tcgen05.mma, M=128 (d), N=32, K=128 tokens,
//                                       V read MN-major from the same staging, P (two
//                                       bf16 terms) stored MN-major, 64-byte swizzled,
//                                       TMEM columns [32, 64)
//   o[q] = o[q] * exp(m_old - m_new) + O^T tile   (thread = d row, registers)
// K and V rows are staged by cp.async (16 lanes per 256-byte row) into the
// canonical 128-byte-swizzled layout; one elected thread issues the MMAs and tcgen05.commit signals an
// mbarrier whose waits are bounded (a time-out sets ZHA_DEV_TIMEOUT and the CTA
// releases its TMEM and returns).
#include "zha_internal.cuh"
#include "zha_tc.cuh"

namespace zha {

constexpr int kTcTok = 128;
constexpr int kTcQ = 32;
constexpr int kTcD = 128;
constexpr int kTcThreads = 128;
constexpr uint32_t kTcWaitTries = 1u << 22;

// Shared-memory plan (bytes from a 1024-byte aligned base).
constexpr int kOffK = 0;                      // [2 column blocks][128 rows][128 B]
constexpr int kOffV = 32768;
constexpr int kOffQ = 65536;                  // 3 terms x [2][32][128 B]
constexpr int kOffP = kOffQ + 3 * 8192;       // 2 terms x [2 token blocks][32][128 B]
constexpr int kOffMisc = kOffP + 2 * 8192;    // 106496

struct TcMisc {
  uint64_t mbar;
  uint32_t tmem_base;
  uint32_t any, mask0, nsel, err;
  float m[kTcQ], l[kTcQ], scale[kTcQ], mnew[kTcQ];
  float red[4][kTcQ];
  uint32_t tmask[2][kTcTok];
  uint32_t scan[33];
};

__host__ inline size_t attend_tc_smem_bytes(int range_chunks) {
  // tiles + misc + per-range chunk offsets and masks + the item's token table + alignment
  return size_t(kOffMisc) + sizeof(TcMisc) + 8 * size_t(range_chunks) +
         2 * size_t(kAttendRangeTokens) + 1024;
}

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

__device__ __forceinline__ int lower_bound_ids(const int32_t* a, int n, int64_t x) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (int64_t(a[mid]) < x) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// Per query head: where each range's entries start in its chunk list, so
// that the work-item pass reads two offsets instead of searching the list.
// Block 0 also clears the two work-item counters.
__global__ void __launch_bounds__(128)
attend_prep_kernel(const int32_t* __restrict__ chunk_ids, const int32_t* __restrict__ n_chunks,
                   int32_t max_sel, int32_t range_chunks, int64_t n_ranges, int64_t n_chunk_total,
                   int32_t* __restrict__ ptr, int64_t ptr_stride, uint32_t* __restrict__ counters) {
  const int64_t bh = blockIdx.x;
  const int32_t* list = chunk_ids + bh * max_sel;
  const int n = max(0, min(n_chunks[bh], max_sel));
  int32_t* out = ptr + bh * ptr_stride;
  for (int64_t r = threadIdx.x; r <= n_ranges; r += blockDim.x)
    out[r] = lower_bound_ids(list, n, r < n_ranges ? r * range_chunks : n_chunk_total);
  if (threadIdx.x == 0) out[n_ranges + 1] = (n > 0 && list[0] == 0) ? 1 : 0;
  if (bh == 0 && threadIdx.x < 2) counters[threadIdx.x] = 0u;
}

// One warp per (range, KV head, block of 32 query heads): which chunks of the
// range any head of the block selected, and by which heads; appends a work
// item when there is something to attend (always for the sink/tail range).
// Item: [g | qb << 16, range, n_sel | tail << 31, head mask | offsets[W] | masks[W]].
__global__ void __launch_bounds__(32)
attend_items_kernel(Geom G, int32_t batch, int64_t nb, const int32_t* __restrict__ chunk_ids,
                    const int32_t* __restrict__ ptr, int64_t ptr_stride, int32_t max_sel,
                    int32_t range_chunks, int64_t n_ranges, uint32_t* __restrict__ counters,
                    uint32_t* __restrict__ items, int64_t item_words) {
  extern __shared__ uint32_t s_m[];      // [W]
  const int g = blockIdx.y, qb = blockIdx.z;
  const int64_t rho = blockIdx.x;
  const bool tail = rho == n_ranges;
  const int GQ = G.group, C = G.chunk;
  const int qb0 = qb * kTcQ;
  const int nq = min(kTcQ, batch * GQ - qb0);
  const int lane = threadIdx.x;
  const int64_t c_lo = rho * range_chunks;
  const int64_t c_hi = min64(c_lo + range_chunks, nb / C);
  for (int i = lane; i < range_chunks; i += 32) s_m[i] = 0u;
  __syncwarp();
  bool mine = false;
  if (lane < nq) {
    const int qi = qb0 + lane;
    const int64_t bh = int64_t(qi / GQ) * G.hq + g * GQ + qi % GQ;
    const int32_t* pr = ptr + bh * ptr_stride;
    if (!tail) {
      const int32_t* list = chunk_ids + bh * max_sel;
      const int lo = pr[rho], hi = pr[rho + 1];
      for (int i = lo; i < hi; ++i) {
        const int64_t c = list[i];
        if (c >= c_lo && c < c_hi) { atomicOr(&s_m[c - c_lo], 1u << lane); mine = true; }
      }
    } else {
      mine = nb > 0 && pr[n_ranges + 1] == 0;      // this head needs the sink token
    }
  }
  const uint32_t heads = __ballot_sync(0xffffffffu, mine);
  __syncwarp();
  if (!tail && heads == 0u) return;
  uint32_t slot = 0;
  if (lane == 0) slot = atomicAdd(&counters[0], 1u);
  slot = __shfl_sync(0xffffffffu, slot, 0);
  uint32_t* it = items + int64_t(slot) * item_words;
  uint32_t n_sel = 0;
  for (int i0 = 0; i0 < range_chunks; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t m = i < range_chunks ? s_m[i] : 0u;
    const uint32_t ball = __ballot_sync(0xffffffffu, m != 0u);
    if (m != 0u) {
      const uint32_t pos = n_sel + __popc(ball & ((1u << lane) - 1u));
      it[4 + pos] = uint32_t(i);
      it[4 + range_chunks + pos] = m;
    }
    n_sel += __popc(ball);
  }
  if (lane == 0) {
    it[0] = uint32_t(g) | (uint32_t(qb) << 16);
    it[1] = uint32_t(rho);
    it[2] = n_sel | (tail ? 0x80000000u : 0u);
    it[3] = heads;
  }
}

// Persistent: each CTA takes work items from the queue until it is empty.
// Scores are kept in base-2 units (s * log2(e) / sqrt(d)) so that the softmax
// uses exp2; the running maximum is converted back to natural-log units when
// the item's state is written.
__global__ void __launch_bounds__(kTcThreads, 2)
attend_tc_kernel(Geom G, int32_t batch, int64_t n_tokens, int64_t nb, const float* __restrict__ Q,
                 const __nv_bfloat16* __restrict__ K, const __nv_bfloat16* __restrict__ V, int64_t ld,
                 int32_t range_chunks, const uint32_t* __restrict__ items, int64_t item_words,
                 uint32_t* __restrict__ counters, float* __restrict__ partial, int64_t slots_per_head,
                 int32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  TcMisc& ms = *reinterpret_cast<TcMisc*>(smem + kOffMisc);
  uint32_t* s_mask = reinterpret_cast<uint32_t*>(smem + kOffMisc + sizeof(TcMisc));
  uint32_t* s_sel = s_mask + range_chunks;
  int16_t* s_tok = reinterpret_cast<int16_t*>(s_sel + range_chunks);   // [kAttendRangeTokens]
  const uint32_t sK = tc::smem_u32(smem + kOffK), sV = tc::smem_u32(smem + kOffV);
  const uint32_t sQ = tc::smem_u32(smem + kOffQ), sP = tc::smem_u32(smem + kOffP);
  const int GQ = G.group;
  const int C = G.chunk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t n_items = counters[0];
  const float scale2 = G.scale * 1.4426950408889634f;      // 1/sqrt(d) * log2(e)

  if (tid == 0) { ms.err = 0u; tc::mbar_init(&ms.mbar, 1); }
  if (warp == 0) tc::tmem_alloc(&ms.tmem_base, 64);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = ms.tmem_base;
  const uint32_t t_lane = uint32_t(warp * 32) << 16;
  constexpr uint32_t idesc_s = tc::idesc_bf16(kTcTok, kTcQ, 0, 0);
  constexpr uint32_t idesc_pv = tc::idesc_bf16(kTcD, kTcQ, 1, 1);
  uint32_t phase = 0;
  bool failed = false;
  // Copy mapping: 16 lanes per 256-byte row, rows r0, r0 + 8, ..., r0 + 120.
  const int piece = tid & 15, r0 = tid >> 4;

  while (!failed) {
    if (tid == 0) ms.any = atomicAdd(&counters[1], 1u);
    __syncthreads();
    const uint32_t item = ms.any;
    if (item >= n_items) break;
    const uint32_t* it = items + int64_t(item) * item_words;
    const uint32_t h0 = it[0], h2 = it[2];
    const int g = int(h0 & 0xffffu), qb = int(h0 >> 16);
    const int64_t rho = int64_t(it[1]);
    const bool tail = (h2 >> 31) != 0u;
    const int n_sel = int(h2 & 0x7fffffffu);
    const uint32_t heads = it[3];
    for (int i = tid; i < n_sel; i += blockDim.x) {
      s_sel[i] = it[4 + i];
      s_mask[i] = it[4 + range_chunks + i];
    }
    const int qb0 = qb * kTcQ;
    const int nq = min(kTcQ, batch * GQ - qb0);
    const uint32_t all_q = nq == 32 ? 0xffffffffu : ((1u << nq) - 1u);
    const int64_t n_tail = n_tokens - nb;
    const int n_tok = tail ? int(n_tail) + (heads != 0u ? 1 : 0) : n_sel * C;
    const int n_tiles = (n_tok + kTcTok - 1) / kTcTok;
    // Token table of the item: offset from the item's first token (-1 = the sink).
    const int64_t tok_base = tail ? nb : rho * range_chunks * C;
    __syncthreads();
    for (int u = tid; u < n_tok; u += blockDim.x)
      s_tok[u] = tail ? int16_t(u < n_tail ? u : -1) : int16_t(int(s_sel[u / C]) * C + u % C);
    __syncthreads();

    // Rows of tile `tile` into the K (or V) staging, one cp.async group; the
    // K call also records the head mask of row `tid` for the softmax.
    auto issue_rows = [&](int tile, bool is_v) {
      const __nv_bfloat16* src = (is_v ? V : K) + int64_t(g) * ld * kTcD;
      const uint32_t dst = is_v ? sV : sK;
#pragma unroll
      for (int k = 0; k < kTcTok / 8; ++k) {
        const int row = r0 + 8 * k;
        const int u = tile * kTcTok + row;
        const bool valid = u < n_tok;
        const int rel = valid ? int(s_tok[u]) : 0;
        const int64_t tok = rel < 0 ? 0 : tok_base + rel;
        tc::cp_async16(dst + tc::sw128_offset(row, 8 * piece, kTcTok), src + tok * kTcD + 8 * piece,
                       valid ? 16u : 0u);
      }
      tc::cp_async_commit();
      if (!is_v) {
        const int u = tile * kTcTok + tid;
        uint32_t msk = 0u;
        if (u < n_tok) msk = tail ? (u < n_tail ? all_q : heads) : s_mask[u / C];
        ms.tmask[tile & 1][tid] = msk;
      }
    };

    if (n_tiles > 0) {
      issue_rows(0, false);
      issue_rows(0, true);
    }
    // Query block -> three bf16 terms, K-major rows (row = query head).
    for (int v = tid; v < kTcQ * (kTcD / 8); v += blockDim.x) {
      const int q = v / (kTcD / 8), col = (v % (kTcD / 8)) * 8;
      float x[8];
      if (q < nq) {
        const int qi = qb0 + q;
        const int64_t bh = int64_t(qi / GQ) * G.hq + g * GQ + qi % GQ;
        const float4 a = *reinterpret_cast<const float4*>(Q + bh * kTcD + col);
        const float4 b = *reinterpret_cast<const float4*>(Q + bh * kTcD + col + 4);
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = 0.f;
      }
      const uint32_t off = tc::sw128_offset(q, col, kTcQ);
#pragma unroll
      for (int term = 0; term < 3; ++term) {
        __align__(16) __nv_bfloat16 h[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          h[i] = __float2bfloat16_rn(x[i]);
          x[i] -= __bfloat162float(h[i]);
        }
        *reinterpret_cast<uint4*>(smem + kOffQ + term * 8192 + off) = *reinterpret_cast<uint4*>(h);
      }
    }
    if (tid < kTcQ) { ms.m[tid] = -INFINITY; ms.l[tid] = 0.f; }
    float acc[kTcQ];
#pragma unroll
    for (int q = 0; q < kTcQ; ++q) acc[q] = 0.f;

    // Pipeline: tile i's S MMA runs once its K rows have landed; tile i+1's K
    // rows are requested as soon as that MMA has consumed the K staging, and
    // its V rows once the P.V MMA of tile i has consumed the V staging.
    for (int i = 0; i < n_tiles && !failed; ++i) {
      const bool has_next = i + 1 < n_tiles;
      tc::cp_async_wait_pending1();          // K_i done (V_i may still be in flight)
      tc::fence_async_smem();
      __syncthreads();
      if (tid == 0) {
        tc::fence_after_sync();
#pragma unroll
        for (int term = 0; term < 3; ++term)
#pragma unroll
          for (int ks = 0; ks < kTcD / 16; ++ks) {
            const uint64_t a = tc::desc_sw128(sK + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
            const uint64_t b = tc::desc_sw128(sQ + term * 8192 + (ks >> 2) * 4096 + (ks & 3) * 32, 16, 1024);
            tc::mma_bf16(tbase, a, b, idesc_s, (term | ks) != 0);
          }
        tc::mma_commit(&ms.mbar);
      }
      if (!tc::mbar_wait(&ms.mbar, phase, kTcWaitTries)) atomicOr(&ms.err, 1u);
      phase ^= 1u;
      tc::fence_after_sync();
      const uint32_t tm = ms.tmask[i & 1][tid];
      if (has_next) issue_rows(i + 1, false);     // the K staging is free again

      float s[kTcQ];
      tc::tmem_ld32(tbase + t_lane, s);
#pragma unroll
      for (int q = 0; q < kTcQ; ++q) s[q] = ((tm >> q) & 1u) ? s[q] * scale2 : -INFINITY;
      {
        float v[kTcQ];
#pragma unroll
        for (int q = 0; q < kTcQ; ++q) v[q] = s[q];
        ms.red[warp][lane] = transpose_reduce32<true>(v);
      }
      __syncthreads();
      if (tid < kTcQ) {
        const float mt = fmaxf(fmaxf(ms.red[0][tid], ms.red[1][tid]), fmaxf(ms.red[2][tid], ms.red[3][tid]));
        const float mo = ms.m[tid];
        const float mn = fmaxf(mo, mt);
        ms.mnew[tid] = mn;
        ms.scale[tid] = mn == -INFINITY ? 1.f : exp2f(mo - mn);
      }
      __syncthreads();
      {
        // p = 2^(s - m_new); P stored MN-major (token row, 32 heads = 64 B) in
        // two bf16 terms, 16 bytes (8 heads) per store.
        float v[kTcQ];
#pragma unroll
        for (int c = 0; c < kTcQ / 8; ++c) {
          __align__(16) __nv_bfloat16 hi[8], lo[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int q = 8 * c + j;
            const float mn = ms.mnew[q];
            const float p = (mn == -INFINITY) ? 0.f : exp2f(s[q] - mn);
            v[q] = p;
            hi[j] = __float2bfloat16_rn(p);
            lo[j] = __float2bfloat16_rn(p - __bfloat162float(hi[j]));
          }
          const uint32_t off = tc::sw64_mn_chunk(tid, c);
          *reinterpret_cast<uint4*>(smem + kOffP + off) = *reinterpret_cast<uint4*>(hi);
          *reinterpret_cast<uint4*>(smem + kOffP + 8192 + off) = *reinterpret_cast<uint4*>(lo);
        }
        ms.red[warp][lane] = transpose_reduce32<false>(v);
      }
      if (has_next) tc::cp_async_wait_pending1(); else tc::cp_async_wait_pending0();   // V_i done
      tc::fence_async_smem();
      tc::fence_before_sync();
      __syncthreads();
      if (tid < kTcQ) {
        ms.l[tid] = ms.l[tid] * ms.scale[tid] + (ms.red[0][tid] + ms.red[1][tid] + ms.red[2][tid] + ms.red[3][tid]);
        ms.m[tid] = ms.mnew[tid];
      }
      if (tid == 0) {
        tc::fence_after_sync();
#pragma unroll
        for (int term = 0; term < 2; ++term)
#pragma unroll
          for (int ks = 0; ks < kTcTok / 16; ++ks) {
            const uint64_t a = tc::desc_sw128(sV + ks * 2048, 16384, 1024);
            const uint64_t b = tc::desc_sw64(sP + term * 8192 + ks * 1024, 8192, 512);
            tc::mma_bf16(tbase + 32, a, b, idesc_pv, (term | ks) != 0);
          }
        tc::mma_commit(&ms.mbar);
      }
      if (!tc::mbar_wait(&ms.mbar, phase, kTcWaitTries)) atomicOr(&ms.err, 1u);
      phase ^= 1u;
      tc::fence_after_sync();
      if (has_next) issue_rows(i + 1, true);      // the V staging is free again
      {
        float o[kTcQ];
        tc::tmem_ld32(tbase + t_lane + 32, o);
#pragma unroll
        for (int q = 0; q < kTcQ; ++q) acc[q] = acc[q] * ms.scale[q] + o[q];
      }
      tc::fence_before_sync();
      __syncthreads();
      failed = ms.err != 0u;
    }
    tc::cp_async_wait_pending0();
    if (failed) break;
    const uint32_t active = tail ? all_q : heads;
#pragma unroll
    for (int q = 0; q < kTcQ; ++q) {
      if (q < nq && ((active >> q) & 1u)) {
        const int qi = qb0 + q;
        const int64_t bh = int64_t(qi / GQ) * G.hq + g * GQ + qi % GQ;
        float* slot = partial + (bh * slots_per_head + rho) * (kTcD + 4);
        slot[4 + tid] = acc[q];
        if (tid == 0)   // maximum back to natural-log units
          *reinterpret_cast<float4*>(slot) = make_float4(ms.m[q] * 0.6931471805599453f, ms.l[q], 0.f, 0.f);
      }
    }
    __syncthreads();     // ms.m / ms.l and the item's shared data are reused
  }
  if (failed && tid == 0 && status != nullptr) atomicOr(status, ZHA_DEV_TIMEOUT);
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, 64);
  }
}

// ---------------------------------------------------------------------------
// Combine: one CTA (D threads, thread = output dim) per query head. The head's
// chunk list is scanned in windows; the range states it touched are merged
// with one maximum per window, so the state loads are independent.
// ---------------------------------------------------------------------------
constexpr int kCombineWindow = 4096;

template <int D>
__global__ void __launch_bounds__(D)
combine_ranges_kernel(Geom G, int32_t batch, int64_t n_chunk_total, const int32_t* __restrict__ chunk_ids,
                      const int32_t* __restrict__ n_chunks, int32_t max_sel, int32_t range_chunks,
                      int64_t n_ranges, const float* __restrict__ partial, int64_t slots_per_head,
                      float* __restrict__ O, float* __restrict__ lse, int32_t* status) {
  __shared__ int32_t s_rng[kCombineWindow + 1];
  __shared__ float s_w[kCombineWindow + 1];
  __shared__ float s_red[D / 32 + 1];
  __shared__ uint32_t s_scan[33];
  __shared__ int s_bad;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = D / 32;
  const int64_t bh = blockIdx.x;
  int n = n_chunks[bh];
  if (tid == 0) s_bad = (n < 0 || n > max_sel) ? 1 : 0;
  n = max(0, min(n, max_sel));
  const int32_t* list = chunk_ids + bh * max_sel;
  const float* slots = partial + bh * slots_per_head * (D + 4);
  float M = -INFINITY, L = 0.f, acc = 0.f;

  auto merge_window = [&](int cnt) {
    // window maximum
    float mloc = -INFINITY;
    for (int i = tid; i < cnt; i += D) {
      const float* sl = slots + int64_t(s_rng[i]) * (D + 4);
      if (sl[1] > 0.f) mloc = fmaxf(mloc, sl[0]);
    }
    mloc = warp_max(mloc);
    if (lane == 0) s_red[warp] = mloc;
    __syncthreads();
    float mw = -INFINITY;
    for (int w = 0; w < NW; ++w) mw = fmaxf(mw, s_red[w]);
    __syncthreads();
    const float mn = fmaxf(M, mw);
    if (mn == -INFINITY) return;
    const float r = expf(M - mn);
    acc *= r;
    L *= r;
    float lsum = 0.f;
    for (int i = tid; i < cnt; i += D) {
      const float* sl = slots + int64_t(s_rng[i]) * (D + 4);
      const float w = sl[1] > 0.f ? expf(sl[0] - mn) : 0.f;
      s_w[i] = w;
      lsum += w * sl[1];
    }
    lsum = warp_sum(lsum);
    if (lane == 0) s_red[warp] = lsum;
    __syncthreads();
    for (int w = 0; w < NW; ++w) L += s_red[w];
    int i = 0;
    for (; i + 4 <= cnt; i += 4) {
      const float o0 = slots[int64_t(s_rng[i]) * (D + 4) + 4 + tid];
      const float o1 = slots[int64_t(s_rng[i + 1]) * (D + 4) + 4 + tid];
      const float o2 = slots[int64_t(s_rng[i + 2]) * (D + 4) + 4 + tid];
      const float o3 = slots[int64_t(s_rng[i + 3]) * (D + 4) + 4 + tid];
      acc += s_w[i] * o0 + s_w[i + 1] * o1 + s_w[i + 2] * o2 + s_w[i + 3] * o3;
    }
    for (; i < cnt; ++i) acc += s_w[i] * slots[int64_t(s_rng[i]) * (D + 4) + 4 + tid];
    __syncthreads();
    M = mn;
  };

  for (int w0 = 0; w0 < n; w0 += kCombineWindow) {
    const int w1 = min(n, w0 + kCombineWindow);
    int cnt = 0;
    for (int b0 = w0; b0 < w1; b0 += D) {
      const int i = b0 + tid;
      int64_t id = -1, prev = -1;
      bool start = false;
      if (i < w1) {
        id = list[i];
        prev = i > 0 ? int64_t(list[i - 1]) : -1;
        const bool valid = id >= 0 && id < n_chunk_total && id > prev;
        if (!valid) s_bad = 1;
        start = valid && (i == 0 || prev < 0 || id / range_chunks != prev / range_chunks);
      }
      uint32_t v = start ? 1u : 0u, x = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (lane == 31) s_scan[warp] = x;
      __syncthreads();
      if (tid == 0) {
        uint32_t run = 0;
        for (int w = 0; w < NW; ++w) { const uint32_t t = s_scan[w]; s_scan[w] = run; run += t; }
        s_scan[32] = run;
      }
      __syncthreads();
      if (start) s_rng[cnt + s_scan[warp] + x - v] = int32_t(id / range_chunks);
      cnt += int(s_scan[32]);
      __syncthreads();
    }
    merge_window(cnt);
  }
  if (tid == 0) s_rng[0] = int32_t(n_ranges);
  __syncthreads();
  merge_window(1);
  O[bh * D + tid] = L > 0.f ? acc / L : 0.f;
  if (tid == 0) {
    if (lse != nullptr) lse[bh] = L > 0.f ? M + logf(L) : -INFINITY;
    if (s_bad && status != nullptr) atomicOr(status, ZHA_DEV_BAD_SELECTION);
  }
}

cudaError_t launch_combine(const Geom& G, int32_t batch, const int32_t* chunk_ids,
                           const int32_t* n_chunks, int32_t max_sel, float* O, float* lse,
                           const float* partial, const AttendLayout& lay, int32_t* status,
                           cudaStream_t s) {
  const unsigned heads = unsigned(int64_t(batch) * G.hq);
  if (G.d == 128)
    combine_ranges_kernel<128><<<heads, 128, 0, s>>>(G, batch, lay.n_chunks, chunk_ids, n_chunks,
                                                     max_sel, lay.range_chunks, lay.n_ranges,
                                                     partial, lay.slots_per_head, O, lse, status);
  else
    combine_ranges_kernel<64><<<heads, 64, 0, s>>>(G, batch, lay.n_chunks, chunk_ids, n_chunks,
                                                   max_sel, lay.range_chunks, lay.n_ranges, partial,
                                                   lay.slots_per_head, O, lse, status);
  zha_count_launch();
  return cudaGetLastError();
}

cudaError_t launch_attend_tc(const Geom& G, const float* Q, const void* K, const void* V, int64_t ld,
                             int64_t n_tokens, int32_t batch, const int32_t* chunk_ids,
                             const int32_t* n_chunks, int32_t max_sel, float* partial,
                             const AttendLayout& lay, int32_t* status, cudaStream_t s) {
  const size_t smem = attend_tc_smem_bytes(lay.range_chunks);
  cudaError_t e = cudaFuncSetAttribute(attend_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int64_t nb = int64_t(G.chunk) * (n_tokens / G.chunk);
  char* base = reinterpret_cast<char*>(partial);
  int32_t* ptr = reinterpret_cast<int32_t*>(base + lay.ptr_offset_bytes);
  uint32_t* counters = reinterpret_cast<uint32_t*>(base + lay.counter_offset_bytes);
  uint32_t* items = reinterpret_cast<uint32_t*>(base + lay.item_offset_bytes);
  attend_prep_kernel<<<unsigned(int64_t(batch) * G.hq), 128, 0, s>>>(
      chunk_ids, n_chunks, max_sel, lay.range_chunks, lay.n_ranges, lay.n_chunks, ptr, lay.ptr_stride,
      counters);
  zha_count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  dim3 grid_items(unsigned(lay.n_ranges + 1), unsigned(G.hkv), unsigned(lay.q_blocks));
  attend_items_kernel<<<grid_items, 32, size_t(lay.range_chunks) * 4, s>>>(
      G, batch, nb, chunk_ids, ptr, lay.ptr_stride, max_sel, lay.range_chunks, lay.n_ranges, counters,
      items, lay.item_words);
  zha_count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int64_t want = lay.max_items;
  const unsigned ctas = unsigned(want < 2 * sms ? want : 2 * sms);
  attend_tc_kernel<<<ctas, kTcThreads, smem, s>>>(
      G, batch, n_tokens, nb, Q, static_cast<const __nv_bfloat16*>(K),
      static_cast<const __nv_bfloat16*>(V), ld, lay.range_chunks, items, lay.item_words, counters,
      partial, lay.slots_per_head, status);
  zha_count_launch();
  return cudaGetLastError();
}

}  // namespace zha
