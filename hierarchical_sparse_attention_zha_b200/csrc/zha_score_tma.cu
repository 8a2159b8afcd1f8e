// zha_score_tma.cu -- node scoring for head_dim 128 and R = 16 reference
// queries per tree, fed by tensor copies and computed on the sm_100a tensor
// cores.
//
// Citations: [ZHA: 무엇과 다른가 / 전제와 한계] = page "ZHA는 KV 캐시를 트리로 요약해
// 어텐션 비용을 준(sub)이차로 낮춘다" (onedev.kr/papers/1556): a node's estimated log
// mass for a query is the maximum of its R tangent planes,
// sigma = max_r (q . khat_r / sqrt(d) + bhat_r); each level scores the
// candidates passed down from the level above.
//
// Work: tiles of 8 nodes of one group (KV head g, block of up to 32 of its
// query heads). The tiles of all groups form one sequence that is split evenly
// over one persistent CTA per SM. Roles inside a CTA:
//   producer (warp 0)       per tile, the candidate mask of each node (bit q =
//                           query head q has the node's parent kept, or the
//                           node is an orphan); tiles without any candidate are
//                           skipped. For the others it issues tensor copies of
//                           the fp32 node records, one half of the columns (64)
//                           at a time: box = 32 columns x 16 planes x 8 nodes,
//                           128-byte swizzled, rows (node, plane) = MMA rows.
//   converters (warps 4-11) thread = (row, 32-column box): each fp32 value ->
//                           two fp16 terms, t0 = x rounded to fp16 and t1 = the
//                           remainder rounded to fp16 (x = t0 + t1 to 2^-22 |x|,
//                           rounded to nearest), stored from registers into tensor memory,
//                           where the MMA reads its A operand (shared memory only
//                           carries the raw tiles and Q, split the same way)
//   MMA issuer (warp 1)     S^T[(node, plane)][head] over the half's 4 K-steps:
//                           A_t0 . [q0 | q1]^T (N = 64) and A_t1 . q0^T (N = 32)
//                           into one of two TMEM buffers -- the three products
//                           above 2^-22 of the result; A and B are both fp16
//   epilogue (warps 12-15)  thread = (node, plane) row: sum of the two column
//                           groups, x 1/sqrt(d) + bhat, maximum over the node's 16
//                           planes, scores of the candidate (node, head) pairs.
//                           An element beyond the fp16 range (|x| >= 65520) makes
//                           its products non-finite; a row that shows one is
//                           recomputed in fp32 from the node record and Q
// The fp16 terms keep each product to about 2^-21 relative (unbiased), the
// order of the fp32 accumulation's own rounding, for every element of
// magnitude up to 65504; below 2^-14 they lose relative, not absolute,
// precision (an absolute error below 2^-25 per element).
// Every wait is bounded; a time-out sets ZHA_DEV_TIMEOUT and the roles stop.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include "zha_host.cuh"
#include "zha_internal.cuh"
#include "zha_tc.cuh"

namespace zha {

namespace {

constexpr int kNodes = 8;                 // nodes per tile (x 16 planes = 128 MMA rows)
constexpr int kR = 16;
constexpr int kQn = 32;                   // query heads per group
constexpr int kD = 128;
constexpr int kRawSlots = 5;              // raw fp32 half-tiles in flight
constexpr int kRawBytes = 32768;          // [2 boxes][128 rows][128 B]
constexpr int kOffRaw = 0;
constexpr int kQHalf = 2 * kQn * 128;                 // [64 rows = term x 32 heads][128 B]
constexpr int kOffQ = kRawSlots * kRawBytes;          // 2 halves x kQHalf
constexpr int kOffMisc = kOffQ + 2 * kQHalf;
constexpr int kThreads = 512;             // warps: 0 producer, 1 MMA, 2-3 idle, 4-11 convert, 12-15 epilogue
constexpr int kConv = 256;                // converter threads (warps 4-11)
constexpr int kEpiWarp0 = 12;
constexpr uint32_t kTmemCols = 512;       // D buffers (64 columns) at 0 and 64; A half-buffers
constexpr uint32_t kTmemA = 128;          // (2 terms x 32 columns) at 128, 192 and 256
constexpr uint32_t kDCols = 64, kACols = 64;
constexpr int kABufs = 3;

struct Meta {                             // one half-tile, producer -> converters
  int32_t node0, group, half, flags;      // flags: 1 = first tile of a group, 2 = end
  uint32_t mask[kNodes];
};
struct CMeta {                            // converters -> MMA issuer
  int32_t half, flags;
};
struct EMeta {                            // converters -> epilogue, per tile
  int32_t node0, group, flags, pad;
  uint32_t mask[kNodes];
  float bhat[kNodes * kR];                // bhat of the tile's (node, plane) rows
};

struct Misc {
  uint64_t raw_full[kRawSlots], raw_empty[kRawSlots];
  uint64_t conv_done[kABufs], a_free[kABufs], d_full[2], d_free[2], q_ready, drain;
  uint32_t tmem_base, err;
  Meta meta[kRawSlots];
  alignas(128) float bhat_raw[kRawSlots][kNodes * kR];  // tensor-copied with the first half of a tile
  CMeta cmeta[kABufs];
  EMeta emeta[2];
};

__host__ inline size_t score_tma_smem_bytes() { return size_t(kOffMisc) + sizeof(Misc) + 1024; }

// Query head (flattened b * hq + h) of query q of group v.
__device__ __forceinline__ int64_t head_of(const Geom& G, int q_blocks, int v, int q) {
  const int g = v / q_blocks, qi = (v % q_blocks) * kQn + q;
  return int64_t(qi / G.group) * G.hq + g * G.group + qi % G.group;
}

__device__ __forceinline__ int group_width(const Geom& G, int batch, int q_blocks, int v) {
  return min(kQn, batch * G.group - (v % q_blocks) * kQn);
}

// Two fp32 values -> two packed fp16x2 terms, x = t0 + t1 + e (x0 in the low
// halves): t0 rounds x to fp16 (11 significant bits), the remainder x - t0 is
// exact in fp32 and t1 rounds it to fp16, so |e| <= 2^-22 |x| while x and the
// remainder are normal fp16 numbers.
__device__ __forceinline__ void split2_x2(float x0, float x1, uint32_t& t0, uint32_t& t1) {
  const __half2 h = __floats2half2_rn(x0, x1);
  const float2 f = __half22float2(h);
  const __half2 l = __floats2half2_rn(x0 - f.x, x1 - f.y);
  t0 = *reinterpret_cast<const uint32_t*>(&h);
  t1 = *reinterpret_cast<const uint32_t*>(&l);
}

// Eight fp32 values -> two fp16x8 terms.
__device__ __forceinline__ void split2_x8(const float4& a, const float4& b, uint4& t0, uint4& t1) {
  split2_x2(a.x, a.y, t0.x, t1.x);
  split2_x2(a.z, a.w, t0.y, t1.y);
  split2_x2(b.x, b.y, t0.z, t1.z);
  split2_x2(b.z, b.w, t0.w, t1.w);
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
score_tma_kernel(const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmB, Geom G, int level, int64_t n_nodes,
                 int64_t n_par, int32_t batch, int32_t q_blocks, int32_t groups,
                 const float* __restrict__ Q, const uint32_t* __restrict__ kept_up, int64_t words_up,
                 float* __restrict__ sigma, const float* __restrict__ level_base, int32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Misc& ms = *reinterpret_cast<Misc*>(smem + kOffMisc);
  __shared__ uint64_t emeta_full[2];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t nt = (n_nodes + kNodes - 1) / kNodes;        // tiles per group
  const int64_t T = nt * groups;
  const int nct = int(gridDim.x), cta = int(blockIdx.x);
  const int64_t t0 = int64_t(cta) * T / nct, t1 = int64_t(cta + 1) * T / nct;

  if (tid == 0) {
    ms.err = 0u;
    for (int s = 0; s < kRawSlots; ++s) {
      tc::mbar_init(&ms.raw_full[s], 1);
      tc::mbar_init(&ms.raw_empty[s], kConv / 32);      // one arrival per converter warp
    }
    for (int b = 0; b < kABufs; ++b) {
      tc::mbar_init(&ms.conv_done[b], kConv / 32);
      tc::mbar_init(&ms.a_free[b], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&ms.d_full[b], 1);
      tc::mbar_init(&ms.d_free[b], 128);
      tc::mbar_init(&emeta_full[b], kNodes * kR / 32);  // the warps copying bhat
    }
    tc::mbar_init(&ms.q_ready, kConv / 32);
    tc::mbar_init(&ms.drain, 1);
  }
  pdl_trigger();
  if (warp == 1) tc::tmem_alloc(&ms.tmem_base, kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = ms.tmem_base;
  pdl_wait();                                      // inputs of the previous kernel from here on

  if (warp == 0) {
    // ---------------- producer ----------------
    const int64_t orphan0 = int64_t(G.chunk) * n_par;
    int64_t k = 0;                     // half-tiles emitted
    int prev_v = -1;
    bool failed = false;
    // Lane q's kept words for the parents of tile t (8 nodes span at most two
    // words of parents), loaded one tile ahead of their use. Tile and node
    // indices fit 32 bits (node capacities are below 2^31).
    const int32_t C = G.chunk, nt32 = int32_t(nt), nn = int32_t(n_nodes), orph = int32_t(orphan0);
    auto load_words = [&](int32_t t, uint32_t& w0, uint32_t& w1) {
      w0 = w1 = 0u;
      if (int64_t(t) >= t1) return;
      const int v = t / nt32;
      const int32_t node0 = (t - v * nt32) * kNodes;
      const int nq = group_width(G, batch, q_blocks, v);
      if (lane >= nq || node0 >= orph) return;
      const int64_t base = head_of(G, q_blocks, v, lane) * words_up;
      const int32_t p0 = node0 / C, p1 = min(node0 + kNodes - 1, orph - 1) / C;
      w0 = kept_up[base + (p0 >> 5)];
      w1 = (p1 >> 5) != (p0 >> 5) ? kept_up[base + (p1 >> 5)] : w0;
    };
    uint32_t nw0 = 0u, nw1 = 0u;
    if (t0 < t1) load_words(int32_t(t0), nw0, nw1);
    // Test hook: send nothing, so that every consumer's bounded wait runs out.
    const int32_t t_stop = G.debug_withhold ? int32_t(t0) : int32_t(t1);
    for (int32_t t = int32_t(t0); t < t_stop && !failed; ++t) {
      const uint32_t w0 = nw0, w1 = nw1;
      load_words(t + 1, nw0, nw1);
      const int v = t / nt32;
      const int32_t node0 = (t - v * nt32) * kNodes;
      const int nq = group_width(G, batch, q_blocks, v);
      int32_t par = node0 / C, rem = node0 - par * C;         // parent of node0 and its offset
      const int32_t pw0 = par >> 5;
      uint32_t m[kNodes], any = 0u;
#pragma unroll
      for (int j = 0; j < kNodes; ++j) {
        const int32_t node = node0 + j;
        bool cand = false;
        if (node < nn && lane < nq)
          cand = node >= orph || ((((par >> 5) == pw0 ? w0 : w1) >> (par & 31)) & 1u) != 0u;
        m[j] = __ballot_sync(0xffffffffu, cand);
        any |= m[j];
        if (++rem == C) { rem = 0; ++par; }
      }
      if (any == 0u) continue;                     // no candidate in the tile
      const bool first = v != prev_v;
      prev_v = v;
      const int32_t z = int32_t(int64_t(v / q_blocks) * G.cap[level] + node0);
      for (int h = 0; h < 2; ++h, ++k) {
        const int slot = int(k % kRawSlots);
        const int64_t use = k / kRawSlots;
        bool bad = false;
        if (use > 0) bad = !tc::mbar_wait(&ms.raw_empty[slot], uint32_t((use - 1) & 1), G.wait_polls);
        if (__any_sync(0xffffffffu, bad)) { failed = true; break; }
        if (lane == 0) {
          Meta& mt = ms.meta[slot];
          mt.node0 = int32_t(node0);
          mt.group = v;
          mt.half = h;
          mt.flags = (first && h == 0) ? 1 : 0;
#pragma unroll
          for (int j = 0; j < kNodes; ++j) mt.mask[j] = m[j];
          tc::mbar_arrive_expect_tx(&ms.raw_full[slot], 2u * 16384u + (h == 0 ? 512u : 0u));
          const uint32_t dst = tc::smem_u32(smem + kOffRaw + slot * kRawBytes);
          tc::tma_load_3d(dst, &tmS, 64 * h, 0, z, &ms.raw_full[slot]);
          tc::tma_load_3d(dst + 16384, &tmS, 64 * h + 32, 0, z, &ms.raw_full[slot]);
          if (h == 0) tc::tma_load_2d(tc::smem_u32(ms.bhat_raw[slot]), &tmB, 0, z, &ms.raw_full[slot]);
        }
        __syncwarp();
      }
    }
    bool sent_end = false;
    if (!failed && !G.debug_withhold) {            // end of the stream
      const int slot = int(k % kRawSlots);
      const int64_t use = k / kRawSlots;
      bool bad = false;
      if (use > 0) bad = !tc::mbar_wait(&ms.raw_empty[slot], uint32_t((use - 1) & 1), G.wait_polls);
      if (__any_sync(0xffffffffu, bad)) {
        failed = true;
      } else {
        sent_end = true;
        if (lane == 0) {
          ms.meta[slot].flags = 2;
          tc::mbar_arrive(&ms.raw_full[slot]);
        }
      }
    }
    // Before the CTA may exit, every tensor copy issued into shared memory has
    // landed: wait for the last copy of each slot (already complete when the
    // converters consumed it). The end marker reused the slot of copy k - 5
    // only after the converters had taken that copy, and moved that slot's
    // phase on, so that copy is not waited for again.
    if (lane == 0) {
      const int64_t j0 = (k > kRawSlots ? k - kRawSlots : 0) + (sent_end && k >= kRawSlots ? 1 : 0);
      for (int64_t j = j0; j < k; ++j)
        if (!tc::mbar_wait(&ms.raw_full[j % kRawSlots], uint32_t((j / kRawSlots) & 1), G.wait_polls))
          failed = true;
    }
    if (failed && lane == 0) atomicOr(&ms.err, 1u);
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc64 = tc::idesc_f16(128, 64, 0, 0);
      constexpr uint32_t idesc32 = tc::idesc_f16(128, 32, 0, 0);
      int64_t k = 0, tile_i = 0;
      int seg = 0;
      bool failed = false;
      while (true) {
        const int ab = int(k % kABufs);
        if (!tc::mbar_wait(&ms.conv_done[ab], uint32_t((k / kABufs) & 1), G.wait_polls)) { failed = true; break; }
        const CMeta cm = ms.cmeta[ab];
        if (cm.half == 0 || (cm.flags & 2)) {
          // The D buffer of this tile must have been read by the epilogue.
          if (tile_i >= 2 &&
              !tc::mbar_wait(&ms.d_free[tile_i & 1], uint32_t(((tile_i >> 1) - 1) & 1), G.wait_polls)) {
            failed = true;
            break;
          }
        }
        if (cm.flags & 2) {                        // end: let the epilogue see it
          tc::mma_commit(&ms.d_full[tile_i & 1]);
          break;
        }
        if (cm.half == 0 && (cm.flags & 1)) {
          if (!tc::mbar_wait(&ms.q_ready, uint32_t(seg & 1), G.wait_polls)) { failed = true; break; }
          ++seg;
        }
        tc::fence_after_sync();
        const uint32_t d = tbase + uint32_t(tile_i & 1) * kDCols;
        const uint32_t tA = tbase + kTmemA + uint32_t(ab) * kACols;   // term t at + 32 t
        const uint32_t sQ = tc::smem_u32(smem + kOffQ) + uint32_t(cm.half) * kQHalf;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {           // K-step = 16 fp16 = 8 TMEM columns
          const uint64_t b = tc::desc_sw128(sQ + ks * 32, 16, 1024);   // rows: q0 heads, then q1
          tc::mma_f16_ta(d, tA + ks * 8, b, idesc64, (cm.half == 0 && ks == 0) ? 0u : 1u);
          tc::mma_f16_ta(d, tA + 32 + ks * 8, b, idesc32, 1u);
        }
        tc::mma_commit(&ms.a_free[ab]);
        if (cm.half == 1) {
          tc::mma_commit(&ms.d_full[tile_i & 1]);
          ++tile_i;
        }
        ++k;
      }
      // Every MMA issued so far completes before TMEM is released.
      tc::mma_commit(&ms.drain);
      if (!tc::mbar_wait(&ms.drain, 0u, G.wait_polls)) failed = true;
      if (failed) atomicOr(&ms.err, 1u);
    }
  } else if (warp >= 4 && warp < kEpiWarp0) {
    // ---------------- converters ----------------
    const int ctid = tid - 128;                     // 0..255
    const int cq = warp & 3;                        // TMEM lane quadrant
    const int cr = cq * 32 + lane;                  // MMA row = (node, plane)
    const int cb = (warp - 4) >> 2;                 // 32-column box of the half
    int64_t k = 0, tile_i = 0;
    int slot = 0, ab = 0, prev_ab = kABufs - 1;    // k % kRawSlots, k % kABufs, (k - 1) % kABufs
    uint32_t slot_par = 0u, ab_par = 0u, prev_par = 1u;   // the matching (k / n) & 1
    bool failed = false;
    while (true) {
      bool bad = !tc::mbar_wait(&ms.raw_full[slot], slot_par, G.wait_polls);
      // (after a failed wait these fields are stale: they then only steer
      // bounded waits before the warp stops)
      const int32_t m_flags = ms.meta[slot].flags, m_half = ms.meta[slot].half;
      const bool end = (m_flags & 2) != 0;
      // A half-buffer ab was last read by the MMAs of half k - kABufs; the
      // tile's metadata slot by the epilogue of tile_i - 2.
      // (also before the end marker: the MMA issuer reads cmeta[ab] first)
      if (k >= kABufs) bad |= !tc::mbar_wait(&ms.a_free[ab], ab_par ^ 1u, G.wait_polls);
      if ((end || m_half == 0) && tile_i >= 2)
        bad |= !tc::mbar_wait(&ms.d_free[tile_i & 1], uint32_t(((tile_i >> 1) - 1) & 1), G.wait_polls);
      // A new group's Q replaces the old one once every MMA that reads it (the
      // previous half's) is complete.
      const bool new_q = !end && m_half == 0 && (m_flags & 1);
      if (new_q && k >= 1) bad |= !tc::mbar_wait(&ms.a_free[prev_ab], prev_par, G.wait_polls);
      // A warp stops as a whole; the other roles' bounded waits then run out.
      if (__any_sync(0xffffffffu, bad)) { failed = true; break; }
      if (end) {
        if (ctid == 0) {
          ms.cmeta[ab].half = 0;
          ms.cmeta[ab].flags = 2;
          ms.emeta[tile_i & 1].flags = 2;
        }
        __syncwarp();
        if (lane == 0) {
          if (ctid < kNodes * kR) tc::mbar_arrive(&emeta_full[tile_i & 1]);
          tc::mbar_arrive(&ms.conv_done[ab]);
        }
        break;
      }
      if (new_q) {
        // Q of the slot's group -> two fp16 terms, rows term * 32 + q of a
        // [2 halves][64 rows][128 B] K-major 128-byte-swizzled operand.
        const int v = ms.meta[slot].group;
        const int nq = group_width(G, batch, q_blocks, v);
        const int q = ctid >> 3, part = ctid & 7;
#pragma unroll
        for (int c8 = 0; c8 < 2; ++c8) {
          const int col = part * 16 + c8 * 8;
          float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
          if (q < nq) {
            const float* src = Q + head_of(G, q_blocks, v, q) * kD + col;
            a = *reinterpret_cast<const float4*>(src);
            b = *reinterpret_cast<const float4*>(src + 4);
          }
          uint4 t[2];
          split2_x8(a, b, t[0], t[1]);
          const int half = col >> 6, c16 = (col & 63) >> 3;
#pragma unroll
          for (int term = 0; term < 2; ++term) {
            const int row = term * kQn + q;
            const uint32_t off = uint32_t(half * kQHalf + (row >> 3) * 1024 + (row & 7) * 128 +
                                          ((c16 ^ (row & 7)) << 4));
            *reinterpret_cast<uint4*>(smem + kOffQ + off) = t[term];
          }
        }
        tc::fence_async_smem();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&ms.q_ready);
      }
      // The tile's metadata (lanes of warp 4, one field each) and bhat (warps
      // 4-7) reach the epilogue through one arrival per copying warp.
      if (m_half == 0 && ctid < kNodes * kR) {
        EMeta& em = ms.emeta[tile_i & 1];
        if (ctid < kNodes) em.mask[ctid] = ms.meta[slot].mask[ctid];
        else if (ctid == kNodes) em.node0 = ms.meta[slot].node0;
        else if (ctid == kNodes + 1) em.group = ms.meta[slot].group;
        else if (ctid == kNodes + 2) em.flags = m_flags;
        em.bhat[ctid] = ms.bhat_raw[slot][ctid];
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&emeta_full[tile_i & 1]);
      }
      // Raw half: [2 boxes of 32 columns][128 rows][128 B] fp32, 128-byte
      // swizzled. Thread = (row cr, box cb): its 32 values -> two terms of 16
      // packed fp16 pairs -> TMEM columns [term * 32 + cb * 16, + 16) of the A
      // half-buffer, lane cr.
      tc::fence_after_sync();                      // after a_free: the MMAs that read this A are done
      {
        const int sw = cr & 7;
        const uint8_t* rrow = smem + kOffRaw + slot * kRawBytes + cb * 16384 + (cr >> 3) * 1024 + sw * 128;
        uint32_t t0[16], t1[16];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float4 x = *reinterpret_cast<const float4*>(rrow + ((c ^ sw) << 4));
          split2_x2(x.x, x.y, t0[2 * c], t1[2 * c]);
          split2_x2(x.z, x.w, t0[2 * c + 1], t1[2 * c + 1]);
        }
        const uint32_t tA = tbase + (uint32_t(cq * 32) << 16) + kTmemA + uint32_t(ab) * kACols + cb * 16;
        tc::tmem_st16u(tA, t0);
        tc::tmem_st16u(tA + 32, t1);
        tc::tmem_wait_st();
      }
      if (ctid == 0) {
        ms.cmeta[ab].half = m_half;
        ms.cmeta[ab].flags = m_flags & 1;
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) {                             // for the warp's 32 threads
        tc::mbar_arrive(&ms.raw_empty[slot]);
        tc::mbar_arrive(&ms.conv_done[ab]);
      }
      if (m_half == 1) ++tile_i;
      ++k;
      prev_ab = ab;
      prev_par = ab_par;
      if (++slot == kRawSlots) { slot = 0; slot_par ^= 1u; }
      if (++ab == kABufs) { ab = 0; ab_par ^= 1u; }
    }
    if (failed && lane == 0) atomicOr(&ms.err, 1u);
  } else if (warp >= kEpiWarp0) {
    // ---------------- epilogue: thread = TMEM lane = (node, plane) row ----------------
    const int eq = warp & 3;
    const int r = eq * 32 + lane, nj = r >> 4, plane = r & 15;
    const uint32_t t_lane = uint32_t(eq * 32) << 16;
    int64_t tile_i = 0;
    bool failed = false;
    int row_group = -1;                            // group of the cached score rows
    int64_t srow[2] = {0, 0};                      // sigma rows of heads 2 plane, 2 plane + 1
    while (true) {
      const int b = int(tile_i & 1);
      const uint32_t ph = uint32_t((tile_i >> 1) & 1);
      bool bad = !tc::mbar_wait(&emeta_full[b], ph, G.wait_polls);
      bad |= !tc::mbar_wait(&ms.d_full[b], ph, G.wait_polls);
      if (tc::named_sync_or(3, 128, bad)) { failed = true; break; }
      tc::fence_after_sync();
      const int32_t em_flags = ms.emeta[b].flags, em_node0 = ms.emeta[b].node0, em_group = ms.emeta[b].group;
      const uint32_t node_mask = ms.emeta[b].mask[nj];
      const float bhat_r = ms.emeta[b].bhat[r];
      if (em_flags & 2) break;
      float v[kQn];
      tc::tmem_ld32(tbase + t_lane + uint32_t(b) * kDCols, v);
#pragma unroll
      for (int g2 = 0; g2 < 2; ++g2) {            // + column group 32..63, 16 at a time
        float w[16];
        tc::tmem_ld16(tbase + t_lane + uint32_t(b) * kDCols + 32 + 16 * g2, w);
#pragma unroll
        for (int i = 0; i < 16; ++i) v[16 * g2 + i] += w[i];
      }
      tc::fence_before_sync();
      tc::mbar_arrive(&ms.d_free[b]);
      const int64_t node = int64_t(em_node0) + nj;
      const bool live = node < n_nodes;
      // A non-finite product means an element beyond the fp16 range (or a
      // non-finite input): this row's dot products are recomputed in fp32.
      // (Finite products stay far below the fp32 range, so the sum of the
      // row's values is finite exactly when every value is.)
      float vsum = 0.f;
#pragma unroll
      for (int q = 0; q < kQn; ++q) vsum += v[q];
      if (!isfinite(vsum) && live) {
        const int gq = em_group / q_blocks;
        const float* krow = level_base + (int64_t(gq) * G.cap[level] + node) * G.node_floats + plane * kD;
        const int nq = group_width(G, batch, q_blocks, em_group);
#pragma unroll
        for (int q = 0; q < kQn; ++q) {
          float acc = 0.f;
          if (q < nq) {
            const float* qrow = Q + head_of(G, q_blocks, em_group, q) * kD;
#pragma unroll 1
            for (int dd = 0; dd < kD; ++dd) acc = fmaf(qrow[dd], krow[dd], acc);
          }
          v[q] = acc;
        }
      }
      const float bh_ = bhat_r;
#pragma unroll
      for (int q = 0; q < kQn; ++q) v[q] = live ? v[q] * G.scale + bh_ : -INFINITY;
      // maximum over the node's 16 lanes; lane `plane` ends with heads 2 plane, 2 plane + 1
#pragma unroll
      for (int o = 8, half = 16; o > 0; o >>= 1, half >>= 1) {
        const bool upper = (plane & o) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
          const float send = upper ? v[i] : v[i + half];
          const float keep = upper ? v[i + half] : v[i];
          v[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, o));
        }
      }
      if (live) {
        if (em_group != row_group) {
          row_group = em_group;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) srow[kk] = head_of(G, q_blocks, em_group, 2 * plane + kk) * n_nodes;
        }
        const uint32_t m = node_mask;
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          if ((m >> (2 * plane + kk)) & 1u) sigma[srow[kk] + node] = v[kk];
      }
      ++tile_i;
    }
    if (failed && lane == 0 && eq == 0) atomicOr(&ms.err, 1u);
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, kTmemCols);
  }
  if (tid == 0 && ms.err != 0u && status != nullptr) atomicOr(status, ZHA_DEV_TIMEOUT);
}

// Level `level` of the summary store as a 3-D fp32 tensor {d, R, Hkv * cap}:
// box 32 columns (128 B) x 16 planes x 8 nodes, 128-byte swizzled.
bool score_tma_supported(const Geom& G) { return G.d == kD && G.nref == kR; }

cudaError_t launch_score_tma(const Geom& G, int level, int64_t n_nodes, int64_t n_par, int32_t batch,
                             const float* Q, const uint32_t* kept_up, int64_t words_up, float* sigma,
                             const float* store, int32_t* status, cudaStream_t s, bool* used) {
  *used = false;
  const PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (fn == nullptr || n_nodes <= 0) return cudaSuccess;
  const float* level_base = store + G.off[level];
  CUtensorMap map{};
  const cuuint64_t dims[3] = {cuuint64_t(kD), cuuint64_t(kR), cuuint64_t(G.hkv) * cuuint64_t(G.cap[level])};
  const cuuint64_t strides[2] = {cuuint64_t(kD) * 4, cuuint64_t(G.node_floats) * 4};
  const cuuint32_t box[3] = {32u, cuuint32_t(kR), cuuint32_t(kNodes)};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  if (fn(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(level_base), dims, strides, box,
         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaSuccess;
  // bhat of each node: 16 floats after the node's khat, as a 2-D tensor {R, Hkv * cap}.
  CUtensorMap bmap{};
  const cuuint64_t bdims[2] = {cuuint64_t(kR), cuuint64_t(G.hkv) * cuuint64_t(G.cap[level])};
  const cuuint64_t bstrides[1] = {cuuint64_t(G.node_floats) * 4};
  const cuuint32_t bbox[2] = {cuuint32_t(kR), cuuint32_t(kNodes)};
  const cuuint32_t bestr[2] = {1u, 1u};
  if (fn(&bmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(level_base + kR * kD), bdims,
         bstrides, bbox, bestr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
         CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaSuccess;
  const size_t smem = score_tma_smem_bytes();
  cudaError_t e = ensure_dynamic_smem(score_tma_kernel, smem);
  if (e != cudaSuccess) return e;
  int sms = 148;
  if ((e = device_sm_count(&sms)) != cudaSuccess) return e;
  const int32_t q_blocks = int32_t((int64_t(batch) * G.group + kQn - 1) / kQn);
  const int32_t groups = G.hkv * q_blocks;
  const int64_t tiles = groups * ((n_nodes + kNodes - 1) / kNodes);
  const unsigned ctas = unsigned(tiles < sms ? tiles : sms);
  TraceScope ts("score_tma_kernel", level, s);
  e = launch_pdl(score_tma_kernel, dim3(ctas), dim3(kThreads), smem, s, map, bmap, G, level, n_nodes,
                 n_par, batch, q_blocks, groups, Q, kept_up, words_up, sigma, level_base, status);
  zha_count_launch();
  *used = true;
  return e;
}

}  // namespace zha
