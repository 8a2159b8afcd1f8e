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
// Operand. For this shape the store keeps every level's planes twice: the
// fp32 summary, and two fp16 terms per value, t0 = x rounded to fp16 and t1 =
// (x - t0) rounded to fp16 (x = t0 + t1 to 2^-22 |x|, rounded to nearest).
// plane_terms_kernel writes the terms of the nodes that zha_build and
// zha_append_chunk have just summarised. The terms are the A operand of the
// tensor cores exactly as they arrive from HBM: between the tensor copy and the
// MMA no thread touches a plane value.
//
// Work: tiles of 8 nodes of one group (KV head g, block of up to 32 of its
// query heads). The tiles of all groups form one sequence that is split evenly
// over one persistent CTA per SM. Roles inside a CTA:
//   producer (warp 0)       per tile, the candidate mask of each node (bit q =
//                           query head q has the node's parent kept, or the
//                           node is an orphan); tiles without any candidate are
//                           skipped. For the others the tile's metadata goes
//                           into its stage of a 3-stage ring, then tensor
//                           copies of both terms (box = 64 columns x 16 planes
//                           x 8 nodes, fp16, 128-byte swizzled, rows (node,
//                           plane) = MMA rows; one box per term and half of the
//                           columns, 64 KB a tile) and of bhat
//   MMA issuer (warp 1)     S^T[(node, plane)][head] over 8 K-steps:
//                           A_t0 . [q0 | q1]^T (N = 64) and A_t1 . q0^T (N = 32)
//                           into one of two TMEM buffers -- the three products
//                           above 2^-22 of the result; A and B both fp16 in
//                           shared memory
//   Q writer (warps 2-3)    at a group's first tile, once every MMA of the
//                           previous group is complete: the group's queries as
//                           two fp16 terms (q0, q1) in the B operand's layout
//   epilogue (warps 4-7)    thread = (node, plane) row: sum of the two column
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
constexpr int kStages = 3;
constexpr int kStageBytes = 65536;        // [2 terms][2 column halves][128 rows][128 B]
constexpr int kQHalf = 2 * kQn * 128;     // [64 rows = term x 32 heads][128 B]
constexpr int kOffQ = kStages * kStageBytes;          // 2 column halves x kQHalf
constexpr int kOffMisc = kOffQ + 2 * kQHalf;
constexpr int kThreads = 256;             // warps: 0 producer, 1 MMA, 2-3 Q writer, 4-7 epilogue
constexpr int kEpiWarp0 = 4;
constexpr uint32_t kTmemCols = 128;       // D buffers (64 columns) at 0 and 64
constexpr uint32_t kDCols = 64;

struct Meta {                             // one tile, producer -> MMA issuer and epilogue
  int32_t node0, group, flags, pad;       // flags: 1 = first tile of a group, 2 = end
  uint32_t mask[kNodes];
};

struct Misc {
  uint64_t full[kStages], empty[kStages], d_full[2], d_free[2], q_req, q_free, q_ready, drain;
  uint32_t tmem_base, err;
  int32_t q_group, pad;                   // the group whose queries the MMA issuer asks for (-1: stop)
  Meta meta[kStages];
  alignas(128) float bhat[kStages][kNodes * kR];  // tensor-copied with the tile
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

// Level `level`'s planes of nodes [n0, n1) of every KV head -> the two fp16
// terms of the store's second copy. Thread = (node, plane, 8 columns).
__global__ void __launch_bounds__(256)
plane_terms_kernel(Geom G, int level, int64_t n0, int64_t n1, float* __restrict__ store) {
  const int g = blockIdx.y;
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= (n1 - n0) * (kR * kD / 8)) return;
  const int64_t node = n0 + i / (kR * kD / 8);
  const int plane = int(i / (kD / 8)) % kR, c8 = int(i % (kD / 8));
  const float* src = store + G.off[level] + (int64_t(g) * G.cap[level] + node) * G.node_floats +
                     plane * kD + 8 * c8;
  const float4 a = *reinterpret_cast<const float4*>(src);
  const float4 b = *reinterpret_cast<const float4*>(src + 4);
  uint4 t0, t1;
  split2_x8(a, b, t0, t1);
  __half* dst = reinterpret_cast<__half*>(reinterpret_cast<uint8_t*>(store) + G.split_off[level]);
  const int64_t term = G.cap[level] * (kR * kD);                  // elements per term of a KV head
  const int64_t e = int64_t(g) * 2 * term + node * (kR * kD) + plane * kD + 8 * c8;
  *reinterpret_cast<uint4*>(dst + e) = t0;
  *reinterpret_cast<uint4*>(dst + e + term) = t1;
}

__global__ void __launch_bounds__(kThreads, 1)
score_tma_kernel(const __grid_constant__ CUtensorMap tmT, const __grid_constant__ CUtensorMap tmB, Geom G,
                 int level, int64_t n_nodes, int64_t n_par, int32_t batch, int32_t q_blocks, int32_t groups,
                 const float* __restrict__ Q, const uint32_t* __restrict__ kept_up, int64_t words_up,
                 float* __restrict__ sigma, const float* __restrict__ level_base, int32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Misc& ms = *reinterpret_cast<Misc*>(smem + kOffMisc);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t nt = (n_nodes + kNodes - 1) / kNodes;        // tiles per group
  const int64_t T = nt * groups;
  const int nct = int(gridDim.x), cta = int(blockIdx.x);
  const int64_t t0 = int64_t(cta) * T / nct, t1 = int64_t(cta + 1) * T / nct;

  if (tid == 0) {
    ms.err = 0u;
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&ms.full[s], 1);
      tc::mbar_init(&ms.empty[s], 1 + 4);          // the MMAs' commit, one arrival per epilogue warp
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&ms.d_full[b], 1);
      tc::mbar_init(&ms.d_free[b], 4);             // one arrival per epilogue warp
    }
    tc::mbar_init(&ms.q_req, 1);
    tc::mbar_init(&ms.q_free, 1);
    tc::mbar_init(&ms.q_ready, 2);                 // one arrival per Q writer warp
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
    int64_t k = 0;                     // tiles emitted
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
    for (int32_t t = int32_t(t0); t < t_stop; ++t) {
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
      const int st = int(k % kStages);
      const int64_t use = k / kStages;
      bool bad = false;
      if (use > 0) bad = !tc::mbar_wait(&ms.empty[st], uint32_t((use - 1) & 1), G.wait_polls);
      if (__any_sync(0xffffffffu, bad)) { failed = true; break; }
      if (lane == 0) {
        Meta& mt = ms.meta[st];
        mt.node0 = node0;
        mt.group = v;
        mt.flags = first ? 1 : 0;
#pragma unroll
        for (int j = 0; j < kNodes; ++j) mt.mask[j] = m[j];
        tc::mbar_arrive_expect_tx(&ms.full[st], 4u * 16384u + 512u);
        const uint32_t dst = tc::smem_u32(smem + st * kStageBytes);
        const int32_t zt = 2 * (v / q_blocks);    // term 0 of KV head g; term 1 follows
        tc::tma_load_4d(dst, &tmT, 0, 0, node0, zt, &ms.full[st]);
        tc::tma_load_4d(dst + 16384, &tmT, 64, 0, node0, zt, &ms.full[st]);
        tc::tma_load_4d(dst + 32768, &tmT, 0, 0, node0, zt + 1, &ms.full[st]);
        tc::tma_load_4d(dst + 49152, &tmT, 64, 0, node0, zt + 1, &ms.full[st]);
        const int32_t zb = int32_t(int64_t(v / q_blocks) * G.cap[level] + node0);
        tc::tma_load_2d(tc::smem_u32(ms.bhat[st]), &tmB, 0, zb, &ms.full[st]);
      }
      __syncwarp();
      ++k;
    }
    bool sent_end = false;
    if (!failed && !G.debug_withhold) {            // end of the stream
      const int st = int(k % kStages);
      const int64_t use = k / kStages;
      bool bad = false;
      if (use > 0) bad = !tc::mbar_wait(&ms.empty[st], uint32_t((use - 1) & 1), G.wait_polls);
      if (__any_sync(0xffffffffu, bad)) {
        failed = true;
      } else {
        sent_end = true;
        if (lane == 0) {
          ms.meta[st].flags = 2;
          tc::mbar_arrive(&ms.full[st]);
        }
      }
    }
    // Before the CTA may exit, every tensor copy issued into shared memory has
    // landed: wait for the copies of each stage's last tile. The end marker
    // reused the stage of tile k - 3 only after that tile was consumed, and
    // moved the stage's phase on, so that tile is not waited for again.
    if (lane == 0) {
      const int64_t j0 = (k > kStages ? k - kStages : 0) + (sent_end && k >= kStages ? 1 : 0);
      for (int64_t j = j0; j < k; ++j)
        if (!tc::mbar_wait(&ms.full[j % kStages], uint32_t((j / kStages) & 1), G.wait_polls))
          failed = true;
    }
    if (failed && lane == 0) atomicOr(&ms.err, 1u);
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc64 = tc::idesc_f16(128, 64, 0, 0);
      constexpr uint32_t idesc32 = tc::idesc_f16(128, 32, 0, 0);
      const uint32_t sQ = tc::smem_u32(smem + kOffQ);
      int64_t k = 0;
      int seg = 0;                     // groups whose queries have been written
      bool failed = false;
      while (true) {
        const int st = int(k % kStages), b = int(k & 1);
        if (!tc::mbar_wait(&ms.full[st], uint32_t((k / kStages) & 1), G.wait_polls)) { failed = true; break; }
        const int32_t flags = ms.meta[st].flags, v = ms.meta[st].group;
        // The D buffer of this tile must have been read by the epilogue.
        if (k >= 2 && !tc::mbar_wait(&ms.d_free[b], uint32_t(((k >> 1) - 1) & 1), G.wait_polls)) {
          failed = true;
          break;
        }
        if (flags & 2) {                           // end: let the epilogue see it
          tc::mma_commit(&ms.d_full[b]);
          break;
        }
        if (flags & 1) {
          // A new group: its queries replace the previous group's once every
          // MMA issued so far is complete (the commit tracks them all).
          if (seg > 0) tc::mma_commit(&ms.q_free);
          ms.q_group = v;
          tc::mbar_arrive(&ms.q_req);
          if (!tc::mbar_wait(&ms.q_ready, uint32_t(seg & 1), G.wait_polls)) { failed = true; break; }
          ++seg;
        }
        tc::fence_after_sync();
        const uint32_t d = tbase + uint32_t(b) * kDCols;
        const uint32_t sA = tc::smem_u32(smem + st * kStageBytes);
#pragma unroll
        for (int kh = 0; kh < 2; ++kh) {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {         // K-step = 16 fp16 = 32 bytes of a row
            const uint64_t a0 = tc::desc_sw128(sA + kh * 16384 + ks * 32, 16, 1024);
            const uint64_t a1 = tc::desc_sw128(sA + 32768 + kh * 16384 + ks * 32, 16, 1024);
            const uint64_t bq = tc::desc_sw128(sQ + kh * kQHalf + ks * 32, 16, 1024);  // q0 rows, then q1
            tc::mma_f16(d, a0, bq, idesc64, (kh | ks) != 0 ? 1u : 0u);
            tc::mma_f16(d, a1, bq, idesc32, 1u);
          }
        }
        tc::mma_commit(&ms.empty[st]);
        tc::mma_commit(&ms.d_full[b]);
        ++k;
      }
      ms.q_group = -1;                             // the Q writer stops
      tc::mbar_arrive(&ms.q_req);
      // Every MMA issued so far completes before TMEM is released.
      tc::mma_commit(&ms.drain);
      if (!tc::mbar_wait(&ms.drain, 0u, G.wait_polls)) failed = true;
      if (failed) atomicOr(&ms.err, 1u);
    }
  } else if (warp < kEpiWarp0) {
    // ---------------- Q writer: thread = (head q, half of the columns) ----------------
    const int qt = tid - 64, q = qt >> 1, hf = qt & 1;
    bool failed = false;
    for (int j = 0;; ++j) {
      bool bad = !tc::mbar_wait(&ms.q_req, uint32_t(j & 1), G.wait_polls);
      const int v = ms.q_group;
      if (!bad && v >= 0 && j > 0) bad = !tc::mbar_wait(&ms.q_free, uint32_t((j - 1) & 1), G.wait_polls);
      if (__any_sync(0xffffffffu, bad)) { failed = true; break; }
      if (v < 0) break;
      // Q of head q, columns [64 hf, + 64) -> rows term * 32 + q of column
      // half hf of the [2 halves][64 rows][128 B] K-major 128-byte-swizzled
      // operand.
      const int nq = group_width(G, batch, q_blocks, v);
      const float* src = Q + head_of(G, q_blocks, v, q < nq ? q : 0) * kD + 64 * hf;
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
        if (q < nq) {
          a = *reinterpret_cast<const float4*>(src + 8 * c8);
          b = *reinterpret_cast<const float4*>(src + 8 * c8 + 4);
        }
        uint4 t[2];
        split2_x8(a, b, t[0], t[1]);
#pragma unroll
        for (int term = 0; term < 2; ++term) {
          const int row = term * kQn + q;
          const uint32_t off = uint32_t(hf * kQHalf + (row >> 3) * 1024 + (row & 7) * 128 +
                                        ((c8 ^ (row & 7)) << 4));
          *reinterpret_cast<uint4*>(smem + kOffQ + off) = t[term];
        }
      }
      tc::fence_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&ms.q_ready);
    }
    if (failed && lane == 0) atomicOr(&ms.err, 1u);
  } else {
    // ---------------- epilogue: thread = TMEM lane = (node, plane) row ----------------
    const int eq = warp & 3;
    const int r = eq * 32 + lane, nj = r >> 4, plane = r & 15;
    const uint32_t t_lane = uint32_t(eq * 32) << 16;
    int64_t k = 0;
    bool failed = false;
    int row_group = -1;                            // group of the cached score rows
    int64_t srow[2] = {0, 0};                      // sigma rows of heads 2 plane, 2 plane + 1
    while (true) {
      const int st = int(k % kStages), b = int(k & 1);
      bool bad = !tc::mbar_wait(&ms.d_full[b], uint32_t((k >> 1) & 1), G.wait_polls);
      // (the stage's metadata was written before the producer's arrival)
      bad |= !tc::mbar_wait(&ms.full[st], uint32_t((k / kStages) & 1), G.wait_polls);
      if (tc::named_sync_or(3, 128, bad)) { failed = true; break; }
      const Meta& mt = ms.meta[st];
      if (mt.flags & 2) break;
      const int32_t em_node0 = mt.node0, em_group = mt.group;
      const uint32_t node_mask = mt.mask[nj];
      const float bhat_r = ms.bhat[st][r];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&ms.empty[st]);      // the warp is done with the stage
      tc::fence_after_sync();
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
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&ms.d_free[b]);
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
      ++k;
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

bool score_tma_supported(const Geom& G) { return has_plane_terms(G) && G.d == kD && G.nref == kR; }

// The fp16 terms of nodes [nb_old / C^l, nb_new / C^l) of every level, after
// the fp32 planes of those nodes have been written.
cudaError_t launch_plane_terms(const Geom& G, float* store, int64_t nb_old, int64_t nb_new, cudaStream_t s) {
  if (!score_tma_supported(G)) return cudaSuccess;
  for (int l = 1; l <= G.levels; ++l) {
    const int64_t n0 = nodes_at(nb_old, G.chunk, l), n1 = nodes_at(nb_new, G.chunk, l);
    if (n1 <= n0) continue;
    const int64_t threads = (n1 - n0) * (kR * kD / 8);
    plane_terms_kernel<<<dim3(unsigned((threads + 255) / 256), unsigned(G.hkv)), 256, 0, s>>>(G, l, n0, n1,
                                                                                                 store);
    zha_count_launch();
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_score_tma(const Geom& G, int level, int64_t n_nodes, int64_t n_par, int32_t batch,
                             const float* Q, const uint32_t* kept_up, int64_t words_up, float* sigma,
                             const float* store, int32_t* status, cudaStream_t s, bool* used) {
  *used = false;
  const PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (fn == nullptr || n_nodes <= 0 || G.split_off[level] == 0) return cudaSuccess;
  const float* level_base = store + G.off[level];
  // The level's fp16 terms as a 4-D tensor {d, R, cap, Hkv * 2 terms}: box 64
  // columns (128 B) x 16 planes x 8 nodes, 128-byte swizzled.
  CUtensorMap map{};
  const void* terms = reinterpret_cast<const uint8_t*>(store) + G.split_off[level];
  const cuuint64_t dims[4] = {cuuint64_t(kD), cuuint64_t(kR), cuuint64_t(G.cap[level]), cuuint64_t(G.hkv) * 2};
  const cuuint64_t strides[3] = {cuuint64_t(kD) * 2, cuuint64_t(kR) * kD * 2,
                                 cuuint64_t(G.cap[level]) * kR * kD * 2};
  const cuuint32_t box[4] = {64u, cuuint32_t(kR), cuuint32_t(kNodes), 1u};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  if (fn(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void*>(terms), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
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
