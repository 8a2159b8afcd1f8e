// zha_score_tc.cu -- node scoring on the sm_100a tensor cores for head_dim 128
// and fewer than 16 reference queries per tree (R = 16 goes to the tensor-copy
// kernel in zha_score_tma.cu).
//
// Citations: [ZHA: 무엇과 다른가 / 전제와 한계] = page "ZHA는 KV 캐시를 트리로 요약해
// 어텐션 비용을 준(sub)이차로 낮춘다" (onedev.kr/papers/1556): a node's estimated log
// mass for a query is the maximum of its R tangent planes,
// sigma = max_r (q . khat_r / sqrt(d) + bhat_r); each level scores the
// candidates passed down from the level above.
//
// A CTA (128 threads) takes a tile of nodes of one KV head; nodes that are a
// candidate of no query head of the block are skipped in groups of 8. For 8
// nodes the planes form A = [128 rows = (node, plane)][128 = d] and the block's
// query heads B = [32][128]; S^T = A . B^T lands in TMEM (128 lanes x 32
// columns). fp32 accuracy with bf16 tensor cores: khat and q are each split
// into three bf16 terms (x = x1 + x2 + x3, exact to fp32's 24 bits) and the
// six products with term indices summing to <= 2 are accumulated; the three
// dropped products are below fp32 rounding. The K dimension is processed in
// two halves of 64 so that the three A terms of a half take 48 KB (the split
// uses packed bf16x2 conversions, 8 elements per 16-byte store); the next
// half's node rows are loaded into registers while the MMAs of the current
// one run. Epilogue: thread = TMEM lane = (node, plane) adds bhat and takes
// the maximum over its node's 16 lanes (a transpose-reduction leaves lane p
// of the node with heads 2p and 2p+1), then writes the scores of the
// (node, head) pairs that are candidates.
#include "zha_host.cuh"
#include "zha_internal.cuh"
#include "zha_tc.cuh"

namespace zha {

constexpr int kStThreads = 128;
constexpr int kStNodes = 8;                // nodes per MMA tile (8 x 16 planes = 128 rows)
constexpr int kStQ = 32;                   // query heads per CTA (MMA N)
constexpr int kStD = 128;
constexpr int kStTile = 64;                // nodes per CTA at most
constexpr uint32_t kStWaitTries = tc::kWaitPolls;
constexpr int kStOffA = 0;                 // 3 terms x [128 rows][64 cols] bf16 = 3 x 16 KB
constexpr int kStOffQ = 3 * 16384;         // 3 terms x [2 col blocks][32 rows][128 B] = 3 x 8 KB
constexpr int kStOffMisc = kStOffQ + 3 * 8192;

struct StMisc {
  uint64_t mbar;
  uint32_t tmem_base;
  uint32_t err;
  unsigned long long any;
  uint32_t mask[kStTile];
  uint32_t kw[kStQ][3];
  int64_t out[kStQ];
};

__host__ inline size_t score_tc_smem_bytes() { return size_t(kStOffMisc) + sizeof(StMisc) + 1024; }

__device__ __forceinline__ void split3(float x, __nv_bfloat16& a, __nv_bfloat16& b, __nv_bfloat16& c) {
  a = __float2bfloat16_rn(x);
  x -= __bfloat162float(a);
  b = __float2bfloat16_rn(x);
  x -= __bfloat162float(b);
  c = __float2bfloat16_rn(x);
}

// Two fp32 values -> three packed bf16x2 terms (x = t1 + t2 + t3 per lane of
// the pair): one cvt.rn.bf16x2.f32 per term, the widening back to fp32 is a
// shift or a mask.
__device__ __forceinline__ void split3_x2(float x0, float x1, uint32_t& t1, uint32_t& t2, uint32_t& t3) {
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(t1) : "f"(x1), "f"(x0));
  x0 -= __uint_as_float(t1 << 16);
  x1 -= __uint_as_float(t1 & 0xffff0000u);
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(t2) : "f"(x1), "f"(x0));
  x0 -= __uint_as_float(t2 << 16);
  x1 -= __uint_as_float(t2 & 0xffff0000u);
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(t3) : "f"(x1), "f"(x0));
}

__global__ void __launch_bounds__(kStThreads)
score_tc_kernel(Geom G, int level, int64_t n_nodes, int64_t n_par, int32_t batch, int tile,
                const float* __restrict__ Q, const uint32_t* __restrict__ kept_up, int64_t words_up,
                float* __restrict__ sigma, const float* __restrict__ store, int32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  pdl_trigger();
  pdl_wait();
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  StMisc& ms = *reinterpret_cast<StMisc*>(smem + kStOffMisc);
  const uint32_t sA = tc::smem_u32(smem + kStOffA), sQ = tc::smem_u32(smem + kStOffQ);
  const int g = blockIdx.y;
  const int64_t n0 = int64_t(blockIdx.x) * tile;
  const int GQ = G.group;
  const int qb0 = blockIdx.z * kStQ;
  const int nq = min(kStQ, batch * GQ - qb0);
  const int C = G.chunk, R = G.nref;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int64_t orphan0 = int64_t(C) * n_par;
  const int64_t w_lo = (n0 / C) >> 5;

  // Which query heads of the block have each node of the tile as candidate.
  if (tid == 0) { ms.any = 0ull; ms.err = 0u; }
  if (tid < nq) {
    const int qi = qb0 + tid;
    const int64_t bh = int64_t(qi / GQ) * G.hq + g * GQ + qi % GQ;
    ms.out[tid] = bh * n_nodes;
    if (n0 < orphan0) {
      const uint32_t* kw = kept_up + bh * words_up;
#pragma unroll
      for (int k = 0; k < 3; ++k) ms.kw[tid][k] = (w_lo + k < words_up) ? kw[w_lo + k] : 0u;
    }
  }
  __syncthreads();
  if (tid < tile) {
    const int64_t n = n0 + tid;
    uint32_t m = 0u;
    if (n < n_nodes) {
      if (n >= orphan0) {
        m = nq == 32 ? 0xffffffffu : ((1u << nq) - 1u);
      } else {
        const int64_t pnode = n / C;
        const int slot = int((pnode >> 5) - w_lo);
        const int bit = int(pnode & 31);
        for (int q = 0; q < nq; ++q) m |= ((ms.kw[q][slot] >> bit) & 1u) << q;
      }
    }
    ms.mask[tid] = m;
    if (m) atomicOr(&ms.any, 1ull << (tid / kStNodes));
  }
  __syncthreads();
  unsigned long long tiles_left = ms.any;      // bit s = sub-tile s has work
  if (tiles_left == 0ull) return;

  // Query heads of the block -> three bf16 terms, K-major rows (row = head).
  for (int v = tid; v < kStQ * (kStD / 8); v += blockDim.x) {
    const int q = v / (kStD / 8), col = (v % (kStD / 8)) * 8;
    float x[8];
    if (q < nq) {
      const int qi = qb0 + q;
      const int64_t bh = int64_t(qi / GQ) * G.hq + g * GQ + qi % GQ;
      const float4 a = *reinterpret_cast<const float4*>(Q + bh * kStD + col);
      const float4 b = *reinterpret_cast<const float4*>(Q + bh * kStD + col + 4);
      x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = 0.f;
    }
    __align__(16) __nv_bfloat16 h[3][8];
#pragma unroll
    for (int i = 0; i < 8; ++i) split3(x[i], h[0][i], h[1][i], h[2][i]);
    const uint32_t off = tc::sw128_offset(q, col, kStQ);
#pragma unroll
    for (int t = 0; t < 3; ++t)
      *reinterpret_cast<uint4*>(smem + kStOffQ + t * 8192 + off) = *reinterpret_cast<uint4*>(h[t]);
  }
  if (tid == 0) tc::mbar_init(&ms.mbar, 1);
  if (warp == 0) tc::tmem_alloc(&ms.tmem_base, 32);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = ms.tmem_base;
  constexpr uint32_t idesc = tc::idesc_bf16(128, kStQ, 0, 0);
  const float* level_base = store + G.off[level] + int64_t(g) * G.cap[level] * G.node_floats;
  uint32_t phase = 0;
  bool pending = false, failed = false;

  // Register-staged half of a sub-tile in chunks of 8 elements: chunk
  // 128j + tid is row (16j + tid/8) (node-major, 16 planes per node), columns
  // 64h + 8 (tid % 8) .. +7.
  float4 buf[16];
  auto load_half = [&](int st, int h) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int row = 16 * j + (tid >> 3);
      const int64_t node = n0 + st * kStNodes + (row >> 4);
      const int plane = row & 15;
      if (node < n_nodes && plane < R) {
        const float4* src = reinterpret_cast<const float4*>(level_base + node * G.node_floats +
                                                            plane * kStD + 64 * h + 8 * (tid & 7));
        buf[2 * j] = __ldg(src);
        buf[2 * j + 1] = __ldg(src + 1);
      } else {
        buf[2 * j] = make_float4(0.f, 0.f, 0.f, 0.f);
        buf[2 * j + 1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  };
  auto store_half = [&]() {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int row = 16 * j + (tid >> 3);
      const float4 a = buf[2 * j], b = buf[2 * j + 1];
      uint4 t1, t2, t3;
      split3_x2(a.x, a.y, t1.x, t2.x, t3.x);
      split3_x2(a.z, a.w, t1.y, t2.y, t3.y);
      split3_x2(b.x, b.y, t1.z, t2.z, t3.z);
      split3_x2(b.z, b.w, t1.w, t2.w, t3.w);
      const uint32_t off = tc::sw128_offset(row, 8 * (tid & 7), 128);
      *reinterpret_cast<uint4*>(smem + kStOffA + off) = t1;
      *reinterpret_cast<uint4*>(smem + kStOffA + 16384 + off) = t2;
      *reinterpret_cast<uint4*>(smem + kStOffA + 32768 + off) = t3;
    }
  };
  auto wait_mma = [&]() {
    if (!tc::mbar_wait(&ms.mbar, phase, kStWaitTries)) atomicOr(&ms.err, 1u);
    phase ^= 1u;
    tc::fence_after_sync();
  };

  int st = __ffsll(tiles_left) - 1;
  tiles_left &= tiles_left - 1ull;
  load_half(st, 0);
  while (st >= 0 && !failed) {
    const int next = tiles_left ? __ffsll(tiles_left) - 1 : -1;
    for (int h = 0; h < 2; ++h) {
      if (pending) { wait_mma(); pending = false; }     // the MMAs reading the A staging are done
      store_half();
      tc::fence_async_smem();
      tc::fence_before_sync();
      __syncthreads();
      if (tid == 0) {
        tc::fence_after_sync();
        constexpr int pa[6] = {0, 0, 1, 0, 1, 2}, pb[6] = {0, 1, 0, 2, 1, 0};
#pragma unroll
        for (int p = 0; p < 6; ++p)
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t a = tc::desc_sw128(sA + pa[p] * 16384 + ks * 32, 16, 1024);
            const uint64_t b = tc::desc_sw128(sQ + pb[p] * 8192 + h * 4096 + ks * 32, 16, 1024);
            tc::mma_bf16(tbase, a, b, idesc, (h | p | ks) != 0);
          }
        tc::mma_commit(&ms.mbar);
      }
      pending = true;
      if (h == 0) load_half(st, 1);                     // in flight while the MMAs run
      else if (next >= 0) load_half(next, 0);
    }
    wait_mma();
    pending = false;

    // Epilogue: lane = (node, plane); + bhat, max over the node's 16 planes.
    float v[kStQ];
    tc::tmem_ld32(tbase + (uint32_t(warp * 32) << 16), v);
    const int nl = tid >> 4, plane = tid & 15;
    const int64_t node = n0 + st * kStNodes + nl;
    const bool live = plane < R && node < n_nodes;
    const float b = live ? __ldg(level_base + node * G.node_floats + R * kStD + plane) : 0.f;
#pragma unroll
    for (int q = 0; q < kStQ; ++q) v[q] = live ? v[q] * G.scale + b : -INFINITY;
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
    // lane `plane` of the node now holds heads 2*plane and 2*plane + 1
    if (node < n_nodes) {
      const uint32_t m = ms.mask[st * kStNodes + nl];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int q = 2 * plane + k;
        if ((m >> q) & 1u) sigma[ms.out[q] + node] = v[k];
      }
    }
    tc::fence_before_sync();
    __syncthreads();                                    // TMEM and A staging are reused
    failed = ms.err != 0u;
    st = next;
    if (next >= 0) tiles_left &= tiles_left - 1ull;
  }
  if (failed && tid == 0 && status != nullptr) atomicOr(status, ZHA_DEV_TIMEOUT);
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, 32);
  }
}

cudaError_t launch_score_tc(const Geom& G, int level, int64_t n_nodes, int64_t n_par, int32_t batch,
                            const float* Q, const uint32_t* kept_up, int64_t words_up, float* sigma,
                            const float* store, int32_t* status, cudaStream_t s) {
  const size_t smem = score_tc_smem_bytes();
  cudaError_t e = ensure_dynamic_smem(score_tc_kernel, smem);
  if (e != cudaSuccess) return e;
  const int qn = batch * G.group;
  // Nodes per CTA: enough CTAs to fill the GPU twice over, at most kStTile.
  int tile = kStTile;
  while (tile > kStNodes && (n_nodes * G.hkv) / tile < 2 * 148) tile >>= 1;
  dim3 grid(unsigned((n_nodes + tile - 1) / tile), unsigned(G.hkv), unsigned((qn + kStQ - 1) / kStQ));
  TraceScope ts("score_tc_kernel", level, s);
  e = launch_pdl(score_tc_kernel, grid, dim3(kStThreads), smem, s, G, level, n_nodes, n_par, batch,
                 tile, Q, kept_up, words_up, sigma, store, status);
  zha_count_launch();
  return e;
}

}  // namespace zha
