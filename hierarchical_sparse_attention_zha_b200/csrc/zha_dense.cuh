// zha_dense.cuh -- dense scoring of whole tree levels on the CUDA cores: every
// node of each given level for every query head of a block of up to 32 heads,
// sigma = max_r (q . khat_r / sqrt(d) + bhat_r) [ZHA: 무엇과 다른가] (page "ZHA는
// KV 캐시를 트리로 요약해 어텐션 비용을 준(sub)이차로 낮춘다"). Used for the small top
// levels of a route and, with the argmax-plane count, for routing diagnostics.
#pragma once

#include "zha_internal.cuh"

namespace zha {

// The small top levels scored densely in one launch: every node of each level
// for every query head (a superset of the candidates; selection reads only the
// candidates' scores). A CTA computes one tile of kDenseRows (node, plane) rows
// -- 64 / R consecutive nodes of one level of KV head g -- against a block of
// up to kDenseQ query heads of g's group, as a small fp32 matrix product:
// operands staged in shared memory K-block-major ([k / 4][row][4]), each thread
// a 4-row x 2-query register tile (rows ty + 16 i, queries tx and tx + 16), so
// that the 16-byte loads of a warp are broadcast (rows) or contiguous (queries).
// Then sigma = max over the node's planes of (dot / sqrt(d) + bhat).
// blockIdx.x runs over the levels' tiles in turn.
constexpr int kDenseRows = 64;
constexpr int kDenseQ = 32;
constexpr int kDenseThreads = 256;

struct DenseLevels {
  int32_t count;
  int32_t level[ZHA_MAX_LEVELS];
  int64_t n_nodes[ZHA_MAX_LEVELS];
  int64_t tile0[ZHA_MAX_LEVELS + 1];       // first blockIdx.x of each level
  float* sigma[ZHA_MAX_LEVELS];
};

template <int D>
__host__ __device__ constexpr size_t dense_smem_bytes() {
  return size_t(kDenseRows + kDenseQ) * D * sizeof(float);
}

// kUsage: also count, per level, how often each plane r gives a node's score
// (the argmax plane, lowest r on ties), into usage[level - 1][R] (accumulated).
template <int D, bool kUsage>
__global__ void __launch_bounds__(kDenseThreads)
score_dense_kernel(Geom G, DenseLevels dl, int32_t batch, const float* __restrict__ Q,
                   const float* __restrict__ store, uint32_t* __restrict__ usage) {
  extern __shared__ float4 smem_v4[];
  float4* As = smem_v4;                          // [D / 4][kDenseRows]
  float4* Bs = smem_v4 + (D / 4) * kDenseRows;   // [D / 4][kDenseQ]
  float* Cs = reinterpret_cast<float*>(smem_v4); // [kDenseRows][kDenseQ + 1] after the product
  __shared__ float s_b[kDenseRows];
  __shared__ uint32_t s_use[ZHA_MAX_REF];
  pdl_trigger();
  pdl_wait();
  if (kUsage && threadIdx.x < ZHA_MAX_REF) s_use[threadIdx.x] = 0u;
  int li = 0;
  while (li + 1 < dl.count && int64_t(blockIdx.x) >= dl.tile0[li + 1]) ++li;
  const int level = dl.level[li];
  const int64_t n_nodes = dl.n_nodes[li];
  const int R = G.nref, npt = kDenseRows / R, rows = npt * R;
  const int g = blockIdx.y, qb = blockIdx.z;
  const int64_t n0 = (int64_t(blockIdx.x) - dl.tile0[li]) * npt;
  const int nn = int(min64(npt, n_nodes - n0));
  const int qn = min(kDenseQ, batch * G.group - qb * kDenseQ);
  const int tid = threadIdx.x;
  const float* level_base = store + G.off[level] + int64_t(g) * G.cap[level] * G.node_floats;
  auto head_of = [&](int q) -> int64_t {
    const int qi = qb * kDenseQ + q;
    return int64_t(qi / G.group) * G.hq + g * G.group + qi % G.group;
  };

  // Stage the tile's planes, bhat and the queries.
  for (int v = tid; v < kDenseRows * (D / 4); v += kDenseThreads) {
    const int row = v / (D / 4), kb = v % (D / 4);
    const int j = row / R, r = row % R;
    float4* dst = As + kb * kDenseRows + row;
    if (row < rows && j < nn) {
      const float* src = level_base + (n0 + j) * G.node_floats + r * D + 4 * kb;
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" : : "r"(uint32_t(__cvta_generic_to_shared(dst))),
                   "l"(src) : "memory");
    } else {
      *dst = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  for (int v = tid; v < kDenseQ * (D / 4); v += kDenseThreads) {
    const int q = v / (D / 4), kb = v % (D / 4);
    float4* dst = Bs + kb * kDenseQ + q;
    if (q < qn) {
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" : : "r"(uint32_t(__cvta_generic_to_shared(dst))),
                   "l"(Q + head_of(q) * D + 4 * kb) : "memory");
    } else {
      *dst = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  if (tid < kDenseRows) {
    const int j = tid / R, r = tid % R;
    s_b[tid] = (tid < rows && j < nn) ? level_base[(n0 + j) * G.node_floats + R * D + r] : 0.f;
  }
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
  __syncthreads();

  const int tx = tid & 15, ty = tid >> 4;
  float acc[4][2] = {};
#pragma unroll 4
  for (int kb = 0; kb < D / 4; ++kb) {
    float4 a[4], b[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = As[kb * kDenseRows + ty + 16 * i];
#pragma unroll
    for (int j = 0; j < 2; ++j) b[j] = Bs[kb * kDenseQ + tx + 16 * j];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 2; ++j)
        acc[i][j] += a[i].x * b[j].x + a[i].y * b[j].y + a[i].z * b[j].z + a[i].w * b[j].w;
  }
  __syncthreads();                               // the operands are read; Cs overwrites them
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int row = ty + 16 * i;
      Cs[row * (kDenseQ + 1) + tx + 16 * j] = acc[i][j] * G.scale + s_b[row];
    }
  __syncthreads();
  for (int o = tid; o < npt * kDenseQ; o += kDenseThreads) {
    const int j = o / kDenseQ, q = o % kDenseQ;
    if (j >= nn || q >= qn) continue;
    float m = -INFINITY;
    int arg = 0;
    for (int r = 0; r < R; ++r) {
      const float v = Cs[(j * R + r) * (kDenseQ + 1) + q];
      if (v > m) { m = v; arg = r; }
    }
    dl.sigma[li][head_of(q) * n_nodes + n0 + j] = m;
    if (kUsage) atomicAdd(&s_use[arg], 1u);
  }
  if (kUsage) {
    __syncthreads();
    if (tid < R && s_use[tid] != 0u) atomicAdd(&usage[(level - 1) * R + tid], s_use[tid]);
  }
}

}  // namespace zha
