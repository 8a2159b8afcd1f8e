// zha_build.cu -- tree construction: level-1 tangent-plane summaries, the merge
// of upper levels, and the fused incremental append.
//
// Citations: [ZHA: 무엇과 다른가] = page "ZHA는 KV 캐시를 트리로 요약해 어텐션 비용을
// 준(sub)이차로 낮춘다" (onedev.kr/papers/1556), section "무엇과 다른가": the chunk's
// log mass F_C(q) = LSE_j(q.k_j/sqrt(d)), its tangent plane at reference query
// q_r with khat_r = Attn(q_r, K_C, K_C) and bhat_r = F_C(q_r) - q_r.khat_r/sqrt(d),
// parents merging child summaries "in the same way", level 1 every C steps and
// level 2 every C^2 steps.
#include "zha_host.cuh"
#include "zha_internal.cuh"

namespace zha {
cudaError_t launch_build_level1_tc(const Geom& G, const void* K, int64_t ld, int64_t c_begin,
                                   int64_t c_end, const float* refq, float* store, int32_t* status,
                                   cudaStream_t s);
cudaError_t launch_plane_terms(const Geom& G, float* store, int64_t nb_old, int64_t nb_new, cudaStream_t s);

// ---------------------------------------------------------------------------
// Level 1. One CTA summarises a tile of `nch` consecutive chunks (nch*C <= 128
// tokens) for all R planes. With the tile's keys K_t [TT][d] and the reference
// queries Qr [R][d] staged in shared memory:
//   S[r][t] = q_r . k_t / sqrt(d)                         (all tokens of the tile)
//   per (chunk, r): F = LSE over the chunk's tokens, P = exp(S - F)
//   khat[r] = sum_t P[r][t] k_t,  bhat[r] = F - q_r . khat[r] / sqrt(d)
// ---------------------------------------------------------------------------
constexpr int kL1Tokens = 128;   // tokens per level-1 tile
constexpr int kBuildThreads = 256;

__host__ __device__ inline int l1_chunks_per_tile(int chunk) { return kL1Tokens / chunk; }

template <int D>
__host__ __device__ inline size_t l1_smem_bytes(int nref) {
  // keys [128][D+4], reference queries [R][D+4], scores [R][128], F [R][128/C] (<= R*64),
  // rotations of the tile's chunks [128/C][D/2] (cos, sin) (<= 64 chunks)
  return sizeof(float) * (size_t(kL1Tokens) * (D + 4) + size_t(nref) * (D + 4) +
                          size_t(nref) * kL1Tokens + size_t(nref) * 64 + size_t(64) * D);
}

template <typename T, int D>
__device__ void summarise_tile(const Geom& G, int g, const KvView& kv, int64_t c0, int nch,
                               const float* __restrict__ refq, float* __restrict__ store,
                               float* smem) {
  constexpr int DP = D + 4;
  constexpr int EPL = D / 32;
  const int C = G.chunk, R = G.nref;
  const int TT = nch * C;
  float* ks = smem;                       // [128][DP]
  float* qs = ks + kL1Tokens * DP;        // [R][DP]
  float* ss = qs + R * DP;                // [R][128]
  float* fs = ss + R * kL1Tokens;         // [R][nch]
  float2* rot = reinterpret_cast<float2*>(fs + R * 64);   // [nch][D/2] (cos, sin) of the chunk start
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  const int RP = G.rope_pairs;

  // Stage keys (16-byte vectors, coalesced) and reference queries. A key whose
  // page the block table does not hold reads as zeros and marks the tree.
  {
    constexpr int VEC = 16 / sizeof(T);
    const T* K = static_cast<const T*>(kv.k);
    const int nvec = TT * (D / VEC);
    bool bad = false;
    for (int v = tid; v < nvec; v += blockDim.x) {
      const int row = v / (D / VEC), col = (v % (D / VEC)) * VEC;
      const int64_t kr = kv_row(kv, g, c0 * C + row, C);
      float tmp[VEC];
      if (kr >= 0) {
        load_slice<VEC>(K + kr * D, col, tmp);
      } else {
        bad = true;
#pragma unroll
        for (int i = 0; i < VEC; ++i) tmp[i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < VEC; ++i) ks[row * DP + col + i] = tmp[i];
    }
    if (bad) atomicOr(tree_status_word(G, store), ZHA_DEV_BAD_PAGE);
    const float* qb = refq + int64_t(g) * R * D;
    for (int v = tid; v < R * (D / 4); v += blockDim.x) {
      const int row = v / (D / 4), col = (v % (D / 4)) * 4;
      *reinterpret_cast<float4*>(qs + row * DP + col) =
          *reinterpret_cast<const float4*>(qb + int64_t(row) * D + col);
    }
    for (int v = tid; v < nch * RP; v += blockDim.x) {
      const int cl = v / RP, i = v % RP;
      float c, s;
      rope_cos_sin(G, (c0 + cl) * C, i, &c, &s);
      rot[cl * (D / 2) + i] = make_float2(c, s);
    }
  }
  __syncthreads();
  // Rotary positions: the chunk's summaries at the reference queries turned to
  // the chunk's position equal the position-free summaries of the keys turned
  // back by that position (then khat is turned forward again, below).
  if (RP > 0) {
    for (int v = tid; v < TT * RP; v += blockDim.x) {
      const int t = v / RP, i = v % RP;
      const float2 cs = rot[(t / C) * (D / 2) + i];
      float* k2 = ks + t * DP + 2 * i;
      const float a = k2[0], b = k2[1];
      k2[0] = a * cs.x + b * cs.y;
      k2[1] = b * cs.x - a * cs.y;
    }
    __syncthreads();
  }

  // Scores: warp w takes plane pairs (2w, 2w+1), lane takes tokens lane + 32i.
  for (int rp = warp; 2 * rp < R; rp += nwarps) {
    const int r0 = 2 * rp, r1 = min(2 * rp + 1, R - 1);
    float acc[2][4] = {};
#pragma unroll 4
    for (int e = 0; e < D; e += 4) {
      const float4 qa = *reinterpret_cast<const float4*>(qs + r0 * DP + e);
      const float4 qb = *reinterpret_cast<const float4*>(qs + r1 * DP + e);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 k = *reinterpret_cast<const float4*>(ks + (lane + 32 * i) * DP + e);
        acc[0][i] += qa.x * k.x + qa.y * k.y + qa.z * k.z + qa.w * k.w;
        acc[1][i] += qb.x * k.x + qb.y * k.y + qb.z * k.z + qb.w * k.w;
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = lane + 32 * i;
      if (t < TT) {
        ss[r0 * kL1Tokens + t] = acc[0][i] * G.scale;
        if (2 * rp + 1 < R) ss[r1 * kL1Tokens + t] = acc[1][i] * G.scale;
      }
    }
  }
  __syncthreads();

  // Softmax per (chunk, plane): F = m + log(sum exp(S - m)); P = exp(S - F).
  for (int it = warp; it < nch * R; it += nwarps) {
    const int cl = it / R, r = it % R;
    float* srow = ss + r * kL1Tokens + cl * C;
    float m = -INFINITY;
    for (int j = lane; j < C; j += 32) m = fmaxf(m, srow[j]);
    m = warp_max(m);
    float l = 0.f;
    for (int j = lane; j < C; j += 32) l += expf(srow[j] - m);
    l = warp_sum(l);
    const float F = m + logf(l);
    __syncwarp();
    for (int j = lane; j < C; j += 32) srow[j] = expf(srow[j] - F);
    if (lane == 0) fs[r * nch + cl] = F;
  }
  __syncthreads();

  // khat[r] = sum_t P[r][t] k_t over the chunk; lane owns dims [EPL*lane, EPL*lane+EPL).
  for (int it = warp; it < nch * R; it += nwarps) {
    const int cl = it / R, r = it % R;
    const float* prow = ss + r * kL1Tokens + cl * C;
    float acc[EPL] = {};
    for (int j = 0; j < C; ++j) {
      const float pj = prow[j];
      const float* krow = ks + (cl * C + j) * DP + EPL * lane;
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[e] += pj * krow[e];
    }
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) dot += acc[e] * qs[r * DP + EPL * lane + e];
    dot = warp_sum(dot);
#pragma unroll
    for (int e = 0; e < EPL; e += 2) {            // khat back into the keys' frame
      const int i = (EPL * lane + e) / 2;
      if (i < RP) {
        const float2 cs = rot[cl * (D / 2) + i];
        const float a = acc[e], b = acc[e + 1];
        acc[e] = a * cs.x - b * cs.y;
        acc[e + 1] = a * cs.y + b * cs.x;
      }
    }
    float* rec = store + G.off[1] + (int64_t(g) * G.cap[1] + c0 + cl) * G.node_floats;
#pragma unroll
    for (int e = 0; e < EPL; ++e) rec[r * D + EPL * lane + e] = acc[e];
    if (lane == 0) rec[R * D + r] = fs[r * nch + cl] - dot * G.scale;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kBuildThreads)
build_level1_kernel(Geom G, KvView kv, int64_t c_begin, int64_t c_end,
                    const float* __restrict__ refq, float* __restrict__ store) {
  extern __shared__ float4 smem_v4[];
  const int cpt = l1_chunks_per_tile(G.chunk);
  const int64_t c0 = c_begin + int64_t(blockIdx.x) * cpt;
  if (c0 >= c_end) return;
  const int nch = int(min64(cpt, c_end - c0));
  summarise_tile<T, D>(G, blockIdx.y, kv, c0, nch, refq, store, reinterpret_cast<float*>(smem_v4));
}

// ---------------------------------------------------------------------------
// Upper levels. Item (parent P, plane r), one warp: for children c of P,
//   u_c = q_r . khat_{r,c} / sqrt(d) + bhat_{r,c}
//   F_P = LSE_c u_c;  khat_{r,P} = sum_c softmax(u)_c khat_{r,c}
//   bhat_{r,P} = F_P - q_r . khat_{r,P} / sqrt(d)
// accumulated with a running maximum over batches of 4 children so that four
// child rows are in flight per warp.
// ---------------------------------------------------------------------------
template <int D>
__device__ void merge_item(const Geom& G, int g, int level, int64_t parent, int r,
                           const float* __restrict__ refq, float* __restrict__ store) {
  constexpr int EPL = D / 32;
  const int lane = threadIdx.x & 31;
  const int C = G.chunk, R = G.nref;
  float q[EPL];
  load_slice<EPL>(refq + (int64_t(g) * R + r) * D, EPL * lane, q);
  // Rotary positions: the children are re-evaluated at the parent's rotated
  // reference query (its plane at that query: the tangent value at the child's
  // own rotated query plus the correction 1/sqrt(d) <khat_c, q_P - q_c>).
#pragma unroll
  for (int e = 0; e < EPL; e += 2) {
    const int i = (EPL * lane + e) / 2;
    if (i < G.rope_pairs) {
      float c, s;
      rope_cos_sin(G, parent * span_of(C, level), i, &c, &s);
      const float a = q[e], b = q[e + 1];
      q[e] = a * c - b * s;
      q[e + 1] = a * s + b * c;
    }
  }
  const float* child0 = store + G.off[level - 1] +
                        (int64_t(g) * G.cap[level - 1] + parent * C) * G.node_floats;
  float m = -INFINITY, l = 0.f, acc[EPL] = {};
  for (int c = 0; c < C; c += 4) {
    float kr[4][EPL], u[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (c + k < C) {
        const float* rec = child0 + int64_t(c + k) * G.node_floats;
        load_slice<EPL>(rec + r * D, EPL * lane, kr[k]);
        u[k] = rec[R * D + r];
      } else {
#pragma unroll
        for (int e = 0; e < EPL; ++e) kr[k][e] = 0.f;
        u[k] = 0.f;
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) dot += q[e] * kr[k][e];
      dot = warp_sum(dot);
      u[k] = (c + k < C) ? dot * G.scale + u[k] : -INFINITY;
    }
    const float mb = fmaxf(fmaxf(u[0], u[1]), fmaxf(u[2], u[3]));
    const float mn = fmaxf(m, mb);
    const float sc = expf(m - mn);   // m = -inf on the first batch gives 0
    l *= sc;
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] *= sc;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float w = expf(u[k] - mn);
      l += w;
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[e] += w * kr[k][e];
    }
    m = mn;
  }
  const float inv = 1.f / l;
  float dot = 0.f;
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    acc[e] *= inv;
    dot += acc[e] * q[e];
  }
  dot = warp_sum(dot);
  const float F = m + logf(l);
  float* out = store + G.off[level] + (int64_t(g) * G.cap[level] + parent) * G.node_floats;
#pragma unroll
  for (int e = 0; e < EPL; ++e) out[r * D + EPL * lane + e] = acc[e];
  if (lane == 0) out[R * D + r] = F - dot * G.scale;
}

template <int D>
__global__ void __launch_bounds__(kBuildThreads)
merge_level_kernel(Geom G, int level, int64_t parent0, int64_t n_parents,
                   const float* __restrict__ refq, float* __restrict__ store) {
  const int warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int64_t item = int64_t(blockIdx.x) * nwarps + warp;
  if (item >= n_parents * G.nref) return;
  merge_item<D>(G, blockIdx.y, level, parent0 + item / G.nref, int(item % G.nref), refq, store);
}

// ---------------------------------------------------------------------------
// Append: one CTA per KV head summarises the new chunks [c_begin, c_end), then
// merges the parents they complete, level by level (the CTA barrier orders the
// writes of one level before the reads of the next).
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(kBuildThreads)
append_kernel(Geom G, KvView kv, int64_t nb_old, int64_t nb_new, const float* __restrict__ refq,
              float* __restrict__ store) {
  extern __shared__ float4 smem_v4[];
  float* smem = reinterpret_cast<float*>(smem_v4);
  const int g = blockIdx.x;
  const int C = G.chunk;
  const int cpt = l1_chunks_per_tile(C);
  const int64_t c_begin = nb_old / C, c_end = nb_new / C;
  for (int64_t c0 = c_begin; c0 < c_end; c0 += cpt) {
    const int nch = int(min64(cpt, c_end - c0));
    summarise_tile<T, D>(G, g, kv, c0, nch, refq, store, smem);
    __syncthreads();
  }
  const int warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int level = 2; level <= G.levels; ++level) {
    const int64_t p_begin = nodes_at(nb_old, C, level), p_end = nodes_at(nb_new, C, level);
    const int64_t items = (p_end - p_begin) * G.nref;
    for (int64_t it = warp; it < items; it += nwarps)
      merge_item<D>(G, g, level, p_begin + it / G.nref, int(it % G.nref), refq, store);
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
// Summarise chunks [nb_old/C, nb_new/C) and merge the parents they complete:
// one level-1 launch and one launch per upper level that gains nodes.
template <typename T, int D>
static cudaError_t launch_build_t(const Geom& G, const KvView& kv, int64_t nb_old, int64_t nb_new,
                                  const float* refq, float* store, cudaStream_t s) {
  const size_t smem = l1_smem_bytes<D>(G.nref);
  cudaError_t e = ensure_dynamic_smem(build_level1_kernel<T, D>, smem);
  if (e != cudaSuccess) return e;
  const int64_t c_begin = nb_old / G.chunk, c_end = nb_new / G.chunk;
  // bf16, d = 128, R = 16, C = 64, contiguous cache: the tensor-core level 1 (zha_build_tc.cu).
  const cudaError_t etc =
      kv.table != nullptr
          ? cudaErrorNotSupported
          : launch_build_level1_tc(G, kv.k, kv.ld, c_begin, c_end, refq, store, tree_status_word(G, store), s);
  if (etc != cudaSuccess && etc != cudaErrorNotSupported) return etc;
  if (etc != cudaSuccess && c_end > c_begin) {
    const int cpt = l1_chunks_per_tile(G.chunk);
    dim3 grid(unsigned((c_end - c_begin + cpt - 1) / cpt), unsigned(G.hkv));
    {
      TraceScope ts("build_level1_kernel", 1, s);
      build_level1_kernel<T, D><<<grid, kBuildThreads, smem, s>>>(G, kv, c_begin, c_end, refq, store);
    }
    zha_count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  for (int level = 2; level <= G.levels; ++level) {
    const int64_t p_begin = nodes_at(nb_old, G.chunk, level);
    const int64_t p_end = nodes_at(nb_new, G.chunk, level);
    if (p_end <= p_begin) break;
    const int64_t items = (p_end - p_begin) * G.nref;
    const int per = kBuildThreads / 32;
    dim3 grid(unsigned((items + per - 1) / per), unsigned(G.hkv));
    if ((e = ensure_dynamic_smem(merge_level_kernel<D>, 0)) != cudaSuccess) return e;
    {
      TraceScope ts("merge_level_kernel", level, s);
      merge_level_kernel<D><<<grid, kBuildThreads, 0, s>>>(G, level, p_begin, p_end - p_begin,
                                                            refq, store);
    }
    zha_count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <typename T, int D>
static cudaError_t launch_append_t(const Geom& G, const KvView& kv, int64_t nb_old, int64_t nb_new,
                                   const float* refq, float* store, cudaStream_t s) {
  const size_t smem = l1_smem_bytes<D>(G.nref);
  cudaError_t e = ensure_dynamic_smem(append_kernel<T, D>, smem);
  if (e != cudaSuccess) return e;
  TraceScope ts("append_kernel", 0, s);
  append_kernel<T, D><<<G.hkv, kBuildThreads, smem, s>>>(G, kv, nb_old, nb_new, refq, store);
  zha_count_launch();
  return cudaGetLastError();
}

cudaError_t launch_build(const Geom& G, const KvView& kv, int64_t nb_old, int64_t nb_new,
                         const float* refq, float* store, cudaStream_t s) {
  cudaError_t e;
  if (G.kv_bf16)
    e = G.d == 128 ? launch_build_t<__nv_bfloat16, 128>(G, kv, nb_old, nb_new, refq, store, s)
                   : launch_build_t<__nv_bfloat16, 64>(G, kv, nb_old, nb_new, refq, store, s);
  else
    e = G.d == 128 ? launch_build_t<float, 128>(G, kv, nb_old, nb_new, refq, store, s)
                   : launch_build_t<float, 64>(G, kv, nb_old, nb_new, refq, store, s);
  return e == cudaSuccess ? launch_plane_terms(G, store, nb_old, nb_new, s) : e;
}

cudaError_t launch_append(const Geom& G, const KvView& kv, int64_t nb_old, int64_t nb_new,
                          const float* refq, float* store, cudaStream_t s) {
  cudaError_t e;
  if (G.kv_bf16)
    e = G.d == 128 ? launch_append_t<__nv_bfloat16, 128>(G, kv, nb_old, nb_new, refq, store, s)
                   : launch_append_t<__nv_bfloat16, 64>(G, kv, nb_old, nb_new, refq, store, s);
  else
    e = G.d == 128 ? launch_append_t<float, 128>(G, kv, nb_old, nb_new, refq, store, s)
                   : launch_append_t<float, 64>(G, kv, nb_old, nb_new, refq, store, s);
  return e == cudaSuccess ? launch_plane_terms(G, store, nb_old, nb_new, s) : e;
}

}  // namespace zha
