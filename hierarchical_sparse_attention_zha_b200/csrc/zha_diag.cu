// zha_diag.cu -- routing diagnostics: how well each level's estimate follows
// the dense attention mass, and which reference queries give the scores.
//
// Citations: [ZHA: 어떻게 쓰나] = page "ZHA는 KV 캐시를 트리로 요약해 어텐션 비용을
// 준(sub)이차로 낮춘다" (onedev.kr/papers/1556), section "어떻게 쓰나": the reference
// queries are trained by minimising, at every level, the KL divergence between
// the target p_{l,C}(q) -- the dense attention weights summed chunk by chunk --
// and the estimate p_hat_{l,C}(q); section "전제와 한계": few reference queries
// serve the upper levels, their use evens out towards the leaves.
//
// Three launches:
//  1. diag_chunk_mass_kernel: F_i(q) = LSE_{j in chunk i} q.k_j / sqrt(d) for
//     every complete level-1 chunk and query head: a register-tiled fp32
//     product of a tile of keys (floor(128 / C) chunks of one KV head) with the
//     group's queries, then a log-sum-exp per (chunk, head).
//  2. score_dense_kernel (zha_dense.cuh) over every level: sigma of every node
//     for every head, with the argmax plane counted per level.
//  3. diag_kl_kernel, one CTA per query head: per level, the target's log
//     masses F_n = LSE of the level-1 masses under node n, then
//     KL = sum_n p_n (log p_n - log p_hat_n) with p = softmax(F), p_hat =
//     softmax(sigma) over the level's nodes.
#include <cmath>
#include <cstdio>

#include "zha_dense.cuh"
#include "zha_host.cuh"
#include "zha_internal.cuh"

namespace zha {

namespace {

constexpr int kMassTok = 128;        // keys per tile (at most)
constexpr int kMassQ = 32;           // query heads per CTA
constexpr int kMassThreads = 256;
constexpr int kKlThreads = 512;

template <int D>
constexpr size_t mass_smem_bytes() {
  return size_t(kMassTok + kMassQ) * D * sizeof(float);
}

// Workspace: level-1 masses [B*Hq][n_1] then the route layout's scores.
struct DiagLayout {
  RouteLayout lay;
  int64_t mass_off, sig_off, bytes;
};

DiagLayout diag_layout(const Geom& G, int32_t batch, int64_t n_tokens) {
  DiagLayout d{};
  d.lay = route_layout(G, batch, n_tokens);
  const int64_t heads = int64_t(batch) * G.hq;
  d.mass_off = 0;
  d.sig_off = round_up(heads * (d.lay.n[1] > 0 ? d.lay.n[1] : 1) * 4, 256);
  d.bytes = d.sig_off + round_up(d.lay.sig_floats * 4, 256);
  return d;
}

}  // namespace

template <typename T, int D>
__global__ void __launch_bounds__(kMassThreads)
diag_chunk_mass_kernel(Geom G, int32_t batch, int64_t n_chunks, const float* __restrict__ Q,
                       const T* __restrict__ K, int64_t ld, float* __restrict__ mass) {
  extern __shared__ float4 smem_v4[];
  float4* As = smem_v4;                               // [D / 4][kMassTok] keys
  float4* Bs = smem_v4 + (D / 4) * kMassTok;          // [D / 4][kMassQ] queries
  float* Cs = reinterpret_cast<float*>(smem_v4);      // [kMassTok][kMassQ + 1] after the product
  pdl_trigger();
  pdl_wait();
  const int C = G.chunk, cpt = kMassTok / C;
  const int g = blockIdx.y, qb = blockIdx.z;
  const int64_t c0 = int64_t(blockIdx.x) * cpt;
  const int nch = int(min64(cpt, n_chunks - c0));
  const int qn = min(kMassQ, batch * G.group - qb * kMassQ);
  const int tid = threadIdx.x;
  auto head_of = [&](int q) -> int64_t {
    const int qi = qb * kMassQ + q;
    return int64_t(qi / G.group) * G.hq + g * G.group + qi % G.group;
  };
  const T* kbase = K + (int64_t(g) * ld + c0 * C) * D;
  for (int v = tid; v < kMassTok * (D / 4); v += kMassThreads) {
    const int t = v / (D / 4), kb = v % (D / 4);
    float x[4] = {0.f, 0.f, 0.f, 0.f};
    if (t < nch * C) load_slice<4>(kbase + int64_t(t) * D, 4 * kb, x);
    As[kb * kMassTok + t] = make_float4(x[0], x[1], x[2], x[3]);
  }
  for (int v = tid; v < kMassQ * (D / 4); v += kMassThreads) {
    const int q = v / (D / 4), kb = v % (D / 4);
    Bs[kb * kMassQ + q] = q < qn ? *reinterpret_cast<const float4*>(Q + head_of(q) * D + 4 * kb)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  __syncthreads();
  // thread: keys ty + 16 i (i < 8), queries tx and tx + 16
  const int tx = tid & 15, ty = tid >> 4;
  float acc[8][2] = {};
#pragma unroll 2
  for (int kb = 0; kb < D / 4; ++kb) {
    float4 b[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) b[j] = Bs[kb * kMassQ + tx + 16 * j];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 a = As[kb * kMassTok + ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 2; ++j) acc[i][j] += a.x * b[j].x + a.y * b[j].y + a.z * b[j].z + a.w * b[j].w;
    }
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 2; ++j) Cs[(ty + 16 * i) * (kMassQ + 1) + tx + 16 * j] = acc[i][j] * G.scale;
  __syncthreads();
  for (int o = tid; o < nch * kMassQ; o += kMassThreads) {
    const int cl = o / kMassQ, q = o % kMassQ;
    if (q >= qn) continue;
    float m = -INFINITY;
    for (int j = 0; j < C; ++j) m = fmaxf(m, Cs[(cl * C + j) * (kMassQ + 1) + q]);
    float l = 0.f;
    for (int j = 0; j < C; ++j) l += expf(Cs[(cl * C + j) * (kMassQ + 1) + q] - m);
    mass[head_of(q) * n_chunks + c0 + cl] = m + logf(l);
  }
}

__device__ float kl_block_max(float v, float* tmp) {
  v = warp_max(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) tmp[warp] = v;
  __syncthreads();
  if (warp == 0) {
    float w = lane < int(blockDim.x >> 5) ? tmp[lane] : -INFINITY;
    w = warp_max(w);
    if (lane == 0) tmp[32] = w;
  }
  __syncthreads();
  const float r = tmp[32];
  __syncthreads();
  return r;
}

__device__ float kl_block_sum(float v, float* tmp) {
  v = warp_sum(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) tmp[warp] = v;
  __syncthreads();
  if (warp == 0) {
    float w = lane < int(blockDim.x >> 5) ? tmp[lane] : 0.f;
    w = warp_sum(w);
    if (lane == 0) tmp[32] = w;
  }
  __syncthreads();
  const float r = tmp[32];
  __syncthreads();
  return r;
}

struct KlLevels {
  int32_t levels;
  int64_t n[ZHA_MAX_LEVELS + 2];
  int64_t span[ZHA_MAX_LEVELS + 2];      // level-1 chunks under one node
  const float* sigma[ZHA_MAX_LEVELS + 2];
};

__global__ void __launch_bounds__(kKlThreads)
diag_kl_kernel(KlLevels kl, int64_t n1, const float* __restrict__ mass, float* __restrict__ out,
               int64_t heads) {
  __shared__ float tmp[33];
  pdl_trigger();
  pdl_wait();
  const int64_t bh = blockIdx.x;
  const int tid = threadIdx.x;
  const float* m1 = mass + bh * n1;
  for (int l = 1; l <= kl.levels; ++l) {
    const int64_t n = kl.n[l], span = kl.span[l];
    const float* sg = kl.sigma[l] + bh * n;
    // F_n: log-sum-exp of the level-1 masses under node n
    auto F_of = [&](int64_t i) -> float {
      const float* p = m1 + i * span;
      float m = -INFINITY;
      for (int64_t c = 0; c < span; ++c) m = fmaxf(m, p[c]);
      float s = 0.f;
      for (int64_t c = 0; c < span; ++c) s += expf(p[c] - m);
      return m + logf(s);
    };
    float mf = -INFINITY, ms = -INFINITY;
    for (int64_t i = tid; i < n; i += kKlThreads) {
      mf = fmaxf(mf, F_of(i));
      ms = fmaxf(ms, sg[i]);
    }
    mf = kl_block_max(mf, tmp);
    ms = kl_block_max(ms, tmp);
    float zf = 0.f, zs = 0.f;
    for (int64_t i = tid; i < n; i += kKlThreads) {
      zf += expf(F_of(i) - mf);
      zs += expf(sg[i] - ms);
    }
    zf = kl_block_sum(zf, tmp);
    zs = kl_block_sum(zs, tmp);
    const float lf = mf + logf(zf), ls = ms + logf(zs);
    float acc = 0.f;
    for (int64_t i = tid; i < n; i += kKlThreads) {
      const float lp = F_of(i) - lf;
      acc += expf(lp) * (lp - (sg[i] - ls));
    }
    acc = kl_block_sum(acc, tmp);
    if (tid == 0) out[int64_t(l - 1) * heads + bh] = n > 0 ? acc : 0.f;
  }
}

template <typename T, int D>
static cudaError_t launch_mass_t(const Geom& G, int32_t batch, int64_t n_chunks, const float* Q,
                                 const void* K, int64_t ld, float* mass, cudaStream_t s) {
  const int cpt = kMassTok / G.chunk;
  const int qn = batch * G.group;
  dim3 grid(unsigned((n_chunks + cpt - 1) / cpt), unsigned(G.hkv), unsigned((qn + kMassQ - 1) / kMassQ));
  const size_t smem = mass_smem_bytes<D>();
  cudaError_t e = ensure_dynamic_smem(diag_chunk_mass_kernel<T, D>, smem);
  if (e != cudaSuccess) return e;
  TraceScope ts("diag_chunk_mass_kernel", 1, s);
  e = launch_pdl(diag_chunk_mass_kernel<T, D>, grid, dim3(kMassThreads), smem, s, G, batch, n_chunks, Q,
                 static_cast<const T*>(K), ld, mass);
  zha_count_launch();
  return e;
}

template <int D>
static cudaError_t launch_usage_t(const Geom& G, const DenseLevels& dl, int32_t batch, const float* Q,
                                  const float* store, uint32_t* usage, cudaStream_t s) {
  const int qn = batch * G.group;
  dim3 grid(unsigned(dl.tile0[dl.count]), unsigned(G.hkv), unsigned((qn + kDenseQ - 1) / kDenseQ));
  const size_t smem = dense_smem_bytes<D>();
  cudaError_t e = usage ? ensure_dynamic_smem(score_dense_kernel<D, true>, smem)
                        : ensure_dynamic_smem(score_dense_kernel<D, false>, smem);
  if (e != cudaSuccess) return e;
  TraceScope ts("score_dense_kernel", 0, s);
  e = usage ? launch_pdl(score_dense_kernel<D, true>, grid, dim3(kDenseThreads), smem, s, G, dl, batch, Q,
                         store, usage)
            : launch_pdl(score_dense_kernel<D, false>, grid, dim3(kDenseThreads), smem, s, G, dl, batch,
                         Q, store, usage);
  zha_count_launch();
  return e;
}

}  // namespace zha

extern "C" {

size_t zha_diagnostics_workspace_bytes(const zha_config* cfg, int32_t batch, int64_t n_tokens) {
  if (zha_tree_bytes(cfg) == 0 || batch < 1 || n_tokens < 0) return 0;   // validates cfg
  zha::Geom G{};                   // the layout needs only these fields
  G.hkv = cfg->n_kv_heads;
  G.hq = cfg->n_q_heads;
  G.chunk = cfg->chunk;
  G.levels = cfg->levels;
  return size_t(zha::diag_layout(G, batch, n_tokens).bytes);
}

zha_status zha_route_diagnostics(const zha_tree* tree, const float* d_Q, const void* d_K, int64_t ld,
                                 int32_t batch, int64_t n_tokens, float* d_kl, uint32_t* d_usage,
                                 void* d_ws, size_t ws_bytes, void* stream) {
  if (tree == nullptr) return zha_report_error(ZHA_ERR_INVALID, "zha_route_diagnostics: tree is NULL");
  const zha::Geom& G = tree->geom;
  const uintptr_t a16 = 15;
  if (d_Q == nullptr || d_K == nullptr || d_kl == nullptr || (reinterpret_cast<uintptr_t>(d_Q) & a16) ||
      (reinterpret_cast<uintptr_t>(d_K) & a16) || (d_usage && (reinterpret_cast<uintptr_t>(d_usage) & 3)))
    return zha_report_error(ZHA_ERR_INVALID,
                            "zha_route_diagnostics: Q, K, kl must be non-NULL 16-byte aligned device pointers");
  if (batch < 1 || batch > 65535)
    return zha_report_error(ZHA_ERR_INVALID, "zha_route_diagnostics: batch must be 1..65535");
  if (n_tokens < 1 || n_tokens > G.max_tokens || n_tokens > ld)
    return zha_report_error(ZHA_ERR_INVALID, "zha_route_diagnostics: need 1 <= n_tokens <= min(ld, max_tokens)");
  const int64_t nb = int64_t(G.chunk) * (n_tokens / G.chunk);
  if (nb != tree->nb)
    return zha_report_error(ZHA_ERR_STATE, "zha_route_diagnostics: the tree's built prefix does not match n_tokens");
  const zha::DiagLayout dg = zha::diag_layout(G, batch, n_tokens);
  if (d_ws == nullptr || (reinterpret_cast<uintptr_t>(d_ws) & 255) || int64_t(ws_bytes) < dg.bytes)
    return zha_report_error(ZHA_ERR_CAPACITY, "zha_route_diagnostics: workspace too small or not 256-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(d_ws);
  float* mass = reinterpret_cast<float*>(ws + dg.mass_off);
  float* sigma = reinterpret_cast<float*>(ws + dg.sig_off);
  const int64_t n1 = dg.lay.n[1];
  cudaError_t e = cudaSuccess;
  if (n1 > 0) {
    e = G.kv_bf16 ? (G.d == 128 ? zha::launch_mass_t<__nv_bfloat16, 128>(G, batch, n1, d_Q, d_K, ld, mass, s)
                                : zha::launch_mass_t<__nv_bfloat16, 64>(G, batch, n1, d_Q, d_K, ld, mass, s))
                  : (G.d == 128 ? zha::launch_mass_t<float, 128>(G, batch, n1, d_Q, d_K, ld, mass, s)
                                : zha::launch_mass_t<float, 64>(G, batch, n1, d_Q, d_K, ld, mass, s));
    if (e != cudaSuccess) goto fail;
    zha::DenseLevels dl{};
    int64_t t0 = 0;
    const int npt = zha::kDenseRows / G.nref;
    for (int l = 1; l <= G.levels; ++l) {
      if (dg.lay.n[l] == 0) continue;
      const int i = dl.count++;
      dl.level[i] = l;
      dl.n_nodes[i] = dg.lay.n[l];
      dl.tile0[i] = t0;
      dl.sigma[i] = sigma + dg.lay.sig_off[l];
      t0 += (dg.lay.n[l] + npt - 1) / npt;
    }
    dl.tile0[dl.count] = t0;
    e = G.d == 128 ? zha::launch_usage_t<128>(G, dl, batch, d_Q, tree->store, d_usage, s)
                   : zha::launch_usage_t<64>(G, dl, batch, d_Q, tree->store, d_usage, s);
    if (e != cudaSuccess) goto fail;
  }
  {
    zha::KlLevels kl{};
    kl.levels = G.levels;
    for (int l = 1; l <= G.levels; ++l) {
      kl.n[l] = dg.lay.n[l];
      kl.span[l] = zha::span_of(G.chunk, l - 1);
      kl.sigma[l] = sigma + dg.lay.sig_off[l];
    }
    const int64_t heads = int64_t(batch) * G.hq;
    if ((e = zha::ensure_dynamic_smem(zha::diag_kl_kernel, 0)) != cudaSuccess) goto fail;
    {
      zha::TraceScope ts("diag_kl_kernel", 0, s);
      e = zha::launch_pdl(zha::diag_kl_kernel, dim3(unsigned(heads)), dim3(zha::kKlThreads), 0, s, kl,
                          n1 > 0 ? n1 : 1, mass, d_kl, heads);
    }
    zha_count_launch();
    if (e != cudaSuccess) goto fail;
  }
  return ZHA_OK;
fail : {
  char msg[256];
  snprintf(msg, sizeof msg, "zha_route_diagnostics: %s", cudaGetErrorString(e));
  return zha_report_error(ZHA_ERR_CUDA, msg);
}
}

}  // extern "C"
