// zha_attend.cu -- exact softmax attention over the routed leaf tokens.
//
// Citations: [Attention: ...] = page "Attention"
// (zzong2006.github.io/machine_learning/nlp/attention-function):
//   "Scaled dot-product attention 의 식" -- o = softmax(q K^T / sqrt(d)) V;
//   "FlashAttention 계열" -- online softmax with running maximum m, sum l and
//   unnormalised output o rescaled by exp(m_old - m_new); Flash-Decoding's split
//   of the cache along its length, combined with the per-split max and sum.
// [ZHA: 전제와 한계] = page "ZHA는 KV 캐시를 트리로 요약해 어텐션 비용을
// 준(sub)이차로 낮춘다" (onedev.kr/papers/1556): token 0 (the attention sink) and
// the visible keys of the chunk in progress are always included.
//
// Split: the complete chunks of a KV head are cut into ranges of W chunks
// (W*C ~ 1024 tokens). attend_kernel runs one CTA per (range, KV head, block of
// up to 32 query heads of that KV head): it gathers the chunks any of those
// heads selected inside the range, streams them once through shared memory and
// updates a per-head online-softmax state for the heads that selected each
// chunk. One more CTA per (KV head, block) covers the tail [N_b, N) and the
// sink. The range states are merged by combine_ranges_kernel (below).
// This CUDA-core kernel serves fp32 caches and head_dim 64; bf16 caches with
// head_dim 128 go to the tensor-core kernels in zha_attend_tc.cu.
#include "zha_host.cuh"
#include "zha_internal.cuh"

namespace zha {

constexpr int kAttThreads = 256;
constexpr int kAttQ = 32;       // query heads per CTA
constexpr int kAttT = 64;       // tokens per tile

cudaError_t launch_combine(const Geom& G, int32_t batch, const int32_t* chunk_ids,
                           const int32_t* n_chunks, int32_t max_sel, float* O, float* lse,
                           const float* partial, const AttendLayout& lay, int32_t* status,
                           cudaStream_t s);


template <int D>
__host__ __device__ inline size_t attend_smem_bytes(int range_chunks) {
  constexpr int DP = D + 4;
  return sizeof(float) * (size_t(kAttQ) * DP + 2 * size_t(kAttT) * DP + size_t(kAttQ) * (kAttT + 1)) +
         sizeof(uint32_t) * 2 * size_t(range_chunks) + 16;
}

__device__ __forceinline__ int lower_bound_i32(const int32_t* a, int n, int64_t x) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (int64_t(a[mid]) < x) lo = mid + 1; else hi = mid;
  }
  return lo;
}

template <typename T, int D>
__global__ void __launch_bounds__(kAttThreads)
attend_kernel(Geom G, int32_t batch, int64_t n_tokens, int64_t nb, const float* __restrict__ Q,
              KvView kv, const int32_t* __restrict__ chunk_ids, const int32_t* __restrict__ n_chunks,
              int32_t max_sel, int32_t range_chunks, int64_t n_ranges,
              float* __restrict__ partial, int64_t slots_per_head, int32_t* status) {
  const T* __restrict__ K = static_cast<const T*>(kv.k);
  const T* __restrict__ V = static_cast<const T*>(kv.v);
  constexpr int DP = D + 4;
  constexpr int VEC = 16 / sizeof(T);
  constexpr int NV = D / 32;            // float4 groups per thread in the output update
  extern __shared__ float4 smem_v4[];
  float* s_q = reinterpret_cast<float*>(smem_v4);          // [32][DP]
  float* s_k = s_q + kAttQ * DP;                           // [64][DP]
  float* s_v = s_k + kAttT * DP;                           // [64][DP]
  float* s_p = s_v + kAttT * DP;                           // [32][65]
  uint32_t* s_mask = reinterpret_cast<uint32_t*>(s_p + kAttQ * (kAttT + 1));  // [W]
  uint32_t* s_sel = s_mask + range_chunks;                 // [W]
  __shared__ uint32_t s_tmask[kAttT];
  __shared__ int64_t s_tok[kAttT];
  __shared__ float s_m[kAttQ], s_l[kAttQ], s_scale[kAttQ];
  __shared__ uint32_t s_any, s_nsel, s_mask0, s_w[33];

  const int g = blockIdx.y;
  const int64_t rho = blockIdx.x;
  const bool tail = rho == n_ranges;
  const int GQ = G.group;
  const int qn_total = batch * GQ;
  const int qb0 = blockIdx.z * kAttQ;
  const int nq = min(kAttQ, qn_total - qb0);
  const int C = G.chunk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t c_lo = rho * range_chunks;
  const int64_t c_hi = min64(c_lo + range_chunks, nb / C);

  if (tid == 0) { s_any = 0u; s_mask0 = 0u; }
  for (int i = tid; i < range_chunks; i += blockDim.x) s_mask[i] = 0u;
  __syncthreads();

  // Which chunks of this range each query head selected.
  if (tid < nq) {
    const int qi = qb0 + tid;
    const int64_t bh = int64_t(qi / GQ) * G.hq + g * GQ + qi % GQ;
    const int32_t* list = chunk_ids + bh * max_sel;
    const int n = min(n_chunks[bh], max_sel);
    if (!tail) {
      const int lo = lower_bound_i32(list, n, c_lo), hi = lower_bound_i32(list, n, c_hi);
      bool any = false;
      for (int i = lo; i < hi; ++i) {
        const int64_t c = list[i];
        if (c >= c_lo && c < c_hi) { atomicOr(&s_mask[c - c_lo], 1u << tid); any = true; }
      }
      if (any) atomicOr(&s_any, 1u << tid);
    } else {
      const bool has0 = n > 0 && list[0] == 0;
      if (nb > 0 && !has0) atomicOr(&s_mask0, 1u << tid);
    }
  }
  __syncthreads();
  const uint32_t all_q = nq == 32 ? 0xffffffffu : ((1u << nq) - 1u);
  const uint32_t active = tail ? all_q : s_any;
  if (active == 0u) return;

  // Ordered list of the selected chunks of the range (tail: none).
  int64_t n_tok;
  if (!tail) {
    uint32_t base = 0;
    for (int i0 = 0; i0 < range_chunks; i0 += blockDim.x) {
      const int i = i0 + tid;
      const uint32_t f = (i < range_chunks && s_mask[i] != 0u) ? 1u : 0u;
      // block exclusive scan of f
      uint32_t v = f;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t nv = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += nv;
      }
      if (lane == 31) s_w[warp] = v;
      __syncthreads();
      if (warp == 0) {
        const uint32_t w = lane < (blockDim.x >> 5) ? s_w[lane] : 0u;
        uint32_t wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t nv = __shfl_up_sync(0xffffffffu, wi, o);
          if (lane >= o) wi += nv;
        }
        if (lane < (blockDim.x >> 5)) s_w[lane] = wi - w;
        if (lane == 31) s_w[32] = wi;
      }
      __syncthreads();
      if (f) s_sel[base + s_w[warp] + v - f] = uint32_t(i);
      base += s_w[32];
      __syncthreads();
    }
    if (tid == 0) s_nsel = base;
    __syncthreads();
    n_tok = int64_t(s_nsel) * C;
  } else {
    n_tok = (n_tokens - nb) + (s_mask0 != 0u ? 1 : 0);
  }

  // Query block and running state.
  for (int v = tid; v < kAttQ * (D / 4); v += blockDim.x) {
    const int q = v / (D / 4), col = (v % (D / 4)) * 4;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (q < nq) {
      const int qi = qb0 + q;
      const int64_t bh = int64_t(qi / GQ) * G.hq + g * GQ + qi % GQ;
      x = *reinterpret_cast<const float4*>(Q + bh * D + col);
    }
    *reinterpret_cast<float4*>(s_q + q * DP + col) = x;
  }
  if (tid < kAttQ) { s_m[tid] = -INFINITY; s_l[tid] = 0.f; }
  const int qo = tid >> 3, l8 = tid & 7;     // output update: query qo, dims l8*4 + 32k
  float acc[NV][4] = {};
  __syncthreads();

  for (int64_t t0 = 0; t0 < n_tok; t0 += kAttT) {
    const int nt = int(min64(kAttT, n_tok - t0));
    if (tid < kAttT) {
      int64_t tok = 0;
      uint32_t msk = 0u;
      if (tid < nt) {
        const int64_t u = t0 + tid;
        if (!tail) {
          const uint32_t k = s_sel[u / C];
          tok = (c_lo + k) * C + u % C;
          msk = s_mask[k];
        } else if (u < n_tokens - nb) {
          tok = nb + u;
          msk = all_q;
        } else {
          tok = 0;
          msk = s_mask0;
        }
      }
      if (tid < nt && kv.table != nullptr && kv_row(kv, g, tok, C) < 0) {
        msk = 0u;                     // page outside the pool: not read, not attended
        if (status != nullptr) atomicOr(status, ZHA_DEV_BAD_PAGE);
      }
      s_tok[tid] = tok;
      s_tmask[tid] = msk;
    }
    __syncthreads();
    // Stage K and V rows of the tile (16-byte vectors); a token on a page the
    // block table does not hold reads as zeros and no head attends it.
    for (int v = tid; v < kAttT * (D / VEC); v += blockDim.x) {
      const int row = v / (D / VEC), col = (v % (D / VEC)) * VEC;
      float kt[VEC], vt[VEC];
      const int64_t kr = row < nt ? kv_row(kv, g, s_tok[row], C) : -1;
      if (kr >= 0) {
        const int64_t off = kr * D;
        load_slice<VEC>(K + off, col, kt);
        load_slice<VEC>(V + off, col, vt);
      } else {
#pragma unroll
        for (int i = 0; i < VEC; ++i) { kt[i] = 0.f; vt[i] = 0.f; }
      }
#pragma unroll
      for (int i = 0; i < VEC; ++i) {
        s_k[row * DP + col + i] = kt[i];
        s_v[row * DP + col + i] = vt[i];
      }
    }
    __syncthreads();
    // Scores: thread takes queries (2*qg, 2*qg+1) and tokens jg + 16 i.
    {
      const int qg = tid >> 4, jg = tid & 15;
      float sacc[2][4] = {};
#pragma unroll 4
      for (int e = 0; e < D; e += 4) {
        const float4 qa = *reinterpret_cast<const float4*>(s_q + (2 * qg) * DP + e);
        const float4 qb = *reinterpret_cast<const float4*>(s_q + (2 * qg + 1) * DP + e);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 k = *reinterpret_cast<const float4*>(s_k + (jg + 16 * i) * DP + e);
          sacc[0][i] += qa.x * k.x + qa.y * k.y + qa.z * k.z + qa.w * k.w;
          sacc[1][i] += qb.x * k.x + qb.y * k.y + qb.z * k.z + qb.w * k.w;
        }
      }
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        const int q = 2 * qg + a;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int j = jg + 16 * i;
          const bool on = (s_tmask[j] >> q) & 1u;
          s_p[q * (kAttT + 1) + j] = on ? sacc[a][i] * G.scale : -INFINITY;
        }
      }
    }
    __syncthreads();
    // Online softmax per query row (warp w: queries 4w .. 4w+3).
    for (int q = 4 * warp; q < 4 * warp + 4; ++q) {
      float* row = s_p + q * (kAttT + 1);
      const float a0 = row[lane], a1 = row[lane + 32];
      const float mt = warp_max(fmaxf(a0, a1));
      const float m_old = s_m[q];
      const float m_new = fmaxf(m_old, mt);
      float p0 = 0.f, p1 = 0.f, sc = 1.f;
      if (m_new != -INFINITY) {
        sc = expf(m_old - m_new);
        p0 = expf(a0 - m_new);
        p1 = expf(a1 - m_new);
      }
      const float ps = warp_sum(p0 + p1);
      row[lane] = p0;
      row[lane + 32] = p1;
      if (lane == 0) {
        s_scale[q] = sc;
        s_m[q] = m_new;
        s_l[q] = s_l[q] * sc + ps;
      }
    }
    __syncthreads();
    // o = o * scale + P V
    {
      const float sc = s_scale[qo];
#pragma unroll
      for (int k = 0; k < NV; ++k)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[k][c] *= sc;
      const float* prow = s_p + qo * (kAttT + 1);
      for (int j = 0; j < nt; ++j) {
        const float pj = prow[j];
#pragma unroll
        for (int k = 0; k < NV; ++k) {
          const float4 v = *reinterpret_cast<const float4*>(s_v + j * DP + 4 * l8 + 32 * k);
          acc[k][0] += pj * v.x; acc[k][1] += pj * v.y; acc[k][2] += pj * v.z; acc[k][3] += pj * v.w;
        }
      }
    }
    __syncthreads();
  }

  // Partial state of each active query head: [m, l, 0, 0, o[D]].
  if (qo < nq && ((active >> qo) & 1u)) {
    const int qi = qb0 + qo;
    const int64_t bh = int64_t(qi / GQ) * G.hq + g * GQ + qi % GQ;
    float* slot = partial + (bh * slots_per_head + rho) * (D + 4);
    if (l8 == 0) {
      *reinterpret_cast<float4*>(slot) = make_float4(s_m[qo], s_l[qo], 0.f, 0.f);
    }
#pragma unroll
    for (int k = 0; k < NV; ++k)
      *reinterpret_cast<float4*>(slot + 4 + 4 * l8 + 32 * k) =
          make_float4(acc[k][0], acc[k][1], acc[k][2], acc[k][3]);
  }
}

template <typename T, int D>
static cudaError_t launch_attend_t(const Geom& G, const float* Q, const KvView& kv, int64_t n_tokens,
                                   int32_t batch, const int32_t* chunk_ids, const int32_t* n_chunks,
                                   int32_t max_sel, float* O, float* lse, float* partial,
                                   const AttendLayout& lay, int32_t* status, cudaStream_t s) {
  const size_t smem = attend_smem_bytes<D>(lay.range_chunks);
  cudaError_t e = ensure_dynamic_smem(attend_kernel<T, D>, smem);
  if (e != cudaSuccess) return e;
  const int64_t nb = int64_t(G.chunk) * (n_tokens / G.chunk);
  const int qn = batch * G.group;
  dim3 grid(unsigned(lay.n_ranges + 1), unsigned(G.hkv), unsigned((qn + kAttQ - 1) / kAttQ));
  {
    TraceScope ts("attend_kernel", 0, s);
    attend_kernel<T, D><<<grid, kAttThreads, smem, s>>>(G, batch, n_tokens, nb, Q, kv, chunk_ids, n_chunks,
                                                        max_sel, lay.range_chunks, lay.n_ranges, partial,
                                                        lay.slots_per_head, status);
  }
  zha_count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return launch_combine(G, batch, chunk_ids, n_chunks, max_sel, O, lse, partial, lay, status, s);
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
  cudaError_t e = G.d == 128 ? ensure_dynamic_smem(combine_ranges_kernel<128>, 0)
                             : ensure_dynamic_smem(combine_ranges_kernel<64>, 0);
  if (e != cudaSuccess) return e;
  TraceScope ts("combine_ranges_kernel", 0, s);
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

cudaError_t launch_attend(const Geom& G, const float* Q, const KvView& kv, int64_t n_tokens,
                          int32_t batch, const int32_t* chunk_ids, const int32_t* n_chunks,
                          int32_t max_sel, float* O, float* lse, float* partial,
                          const AttendLayout& lay, int32_t* status, cudaStream_t s) {
  if (G.kv_bf16)
    return G.d == 128 ? launch_attend_t<__nv_bfloat16, 128>(G, Q, kv, n_tokens, batch, chunk_ids, n_chunks,
                                                            max_sel, O, lse, partial, lay, status, s)
                      : launch_attend_t<__nv_bfloat16, 64>(G, Q, kv, n_tokens, batch, chunk_ids, n_chunks,
                                                           max_sel, O, lse, partial, lay, status, s);
  return G.d == 128 ? launch_attend_t<float, 128>(G, Q, kv, n_tokens, batch, chunk_ids, n_chunks, max_sel,
                                                  O, lse, partial, lay, status, s)
                    : launch_attend_t<float, 64>(G, Q, kv, n_tokens, batch, chunk_ids, n_chunks, max_sel,
                                                 O, lse, partial, lay, status, s);
}

}  // namespace zha
