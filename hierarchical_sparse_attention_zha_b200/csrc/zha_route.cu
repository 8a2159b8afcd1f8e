// zha_route.cu -- per-level top-p routing of decode queries through the trees.
//
// Citations: [ZHA: 무엇과 다른가 / 전제와 한계] = page "ZHA는 KV 캐시를 트리로 요약해
// 어텐션 비용을 준(sub)이차로 낮춘다" (onedev.kr/papers/1556): a node's log mass for
// a future query is estimated by the maximum of its R tangent planes (무엇과 다른가);
// routing runs top-p per level -- sort the candidates by score, keep the minimal
// prefix holding estimated mass p, pass the kept nodes' children and the
// parentless chunks down (전제와 한계).
//
// Per level l = L..1 the host launches two kernels:
//   scoring -- head_dim 128 with R = 16: score_tma_kernel (zha_score_tma.cu,
//              tensor copies + tcgen05); head_dim 128 with R < 16:
//              score_tc_kernel (zha_score_tc.cu); otherwise score_kernel here
//              (one warp per candidate node -- the union over the query heads of
//              a KV head -- its R planes in registers, one score per query head
//              that has the node as candidate);
//   selection -- one CTA per query head: softmax over its candidates, the cut
//              on the key (score desc, node index asc) by fixed-point mass, kept
//              bitmap (and at level 1 the ascending chunk list).
//              select_fast_kernel when the level fits in shared memory
//              (<= 16384 nodes), select_kernel otherwise.
// Both kinds are launched with programmatic dependent launch.
#include "zha_host.cuh"
#include "zha_internal.cuh"

namespace zha {

constexpr int kScoreThreads = 256;
constexpr int kScoreTile = 64;       // nodes per score CTA
constexpr int kScoreQBlock = 64;     // query heads per score CTA (u64 masks)
constexpr int kSelectThreads = 512;
constexpr int kSelectCache = 16384;  // candidate scores cached in shared memory
constexpr int kSelectKpCache = 4096;  // kept parents held in shared memory
constexpr double kMassScale = 1099511627776.0;  // 2^40: fixed-point unit of probability

// ---------------------------------------------------------------------------
// Scoring. A candidate of level l for query head (b, h) of KV head g is a node n
// with n >= C * n_{l+1} (an orphan; every node at the top level) or whose parent
// n / C is kept by (b, h) at level l+1. sigma = max_r (q . khat_r / sqrt(d) + bhat_r).
// ---------------------------------------------------------------------------

// Lane L of a warp holds part (L % P) of plane r = L / P of a node, P = 32 / RP
// lanes per plane (RP = R rounded up to a power of two): EP = D / P
// consecutive elements of khat_r. A query's score is then EP FMAs per lane,
// log2(P) shuffles to finish each plane's dot product and log2(RP) shuffles for
// the maximum over planes. Node records reach shared memory by coalesced
// cp.async into a per-warp buffer whose rows and parts are padded so that the
// lanes' reads in this mapping fall into distinct banks; each warp requests
// its next node before it scores the current one.
template <int D, int RP>
struct ScoreShape {
  static constexpr int P = 32 / RP;
  static constexpr int EP = D / P;
  static constexpr int QS = EP + 4;          // padded stride of one query part in shared memory
  static constexpr int QROW = P * QS;        // floats per staged query
  static constexpr int KROW = P * QS;        // floats per staged plane
  static constexpr int KBUF = RP * KROW;     // floats per staged node (planes only)
  static_assert(EP % 4 == 0, "each lane must hold whole float4s of its plane");
};

__device__ __forceinline__ void cp_async16_ca(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" : : "r"(dst), "l"(src) : "memory");
}

template <int D, int RP>
__global__ void __launch_bounds__(kScoreThreads)
score_kernel(Geom G, int level, int64_t n_nodes, int64_t n_par, int32_t batch, int tile,
             const float* __restrict__ Q, const uint32_t* __restrict__ kept_up, int64_t words_up,
             float* __restrict__ sigma, const float* __restrict__ store) {
  using S = ScoreShape<D, RP>;
  constexpr int NW = kScoreThreads / 32;
  extern __shared__ float4 smem_v4[];
  float* s_kbuf = reinterpret_cast<float*>(smem_v4);       // [NW][KBUF]
  pdl_trigger();
  pdl_wait();
  float* s_q = s_kbuf + NW * S::KBUF;                       // [nq][P][QS]
  __shared__ unsigned long long s_mask[kScoreTile];
  __shared__ uint32_t s_kw[kScoreQBlock][3];
  __shared__ int64_t s_out[kScoreQBlock];
  __shared__ unsigned long long s_any;
  const int g = blockIdx.y;
  const int64_t n0 = int64_t(blockIdx.x) * tile;
  const int GQ = G.group;
  const int qn_total = batch * GQ;
  const int qb0 = blockIdx.z * kScoreQBlock;
  const int nq = min(kScoreQBlock, qn_total - qb0);
  const int C = G.chunk, R = G.nref;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t orphan0 = int64_t(C) * n_par;
  const int64_t w_lo = (n0 / C) >> 5;

  if (tid == 0) s_any = 0ull;
  if (tid < nq) {
    const int qi = qb0 + tid;
    const int64_t bh = int64_t(qi / GQ) * G.hq + g * GQ + qi % GQ;
    s_out[tid] = bh * n_nodes;
    if (n0 < orphan0) {
      const uint32_t* kw = kept_up + bh * words_up;
#pragma unroll
      for (int k = 0; k < 3; ++k) s_kw[tid][k] = (w_lo + k < words_up) ? kw[w_lo + k] : 0u;
    }
  }
  __syncthreads();
  if (tid < tile) {
    const int64_t n = n0 + tid;
    unsigned long long m = 0ull;
    if (n < n_nodes) {
      if (n >= orphan0) {
        m = nq == 64 ? ~0ull : ((1ull << nq) - 1ull);
      } else {
        const int64_t pnode = n / C;
        const int slot = int((pnode >> 5) - w_lo);
        const int bit = int(pnode & 31);
        for (int q = 0; q < nq; ++q) m |= (unsigned long long)((s_kw[q][slot] >> bit) & 1u) << q;
      }
    }
    s_mask[tid] = m;
    if (m) atomicOr(&s_any, m);
  }
  __syncthreads();
  const unsigned long long any = s_any;
  if (any == 0ull) return;
  // Stage the rows of the query heads this tile needs, split in P parts.
  for (int v = tid; v < nq * (D / 4); v += blockDim.x) {
    const int q = v / (D / 4), e = (v % (D / 4)) * 4;
    if (!((any >> q) & 1ull)) continue;
    const int qi = qb0 + q;
    const int64_t bh = int64_t(qi / GQ) * G.hq + g * GQ + qi % GQ;
    const float4 x = *reinterpret_cast<const float4*>(Q + bh * D + e);
    *reinterpret_cast<float4*>(s_q + q * S::QROW + (e / S::EP) * S::QS + e % S::EP) = x;
  }
  __syncthreads();

  float* kb = s_kbuf + warp * S::KBUF;
  const uint32_t kb_s = static_cast<uint32_t>(__cvta_generic_to_shared(kb));
  const float* level_base = store + G.off[level] + int64_t(g) * G.cap[level] * G.node_floats;
  // Copy the planes of node n (R * D floats) into this warp's buffer.
  auto stage = [&](int t) {
    const float* rec = level_base + (n0 + t) * G.node_floats;
    for (int c = lane; c < R * (D / 4); c += 32) {
      const int e = 4 * c, r = e / D, col = e % D;
      cp_async16_ca(kb_s + 4u * uint32_t(r * S::KROW + (col / S::EP) * S::QS + col % S::EP), rec + e);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  auto next_node = [&](int t) {
    for (t += NW; t < tile; t += NW)
      if (s_mask[t] != 0ull) return t;
    return tile;
  };

  const int r = lane / S::P, part = lane % S::P;
  const bool live = r < R;
  int t = warp < tile && s_mask[warp] != 0ull ? warp : next_node(warp);
  if (t < tile) stage(t);
  while (t < tile) {
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncwarp();
    float kr[S::EP];
    if (live) {
#pragma unroll
      for (int e = 0; e < S::EP; e += 4) {
        const float4 x = *reinterpret_cast<const float4*>(kb + r * S::KROW + part * S::QS + e);
        kr[e] = x.x; kr[e + 1] = x.y; kr[e + 2] = x.z; kr[e + 3] = x.w;
      }
    } else {
#pragma unroll
      for (int e = 0; e < S::EP; ++e) kr[e] = 0.f;
    }
    const int64_t n = n0 + t;
    const float b = live ? __ldg(level_base + n * G.node_floats + R * D + r) : 0.f;
    unsigned long long m = s_mask[t];
    __syncwarp();
    const int tn = next_node(t);
    if (tn < tile) stage(tn);          // overlaps the scoring below
    while (m) {
      const int q = __ffsll(m) - 1;
      m &= m - 1ull;
      const float* qs = s_q + q * S::QROW + part * S::QS;
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < S::EP; e += 4) {
        const float4 x = *reinterpret_cast<const float4*>(qs + e);
        dot += kr[e] * x.x + kr[e + 1] * x.y + kr[e + 2] * x.z + kr[e + 3] * x.w;
      }
#pragma unroll
      for (int o = 1; o < S::P; o <<= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      float tr = live ? dot * G.scale + b : -INFINITY;
#pragma unroll
      for (int o = S::P; o < 32; o <<= 1) tr = fmaxf(tr, __shfl_xor_sync(0xffffffffu, tr, o));
      if (lane == 0) sigma[s_out[q] + n] = tr;
    }
    t = tn;
  }
}

// ---------------------------------------------------------------------------
// Block-wide helpers for the select kernel (blockDim = kSelectThreads).
// ---------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ T warp_incl_scan(T v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    T n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// Exclusive prefix over threads in thread order; returns this thread's offset
// and writes the block total to *total. `tmp` holds >= 33 elements.
template <typename T>
__device__ T block_excl_scan(T v, T* tmp, T* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const T incl = warp_incl_scan(v);
  if (lane == 31) tmp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    T w = lane < nw ? tmp[lane] : T(0);
    T wi = warp_incl_scan(w);
    if (lane < nw) tmp[lane] = wi - w;
    if (lane == 31) tmp[32] = wi;
  }
  __syncthreads();
  const T out = tmp[warp] + incl - v;
  *total = tmp[32];
  __syncthreads();
  return out;
}

__device__ float block_max(float v, float* tmp) {
  v = warp_max(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if (lane == 0) tmp[warp] = v;
  __syncthreads();
  if (warp == 0) {
    float w = lane < nw ? tmp[lane] : -INFINITY;
    w = warp_max(w);
    if (lane == 0) tmp[32] = w;
  }
  __syncthreads();
  const float r = tmp[32];
  __syncthreads();
  return r;
}

__device__ float block_sum(float v, float* tmp) {
  v = warp_sum(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if (lane == 0) tmp[warp] = v;
  __syncthreads();
  if (warp == 0) {
    float w = lane < nw ? tmp[lane] : 0.f;
    w = warp_sum(w);
    if (lane == 0) tmp[32] = w;
  }
  __syncthreads();
  const float r = tmp[32];
  __syncthreads();
  return r;
}

// ---------------------------------------------------------------------------
// Selection for one query head at one level.
// ---------------------------------------------------------------------------
struct SelectArgs {
  int level;
  int64_t n_nodes, n_par;
  const uint32_t* kept_up;   // level l+1 bitmaps, [B*Hq][words_up] (null at the top)
  int64_t words_up;
  uint32_t* kept_here;       // level l bitmaps, [B*Hq][words_here]
  int64_t words_here;
  const float* sigma;        // [B*Hq][n_nodes]
  int32_t* kp;               // scratch [B*Hq][kp_stride]
  int64_t kp_stride;
  unsigned long long p_fixed;    // p in units of 2^-40 (select_kernel)
  unsigned long long p_fixed32;  // p in units of 2^-32 (select_fast_kernel)
  int keep_all;
  int32_t* chunk_ids;        // level 1 only
  int32_t* n_chunks;
  int32_t max_sel;
  int32_t* status;
  const int32_t* tree_status;  // top level only: the tree's build status, OR-ed into *status
};

// The first selection of a route passes the tree's build status on to the
// caller's status word (a build whose bounded wait ran out left the tree invalid).
__device__ __forceinline__ void forward_tree_status(const SelectArgs& a) {
  if (a.tree_status != nullptr && a.status != nullptr && blockIdx.x == 0 && threadIdx.x == 0) {
    const int32_t v = *a.tree_status;
    if (v != 0) atomicOr(a.status, v);
  }
}

__global__ void __launch_bounds__(kSelectThreads)
select_kernel(Geom G, SelectArgs a) {
  extern __shared__ float4 smem_v4[];
  unsigned long long* hist = reinterpret_cast<unsigned long long*>(smem_v4);  // [nwarps][256]
  float* s_sig = reinterpret_cast<float*>(hist + (kSelectThreads / 32) * 256);
  int32_t* s_kp = reinterpret_cast<int32_t*>(s_sig + kSelectCache);           // [kSelectKpCache]
  __shared__ float s_f[33];
  __shared__ unsigned long long s_u[33];
  __shared__ uint32_t s_w[33];
  __shared__ uint32_t s_bucket;
  __shared__ unsigned long long s_before;
  pdl_trigger();
  pdl_wait();
  forward_tree_status(a);

  const int bh = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  const int C = G.chunk;
  uint32_t* bits = a.kept_here + int64_t(bh) * a.words_here;
  for (int64_t w = tid; w < a.words_here; w += blockDim.x) bits[w] = 0u;

  // Kept parents of this head, ascending (compaction of the level-(l+1) bitmap).
  // Parents fit in shared memory unless the level above is very wide.
  const bool kp_in_smem = a.words_up <= kSelectKpCache / 32;
  int32_t* kp = kp_in_smem ? s_kp : a.kp + int64_t(bh) * a.kp_stride;
  uint32_t n_kp = 0;
  if (a.kept_up != nullptr && a.words_up > 0) {
    const uint32_t* up = a.kept_up + int64_t(bh) * a.words_up;
    for (int64_t w0 = 0; w0 < a.words_up; w0 += blockDim.x) {
      const int64_t w = w0 + tid;
      const uint32_t word = w < a.words_up ? up[w] : 0u;
      uint32_t tot;
      uint32_t pos = n_kp + block_excl_scan<uint32_t>(__popc(word), s_w, &tot);
      uint32_t x = word;
      while (x) {
        const int bit = __ffs(x) - 1;
        x &= x - 1u;
        kp[pos++] = int32_t(w * 32 + bit);
      }
      n_kp += tot;
    }
  }
  __syncthreads();   // kp visible to the block

  const int64_t orphan0 = int64_t(C) * a.n_par;
  const int64_t n_child = int64_t(n_kp) * C;
  const int64_t n_c = n_child + (a.n_nodes - orphan0);
  // Candidate i -> node: child (i % C) of kept parent i / C, or an orphan.
  // Candidate and node indices fit 32 bits; the division is 32-bit.
  const uint32_t uC = uint32_t(C), u_nchild = uint32_t(n_child);
  auto node_of = [&](int64_t i) -> int64_t {
    const uint32_t ui = uint32_t(i);
    if (ui < u_nchild) {
      const uint32_t par = ui / uC;
      return int64_t(kp[par]) * C + (ui - par * uC);
    }
    return orphan0 + (ui - u_nchild);
  };
  const float* sig = a.sigma + int64_t(bh) * a.n_nodes;
  const bool cached = n_c <= kSelectCache;
  if (cached) {
    // Eight independent loads in flight per thread.
    for (int64_t i0 = tid; i0 < n_c; i0 += 8 * int64_t(blockDim.x)) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t i = i0 + int64_t(u) * blockDim.x;
        v[u] = i < n_c ? sig[node_of(i)] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t i = i0 + int64_t(u) * blockDim.x;
        if (i < n_c) s_sig[i] = v[u];
      }
    }
  }
  __syncthreads();
  auto sigma_of = [&](int64_t i) -> float { return cached ? s_sig[i] : sig[node_of(i)]; };

  // Softmax statistics over the candidates.
  float mx = -INFINITY;
  for (int64_t i = tid; i < n_c; i += blockDim.x) mx = fmaxf(mx, sigma_of(i));
  mx = block_max(mx, s_f);
  float z = 0.f;
  for (int64_t i = tid; i < n_c; i += blockDim.x) z += expf(sigma_of(i) - mx);
  z = block_sum(z, s_f);
  const float inv_z = 1.f / z;
  auto mass_of = [&](float s) -> unsigned long long {
    return __float2ull_rn(expf(s - mx) * inv_z * float(kMassScale));
  };

  // Cut: smallest key (score desc, index asc) whose cumulative mass reaches p.
  bool keep_all = a.keep_all != 0 || n_c == 0;
  uint32_t key_cut = 0xffffffffu;
  unsigned long long t_keep = 0;
  if (!keep_all) {
    unsigned long long tm = 0;
    for (int64_t i = tid; i < n_c; i += blockDim.x) tm += mass_of(sigma_of(i));
    unsigned long long total;
    block_excl_scan<unsigned long long>(tm, s_u, &total);
    if (total < a.p_fixed) keep_all = true;
  }
  if (!keep_all) {
    uint32_t prefix = 0, pmask = 0;
    unsigned long long before = 0;
    unsigned long long* wh = hist + warp * 256;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int k = lane; k < 256; k += 32) wh[k] = 0ull;
      __syncthreads();
      // Runs of equal buckets are summed in a register and flushed once: the
      // leading digits of nearby scores coincide, and per-element atomics on
      // one bucket would serialise the whole warp.
      uint32_t cb = 0xffffffffu;
      unsigned long long cs = 0ull;
      for (int64_t i = tid; i < n_c; i += blockDim.x) {
        const float s = sigma_of(i);
        const uint32_t key = ~float_order_key(s);
        if ((key & pmask) == prefix) {
          const uint32_t b = (key >> shift) & 255u;
          const unsigned long long mm = mass_of(s);
          if (b == cb) {
            cs += mm;
          } else {
            if (cs != 0ull) atomicAdd(&wh[cb], cs);
            cb = b;
            cs = mm;
          }
        }
      }
      if (cs != 0ull) atomicAdd(&wh[cb], cs);
      __syncthreads();
      // bucket totals into warp 0's histogram
      for (int k = tid; k < 256; k += blockDim.x) {
        unsigned long long v = 0;
        for (int w = 0; w < nw; ++w) v += hist[w * 256 + k];
        hist[k] = v;
      }
      __syncthreads();
      if (warp == 0) {
        // lane owns buckets [8*lane, 8*lane+8)
        unsigned long long loc[8], run = 0;
        for (int k = 0; k < 8; ++k) { loc[k] = hist[8 * lane + k]; run += loc[k]; }
        unsigned long long incl = warp_incl_scan<unsigned long long>(run);
        unsigned long long excl = incl - run;
        // first bucket whose inclusive cumulative mass reaches p
        int found = -1;
        unsigned long long acc = before + excl, acc_before = 0;
        for (int k = 0; k < 8; ++k) {
          if (found < 0 && acc + loc[k] >= a.p_fixed) { found = 8 * lane + k; acc_before = acc; }
          acc += loc[k];
        }
        const unsigned ball = __ballot_sync(0xffffffffu, found >= 0);
        const int src = ball ? __ffs(ball) - 1 : 31;
        const int fb = __shfl_sync(0xffffffffu, found, src);
        const unsigned long long ab = __shfl_sync(0xffffffffu, acc_before, src);
        if (lane == 0) {
          s_bucket = fb < 0 ? 255u : uint32_t(fb);
          s_before = fb < 0 ? before : ab;
        }
      }
      __syncthreads();
      prefix |= s_bucket << shift;
      pmask |= 255u << shift;
      before = s_before;
      __syncthreads();
    }
    key_cut = prefix;
    const unsigned long long pi_cut = mass_of(order_key_float(~key_cut));
    const unsigned long long need = a.p_fixed > before ? a.p_fixed - before : 0ull;
    t_keep = pi_cut > 0 ? (need + pi_cut - 1) / pi_cut : 0ull;
  }

  // Keep flags in candidate order (ascending node index): thread-contiguous
  // ranges so that ties at the cut are taken lowest index first.
  const int64_t per = (n_c + blockDim.x - 1) / blockDim.x;
  const int64_t i_lo = min64(n_c, per * tid), i_hi = min64(n_c, i_lo + per);
  uint32_t my_ties = 0;
  if (!keep_all)
    for (int64_t i = i_lo; i < i_hi; ++i) my_ties += (~float_order_key(sigma_of(i)) == key_cut);
  uint32_t tie_total;
  uint32_t tie_rank = block_excl_scan<uint32_t>(my_ties, s_w, &tie_total);
  uint32_t my_kept = 0;
  {
    uint32_t tr = tie_rank;
    for (int64_t i = i_lo; i < i_hi; ++i) {
      bool k = keep_all;
      if (!k) {
        const uint32_t key = ~float_order_key(sigma_of(i));
        k = key < key_cut || (key == key_cut && tr++ < t_keep);
      }
      my_kept += k;
    }
  }
  uint32_t kept_total;
  uint32_t pos = block_excl_scan<uint32_t>(my_kept, s_w, &kept_total);
  {
    uint32_t tr = tie_rank;
    for (int64_t i = i_lo; i < i_hi; ++i) {
      bool k = keep_all;
      if (!k) {
        const uint32_t key = ~float_order_key(sigma_of(i));
        k = key < key_cut || (key == key_cut && tr++ < t_keep);
      }
      if (k) {
        const int64_t node = node_of(i);
        atomicOr(&bits[node >> 5], 1u << (node & 31));
        if (a.chunk_ids != nullptr && pos < uint32_t(a.max_sel))
          a.chunk_ids[int64_t(bh) * a.max_sel + pos] = int32_t(node);
        ++pos;
      }
    }
  }
  if (a.chunk_ids != nullptr && tid == 0) {
    a.n_chunks[bh] = int32_t(kept_total);
    if (kept_total > uint32_t(a.max_sel) && a.status != nullptr)
      atomicOr(a.status, ZHA_DEV_SELECTION_TRUNCATED);
  }
}

// ---------------------------------------------------------------------------
// Selection for one query head at one level, all candidates in shared memory
// (n_nodes <= kFastMax). Each candidate's order key (score descending, then
// index ascending) and its softmax mass in 2^-32 fixed point are computed once.
//  * up to kFastSmallN candidates: thread i counts the mass of every candidate
//    ordered before it; i is kept iff that mass is below p (the minimal prefix
//    holding mass p). No radix passes, a handful of barriers.
//  * more: the cut key by a radix select over 8-bit digits with per-warp
//    histograms of mass, starting at the first byte in which the candidates'
//    keys differ; runs of equal buckets are summed in registers before the
//    atomic add.
// The rounding of the fixed-point masses adds at most n 2^-33 to any
// cumulative mass (< 2e-6 at n = 16384).
// ---------------------------------------------------------------------------
constexpr int kFastMax = 16384;
constexpr int kFastSmallN = kSelectThreads;
constexpr int kHistBins = (kSelectThreads / 32) * 256;   // per-warp 256-bin histograms

__global__ void __launch_bounds__(kSelectThreads)
select_fast_kernel(Geom G, SelectArgs a) {
  extern __shared__ float4 smem_v4[];
  uint32_t* s_key = reinterpret_cast<uint32_t*>(smem_v4);                    // scores, then keys
  uint32_t* s_m = s_key + kFastMax;                                           // masses
  unsigned long long* hist = reinterpret_cast<unsigned long long*>(s_m + kFastMax);   // [kHistBins]
  int32_t* s_kp = reinterpret_cast<int32_t*>(hist + kHistBins);               // [kSelectKpCache]
  float* s_sig = reinterpret_cast<float*>(s_key);
  __shared__ float s_f[33];
  __shared__ unsigned long long s_u[33];
  __shared__ uint32_t s_w[33];
  __shared__ uint32_t s_bucket;
  __shared__ unsigned long long s_before;
  pdl_trigger();
  pdl_wait();
  forward_tree_status(a);

  const int bh = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int C = G.chunk;
  uint32_t* bits = a.kept_here + int64_t(bh) * a.words_here;
  for (int64_t w = tid; w < a.words_here; w += blockDim.x) bits[w] = 0u;

  // Kept parents of this head, ascending.
  const bool kp_in_smem = a.words_up <= kSelectKpCache / 32;
  int32_t* kp = kp_in_smem ? s_kp : a.kp + int64_t(bh) * a.kp_stride;
  uint32_t n_kp = 0;
  if (a.kept_up != nullptr && a.words_up > 0) {
    const uint32_t* up = a.kept_up + int64_t(bh) * a.words_up;
    for (int64_t w0 = 0; w0 < a.words_up; w0 += blockDim.x) {
      const int64_t w = w0 + tid;
      const uint32_t word = w < a.words_up ? up[w] : 0u;
      uint32_t tot;
      uint32_t pos = n_kp + block_excl_scan<uint32_t>(__popc(word), s_w, &tot);
      uint32_t x = word;
      while (x) {
        const int bit = __ffs(x) - 1;
        x &= x - 1u;
        kp[pos++] = int32_t(w * 32 + bit);
      }
      n_kp += tot;
    }
  }
  __syncthreads();

  const int64_t orphan0 = int64_t(C) * a.n_par;
  const uint32_t uC = uint32_t(C), n_child = n_kp * uC;
  const int n_c = int(n_child + uint32_t(a.n_nodes - orphan0));
  auto node_of = [&](int i) -> int64_t {
    const uint32_t ui = uint32_t(i);
    if (ui < n_child) {
      const uint32_t par = ui / uC;
      return int64_t(kp[par]) * C + (ui - par * uC);
    }
    return orphan0 + (ui - n_child);
  };
  const float* sig = a.sigma + int64_t(bh) * a.n_nodes;
  for (int i0 = tid; i0 < n_c; i0 += 8 * kSelectThreads) {      // eight loads in flight
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * kSelectThreads;
      v[u] = i < n_c ? sig[node_of(i)] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * kSelectThreads;
      if (i < n_c) s_sig[i] = v[u];
    }
  }
  __syncthreads();

  // Softmax statistics, then keys and fixed-point masses (same arithmetic for
  // every use of a candidate's mass).
  float mx = -INFINITY;
  for (int i = tid; i < n_c; i += kSelectThreads) mx = fmaxf(mx, s_sig[i]);
  mx = block_max(mx, s_f);
  float z = 0.f;
  for (int i = tid; i < n_c; i += kSelectThreads) z += expf(s_sig[i] - mx);
  z = block_sum(z, s_f);
  const float scale32 = 4294967296.f / z;
  auto mass_of = [&](float s) -> uint32_t { return __float2uint_rn(expf(s - mx) * scale32); };
  unsigned long long tm = 0;
  for (int i = tid; i < n_c; i += kSelectThreads) {
    const float s = s_sig[i];
    const uint32_t m = mass_of(s);
    s_m[i] = m;
    s_key[i] = ~float_order_key(s);
    tm += m;
  }
  unsigned long long total;
  block_excl_scan<unsigned long long>(tm, s_u, &total);      // its barriers publish s_key / s_m
  const unsigned long long p32 = a.p_fixed32;
  const bool keep_all = a.keep_all != 0 || n_c == 0 || total < p32;

  uint32_t kept_total = 0;
  auto emit = [&](int i, uint32_t pos) {
    const int64_t node = node_of(i);
    atomicOr(&bits[node >> 5], 1u << (node & 31));
    if (a.chunk_ids != nullptr && pos < uint32_t(a.max_sel))
      a.chunk_ids[int64_t(bh) * a.max_sel + pos] = int32_t(node);
  };
  if (keep_all || n_c <= kFastSmallN) {
    // Thread i = candidate i (candidate order = ascending node index).
    bool k = false;
    if (tid < n_c) {
      if (keep_all) {
        k = true;
      } else {
        const uint32_t ki = s_key[tid];
        unsigned long long cb = 0ull;
        for (int j = 0; j < n_c; ++j) {
          const uint32_t kj = s_key[j];
          if (kj < ki || (kj == ki && j < tid)) cb += s_m[j];
        }
        k = cb < p32;
      }
    }
    if (keep_all && n_c > kSelectThreads) {
      // keep everything: thread-contiguous ranges, positions by a scan
      const int per = (n_c + kSelectThreads - 1) / kSelectThreads;
      const int i_lo = min(n_c, per * tid), i_hi = min(n_c, i_lo + per);
      uint32_t pos = block_excl_scan<uint32_t>(uint32_t(i_hi - i_lo), s_w, &kept_total);
      for (int i = i_lo; i < i_hi; ++i) emit(i, pos++);
    } else {
      const uint32_t pos = block_excl_scan<uint32_t>(k ? 1u : 0u, s_w, &kept_total);
      if (k) emit(tid, pos);
    }
  } else {
    // Leading bytes shared by every candidate's key are fixed up front.
    uint32_t k_and = 0xffffffffu, k_or = 0u;
    for (int i = tid; i < n_c; i += kSelectThreads) { k_and &= s_key[i]; k_or |= s_key[i]; }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      k_and &= __shfl_xor_sync(0xffffffffu, k_and, o);
      k_or |= __shfl_xor_sync(0xffffffffu, k_or, o);
    }
    if (lane == 0) { s_w[warp] = k_and; s_w[16 + warp] = k_or; }
    __syncthreads();
    if (tid == 0) {
      uint32_t x = 0xffffffffu, y = 0u;
      for (int w = 0; w < kSelectThreads / 32; ++w) { x &= s_w[w]; y |= s_w[16 + w]; }
      s_w[32] = x;
      s_bucket = y;
    }
    __syncthreads();
    k_and = s_w[32];
    k_or = s_bucket;
    const int lead = (k_and ^ k_or) == 0u ? 32 : __clz(k_and ^ k_or);   // common leading bits
    const int first_byte = min(lead / 8, 3);
    uint32_t pmask = first_byte == 0 ? 0u : ~0u << (32 - 8 * first_byte);
    uint32_t prefix = k_and & pmask;
    unsigned long long before = 0ull;
    unsigned long long* wh = hist + warp * 256;
#pragma unroll 1
    for (int shift = 24 - 8 * first_byte; shift >= 0; shift -= 8) {
      for (int k = lane; k < 256; k += 32) wh[k] = 0ull;
      __syncthreads();
      uint32_t cb = 0xffffffffu;
      unsigned long long cs = 0ull;
      for (int i = tid; i < n_c; i += kSelectThreads) {
        const uint32_t key = s_key[i];
        if ((key & pmask) == prefix) {
          const uint32_t bkt = (key >> shift) & 255u;
          if (bkt == cb) {
            cs += s_m[i];
          } else {
            if (cs != 0ull) atomicAdd(&wh[cb], cs);
            cb = bkt;
            cs = s_m[i];
          }
        }
      }
      if (cs != 0ull) atomicAdd(&wh[cb], cs);
      __syncthreads();
      for (int k = tid; k < 256; k += kSelectThreads) {     // bucket totals into warp 0's histogram
        unsigned long long v = 0ull;
        for (int w = 0; w < kSelectThreads / 32; ++w) v += hist[w * 256 + k];
        hist[k] = v;
      }
      __syncthreads();
      if (warp == 0) {
        // lane owns buckets [8 lane, 8 lane + 8): first bucket whose cumulative
        // mass (with `before`) reaches p
        unsigned long long loc[8], run = 0ull;
#pragma unroll
        for (int k = 0; k < 8; ++k) { loc[k] = hist[8 * lane + k]; run += loc[k]; }
        const unsigned long long incl = warp_incl_scan<unsigned long long>(run);
        unsigned long long acc = before + incl - run, acc_before = 0ull;
        int found = -1;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if (found < 0 && acc + loc[k] >= p32) { found = 8 * lane + k; acc_before = acc; }
          acc += loc[k];
        }
        const unsigned ball = __ballot_sync(0xffffffffu, found >= 0);
        const int src = ball ? __ffs(ball) - 1 : 31;
        const int fb = __shfl_sync(0xffffffffu, found, src);
        const unsigned long long ab = __shfl_sync(0xffffffffu, acc_before, src);
        if (lane == 0) {
          s_bucket = fb < 0 ? 255u : uint32_t(fb);
          s_before = fb < 0 ? before : ab;
        }
      }
      __syncthreads();
      prefix |= s_bucket << shift;
      pmask |= 255u << shift;
      before = s_before;
      __syncthreads();                                      // s_bucket / s_before are reused
    }
    const uint32_t key_cut = prefix;
    const uint32_t m_cut = mass_of(order_key_float(~key_cut));
    const unsigned long long need = p32 > before ? p32 - before : 0ull;
    const unsigned long long t_keep = m_cut > 0u ? (need + m_cut - 1ull) / m_cut : 0ull;
    // Kept flags in candidate order: thread-contiguous ranges so that ties at
    // the cut are taken lowest index first.
    const int per = (n_c + kSelectThreads - 1) / kSelectThreads;
    const int i_lo = min(n_c, per * tid), i_hi = min(n_c, i_lo + per);
    uint32_t my_ties = 0;
    for (int i = i_lo; i < i_hi; ++i) my_ties += (s_key[i] == key_cut);
    uint32_t tie_total;
    const uint32_t tie_rank = block_excl_scan<uint32_t>(my_ties, s_w, &tie_total);
    uint32_t my_kept = 0;
    {
      uint32_t tr = tie_rank;
      for (int i = i_lo; i < i_hi; ++i) {
        const uint32_t key = s_key[i];
        my_kept += (key < key_cut || (key == key_cut && tr++ < t_keep)) ? 1u : 0u;
      }
    }
    uint32_t pos = block_excl_scan<uint32_t>(my_kept, s_w, &kept_total);
    {
      uint32_t tr = tie_rank;
      for (int i = i_lo; i < i_hi; ++i) {
        const uint32_t key = s_key[i];
        if (key < key_cut || (key == key_cut && tr++ < t_keep)) emit(i, pos++);
      }
    }
  }
  if (a.chunk_ids != nullptr && tid == 0) {
    a.n_chunks[bh] = int32_t(kept_total);
    if (kept_total > uint32_t(a.max_sel) && a.status != nullptr)
      atomicOr(a.status, ZHA_DEV_SELECTION_TRUNCATED);
  }
}

size_t select_fast_smem_bytes() {
  return size_t(2 * kFastMax) * sizeof(uint32_t) + size_t(kHistBins) * sizeof(unsigned long long) +
         size_t(kSelectKpCache) * sizeof(int32_t);
}

cudaError_t launch_score_tc(const Geom& G, int level, int64_t n_nodes, int64_t n_par, int32_t batch,
                            const float* Q, const uint32_t* kept_up, int64_t words_up, float* sigma,
                            const float* store, int32_t* status, cudaStream_t s);
bool score_tma_supported(const Geom& G);
cudaError_t launch_score_tma(const Geom& G, int level, int64_t n_nodes, int64_t n_par, int32_t batch,
                             const float* Q, const uint32_t* kept_up, int64_t words_up, float* sigma,
                             const float* store, int32_t* status, cudaStream_t s, bool* used);

// ---------------------------------------------------------------------------
// Host launcher: levels L..1, score then select.
// ---------------------------------------------------------------------------
template <int D, int RP>
static cudaError_t launch_score_t(const Geom& G, int level, int64_t n_nodes, int64_t n_par,
                                  int32_t batch, const float* Q, const uint32_t* kept_up,
                                  int64_t words_up, float* sigma, const float* store,
                                  cudaStream_t s) {
  using S = ScoreShape<D, RP>;
  const int qn = batch * G.group;
  // Nodes per CTA: enough CTAs to fill the GPU twice over, at most kScoreTile.
  int tile = kScoreTile;
  while (tile > kScoreThreads / 32 && (n_nodes * G.hkv) / tile < 2 * 148) tile >>= 1;
  dim3 grid(unsigned((n_nodes + tile - 1) / tile), unsigned(G.hkv),
            unsigned((qn + kScoreQBlock - 1) / kScoreQBlock));
  const size_t smem = (size_t(kScoreThreads / 32) * S::KBUF +
                       size_t(qn < kScoreQBlock ? qn : kScoreQBlock) * S::QROW) * 4;
  cudaError_t e = ensure_dynamic_smem(score_kernel<D, RP>, smem);
  if (e != cudaSuccess) return e;
  TraceScope ts("score_kernel", level, s);
  e = launch_pdl(score_kernel<D, RP>, grid, dim3(kScoreThreads), smem, s, G, level, n_nodes, n_par,
                 batch, tile, Q, kept_up, words_up, sigma, store);
  zha_count_launch();
  return e;
}

template <int D>
static cudaError_t launch_score_d(const Geom& G, int level, int64_t n_nodes, int64_t n_par,
                                  int32_t batch, const float* Q, const uint32_t* kept_up,
                                  int64_t words_up, float* sigma, const float* store,
                                  cudaStream_t s) {
  // Planes are padded to a power of two RP >= 128 / D so that each lane holds
  // at least one float4 of its plane's row.
  const int R = G.nref;
#define ZHA_SCORE_CASE(RP)                                                                      \
  if (R <= RP && RP * D >= 128)                                                                 \
    return launch_score_t<D, RP>(G, level, n_nodes, n_par, batch, Q, kept_up, words_up, sigma, \
                                 store, s);
  if constexpr (D >= 128) ZHA_SCORE_CASE(1)
  ZHA_SCORE_CASE(2)
  ZHA_SCORE_CASE(4)
  ZHA_SCORE_CASE(8)
  ZHA_SCORE_CASE(16)
  ZHA_SCORE_CASE(32)
#undef ZHA_SCORE_CASE
  return cudaErrorInvalidValue;
}

size_t select_smem_bytes() {
  return size_t(kSelectThreads / 32) * 256 * sizeof(unsigned long long) +
         size_t(kSelectCache) * sizeof(float) + size_t(kSelectKpCache) * sizeof(int32_t);
}

cudaError_t launch_route(const Geom& G, const float* Q, int32_t batch, int64_t n_tokens, float p,
                         int32_t* chunk_ids, int32_t* n_chunks, int32_t max_sel, uint32_t* bits,
                         float* sigma, int32_t* kp, const RouteLayout& lay, int32_t* status,
                         const float* store, cudaStream_t s) {
  const size_t smem = select_smem_bytes();
  cudaError_t e = ensure_dynamic_smem(select_kernel, smem);
  if (e != cudaSuccess) return e;
  const int heads = batch * G.hq;
  SelectArgs a{};
  a.p_fixed = (unsigned long long)ceil(double(p) * kMassScale);
  if (a.p_fixed == 0) a.p_fixed = 1;
  a.p_fixed32 = (unsigned long long)ceil(double(p) * 4294967296.0);
  if (a.p_fixed32 == 0) a.p_fixed32 = 1;
  const size_t smem_fast = select_fast_smem_bytes();
  if ((e = ensure_dynamic_smem(select_fast_kernel, smem_fast)) != cudaSuccess)
    return e;
  a.keep_all = p >= 1.0f;
  a.kp = kp;
  int64_t kp_stride = lay.kp_ints / (heads > 0 ? heads : 1);
  a.kp_stride = kp_stride;
  a.max_sel = max_sel;
  a.status = status;
  for (int level = G.levels; level >= 1; --level) {
    const int64_t n_nodes = lay.n[level];
    const int64_t n_par = level < G.levels ? lay.n[level + 1] : 0;
    const uint32_t* up = level < G.levels ? bits + lay.bits_off[level + 1] : nullptr;
    const int64_t words_up = level < G.levels ? lay.words[level + 1] : 0;
    float* sg = sigma + lay.sig_off[level];
    if (n_nodes > 0) {
      bool done = false;
      if (score_tma_supported(G)) {      // tensor copies + tensor cores (zha_score_tma.cu)
        e = launch_score_tma(G, level, n_nodes, n_par, batch, Q, up, words_up, sg, store, status, s,
                             &done);
        if (e != cudaSuccess) return e;
      }
      if (done)
        ;
      else if (G.d == 128 && G.nref <= 16)      // tensor cores (zha_score_tc.cu)
        e = launch_score_tc(G, level, n_nodes, n_par, batch, Q, up, words_up, sg, store, status, s);
      else
        e = G.d == 128 ? launch_score_d<128>(G, level, n_nodes, n_par, batch, Q, up, words_up, sg,
                                             store, s)
                       : launch_score_d<64>(G, level, n_nodes, n_par, batch, Q, up, words_up, sg,
                                            store, s);
      if (e != cudaSuccess) return e;
    }
    a.level = level;
    a.n_nodes = n_nodes;
    a.n_par = n_par;
    a.kept_up = up;
    a.words_up = words_up;
    a.kept_here = bits + lay.bits_off[level];
    a.words_here = lay.words[level];
    a.sigma = sg;
    a.chunk_ids = level == 1 ? chunk_ids : nullptr;
    a.n_chunks = level == 1 ? n_chunks : nullptr;
    a.tree_status = level == G.levels ? tree_status_word(G, const_cast<float*>(store)) : nullptr;
    if (n_nodes <= kFastMax) {
      TraceScope ts("select_fast_kernel", level, s);
      e = launch_pdl(select_fast_kernel, dim3(heads), dim3(kSelectThreads), smem_fast, s, G, a);
    } else {
      TraceScope ts("select_kernel", level, s);
      e = launch_pdl(select_kernel, dim3(heads), dim3(kSelectThreads), smem, s, G, a);
    }
    if (e != cudaSuccess) return e;
    zha_count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace zha
