// zha_route.cu -- per-level top-p routing of decode queries through the trees.
//
// Citations: [ZHA: 무엇과 다른가 / 전제와 한계] = page "ZHA는 KV 캐시를 트리로 요약해
// 어텐션 비용을 준(sub)이차로 낮춘다" (onedev.kr/papers/1556): a node's log mass for
// a future query is estimated by the maximum of its R tangent planes (무엇과 다른가);
// routing runs top-p per level -- sort the candidates by score, keep the minimal
// prefix holding estimated mass p, pass the kept nodes' children and the
// parentless chunks down (전제와 한계).
//
// The small top levels (a few hundred nodes per KV head) are scored densely,
// every node for every query head, by score_dense_kernel (zha_dense.cuh) in one
// launch and selected level after level by select_top_kernel in one launch.
// Every lower level l takes two launches:
//   scoring -- head_dim 128 with R = 16: score_tma_kernel (zha_score_tma.cu,
//              tensor copies + tcgen05); head_dim 128 with R < 16:
//              score_tc_kernel (zha_score_tc.cu); otherwise score_kernel here
//              (one warp per candidate node -- the union over the query heads of
//              a KV head -- its R planes in registers, one score per query head
//              that has the node as candidate);
//   selection -- select_fast_kernel, one CTA per query head: softmax over its
//              candidates, the cut on the key (score desc, node index asc) by
//              fixed-point mass, kept bitmap (and at level 1 the ascending
//              chunk list).
// Both kinds are launched with programmatic dependent launch.
#include "zha_host.cuh"
#include "zha_internal.cuh"
#include "zha_dense.cuh"

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

// One CTA: nodes [tile_i * tile, + tile) of level `level` of KV head g, query
// heads [qblock * kScoreQBlock, + kScoreQBlock) of g's group.
template <int D, int RP>
__device__ __forceinline__ void score_tile(const Geom& G, int level, int64_t n_nodes, int64_t n_par,
                                           int32_t batch, int tile, int64_t tile_i, int g, int qblock,
                                           const float* __restrict__ Q,
                                           const uint32_t* __restrict__ kept_up, int64_t words_up,
                                           float* __restrict__ sigma, const float* __restrict__ store) {
  using S = ScoreShape<D, RP>;
  constexpr int NW = kScoreThreads / 32;
  extern __shared__ float4 smem_v4[];
  float* s_kbuf = reinterpret_cast<float*>(smem_v4);       // [NW][KBUF]
  float* s_q = s_kbuf + NW * S::KBUF;                       // [nq][P][QS]
  __shared__ unsigned long long s_mask[kScoreTile];
  __shared__ uint32_t s_kw[kScoreQBlock][3];
  __shared__ int64_t s_out[kScoreQBlock];
  __shared__ unsigned long long s_any;
  const int64_t n0 = tile_i * tile;
  const int GQ = G.group;
  const int qn_total = batch * GQ;
  const int qb0 = qblock * kScoreQBlock;
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

template <int D, int RP>
__global__ void __launch_bounds__(kScoreThreads)
score_kernel(Geom G, int level, int64_t n_nodes, int64_t n_par, int32_t batch, int tile,
             const float* __restrict__ Q, const uint32_t* __restrict__ kept_up, int64_t words_up,
             float* __restrict__ sigma, const float* __restrict__ store) {
  pdl_trigger();
  pdl_wait();
  score_tile<D, RP>(G, level, n_nodes, n_par, batch, tile, blockIdx.x, blockIdx.y, blockIdx.z, Q,
                    kept_up, words_up, sigma, store);
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
//
// Candidates in candidate order (ascending node index): the children of the
// kept parents (compacted from the level above's bitmap), then the level's
// orphans. With at most kFastMax candidates every candidate's order key (score
// descending, then index ascending) and its softmax mass in 2^-31 fixed point
// are computed once into shared memory. The cut is then found in a window of
// keys [lo, lo + 2^span), narrowed pass by pass: a 2048-bin histogram of mass
// (and count) over the window's keys, the bin where the cumulative mass
// (with everything before the window) reaches p becomes the next window. Once
// the window holds at most kFastSmallN candidates, each of them counts the mass
// ordered before it among them (keys, then candidate index) and is kept iff
// that mass is below p -- the minimal prefix holding mass p. A window of one
// key (all tied) keeps its first candidates in candidate order. The rounding
// of the fixed-point masses adds at most n 2^-32 to any cumulative mass
// (< 4e-6 at n = 16384). Wider candidate sets (generic path): scores cached
// when they fit, masses recomputed per pass in 2^-40 fixed point, four radix
// passes of 8 bits with per-warp histograms. The fixed-budget mode (top-k)
// runs the same cut with a mass of exactly 1 per candidate and the threshold
// k, so it keeps the first
// min(k, n) candidates of the order.
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
  unsigned long long p_fixed;    // p in units of 2^-40 (generic path); top-k: k
  unsigned long long p_fixed31;  // p in units of 2^-31 (shared-memory path); top-k: k
  int keep_all;
  int topk;                  // fixed budget: every candidate weighs 1, the threshold is k
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

constexpr int kFastMax = 16384;
constexpr int kFastSmallN = kSelectThreads / 4;       // window size of the exact count
constexpr int kHistBins = (kSelectThreads / 32) * 256;   // generic path: per-warp 256-bin histograms
constexpr int kCutBins = 2048;                           // splitter histogram of the shared-memory path
constexpr int kBitsSmem = 4096;                          // kept-bitmap words held in shared memory
static_assert(kSelectCache <= kFastMax, "the generic path caches scores in the key array");
static_assert(2 * kCutBins * 4 + kFastSmallN * 4 + (kFastMax / 32) * 4 <= kHistBins * 8,
              "the splitter histograms, window list and flags share the histogram region");

__host__ __device__ constexpr size_t select_smem_bytes() {
  return size_t(2 * kFastMax) * sizeof(uint32_t) + size_t(kHistBins) * sizeof(unsigned long long) +
         size_t(kSelectKpCache) * sizeof(int32_t) + size_t(kBitsSmem) * sizeof(uint32_t);
}

// Shared memory of a select CTA (dynamic, select_smem_bytes()).
struct SelectSmem {
  uint32_t* s_key;               // [kFastMax] keys; the generic path's cached scores
  uint32_t* s_m;                 // [kFastMax] fixed-point masses
  unsigned long long* hist;      // [kHistBins] generic path; the shared-memory path uses the
                                 // region for hm, hc [kCutBins] u32, win [kFastSmallN] i32 and
                                 // flags [kFastMax / 32] u32
  int32_t* s_kp;                 // [kSelectKpCache] kept parents
  uint32_t* s_bits;              // [kBitsSmem] this level's kept bitmap when it fits
};

__device__ __forceinline__ SelectSmem select_smem() {
  extern __shared__ float4 smem_v4[];
  SelectSmem m;
  m.s_key = reinterpret_cast<uint32_t*>(smem_v4);
  m.s_m = m.s_key + kFastMax;
  m.hist = reinterpret_cast<unsigned long long*>(m.s_m + kFastMax);
  m.s_kp = reinterpret_cast<int32_t*>(m.hist + kHistBins);
  m.s_bits = reinterpret_cast<uint32_t*>(m.s_kp + kSelectKpCache);
  return m;
}

__device__ void select_level(const Geom& G, const SelectArgs& a, const SelectSmem& sm) {
  __shared__ float s_f[33];
  __shared__ unsigned long long s_u[33];
  __shared__ uint32_t s_w[33];
  __shared__ uint32_t s_bucket;
  __shared__ unsigned long long s_before;

  const int bh = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  const int C = G.chunk;
  // This level's kept bitmap: built in shared memory when it fits (written out
  // once at the end), else cleared and set in place in global memory.
  uint32_t* gbits = a.kept_here + int64_t(bh) * a.words_here;
  const bool bits_in_smem = a.words_here <= kBitsSmem;
  uint32_t* bits = bits_in_smem ? sm.s_bits : gbits;
  for (int64_t w = tid; w < a.words_here; w += blockDim.x) bits[w] = 0u;

  // Kept parents of this head, ascending (compaction of the level-(l+1) bitmap).
  // Parents fit in shared memory unless the level above is very wide.
  const bool kp_in_smem = a.words_up <= kSelectKpCache / 32;
  int32_t* kp = kp_in_smem ? sm.s_kp : a.kp + int64_t(bh) * a.kp_stride;
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
  __syncthreads();   // kp and the cleared bitmap visible to the block

  const int64_t orphan0 = int64_t(C) * a.n_par;
  const int64_t n_c64 = int64_t(n_kp) * C + (a.n_nodes - orphan0);
  // Candidate i -> node: child (i % C) of kept parent i / C, or an orphan.
  // Candidate and node indices fit 32 bits; the division is 32-bit.
  const uint32_t uC = uint32_t(C), u_nchild = n_kp * uC;
  auto node_of = [&](int64_t i) -> int64_t {
    const uint32_t ui = uint32_t(i);
    if (ui < u_nchild) {
      const uint32_t par = ui / uC;
      return int64_t(kp[par]) * C + (ui - par * uC);
    }
    return orphan0 + (ui - u_nchild);
  };
  const float* sig = a.sigma + int64_t(bh) * a.n_nodes;
  uint32_t kept_total = 0;

  if (n_c64 <= kFastMax) {
    // ---------------- all candidates in shared memory ----------------
    const int n_c = int(n_c64);
    uint32_t* s_key = sm.s_key;
    uint32_t* s_m = sm.s_m;
    float* s_sig = reinterpret_cast<float*>(s_key);
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

    // Softmax statistics, then keys and masses in 2^-31 fixed point (the same
    // arithmetic for every use of a candidate's mass; one candidate holds at
    // most 2^31, all of them together less than 2^32).
    float mx = -INFINITY;
    for (int i = tid; i < n_c; i += kSelectThreads) mx = fmaxf(mx, s_sig[i]);
    mx = block_max(mx, s_f);
    float z = 0.f;
    for (int i = tid; i < n_c; i += kSelectThreads) z += expf(s_sig[i] - mx);
    z = block_sum(z, s_f);
    const float scale31 = 2147483648.f / z;
    auto mass_of = [&](float s) -> uint32_t {
      return a.topk ? 1u : __float2uint_rn(expf(s - mx) * scale31);
    };
    unsigned long long tm = 0;
    uint32_t k_hi = 0u;
    for (int i = tid; i < n_c; i += kSelectThreads) {
      const float s = s_sig[i];
      const uint32_t m = mass_of(s);
      const uint32_t key = ~float_order_key(s);
      s_m[i] = m;
      s_key[i] = key;
      k_hi = max(k_hi, key);
      tm += m;
    }
    k_hi = __reduce_max_sync(0xffffffffu, k_hi);
    if (lane == 0) s_w[warp] = k_hi;
    unsigned long long total;
    block_excl_scan<unsigned long long>(tm, s_u, &total);      // its barriers publish s_key / s_m / s_w
    for (int w = 0; w < nw; ++w) k_hi = max(k_hi, s_w[w]);
    const uint32_t k_lo = ~float_order_key(mx);                 // the highest score has the lowest key
    const unsigned long long p31 = a.p_fixed31;
    const bool keep_all = a.keep_all != 0 || n_c == 0 || total < p31;
    __syncthreads();                                            // s_w is reused below

    // Kept predicate over candidate i, filled in below: key < lo keeps; a key
    // inside the cut window [lo, lo + 2^span) keeps by its flag, or (span 0:
    // one key, all tied) by its tie rank.
    uint32_t lo = 0u;
    int span = 0;
    unsigned long long before = 0ull, t_keep = 0ull;
    uint32_t* hm = reinterpret_cast<uint32_t*>(sm.hist);        // [kCutBins] mass per bin
    uint32_t* hc = hm + kCutBins;                               // [kCutBins] candidates per bin
    int32_t* win = reinterpret_cast<int32_t*>(hc + kCutBins);   // [kFastSmallN] window members
    uint32_t* flag = reinterpret_cast<uint32_t*>(win + kFastSmallN);   // [kFastMax / 32]
    if (!keep_all) {
      lo = k_lo;
      const uint32_t range = k_hi - k_lo;
      span = range == 0u ? 0 : 32 - __clz(range);
      uint32_t n_win = uint32_t(n_c);
      // Narrow the window to the splitter bin that holds the cut until it holds
      // few candidates (or one key). Every pass keeps before < p <= before +
      // (mass in the window).
      while (n_win > uint32_t(kFastSmallN) && span > 0) {
        const int shift = span > 11 ? span - 11 : 0;
        for (int b = tid; b < kCutBins; b += kSelectThreads) { hm[b] = 0u; hc[b] = 0u; }
        __syncthreads();
        for (int i = tid; i < n_c; i += kSelectThreads) {
          const uint32_t d = s_key[i] - lo;
          if (span == 32 || (d >> span) == 0u) {
            const uint32_t b = d >> shift;
            atomicAdd(&hm[b], s_m[i]);
            atomicAdd(&hc[b], 1u);
          }
        }
        __syncthreads();
        // first bin whose cumulative mass (with `before`) reaches p: thread t
        // owns bins [4t, 4t + 4)
        unsigned long long loc = 0ull;
#pragma unroll
        for (int j = 0; j < 4; ++j) loc += hm[4 * tid + j];
        unsigned long long tot_bins;
        unsigned long long acc = before + block_excl_scan<unsigned long long>(loc, s_u, &tot_bins);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t mj = hm[4 * tid + j];
          if (acc < p31 && acc + mj >= p31) {
            s_bucket = uint32_t(4 * tid + j);
            s_before = acc;
            s_w[32] = hc[4 * tid + j];
          }
          acc += mj;
        }
        __syncthreads();
        lo += s_bucket << shift;
        before = s_before;
        n_win = s_w[32];
        span = shift;
        __syncthreads();                                        // s_bucket / s_before / s_w reused
      }
      if (span == 0) {
        // One key in the window: the cut falls among tied candidates, taken in
        // candidate order.
        const uint32_t m_cut = mass_of(order_key_float(~lo));
        const unsigned long long need = p31 > before ? p31 - before : 0ull;
        t_keep = m_cut > 0u ? (need + m_cut - 1ull) / m_cut : 0ull;
      } else {
        // Few candidates in the window: each one counts the mass ordered before
        // it (key, then candidate index) among them.
        if (tid == 0) s_w[32] = 0u;
        for (int w = tid; w < (n_c + 31) / 32; w += kSelectThreads) flag[w] = 0u;
        __syncthreads();
        for (int i = tid; i < n_c; i += kSelectThreads) {
          const uint32_t d = s_key[i] - lo;
          if (span == 32 || (d >> span) == 0u) win[atomicAdd(&s_w[32], 1u)] = i;
        }
        __syncthreads();
        const int nwin = int(s_w[32]);
        // Four threads per window member (lanes 4m .. 4m + 3 of one warp), each
        // over every fourth other member, their partial masses summed by shuffles.
        const int mi = tid >> 2, part = tid & 3;
        unsigned long long cb = 0ull;
        int i = 0;
        if (mi < nwin) {
          i = win[mi];
          const uint32_t ki = s_key[i];
          for (int j = part; j < nwin; j += 4) {
            const int ij = win[j];
            const uint32_t kj = s_key[ij];
            if (kj < ki || (kj == ki && ij < i)) cb += s_m[ij];
          }
        }
        cb += __shfl_xor_sync(0xffffffffu, cb, 1);
        cb += __shfl_xor_sync(0xffffffffu, cb, 2);
        if (mi < nwin && part == 0) {
          cb += before;
          if (cb < p31) atomicOr(&flag[i >> 5], 1u << (i & 31));
        }
        __syncthreads();
      }
    }

    // Kept candidates in candidate order (ascending node index): thread-
    // contiguous ranges, positions by a scan.
    const int per = (n_c + kSelectThreads - 1) / kSelectThreads;
    const int i_lo = min(n_c, per * tid), i_hi = min(n_c, i_lo + per);
    uint32_t tie_rank = 0;
    if (!keep_all && span == 0) {
      uint32_t my_ties = 0, tie_total;
      for (int i = i_lo; i < i_hi; ++i) my_ties += (s_key[i] == lo);
      tie_rank = block_excl_scan<uint32_t>(my_ties, s_w, &tie_total);
    }
    auto kept = [&](int i, uint32_t& tr) -> bool {
      if (keep_all) return true;
      const uint32_t key = s_key[i];
      if (key < lo) return true;
      if (span == 0) return key == lo && tr++ < t_keep;
      return (flag[i >> 5] >> (i & 31)) & 1u;
    };
    uint32_t my_kept = 0;
    {
      uint32_t tr = tie_rank;
      for (int i = i_lo; i < i_hi; ++i) my_kept += kept(i, tr) ? 1u : 0u;
    }
    uint32_t pos = block_excl_scan<uint32_t>(my_kept, s_w, &kept_total);
    {
      uint32_t tr = tie_rank;
      for (int i = i_lo; i < i_hi; ++i) {
        if (!kept(i, tr)) continue;
        const int64_t node = node_of(i);
        atomicOr(&bits[node >> 5], 1u << (node & 31));
        if (a.chunk_ids != nullptr && pos < uint32_t(a.max_sel))
          a.chunk_ids[int64_t(bh) * a.max_sel + pos] = int32_t(node);
        ++pos;
      }
    }
  } else {
    // ---------------- generic path: more candidates than kFastMax ----------------
    const int64_t n_c = n_c64;
    float* s_sig = reinterpret_cast<float*>(sm.s_key);
    const bool cached = n_c <= kSelectCache;
    if (cached) {
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

    float mx = -INFINITY;
    for (int64_t i = tid; i < n_c; i += blockDim.x) mx = fmaxf(mx, sigma_of(i));
    mx = block_max(mx, s_f);
    float z = 0.f;
    for (int64_t i = tid; i < n_c; i += blockDim.x) z += expf(sigma_of(i) - mx);
    z = block_sum(z, s_f);
    const float inv_z = 1.f / z;
    auto mass_of = [&](float s) -> unsigned long long {
      return a.topk ? 1ull : __float2ull_rn(expf(s - mx) * inv_z * float(kMassScale));
    };

    // Cut: smallest key (score desc, index asc) whose cumulative mass reaches p.
    bool keep_all = a.keep_all != 0;
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
      unsigned long long* hist = sm.hist;
      unsigned long long* wh = hist + warp * 256;
      for (int shift = 24; shift >= 0; shift -= 8) {
        for (int k = lane; k < 256; k += 32) wh[k] = 0ull;
        __syncthreads();
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
        for (int k = tid; k < 256; k += blockDim.x) {
          unsigned long long v = 0;
          for (int w = 0; w < nw; ++w) v += hist[w * 256 + k];
          hist[k] = v;
        }
        __syncthreads();
        if (warp == 0) {
          unsigned long long loc[8], run = 0;
          for (int k = 0; k < 8; ++k) { loc[k] = hist[8 * lane + k]; run += loc[k]; }
          unsigned long long incl = warp_incl_scan<unsigned long long>(run);
          unsigned long long excl = incl - run;
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
  }
  if (a.chunk_ids != nullptr && tid == 0) {
    a.n_chunks[bh] = int32_t(kept_total);
    if (kept_total > uint32_t(a.max_sel) && a.status != nullptr)
      atomicOr(a.status, ZHA_DEV_SELECTION_TRUNCATED);
  }
  if (bits_in_smem) {
    __syncthreads();
    for (int64_t w = tid; w < a.words_here; w += blockDim.x) gbits[w] = sm.s_bits[w];
  }
}

// One level, one CTA per query head.
__global__ void __launch_bounds__(kSelectThreads)
select_fast_kernel(Geom G, SelectArgs a) {
  pdl_trigger();
  pdl_wait();
  forward_tree_status(a);
  select_level(G, a, select_smem());
}

// Levels top..bottom of a block of consecutive levels in one launch (the small
// top levels scored densely): each level's kept bitmap, written by this CTA,
// gives the next level's candidates after a CTA barrier.
struct SelectLevels {
  int32_t count;
  SelectArgs lv[ZHA_MAX_LEVELS];
};

__global__ void __launch_bounds__(kSelectThreads)
select_top_kernel(Geom G, SelectLevels t) {
  pdl_trigger();
  pdl_wait();
  forward_tree_status(t.lv[0]);
  const SelectSmem sm = select_smem();
  for (int i = 0; i < t.count; ++i) {
    select_level(G, t.lv[i], sm);
    __syncthreads();                 // this level's bitmap before the next level reads it
  }
}

cudaError_t launch_score_tc(const Geom& G, int level, int64_t n_nodes, int64_t n_par, int32_t batch,
                            const float* Q, const uint32_t* kept_up, int64_t words_up, float* sigma,
                            const float* store, int32_t* status, cudaStream_t s);
bool score_tma_supported(const Geom& G);
cudaError_t launch_score_tma(const Geom& G, int level, int64_t n_nodes, int64_t n_par, int32_t batch,
                             const float* Q, const uint32_t* kept_up, int64_t words_up, float* sigma,
                             const float* store, int32_t* status, cudaStream_t s, bool* used);

// ---------------------------------------------------------------------------
// Host launcher. Levels L..1. The small top levels (at most kDenseMaxNodes
// nodes per KV head each, kDenseMaxTotal nodes over all KV heads together) are
// scored densely in one launch and selected in one launch; every lower level is
// scored over its candidates (score_tma_kernel, score_tc_kernel or
// score_kernel) and then selected.
// ---------------------------------------------------------------------------
constexpr int64_t kDenseMaxNodes = 1024;
constexpr int64_t kDenseMaxTotal = 8192;

template <int D, int RP>
static size_t score_smem_bytes(const Geom& G, int32_t batch) {
  using S = ScoreShape<D, RP>;
  const int qn = batch * G.group;
  return (size_t(kScoreThreads / 32) * S::KBUF +
          size_t(qn < kScoreQBlock ? qn : kScoreQBlock) * S::QROW) * 4;
}

// Nodes per CTA: enough CTAs to fill the GPU twice over, at most kScoreTile.
static int score_tile_for(int64_t n_nodes, int hkv) {
  int tile = kScoreTile;
  while (tile > kScoreThreads / 32 && (n_nodes * hkv) / tile < 2 * 148) tile >>= 1;
  return tile;
}

template <int D, int RP>
static cudaError_t launch_score_t(const Geom& G, int level, int64_t n_nodes, int64_t n_par,
                                  int32_t batch, const float* Q, const uint32_t* kept_up,
                                  int64_t words_up, float* sigma, const float* store,
                                  cudaStream_t s) {
  const int qn = batch * G.group;
  const int tile = score_tile_for(n_nodes, G.hkv);
  dim3 grid(unsigned((n_nodes + tile - 1) / tile), unsigned(G.hkv),
            unsigned((qn + kScoreQBlock - 1) / kScoreQBlock));
  const size_t smem = score_smem_bytes<D, RP>(G, batch);
  cudaError_t e = ensure_dynamic_smem(score_kernel<D, RP>, smem);
  if (e != cudaSuccess) return e;
  TraceScope ts("score_kernel", level, s);
  e = launch_pdl(score_kernel<D, RP>, grid, dim3(kScoreThreads), smem, s, G, level, n_nodes, n_par,
                 batch, tile, Q, kept_up, words_up, sigma, store);
  zha_count_launch();
  return e;
}

template <int D>
static cudaError_t launch_dense_t(const Geom& G, const DenseLevels& dl, int32_t batch, const float* Q,
                                  const float* store, cudaStream_t s) {
  const int qn = batch * G.group;
  dim3 grid(unsigned(dl.tile0[dl.count]), unsigned(G.hkv), unsigned((qn + kDenseQ - 1) / kDenseQ));
  const size_t smem = dense_smem_bytes<D>();
  cudaError_t e = ensure_dynamic_smem(score_dense_kernel<D, false>, smem);
  if (e != cudaSuccess) return e;
  TraceScope ts("score_dense_kernel", dl.level[dl.count - 1], s);
  e = launch_pdl(score_dense_kernel<D, false>, grid, dim3(kDenseThreads), smem, s, G, dl, batch, Q, store,
                 static_cast<uint32_t*>(nullptr));
  zha_count_launch();
  return e;
}

// Planes are padded to a power of two RP >= 128 / D so that each lane holds at
// least one float4 of its plane's row.
#define ZHA_SCORE_DISPATCH(CALL)                      \
  do {                                                \
    const int R = G.nref;                             \
    if (G.d == 128) {                                 \
      constexpr int D = 128;                          \
      if (R <= 1) { constexpr int RP = 1; CALL; }     \
      if (R <= 2) { constexpr int RP = 2; CALL; }     \
      if (R <= 4) { constexpr int RP = 4; CALL; }     \
      if (R <= 8) { constexpr int RP = 8; CALL; }     \
      if (R <= 16) { constexpr int RP = 16; CALL; }   \
      if (R <= 32) { constexpr int RP = 32; CALL; }   \
    } else {                                          \
      constexpr int D = 64;                           \
      if (R <= 2) { constexpr int RP = 2; CALL; }     \
      if (R <= 4) { constexpr int RP = 4; CALL; }     \
      if (R <= 8) { constexpr int RP = 8; CALL; }     \
      if (R <= 16) { constexpr int RP = 16; CALL; }   \
      if (R <= 32) { constexpr int RP = 32; CALL; }   \
    }                                                 \
    return cudaErrorInvalidValue;                     \
  } while (0)

static cudaError_t launch_score_simt(const Geom& G, int level, int64_t n_nodes, int64_t n_par,
                                     int32_t batch, const float* Q, const uint32_t* kept_up,
                                     int64_t words_up, float* sigma, const float* store,
                                     cudaStream_t s) {
  ZHA_SCORE_DISPATCH(return (launch_score_t<D, RP>(G, level, n_nodes, n_par, batch, Q, kept_up,
                                                    words_up, sigma, store, s)));
}

#undef ZHA_SCORE_DISPATCH

static cudaError_t launch_dense(const Geom& G, const DenseLevels& dl, int32_t batch, const float* Q,
                                const float* store, cudaStream_t s) {
  return G.d == 128 ? launch_dense_t<128>(G, dl, batch, Q, store, s)
                    : launch_dense_t<64>(G, dl, batch, Q, store, s);
}

cudaError_t launch_route(const Geom& G, const float* Q, int32_t batch, int64_t n_tokens,
                         const RoutePolicy& pol, int32_t* chunk_ids, int32_t* n_chunks,
                         int32_t max_sel, uint32_t* bits, float* sigma, int32_t* kp,
                         const RouteLayout& lay, int32_t* status, const float* store,
                         cudaStream_t s) {
  const size_t smem = select_smem_bytes();
  cudaError_t e = ensure_dynamic_smem(select_fast_kernel, smem);
  if (e != cudaSuccess) return e;
  if ((e = ensure_dynamic_smem(select_top_kernel, smem)) != cudaSuccess) return e;
  const int heads = batch * G.hq;
  SelectArgs base{};
  base.kp = kp;
  base.kp_stride = lay.kp_ints / (heads > 0 ? heads : 1);
  base.max_sel = max_sel;
  base.status = status;
  auto args_for = [&](int level) {
    SelectArgs a = base;
    a.level = level;
    if (pol.topk) {
      a.topk = 1;
      a.p_fixed = a.p_fixed31 = (unsigned long long)pol.k[level];
      a.keep_all = 0;
    } else {
      const double p = double(pol.p[level]);
      a.p_fixed = (unsigned long long)ceil(p * kMassScale);
      if (a.p_fixed == 0) a.p_fixed = 1;
      a.p_fixed31 = (unsigned long long)ceil(p * 2147483648.0);
      if (a.p_fixed31 == 0) a.p_fixed31 = 1;
      a.keep_all = pol.p[level] >= 1.0f;
    }
    a.n_nodes = lay.n[level];
    a.n_par = level < G.levels ? lay.n[level + 1] : 0;
    a.kept_up = level < G.levels ? bits + lay.bits_off[level + 1] : nullptr;
    a.words_up = level < G.levels ? lay.words[level + 1] : 0;
    a.kept_here = bits + lay.bits_off[level];
    a.words_here = lay.words[level];
    a.sigma = sigma + lay.sig_off[level];
    a.chunk_ids = level == 1 ? chunk_ids : nullptr;
    a.n_chunks = level == 1 ? n_chunks : nullptr;
    a.tree_status = level == G.levels ? tree_status_word(G, const_cast<float*>(store)) : nullptr;
    return a;
  };

  // The dense block: levels L..l0 (l0 >= 2).
  int l0 = G.levels + 1;
  {
    int64_t total = 0;
    for (int level = G.levels; level >= 2; --level) {
      const int64_t n = lay.n[level];
      if (n > kDenseMaxNodes || total + n * G.hkv > kDenseMaxTotal) break;
      total += n * G.hkv;
      l0 = level;
    }
  }
  if (l0 <= G.levels) {
    DenseLevels dl{};
    int64_t t0 = 0;
    for (int level = G.levels; level >= l0; --level) {
      if (lay.n[level] == 0) continue;
      const int i = dl.count++;
      const int npt = kDenseRows / G.nref;              // nodes per tile
      dl.level[i] = level;
      dl.n_nodes[i] = lay.n[level];
      dl.tile0[i] = t0;
      dl.sigma[i] = sigma + lay.sig_off[level];
      t0 += (lay.n[level] + npt - 1) / npt;
    }
    dl.tile0[dl.count] = t0;
    if (dl.count > 0 && (e = launch_dense(G, dl, batch, Q, store, s)) != cudaSuccess) return e;
    SelectLevels sl{};
    for (int level = G.levels; level >= l0; --level) sl.lv[sl.count++] = args_for(level);
    {
      TraceScope ts("select_top_kernel", l0, s);
      e = launch_pdl(select_top_kernel, dim3(heads), dim3(kSelectThreads), smem, s, G, sl);
    }
    if (e != cudaSuccess) return e;
    zha_count_launch();
  }
  for (int level = l0 - 1; level >= 1; --level) {
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
        e = launch_score_simt(G, level, n_nodes, n_par, batch, Q, up, words_up, sg, store, s);
      if (e != cudaSuccess) return e;
    }
    const SelectArgs a = args_for(level);
    {
      TraceScope ts("select_fast_kernel", level, s);
      e = launch_pdl(select_fast_kernel, dim3(heads), dim3(kSelectThreads), smem, s, G, a);
    }
    if (e != cudaSuccess) return e;
    zha_count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace zha
