// zha_build_tc.cu -- level-1 tree build on the sm_100a tensor cores (bf16
// caches, head_dim 128, R = 16, C = 16, 32, 64 or 128).
//
// Citations: [ZHA: 무엇과 다른가] = page "ZHA는 KV 캐시를 트리로 요약해 어텐션 비용을
// 준(sub)이차로 낮춘다" (onedev.kr/papers/1556), section "무엇과 다른가": the chunk's
// log mass F_C(q) = LSE_j(q.k_j/sqrt(d)), its tangent plane at reference query
// q_r with khat_r = Attn(q_r, K_C, K_C) and bhat_r = F_C(q_r) - q_r.khat_r/sqrt(d).
//
// Per tile of 128 tokens (128 / C chunks) of one KV head g:
//   S[t][r]  = k_t . q_r / sqrt(d)          tcgen05.mma, A = K tile (K-major),
//                                           B = q in three bf16 terms stacked
//                                           along N (N = 48), TMEM [128][48]
//   per (chunk, plane): F = LSE_t S, W[t][r] = exp(S - F)   (softmax warps; a
//                                           chunk's rows are half a warp (C = 16),
//                                           one warp or several)
//   khat^T[d][r] = sum_t K[t][d] W[t][r]    tcgen05.mma per chunk, A = the same
//                                           K tile read MN-major (M = d), B = W
//                                           in two bf16 terms (N = 32)
//   bhat_r = F - q_r . khat_r / sqrt(d)     epilogue (thread = d row)
// Roles: warp 0 tensor copies of K (2 stages; rows past the built prefix read
// as zeros), warp 1 MMA issuer, warps 2-5 softmax (thread = token row), warps
// 6-9 epilogue (thread = d row); each group covers the TMEM lane quadrants 2,
// 3, 0, 1. W, F and the khat accumulators are double-buffered (khat when two
// buffers fit in TMEM), so the epilogue of one tile overlaps the softmax of
// the next. Every wait is bounded.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "zha_host.cuh"
#include "zha_internal.cuh"
#include "zha_tc.cuh"

namespace zha {

namespace {

constexpr int bTok = 128, bD = 128, bR = 16;
constexpr int bStages = 2;
constexpr int bStageBytes = 32768;                   // K tile [2 halves][128 rows][128 B]
constexpr int bOffQ = bStages * bStageBytes;         // [2 halves][48 rows][128 B]
constexpr int bWBytes = 8192;                        // W [128 tokens][32 = 16 planes x 2 terms] SW64
constexpr int bOffW = bOffQ + 2 * 6144;              // two W buffers
constexpr int bOffMisc = bOffW + 2 * bWBytes;
constexpr int bThreads = 320;                        // warps: 0 copies, 1 MMA, 2-5 softmax, 6-9 epilogue
constexpr uint32_t bTmemK = 64;                      // S at 0 (48 cols), khat buffers from 64 (32 per chunk)
constexpr int bMaxChunks = bTok / 16;                // chunks per tile at C = 16

// khat buffers in TMEM: two when they fit in 256 columns after S, else one.
__host__ __device__ inline int build_khat_bufs(int chunk) {
  return bTmemK + 2u * uint32_t(bTok / chunk) * 32u <= 256u ? 2 : 1;
}
// TMEM columns of a CTA.
__host__ __device__ inline uint32_t build_tmem_cols(int chunk) {
  return bTmemK + uint32_t(build_khat_bufs(chunk) * (bTok / chunk)) * 32u <= 256u ? 256u : 512u;
}

struct BMisc {
  uint64_t full[bStages], empty[bStages], s_full, s_free, w_ready[2], k_full[2], k_free[2], q_ready, drain;
  uint32_t tmem_base, err;
  float red_max[bMaxChunks][bR];                     // softmax: per reduction unit (half-warp, warp)
  float red_sum[bMaxChunks][bR];
  float F[2][bMaxChunks][bR];                        // per W buffer and chunk of the tile
  float red_e[2][bMaxChunks][4][bR];                 // epilogue: q_r . khat partial sums per warp
};

// Reduction of 16 values (one per plane) over lanes: afterwards lane L holds
// plane L & 15 reduced over its half-warp, or over the whole warp (full).
__device__ __forceinline__ float tr16(float (&v)[16], bool is_max, bool full = true) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 8, half = 8; o > 0; o >>= 1, half >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? v[i] : v[i + half];
      const float keep = upper ? v[i + half] : v[i];
      const float got = __shfl_xor_sync(0xffffffffu, send, o);
      v[i] = is_max ? fmaxf(keep, got) : keep + got;
    }
  }
  if (!full) return v[0];
  const float other = __shfl_xor_sync(0xffffffffu, v[0], 16);
  return is_max ? fmaxf(v[0], other) : v[0] + other;
}

}  // namespace

// Tiles li = 0, 1, ... of the CTA; W and F buffer wb = li & 1, khat buffer
// kb = li % kbufs. Barrier waits and the phases they expect:
//   MMA       S(li + 1): full[stage] and s_free (li);  khat(li): w_ready[wb] (li)
//             and k_free (tile li - kbufs: the epilogue has read that buffer)
//   softmax   s_full (li); k_free (li - kbufs: W[wb], F[wb] and the khat buffer
//             of tile li - 2 or li - 1 are read)
//   epilogue  w_ready[wb] (li: F of the tile), k_full[kb] (li)
// None of these barriers can complete the phase after the awaited one before
// its waiter has passed (each later completion depends on the waiter), so
// parity waits are unambiguous. The MMA order S(0), S(1), khat(0), S(2),
// khat(1), ... waits only on work issued before it.
__global__ void __launch_bounds__(bThreads, 2)
build_l1_tc_kernel(const __grid_constant__ CUtensorMap tmK, Geom G, int64_t c_begin, int64_t c_end,
                   const float* __restrict__ refq, float* __restrict__ store, int32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  BMisc& ms = *reinterpret_cast<BMisc*>(smem + bOffMisc);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = blockIdx.y;
  const int C = G.chunk, cpt = bTok / C;
  const int kbufs = build_khat_bufs(C);
  const int64_t n_tiles = (c_end - c_begin + cpt - 1) / cpt;
  const uint32_t kTries = G.wait_polls;
  const uint32_t tmem_cols = build_tmem_cols(C);

  if (tid == 0) {
    ms.err = 0u;
    for (int s = 0; s < bStages; ++s) {
      tc::mbar_init(&ms.full[s], 1);
      tc::mbar_init(&ms.empty[s], 1);
    }
    tc::mbar_init(&ms.s_full, 1);
    tc::mbar_init(&ms.s_free, 4);                   // one arrival per warp of a warpgroup
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&ms.w_ready[b], 4);
      tc::mbar_init(&ms.k_full[b], 1);
      tc::mbar_init(&ms.k_free[b], 4);
    }
    tc::mbar_init(&ms.q_ready, 4);
    tc::mbar_init(&ms.drain, 1);
  }
  if (warp == 1) tc::tmem_alloc(&ms.tmem_base, tmem_cols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = ms.tmem_base;
  // this CTA's tiles of head g: t = blockIdx.x, blockIdx.x + gridDim.x, ...
  const int64_t my_tiles = n_tiles > blockIdx.x ? (n_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  auto khat_col = [&](int64_t li) -> uint32_t {
    return bTmemK + uint32_t(li % kbufs) * uint32_t(cpt) * 32u;
  };

  if (warp == 0) {
    if (lane == 0) {
      int64_t li = 0;
      for (; li < my_tiles; ++li) {
        const int64_t t = blockIdx.x + li * gridDim.x;
        const int st = int(li % bStages);
        const int64_t use = li / bStages;
        if (use > 0 && !tc::mbar_wait(&ms.empty[st], uint32_t((use - 1) & 1), kTries)) {
          atomicOr(&ms.err, 1u);
          break;
        }
        const int32_t tok0 = int32_t((c_begin + t * cpt) * C);
        const uint32_t dst = tc::smem_u32(smem + st * bStageBytes);
        tc::mbar_arrive_expect_tx(&ms.full[st], uint32_t(bStageBytes));
        tc::tma_load_3d(dst, &tmK, 0, tok0, g, &ms.full[st]);
        tc::tma_load_3d(dst + 16384, &tmK, 64, tok0, g, &ms.full[st]);
      }
      // Every tensor copy issued lands before the CTA may exit.
      for (int64_t j = li > bStages ? li - bStages : 0; j < li; ++j)
        if (!tc::mbar_wait(&ms.full[j % bStages], uint32_t((j / bStages) & 1), kTries)) atomicOr(&ms.err, 1u);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = tc::idesc_bf16(bTok, 3 * bR, 0, 0);
      constexpr uint32_t idesc_k = tc::idesc_bf16(bD, 2 * bR, 1, 1);
      const uint32_t sQ = tc::smem_u32(smem + bOffQ);
      bool failed = my_tiles > 0 && !tc::mbar_wait(&ms.q_ready, 0u, kTries);
      int64_t ns = 0;                                // next tile to score
      auto issue_s = [&]() -> bool {
        const int st = int(ns % bStages);
        if (!tc::mbar_wait(&ms.full[st], uint32_t((ns / bStages) & 1), kTries)) return false;
        if (ns > 0 && !tc::mbar_wait(&ms.s_free, uint32_t((ns - 1) & 1), kTries)) return false;
        tc::fence_after_sync();
        const uint32_t sK = tc::smem_u32(smem + st * bStageBytes);
#pragma unroll
        for (int ks = 0; ks < bD / 16; ++ks) {
          const uint64_t a = tc::desc_sw128(sK + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
          const uint64_t b = tc::desc_sw128(sQ + (ks >> 2) * 6144 + (ks & 3) * 32, 16, 1024);
          tc::mma_bf16(tbase, a, b, idesc_s, ks != 0 ? 1u : 0u);
        }
        tc::mma_commit(&ms.s_full);
        ++ns;
        return true;
      };
      auto issue_k = [&](int64_t li) -> bool {
        const int wb = int(li & 1);
        if (!tc::mbar_wait(&ms.w_ready[wb], uint32_t((li >> 1) & 1), kTries)) return false;
        if (li >= kbufs) {
          const int64_t lp = li - kbufs;
          if (!tc::mbar_wait(&ms.k_free[lp % kbufs], uint32_t((lp / kbufs) & 1), kTries)) return false;
        }
        tc::fence_after_sync();
        const int st = int(li % bStages);
        const uint32_t sK = tc::smem_u32(smem + st * bStageBytes);
        const uint32_t sW = tc::smem_u32(smem + bOffW + wb * bWBytes);
        const uint32_t dk = tbase + khat_col(li);
        for (int c = 0; c < cpt; ++c) {
          for (int kk = 0; kk < C / 16; ++kk) {
            const int ks = c * (C / 16) + kk;              // 16-token K-step of the tile
            const uint64_t a = tc::desc_sw128(sK + ks * 2048, 16384, 1024);
            const uint64_t b = tc::desc_sw64(sW + ks * 1024, 8192, 512);
            tc::mma_bf16(dk + uint32_t(c) * 32, a, b, idesc_k, kk != 0 ? 1u : 0u);
          }
        }
        tc::mma_commit(&ms.k_full[li % kbufs]);
        tc::mma_commit(&ms.empty[st]);
        return true;
      };
      if (!failed && my_tiles > 0) failed = !issue_s();
      for (int64_t li = 0; li < my_tiles && !failed; ++li) {
        if (ns < my_tiles && !issue_s()) { failed = true; break; }
        if (!issue_k(li)) failed = true;
      }
      // Every MMA issued completes before TMEM is released.
      tc::mma_commit(&ms.drain);
      if (!tc::mbar_wait(&ms.drain, 0u, kTries)) failed = true;
      if (failed) atomicOr(&ms.err, 1u);
    }
  } else if (warp < 6) {
    // ---------------- softmax (warps 2-5): thread = token row ----------------
    const int q4 = warp & 3;                        // TMEM lane quadrant
    const int r = q4 * 32 + lane;                   // token row of the tile
    const uint32_t t_lane = uint32_t(q4 * 32) << 16;
    const int stid = tid - 64;                      // 0..127
    const float* qg = refq + int64_t(g) * bR * bD;
    // Q stack: rows term * 16 + plane, 3 bf16 terms, K-major SW128 [2 halves][48][128 B]
    for (int v = stid; v < bR * (bD / 8); v += 128) {
      const int pl = v / (bD / 8), col = (v % (bD / 8)) * 8;
      float x[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = qg[pl * bD + col + i];
#pragma unroll
      for (int term = 0; term < 3; ++term) {
        __align__(16) __nv_bfloat16 h[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          h[i] = __float2bfloat16_rn(x[i]);
          x[i] -= __bfloat162float(h[i]);
        }
        const int row = term * bR + pl;
        const uint32_t off = uint32_t((col >> 6) * 6144 + (row >> 3) * 1024 + (row & 7) * 128 +
                                      ((((col & 63) >> 3) ^ (row & 7)) << 4));
        *reinterpret_cast<uint4*>(smem + bOffQ + off) = *reinterpret_cast<const uint4*>(h);
      }
    }
    tc::fence_async_smem();
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(&ms.q_ready);
    // Reduction units: a chunk of C >= 32 rows spans C / 32 warps (unit = warp),
    // a chunk of 16 rows is half a warp (unit = half-warp).
    const bool half_units = C < 32;
    const int chunk_of_row = r / C, units = half_units ? 1 : C / 32;
    const int unit = half_units ? 2 * q4 + (lane >> 4) : q4, unit0 = chunk_of_row * units;
    bool failed = false;
    for (int64_t li = 0; li < my_tiles; ++li) {
      const int wb = int(li & 1);
      bool bad = !tc::mbar_wait(&ms.s_full, uint32_t(li & 1), kTries);
      tc::fence_after_sync();
      float s[bR];
      {
        float w1[bR], w2[bR];
        tc::tmem_ld16(tbase + t_lane, s);
        tc::tmem_ld16(tbase + t_lane + 16, w1);
        tc::tmem_ld16(tbase + t_lane + 32, w2);
#pragma unroll
        for (int i = 0; i < bR; ++i) s[i] = (s[i] + w1[i] + w2[i]) * G.scale;
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&ms.s_free);
      // W[wb] and F[wb] are free once the epilogue of tile li - kbufs is done
      // (it waited for the khat MMA that read W[wb]).
      if (li >= kbufs) {
        const int64_t lp = li - kbufs;
        bad |= !tc::mbar_wait(&ms.k_free[lp % kbufs], uint32_t((lp / kbufs) & 1), kTries);
      }
      // per (chunk, plane) maximum and sum over the chunk's rows
      float tmp[bR];
#pragma unroll
      for (int i = 0; i < bR; ++i) tmp[i] = s[i];
      const float wm = tr16(tmp, true, !half_units);
      if (half_units || lane < bR) ms.red_max[unit][lane & 15] = wm;
      if (tc::named_sync_or(1, 128, bad)) { failed = true; break; }
      float m[bR];
#pragma unroll
      for (int i = 0; i < bR; ++i) {
        float x = -INFINITY;
        for (int w = 0; w < units; ++w) x = fmaxf(x, ms.red_max[unit0 + w][i]);
        m[i] = x;
      }
#pragma unroll
      for (int i = 0; i < bR; ++i) tmp[i] = expf(s[i] - m[i]);
      const float wl = tr16(tmp, false, !half_units);
      if (half_units || lane < bR) ms.red_sum[unit][lane & 15] = wl;
      tc::named_sync(1, 128);
      float F[bR];
#pragma unroll
      for (int i = 0; i < bR; ++i) {
        float l = 0.f;
        for (int w = 0; w < units; ++w) l += ms.red_sum[unit0 + w][i];
        F[i] = m[i] + logf(l);
      }
      if (r % C == 0) {
#pragma unroll
        for (int i = 0; i < bR; ++i) ms.F[wb][chunk_of_row][i] = F[i];
      }
      // W = exp(S - F) in two bf16 terms, MN-major: token row, 16 planes hi then lo (64 B)
      {
        __align__(16) __nv_bfloat16 hi[bR], lo[bR];
#pragma unroll
        for (int i = 0; i < bR; ++i) {
          const float w = expf(s[i] - F[i]);
          hi[i] = __float2bfloat16_rn(w);
          lo[i] = __float2bfloat16_rn(w - __bfloat162float(hi[i]));
        }
        uint8_t* sW = smem + bOffW + wb * bWBytes;
        *reinterpret_cast<uint4*>(sW + tc::sw64_mn_chunk(r, 0)) = *reinterpret_cast<const uint4*>(hi);
        *reinterpret_cast<uint4*>(sW + tc::sw64_mn_chunk(r, 1)) = *reinterpret_cast<const uint4*>(hi + 8);
        *reinterpret_cast<uint4*>(sW + tc::sw64_mn_chunk(r, 2)) = *reinterpret_cast<const uint4*>(lo);
        *reinterpret_cast<uint4*>(sW + tc::sw64_mn_chunk(r, 3)) = *reinterpret_cast<const uint4*>(lo + 8);
      }
      tc::fence_async_smem();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&ms.w_ready[wb]);
    }
    if (failed && stid == 0) atomicOr(&ms.err, 1u);
  } else {
    // ---------------- epilogue (warps 6-9): thread = output dim d ----------------
    const int q4 = warp & 3;                        // TMEM lane quadrant
    const int r = q4 * 32 + lane;                   // d row
    const uint32_t t_lane = uint32_t(q4 * 32) << 16;
    const int etid = tid - 192;                     // 0..127
    const float* qg = refq + int64_t(g) * bR * bD;
    float qd[bR];                                   // q_r[d] for this thread's d row
#pragma unroll
    for (int pl = 0; pl < bR; ++pl) qd[pl] = qg[pl * bD + r];
    bool failed = false;
    for (int64_t li = 0; li < my_tiles; ++li) {
      const int64_t t = blockIdx.x + li * gridDim.x;
      const int64_t chunk0 = c_begin + t * cpt;
      const int wb = int(li & 1), kb = int(li % kbufs);
      bool bad = !tc::mbar_wait(&ms.w_ready[wb], uint32_t((li >> 1) & 1), kTries);   // F of the tile
      bad |= !tc::mbar_wait(&ms.k_full[kb], uint32_t((li / kbufs) & 1), kTries);
      tc::fence_after_sync();
      const uint32_t dk = tbase + t_lane + khat_col(li);
      for (int c = 0; c < cpt; ++c) {
        float kh[bR], kl[bR], tmp[bR];
        tc::tmem_ld16(dk + uint32_t(c) * 32, kh);
        tc::tmem_ld16(dk + uint32_t(c) * 32 + 16, kl);
        const int64_t node = chunk0 + c;
        const bool live = !bad && node < c_end;
        float* rec = store + G.off[1] + (int64_t(g) * G.cap[1] + node) * G.node_floats;
#pragma unroll
        for (int i = 0; i < bR; ++i) {
          kh[i] += kl[i];
          if (live) rec[i * bD + r] = kh[i];
          tmp[i] = kh[i] * qd[i];
        }
        const float dsum = tr16(tmp, false);
        if (lane < bR) ms.red_e[wb][c][q4][lane] = dsum;
      }
      if (tc::named_sync_or(2, 128, bad)) { failed = true; break; }
      // bhat_r = F - q_r . khat_r / sqrt(d) for every (chunk, plane) of the tile
      for (int v = etid; v < cpt * bR; v += 128) {
        const int c = v / bR, i = v % bR;
        const int64_t node = chunk0 + c;
        if (node < c_end) {
          const float dot = ms.red_e[wb][c][0][i] + ms.red_e[wb][c][1][i] + ms.red_e[wb][c][2][i] +
                            ms.red_e[wb][c][3][i];
          store[G.off[1] + (int64_t(g) * G.cap[1] + node) * G.node_floats + bR * bD + i] =
              ms.F[wb][c][i] - dot * G.scale;
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&ms.k_free[kb]);
    }
    if (failed && etid == 0) atomicOr(&ms.err, 1u);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, tmem_cols);
  }
  if (tid == 0 && ms.err != 0u && status != nullptr) atomicOr(status, ZHA_DEV_TIMEOUT);
}

// Level-1 summaries of chunks [c_begin, c_end) with the tensor cores; returns
// cudaErrorNotSupported when the configuration is not covered (the caller then
// uses the CUDA-core build).
cudaError_t launch_build_level1_tc(const Geom& G, const void* K, int64_t ld, int64_t c_begin,
                                   int64_t c_end, const float* refq, float* store, int32_t* status,
                                   cudaStream_t s) {
  const bool chunk_ok = G.chunk == 16 || G.chunk == 32 || G.chunk == 64 || G.chunk == 128;
  if (!(G.kv_bf16 && G.d == bD && G.nref == bR && chunk_ok && G.rope_pairs == 0))
    return cudaErrorNotSupported;
  if (c_end <= c_begin) return cudaSuccess;
  const PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (fn == nullptr) return cudaErrorNotSupported;
  CUtensorMap map{};
  const cuuint64_t dims[3] = {cuuint64_t(bD), cuuint64_t(c_end * G.chunk), cuuint64_t(G.hkv)};
  const cuuint64_t strides[2] = {cuuint64_t(bD) * 2, cuuint64_t(ld) * bD * 2};
  const cuuint32_t box[3] = {64u, cuuint32_t(bTok), 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  if (fn(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(K), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorNotSupported;
  const size_t smem = size_t(bOffMisc) + sizeof(BMisc) + 1024;
  cudaError_t e = ensure_dynamic_smem(build_l1_tc_kernel, smem);
  if (e != cudaSuccess) return e;
  int sms = 148;
  if ((e = device_sm_count(&sms)) != cudaSuccess) return e;
  const int cpt = bTok / G.chunk;
  const int64_t tiles = (c_end - c_begin + cpt - 1) / cpt;
  // two CTAs per SM when both fit in tensor memory, else one
  const int per_sm = build_tmem_cols(G.chunk) <= 256u ? 2 : 1;
  int64_t per_head = (per_sm * int64_t(sms) + G.hkv - 1) / G.hkv;
  if (per_head > tiles) per_head = tiles;
  TraceScope ts("build_l1_tc_kernel", 1, s);
  build_l1_tc_kernel<<<dim3(unsigned(per_head), unsigned(G.hkv)), bThreads, smem, s>>>(
      map, G, c_begin, c_end, refq, store, status);
  zha_count_launch();
  return cudaGetLastError();
}

}  // namespace zha
