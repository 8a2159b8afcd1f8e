// zha_internal.cuh -- geometry, layouts and device helpers shared by the
// kernels and the C-ABI host code of libzha (not part of the public ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "zha.h"

#define ZHA_MAX_LEVELS 8
#define ZHA_MAX_REF 32
#define ZHA_MAX_CHUNK 128

namespace zha {

// ---------------------------------------------------------------------------
// Geometry of one tree configuration, passed by value to kernels.
// ---------------------------------------------------------------------------
struct Geom {
  int32_t hkv, hq, group, d, chunk, levels, nref, node_floats;
  int32_t kv_bf16;
  float scale;                           // 1 / sqrt(d)
  int32_t rope_pairs;                    // rotated element pairs (0: position-free)
  double rope_log2_base;                 // log2 of the rotation base
  uint32_t wait_polls;                   // polls of a bounded mbarrier wait before it gives up
  int32_t debug_withhold;                // test hook: the level scoring's producer sends nothing
  int64_t max_tokens;
  int64_t cap[ZHA_MAX_LEVELS + 2];       // node capacity per KV head, index by level
  int64_t off[ZHA_MAX_LEVELS + 2];       // float offset of level l's [hkv][cap][node] block
  int64_t status_off;                    // float offset of the tree's device status word
  // Byte offset of level l's planes as two fp16 terms, [hkv][2][cap][R][d]
  // (t0 = x rounded to fp16, t1 = x - t0 rounded to fp16), for the tensor-core
  // scoring of head_dim 128, R = 16; 0 when the store has no such copy.
  int64_t split_off[ZHA_MAX_LEVELS + 2];
};

// Whether the store carries fp16 plane terms (the tensor-core scoring's operand).
__host__ __device__ inline bool has_plane_terms(const Geom& g) { return g.d == 128 && g.nref == 16; }

// The tree's device status word (ZHA_DEV_* bits of the build kernels), in the
// 256-byte block that follows the summary levels in the store.
__host__ __device__ inline int32_t* tree_status_word(const Geom& g, float* store) {
  return reinterpret_cast<int32_t*>(store + g.status_off);
}

// Rotation of element pair i at position pos: angle pos * base^(-2i/d),
// formed and reduced modulo 2 pi in double precision (positions reach 2^34),
// then turned into the cosine and sine. Pairs from G.rope_pairs on do not turn.
__device__ __forceinline__ void rope_cos_sin(const Geom& G, int64_t pos, int pair, float* c, float* s) {
  if (pair >= G.rope_pairs || pos == 0) {
    *c = 1.f;
    *s = 0.f;
    return;
  }
  const double theta = exp2(-2.0 * double(pair) / double(G.d) * G.rope_log2_base);
  const double two_pi = 6.283185307179586476925286766559;
  double ang = double(pos) * theta;
  ang -= two_pi * floor(ang / two_pi);
  double sd, cd;
  sincos(ang, &sd, &cd);
  *c = float(cd);
  *s = float(sd);
}

// ---------------------------------------------------------------------------
// A K/V cache as the kernels see it: contiguous [Hkv][ld][d], or paged -- a
// pool of pages of C tokens [n_pages][C][d] and a block table [Hkv][max_blocks]
// giving the page of each chunk of each KV head (ld then counts the pages).
// ---------------------------------------------------------------------------
struct KvView {
  const void* k;
  const void* v;
  int64_t ld;                  // contiguous: tokens per KV head block; paged: pages in the pool
  const int32_t* table;        // nullptr: contiguous
  int64_t max_blocks;
};

// Row (token slot) of token `tok` of KV head g in the cache's row space, or -1
// when the block table names a page outside the pool (nothing is read then).
__host__ __device__ inline int64_t kv_row(const KvView& kv, int g, int64_t tok, int chunk) {
  if (kv.table == nullptr) return int64_t(g) * kv.ld + tok;
  const int64_t c = tok / chunk;
  if (c >= kv.max_blocks) return -1;
  const int32_t page = kv.table[int64_t(g) * kv.max_blocks + c];
  if (page < 0 || int64_t(page) >= kv.ld) return -1;
  return int64_t(page) * chunk + (tok - c * chunk);
}

// C^l, saturating at a value above any token count.
__host__ __device__ inline int64_t span_of(int32_t chunk, int32_t level) {
  int64_t s = 1;
  for (int i = 0; i < level; ++i) {
    if (s > (int64_t(1) << 40)) return int64_t(1) << 50;
    s *= chunk;
  }
  return s;
}

// Nodes of level l that exist when N_b tokens are covered by complete chunks.
__host__ __device__ inline int64_t nodes_at(int64_t nb, int32_t chunk, int32_t level) {
  return nb / span_of(chunk, level);
}

__host__ __device__ inline int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }
__host__ __device__ inline int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ inline int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

// ---------------------------------------------------------------------------
// Route workspace layout: per level, sigma [B][Hq][n_l] float and (unless the
// caller passes its own buffer) kept bitmaps [B][Hq][W_l] uint32, plus the
// compacted kept parents [B][Hq][n_max] int32 used to enumerate candidates.
// ---------------------------------------------------------------------------
struct RouteLayout {
  int64_t n[ZHA_MAX_LEVELS + 2];         // nodes per level at n_tokens
  int64_t words[ZHA_MAX_LEVELS + 2];     // bitmap words per head per level
  int64_t sig_off[ZHA_MAX_LEVELS + 2];   // float offsets into sigma region
  int64_t bits_off[ZHA_MAX_LEVELS + 2];  // word offsets into the bitmap region
  int64_t sig_floats, bits_words, kp_ints;
  int64_t bytes;                          // total workspace (bitmaps included)
  int64_t bytes_no_bits;                  // when the caller supplies the bitmaps
};

inline RouteLayout route_layout(const Geom& g, int32_t batch, int64_t n_tokens) {
  RouteLayout r{};
  const int64_t nb = int64_t(g.chunk) * (n_tokens / g.chunk);
  const int64_t heads = int64_t(batch) * g.hq;
  int64_t sig = 0, bits = 0, nmax = 0;
  for (int l = 1; l <= g.levels; ++l) {
    r.n[l] = nodes_at(nb, g.chunk, l);
    r.words[l] = (r.n[l] + 31) / 32;
    r.sig_off[l] = sig;
    r.bits_off[l] = bits;
    sig += round_up(heads * r.n[l], 64);
    bits += heads * r.words[l];
    if (l >= 2 && r.n[l] > nmax) nmax = r.n[l];
  }
  r.sig_floats = sig;
  r.bits_words = bits;
  r.kp_ints = round_up(heads * (nmax > 0 ? nmax : 1), 64);
  r.bytes_no_bits = round_up(sig * 4, 256) + round_up(r.kp_ints * 4, 256);
  r.bytes = r.bytes_no_bits + round_up(bits * 4, 256);
  return r;
}

// ---------------------------------------------------------------------------
// Attend workspace: one partial state per (query head, range of W chunks) plus
// one for the sink-and-tail pass; each slot is [m, l, 0, 0, o[d]] floats.
// ---------------------------------------------------------------------------
constexpr int kAttendRangeTokens = 1024;

inline int32_t attend_range_chunks(int32_t chunk) {
  int32_t w = kAttendRangeTokens / chunk;
  return w < 1 ? 1 : w;
}

constexpr int kAttendHeadsPerBlock = 32;   // query heads per attention group

struct AttendLayout {
  int64_t n_chunks, n_ranges, slots_per_head, slot_floats, bytes;
  int32_t range_chunks, q_blocks;
};

inline AttendLayout attend_layout(const Geom& g, int32_t batch, int64_t n_tokens) {
  AttendLayout a{};
  const int64_t nb = int64_t(g.chunk) * (n_tokens / g.chunk);
  const int64_t heads = int64_t(batch) * g.hq;
  a.n_chunks = nb / g.chunk;
  a.range_chunks = attend_range_chunks(g.chunk);
  a.n_ranges = (a.n_chunks + a.range_chunks - 1) / a.range_chunks;
  a.slots_per_head = a.n_ranges + 1;
  a.slot_floats = g.d + 4;
  a.q_blocks = int32_t((int64_t(batch) * g.group + kAttendHeadsPerBlock - 1) / kAttendHeadsPerBlock);
  a.bytes = round_up(heads * a.slots_per_head * a.slot_floats * 4, 256);
  return a;
}

// ---------------------------------------------------------------------------
// Tensor-core attend workspace (bf16 caches, d = 128). A "group" v is a KV head
// g and a block of up to 32 of its query heads (v = g * q_blocks + qb). The
// chunk range [0, N_b / C) is cut into n_blocks blocks of block_chunks chunks;
// a "unit" u = v * n_blocks + b is one group's union inside one block.
//   ids   [groups][cap] int32   per unit, at offset b * block_chunks: the
//                               ascending union of the chunks the group's heads
//                               listed in block b (chunk 0 always present when
//                               N_b > 0); cap = n_blocks * block_chunks
//   masks [groups][cap] uint32  bit q = query q of the group listed that chunk
//   counts[units] int32         union entries per unit
//   split [units + 1 + 2] int32 tile offsets of the units, then the CTA count
//                               (written by the attend kernel for the combine)
//   slots [(kTcMaxCtas + groups) * 32][d + 4] float  per (CTA span piece, query)
//                               state [m, l, 0, 0, o[d]]; the piece of CTA c
//                               inside group v has index c + v
// ---------------------------------------------------------------------------
constexpr int kTcMaxCtas = 296;
constexpr int kTcMaxGroups = 1024;
constexpr int kTcMaxUnits = 1024;
constexpr int64_t kTcBlockChunks = 2048;

struct TcAttendLayout {
  int64_t n_chunks, block_chunks, cap, groups, units;
  int64_t ids_off, masks_off, counts_off, split_off, slots_off, bytes;
  int32_t q_blocks, n_blocks;
};

inline TcAttendLayout tc_attend_layout(const Geom& g, int32_t batch, int64_t n_tokens) {
  TcAttendLayout a{};
  a.n_chunks = n_tokens / g.chunk;
  a.q_blocks = int32_t((int64_t(batch) * g.group + kAttendHeadsPerBlock - 1) / kAttendHeadsPerBlock);
  a.groups = int64_t(g.hkv) * a.q_blocks;
  int64_t nblk = (a.n_chunks + kTcBlockChunks - 1) / kTcBlockChunks;
  const int64_t lim = kTcMaxUnits / a.groups;
  if (nblk > lim) nblk = lim;
  if (nblk < 1) nblk = 1;
  a.n_blocks = int32_t(nblk);
  int64_t per = (a.n_chunks + nblk - 1) / nblk;
  a.block_chunks = round_up(per < 1 ? 1 : per, 32);
  a.cap = nblk * a.block_chunks;
  a.units = a.groups * nblk;
  a.ids_off = 0;
  a.masks_off = round_up(a.groups * a.cap * 4, 256);
  a.counts_off = a.masks_off + round_up(a.groups * a.cap * 4, 256);
  a.split_off = a.counts_off + round_up(a.units * 4, 256);
  a.slots_off = a.split_off + round_up((a.units + 3) * 4, 256);
  a.bytes = a.slots_off + round_up((kTcMaxCtas + a.groups) * 32 * int64_t(g.d + 4) * 4, 256);
  return a;
}

inline bool use_tc_attend(const Geom& g) { return g.kv_bf16 && g.d == 128; }

// ---------------------------------------------------------------------------
// Optional kernel timing (zha_trace.cu): a TraceScope around a launch records
// CUDA events before and after it on the stream while tracing is enabled.
// `tag` distinguishes launches of one kernel (the tree level for routing).
// ---------------------------------------------------------------------------
int trace_begin(const char* name, int32_t tag, cudaStream_t s);
void trace_end(int idx, cudaStream_t s);

struct TraceScope {
  int idx;
  cudaStream_t s;
  TraceScope(const char* name, int32_t tag, cudaStream_t stream)
      : idx(trace_begin(name, tag, stream)), s(stream) {}
  ~TraceScope() { trace_end(idx, s); }
  TraceScope(const TraceScope&) = delete;
  TraceScope& operator=(const TraceScope&) = delete;
};

// ---------------------------------------------------------------------------
// Programmatic dependent launch: a kernel launched with launch_pdl may be
// scheduled while the previous kernel on the stream is finishing. It calls
// pdl_trigger() on entry (its own dependents may then be scheduled once all of
// its CTAs are resident) and pdl_wait() before it touches anything the previous
// kernel wrote (pdl_wait returns once that kernel has completed and its memory
// is visible). Both are no-ops for a kernel launched the ordinary way.
// ---------------------------------------------------------------------------
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// EPL consecutive elements of a row, starting at element `e0`, widened to fp32.
// The row start is 16-byte aligned; e0 is a multiple of EPL.
template <int EPL>
__device__ __forceinline__ void load_slice(const float* row, int e0, float (&out)[EPL]) {
  if constexpr (EPL == 4) {
    float4 v = *reinterpret_cast<const float4*>(row + e0);
    out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
  } else if constexpr (EPL == 2) {
    float2 v = *reinterpret_cast<const float2*>(row + e0);
    out[0] = v.x; out[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < EPL; ++i) out[i] = row[e0 + i];
  }
}

template <int EPL>
__device__ __forceinline__ void load_slice(const __nv_bfloat16* row, int e0, float (&out)[EPL]) {
  if constexpr (EPL == 8) {
    uint4 v = *reinterpret_cast<const uint4*>(row + e0);
    out[0] = __uint_as_float(v.x << 16); out[1] = __uint_as_float(v.x & 0xffff0000u);
    out[2] = __uint_as_float(v.y << 16); out[3] = __uint_as_float(v.y & 0xffff0000u);
    out[4] = __uint_as_float(v.z << 16); out[5] = __uint_as_float(v.z & 0xffff0000u);
    out[6] = __uint_as_float(v.w << 16); out[7] = __uint_as_float(v.w & 0xffff0000u);
  } else if constexpr (EPL == 4) {
    uint2 v = *reinterpret_cast<const uint2*>(row + e0);
    out[0] = __uint_as_float(v.x << 16); out[1] = __uint_as_float(v.x & 0xffff0000u);
    out[2] = __uint_as_float(v.y << 16); out[3] = __uint_as_float(v.y & 0xffff0000u);
  } else if constexpr (EPL == 2) {
    uint32_t v = *reinterpret_cast<const uint32_t*>(row + e0);
    out[0] = __uint_as_float(v << 16); out[1] = __uint_as_float(v & 0xffff0000u);
  } else {
#pragma unroll
    for (int i = 0; i < EPL; ++i) out[i] = __bfloat162float(row[e0 + i]);
  }
}

// Monotone map float -> uint32 (ascending floats give ascending keys).
__device__ __forceinline__ uint32_t float_order_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float order_key_float(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(u);
}

// Per-level selection rule of a route: top-p with mass p[l], or top-k keeping
// k[l] nodes, for levels l = 1..L (index l).
struct RoutePolicy {
  int32_t topk;
  float p[ZHA_MAX_LEVELS + 1];
  int32_t k[ZHA_MAX_LEVELS + 1];
};

inline RoutePolicy uniform_top_p(float p) {
  RoutePolicy r{};
  for (int l = 0; l <= ZHA_MAX_LEVELS; ++l) r.p[l] = p;
  return r;
}

cudaError_t launch_route(const Geom& G, const float* Q, int32_t batch, int64_t n_tokens,
                         const RoutePolicy& pol, int32_t* chunk_ids, int32_t* n_chunks,
                         int32_t max_sel, uint32_t* bits, float* sigma, int32_t* kp,
                         const RouteLayout& lay, int32_t* status, const float* store,
                         cudaStream_t s);

}  // namespace zha

// The host handle behind the opaque zha_tree of the C ABI.
struct zha_tree {
  zha_config cfg;
  zha::Geom geom;
  float* store;
  size_t store_bytes;
  const float* ref_q;
  int64_t nb;  // tokens covered by complete level-1 chunks
};

// Launch bookkeeping and error reporting shared by the host wrappers.
void zha_count_launch();
zha_status zha_report_error(zha_status s, const char* msg);
zha_status zha_check_route_args(const zha_tree* tree, const float* d_Q, int32_t batch,
                                int64_t n_tokens, const int32_t* d_chunk_ids,
                                const int32_t* d_n_chunks, int32_t max_sel, const char* who);
zha_status zha_check_p(float p, const char* who);
