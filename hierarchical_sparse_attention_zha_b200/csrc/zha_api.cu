// zha_api.cu -- the extern "C" entry points of libzha: argument checks, layouts
// and kernel launches. Semantics and citations of every call are in include/zha.h.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <string>

#include "zha_internal.cuh"

namespace zha {
cudaError_t launch_build(const Geom& G, const KvView& kv, int64_t nb_old, int64_t nb_new,
                         const float* refq, float* store, cudaStream_t s);
cudaError_t launch_append(const Geom& G, const KvView& kv, int64_t nb_old, int64_t nb_new,
                          const float* refq, float* store, cudaStream_t s);
cudaError_t launch_attend_tc(const Geom& G, const float* Q, const KvView& kv, int64_t n_tokens,
                             int32_t batch, const int32_t* chunk_ids, const int32_t* n_chunks,
                             int32_t max_sel, float* O, float* lse, void* ws, const TcAttendLayout& lay,
                             int32_t* status, cudaStream_t s);
cudaError_t launch_attend(const Geom& G, const float* Q, const KvView& kv, int64_t n_tokens,
                          int32_t batch, const int32_t* chunk_ids, const int32_t* n_chunks,
                          int32_t max_sel, float* O, float* lse, float* partial,
                          const AttendLayout& lay, int32_t* status, cudaStream_t s);
}  // namespace zha

static std::atomic<uint64_t> g_launches{0};
void zha_count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

static thread_local std::string g_err;

static zha_status fail(zha_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

zha_status zha_report_error(zha_status s, const char* msg) { return fail(s, "%s", msg); }

static zha_status cuda_fail(cudaError_t e, const char* where) {
  return fail(ZHA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

static bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Validate a configuration and derive its geometry and store size.
static zha_status make_geom(const zha_config* c, zha::Geom* g, size_t* bytes) {
  if (c == nullptr) return fail(ZHA_ERR_INVALID, "config is NULL");
  if (c->n_kv_heads < 1) return fail(ZHA_ERR_INVALID, "n_kv_heads must be >= 1");
  if (c->n_q_heads < 1 || c->n_q_heads % c->n_kv_heads != 0)
    return fail(ZHA_ERR_INVALID, "n_q_heads must be a positive multiple of n_kv_heads");
  if (c->head_dim != 64 && c->head_dim != 128)
    return fail(ZHA_ERR_UNSUPPORTED, "head_dim %d: 64 and 128 are supported", c->head_dim);
  if (c->chunk < 2 || c->chunk > ZHA_MAX_CHUNK)
    return fail(ZHA_ERR_UNSUPPORTED, "chunk %d: 2..%d supported", c->chunk, ZHA_MAX_CHUNK);
  if (c->levels < 1 || c->levels > ZHA_MAX_LEVELS)
    return fail(ZHA_ERR_UNSUPPORTED, "levels %d: 1..%d supported", c->levels, ZHA_MAX_LEVELS);
  if (c->n_ref < 1 || c->n_ref > ZHA_MAX_REF)
    return fail(ZHA_ERR_UNSUPPORTED, "n_ref %d: 1..%d supported", c->n_ref, ZHA_MAX_REF);
  if (c->kv_dtype != ZHA_F32 && c->kv_dtype != ZHA_BF16)
    return fail(ZHA_ERR_INVALID, "kv_dtype %d unknown", c->kv_dtype);
  if (c->reserved != 0) return fail(ZHA_ERR_INVALID, "reserved must be 0");
  if (c->rope_pairs < 0 || c->rope_pairs > c->head_dim / 2)
    return fail(ZHA_ERR_INVALID, "rope_pairs %d outside [0, head_dim / 2]", c->rope_pairs);
  if (c->rope_pairs > 0 && !(c->rope_base > 1.f && std::isfinite(c->rope_base)))
    return fail(ZHA_ERR_INVALID, "rope_base must be finite and > 1 with rotary positions");
  if (c->max_tokens < 1 || c->max_tokens > (int64_t(1) << 34))
    return fail(ZHA_ERR_INVALID, "max_tokens %lld out of range", (long long)c->max_tokens);
  zha::Geom G{};
  G.hkv = c->n_kv_heads;
  G.hq = c->n_q_heads;
  G.group = c->n_q_heads / c->n_kv_heads;
  G.d = c->head_dim;
  G.chunk = c->chunk;
  G.levels = c->levels;
  G.nref = c->n_ref;
  G.node_floats = int32_t(c->n_ref * c->head_dim + zha::round_up(c->n_ref, 4));
  G.kv_bf16 = c->kv_dtype == ZHA_BF16;
  G.scale = float(1.0 / std::sqrt(double(c->head_dim)));
  G.max_tokens = c->max_tokens;
  G.wait_polls = 1u << 15;                     // ~2 s with the waits' suspend hint
  G.debug_withhold = 0;
  G.rope_pairs = c->rope_pairs;
  G.rope_log2_base = c->rope_pairs > 0 ? std::log2(double(c->rope_base)) : 0.0;
  int64_t off = 0;
  for (int l = 1; l <= G.levels; ++l) {
    G.cap[l] = zha::nodes_at(c->max_tokens, c->chunk, l);
    G.off[l] = off;
    off += int64_t(G.hkv) * G.cap[l] * G.node_floats;
  }
  G.status_off = zha::round_up(off, 64);           // 256-byte aligned, one 256-byte block
  int64_t end = G.status_off * 4 + 256;            // bytes
  for (int l = 0; l <= ZHA_MAX_LEVELS + 1; ++l) G.split_off[l] = 0;
  if (zha::has_plane_terms(G)) {
    for (int l = 1; l <= G.levels; ++l) {
      G.split_off[l] = end;                        // multiples of 8 KiB after a 256-byte boundary
      end += int64_t(G.hkv) * 2 * G.cap[l] * G.nref * G.d * 2;
    }
  }
  *g = G;
  if (bytes) *bytes = size_t(end);
  return ZHA_OK;
}

extern "C" {

int32_t zha_abi_version(void) { return ZHA_ABI_VERSION; }

const char* zha_status_str(int32_t s) {
  switch (s) {
    case ZHA_OK: return "ok";
    case ZHA_ERR_INVALID: return "invalid argument";
    case ZHA_ERR_CAPACITY: return "buffer too small";
    case ZHA_ERR_STATE: return "tree state does not match the token count";
    case ZHA_ERR_CUDA: return "CUDA error";
    case ZHA_ERR_UNSUPPORTED: return "unsupported configuration";
    default: return "unknown status";
  }
}

const char* zha_last_error(void) { return g_err.c_str(); }

uint64_t zha_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

size_t zha_tree_bytes(const zha_config* cfg) {
  zha::Geom G;
  size_t bytes = 0;
  return make_geom(cfg, &G, &bytes) == ZHA_OK ? bytes : 0;
}

zha_status zha_tree_create(const zha_config* cfg, void* d_store, size_t store_bytes,
                           const float* d_ref_q, zha_tree** out) {
  if (out == nullptr) return fail(ZHA_ERR_INVALID, "out is NULL");
  zha::Geom G;
  size_t need = 0;
  zha_status st = make_geom(cfg, &G, &need);
  if (st != ZHA_OK) return st;
  if (d_store == nullptr || !aligned(d_store, 256))
    return fail(ZHA_ERR_INVALID, "store must be a non-NULL 256-byte aligned device pointer");
  if (store_bytes < need)
    return fail(ZHA_ERR_CAPACITY, "store has %zu bytes, %zu needed", store_bytes, need);
  if (d_ref_q == nullptr || !aligned(d_ref_q, 16))
    return fail(ZHA_ERR_INVALID, "ref_q must be a non-NULL 16-byte aligned device pointer");
  zha_tree* t = new zha_tree{};
  t->cfg = *cfg;
  t->geom = G;
  t->store = static_cast<float*>(d_store);
  t->store_bytes = store_bytes;
  t->ref_q = d_ref_q;
  t->nb = 0;
  *out = t;
  return ZHA_OK;
}

void zha_tree_destroy(zha_tree* tree) { delete tree; }

zha_status zha_tree_debug(zha_tree* tree, uint32_t wait_polls, int32_t withhold) {
  if (tree == nullptr) return fail(ZHA_ERR_INVALID, "zha_tree_debug: tree is NULL");
  tree->geom.wait_polls = wait_polls == 0 ? 1u << 15 : wait_polls;
  tree->geom.debug_withhold = withhold != 0;
  return ZHA_OK;
}

int64_t zha_tree_built_tokens(const zha_tree* tree) { return tree ? tree->nb : -1; }

zha_status zha_tree_level_layout(const zha_tree* tree, int32_t level, int64_t* offset_floats,
                                 int64_t* capacity, int32_t* node_floats) {
  if (tree == nullptr) return fail(ZHA_ERR_INVALID, "tree is NULL");
  if (level < 1 || level > tree->geom.levels) return fail(ZHA_ERR_INVALID, "level out of range");
  if (offset_floats) *offset_floats = tree->geom.off[level];
  if (capacity) *capacity = tree->geom.cap[level];
  if (node_floats) *node_floats = tree->geom.node_floats;
  return ZHA_OK;
}

}  // extern "C"

// A zha_kv_cache checked against the tree and turned into the kernels' view.
// `need_v`: the call reads values too. Contiguous: ld rows per KV head, at
// least n_tokens; paged: ld pages, a block table with >= ceil(n_tokens / C)
// entries per KV head.
static zha_status kv_view(const zha_tree* tree, const zha_kv_cache* kv, int64_t n_tokens, bool need_v,
                          const char* what, zha::KvView* out) {
  if (tree == nullptr) return fail(ZHA_ERR_INVALID, "%s: tree is NULL", what);
  if (kv == nullptr) return fail(ZHA_ERR_INVALID, "%s: cache is NULL", what);
  if (kv->k == nullptr || !aligned(kv->k, 16) || (need_v && (kv->v == nullptr || !aligned(kv->v, 16))))
    return fail(ZHA_ERR_INVALID, "%s: K%s must be non-NULL 16-byte aligned device pointers", what,
                need_v ? " and V" : "");
  if (kv->ld < 1) return fail(ZHA_ERR_INVALID, "%s: ld must be >= 1", what);
  if (n_tokens < 0 || n_tokens > tree->geom.max_tokens)
    return fail(ZHA_ERR_INVALID, "%s: n_tokens %lld outside [0, max_tokens]", what, (long long)n_tokens);
  if (kv->block_table == nullptr) {
    if (n_tokens > kv->ld)
      return fail(ZHA_ERR_INVALID, "%s: n_tokens %lld outside [0, min(ld, max_tokens)]", what,
                  (long long)n_tokens);
  } else {
    const int64_t blocks = (n_tokens + tree->geom.chunk - 1) / tree->geom.chunk;
    if (!aligned(kv->block_table, 4) || kv->max_blocks < blocks)
      return fail(ZHA_ERR_INVALID, "%s: the block table needs >= %lld entries per KV head", what,
                  (long long)blocks);
    if (kv->ld > (int64_t(1) << 31) / tree->geom.chunk)
      return fail(ZHA_ERR_UNSUPPORTED, "%s: more than 2^31 token slots in the page pool", what);
  }
  out->k = kv->k;
  out->v = kv->v;
  out->ld = kv->ld;
  out->table = kv->block_table;
  out->max_blocks = kv->block_table ? kv->max_blocks : 0;
  return ZHA_OK;
}

static zha_kv_cache contiguous(const void* k, const void* v, int64_t ld) {
  zha_kv_cache c{};
  c.k = k;
  c.v = v;
  c.ld = ld;
  return c;
}

extern "C" {

zha_status zha_build_kv(zha_tree* tree, const zha_kv_cache* kv, int64_t n_tokens, void* stream) {
  zha::KvView view{};
  zha_status st = kv_view(tree, kv, n_tokens, false, "zha_build", &view);
  if (st != ZHA_OK) return st;
  const int64_t nb = int64_t(tree->geom.chunk) * (n_tokens / tree->geom.chunk);
  // A full build starts the tree's status afresh.
  cudaError_t e = cudaMemsetAsync(zha::tree_status_word(tree->geom, tree->store), 0, sizeof(int32_t),
                                  static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "zha_build");
  e = zha::launch_build(tree->geom, view, 0, nb, tree->ref_q, tree->store,
                        static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "zha_build");
  tree->nb = nb;
  return ZHA_OK;
}

zha_status zha_build(zha_tree* tree, const void* d_K, int64_t ld, int64_t n_tokens, void* stream) {
  const zha_kv_cache kv = contiguous(d_K, nullptr, ld);
  return zha_build_kv(tree, &kv, n_tokens, stream);
}

zha_status zha_append_chunk_kv(zha_tree* tree, const zha_kv_cache* kv, int64_t n_tokens, void* stream) {
  zha::KvView view{};
  zha_status st = kv_view(tree, kv, n_tokens, false, "zha_append_chunk", &view);
  if (st != ZHA_OK) return st;
  const int64_t nb_new = int64_t(tree->geom.chunk) * (n_tokens / tree->geom.chunk);
  if (nb_new < tree->nb)
    return fail(ZHA_ERR_STATE, "zha_append_chunk: n_tokens %lld is below the built prefix %lld",
                (long long)n_tokens, (long long)tree->nb);
  if (nb_new == tree->nb) return ZHA_OK;
  const int64_t new_chunks = (nb_new - tree->nb) / tree->geom.chunk;
  cudaError_t e = new_chunks <= 8
                      ? zha::launch_append(tree->geom, view, tree->nb, nb_new, tree->ref_q, tree->store,
                                           static_cast<cudaStream_t>(stream))
                      : zha::launch_build(tree->geom, view, tree->nb, nb_new, tree->ref_q, tree->store,
                                          static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "zha_append_chunk");
  tree->nb = nb_new;
  return ZHA_OK;
}

zha_status zha_append_chunk(zha_tree* tree, const void* d_K, int64_t ld, int64_t n_tokens,
                            void* stream) {
  const zha_kv_cache kv = contiguous(d_K, nullptr, ld);
  return zha_append_chunk_kv(tree, &kv, n_tokens, stream);
}

size_t zha_route_workspace_bytes(const zha_config* cfg, int32_t batch, int64_t n_tokens) {
  zha::Geom G;
  if (make_geom(cfg, &G, nullptr) != ZHA_OK || batch < 1 || n_tokens < 0) return 0;
  return size_t(zha::route_layout(G, batch, n_tokens).bytes);
}

size_t zha_route_kept_words(const zha_config* cfg, int32_t batch, int64_t n_tokens) {
  zha::Geom G;
  if (make_geom(cfg, &G, nullptr) != ZHA_OK || batch < 1 || n_tokens < 0) return 0;
  return size_t(zha::route_layout(G, batch, n_tokens).bits_words);
}

}  // extern "C"

// Argument checks of a routing call (zha_route and zha_route_noalloc share them).
zha_status zha_check_p(float p, const char* who) {
  if (!(p > 0.f) || !std::isfinite(p)) return fail(ZHA_ERR_INVALID, "%s: p must be > 0", who);
  return ZHA_OK;
}

zha_status zha_check_route_args(const zha_tree* tree, const float* d_Q, int32_t batch,
                                int64_t n_tokens, const int32_t* d_chunk_ids,
                                const int32_t* d_n_chunks, int32_t max_sel, const char* who) {
  if (tree == nullptr) return fail(ZHA_ERR_INVALID, "%s: tree is NULL", who);
  const zha::Geom& G = tree->geom;
  if (d_Q == nullptr || !aligned(d_Q, 16))
    return fail(ZHA_ERR_INVALID, "%s: Q must be a non-NULL 16-byte aligned device pointer", who);
  if (batch < 1 || batch > 65535) return fail(ZHA_ERR_INVALID, "%s: batch must be 1..65535", who);
  if (n_tokens < 1 || n_tokens > G.max_tokens)
    return fail(ZHA_ERR_INVALID, "%s: n_tokens %lld outside [1, max_tokens]", who,
                (long long)n_tokens);
  const int64_t nb = int64_t(G.chunk) * (n_tokens / G.chunk);
  if (nb != tree->nb)
    return fail(ZHA_ERR_STATE, "%s: tree covers %lld tokens, n_tokens %lld needs %lld", who,
                (long long)tree->nb, (long long)n_tokens, (long long)nb);
  if (d_chunk_ids == nullptr || d_n_chunks == nullptr || max_sel < 1)
    return fail(ZHA_ERR_INVALID, "%s: chunk_ids / n_chunks NULL or max_sel < 1", who);
  return ZHA_OK;
}

extern "C" {

// zha_route and zha_route_ex after their own argument checks.
static zha_status route_impl(const zha_tree* tree, const float* d_Q, int32_t batch, int64_t n_tokens,
                             const zha::RoutePolicy& pol, int32_t* d_chunk_ids, int32_t* d_n_chunks,
                             int32_t max_sel, uint32_t* d_kept_bits, void* d_ws, size_t ws_bytes,
                             int32_t* d_status, void* stream, const char* who) {
  const zha::Geom& G = tree->geom;
  const zha::RouteLayout lay = zha::route_layout(G, batch, n_tokens);
  const int64_t need = d_kept_bits ? lay.bytes_no_bits : lay.bytes;
  if (d_ws == nullptr || !aligned(d_ws, 256) || int64_t(ws_bytes) < need)
    return fail(ZHA_ERR_CAPACITY, "%s: workspace must be 256-byte aligned with %lld bytes", who,
                (long long)need);
  char* ws = static_cast<char*>(d_ws);
  float* sigma = reinterpret_cast<float*>(ws);
  int32_t* kp = reinterpret_cast<int32_t*>(ws + zha::round_up(lay.sig_floats * 4, 256));
  uint32_t* bits = d_kept_bits ? d_kept_bits : reinterpret_cast<uint32_t*>(ws + lay.bytes_no_bits);
  cudaError_t e = zha::launch_route(G, d_Q, batch, n_tokens, pol, d_chunk_ids, d_n_chunks, max_sel,
                                    bits, sigma, kp, lay, d_status, tree->store,
                                    static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, who);
  return ZHA_OK;
}

zha_status zha_route(const zha_tree* tree, const float* d_Q, int32_t batch, int64_t n_tokens,
                     float p, int32_t* d_chunk_ids, int32_t* d_n_chunks, int32_t max_sel,
                     uint32_t* d_kept_bits, void* d_ws, size_t ws_bytes, int32_t* d_status,
                     void* stream) {
  zha_status st = zha_check_route_args(tree, d_Q, batch, n_tokens, d_chunk_ids, d_n_chunks, max_sel,
                                       "zha_route");
  if (st != ZHA_OK) return st;
  if ((st = zha_check_p(p, "zha_route")) != ZHA_OK) return st;
  return route_impl(tree, d_Q, batch, n_tokens, zha::uniform_top_p(p), d_chunk_ids, d_n_chunks,
                    max_sel, d_kept_bits, d_ws, ws_bytes, d_status, stream, "zha_route");
}

zha_status zha_route_ex(const zha_tree* tree, const float* d_Q, int32_t batch, int64_t n_tokens,
                        const zha_route_policy* policy, int32_t* d_chunk_ids, int32_t* d_n_chunks,
                        int32_t max_sel, uint32_t* d_kept_bits, void* d_ws, size_t ws_bytes,
                        int32_t* d_status, void* stream) {
  zha_status st = zha_check_route_args(tree, d_Q, batch, n_tokens, d_chunk_ids, d_n_chunks, max_sel,
                                       "zha_route_ex");
  if (st != ZHA_OK) return st;
  if (policy == nullptr) return fail(ZHA_ERR_INVALID, "zha_route_ex: policy is NULL");
  if (policy->reserved != 0) return fail(ZHA_ERR_INVALID, "zha_route_ex: policy.reserved must be 0");
  zha::RoutePolicy pol{};
  if (policy->mode == ZHA_SELECT_TOP_P) {
    for (int l = 1; l <= tree->geom.levels; ++l) {
      if ((st = zha_check_p(policy->p[l - 1], "zha_route_ex")) != ZHA_OK) return st;
      pol.p[l] = policy->p[l - 1];
    }
  } else if (policy->mode == ZHA_SELECT_TOP_K) {
    pol.topk = 1;
    for (int l = 1; l <= tree->geom.levels; ++l) {
      if (policy->k[l - 1] < 1)
        return fail(ZHA_ERR_INVALID, "zha_route_ex: k of level %d must be >= 1", l);
      pol.k[l] = policy->k[l - 1];
    }
  } else {
    return fail(ZHA_ERR_INVALID, "zha_route_ex: unknown policy mode %d", policy->mode);
  }
  return route_impl(tree, d_Q, batch, n_tokens, pol, d_chunk_ids, d_n_chunks, max_sel, d_kept_bits,
                    d_ws, ws_bytes, d_status, stream, "zha_route_ex");
}

size_t zha_attend_workspace_bytes(const zha_config* cfg, int32_t batch, int64_t n_tokens) {
  zha::Geom G;
  if (make_geom(cfg, &G, nullptr) != ZHA_OK || batch < 1 || n_tokens < 0) return 0;
  if (zha::use_tc_attend(G)) return size_t(zha::tc_attend_layout(G, batch, n_tokens).bytes);
  return size_t(zha::attend_layout(G, batch, n_tokens).bytes);
}

zha_status zha_sparse_attend_kv(const zha_tree* tree, const float* d_Q, const zha_kv_cache* kv,
                                int64_t n_tokens, int32_t batch, const int32_t* d_chunk_ids,
                                const int32_t* d_n_chunks, int32_t max_sel, float* d_O, float* d_lse,
                                void* d_ws, size_t ws_bytes, int32_t* d_status, void* stream) {
  zha::KvView view{};
  zha_status st = kv_view(tree, kv, n_tokens, true, "zha_sparse_attend", &view);
  if (st != ZHA_OK) return st;
  const zha::Geom& G = tree->geom;
  if (d_Q == nullptr || d_O == nullptr || !aligned(d_Q, 16) || !aligned(d_O, 16))
    return fail(ZHA_ERR_INVALID,
                "zha_sparse_attend: Q, K, V, O must be non-NULL 16-byte aligned device pointers");
  if (batch < 1 || batch > 65535)
    return fail(ZHA_ERR_INVALID, "zha_sparse_attend: batch must be 1..65535");
  if (n_tokens < 1) return fail(ZHA_ERR_INVALID, "zha_sparse_attend: need 1 <= n_tokens <= ld");
  if (d_chunk_ids == nullptr || d_n_chunks == nullptr || max_sel < 1)
    return fail(ZHA_ERR_INVALID, "zha_sparse_attend: chunk_ids / n_chunks NULL or max_sel < 1");
  if (zha::use_tc_attend(G)) {
    const zha::TcAttendLayout lay = zha::tc_attend_layout(G, batch, n_tokens);
    if (lay.groups > zha::kTcMaxGroups || n_tokens > 2147483647LL - 256)
      return fail(ZHA_ERR_UNSUPPORTED,
                  "zha_sparse_attend: more than %d (KV head, 32-query block) groups or 2^31 tokens",
                  zha::kTcMaxGroups);
    if (d_ws == nullptr || !aligned(d_ws, 256) || int64_t(ws_bytes) < lay.bytes)
      return fail(ZHA_ERR_CAPACITY,
                  "zha_sparse_attend: workspace must be 256-byte aligned with %lld bytes",
                  (long long)lay.bytes);
    cudaError_t e = zha::launch_attend_tc(G, d_Q, view, n_tokens, batch, d_chunk_ids, d_n_chunks, max_sel,
                                          d_O, d_lse, d_ws, lay, d_status, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "zha_sparse_attend");
    return ZHA_OK;
  }
  const zha::AttendLayout lay = zha::attend_layout(G, batch, n_tokens);
  if (lay.n_ranges + 1 > 2147483647LL)
    return fail(ZHA_ERR_UNSUPPORTED, "zha_sparse_attend: too many tokens");
  if (d_ws == nullptr || !aligned(d_ws, 256) || int64_t(ws_bytes) < lay.bytes)
    return fail(ZHA_ERR_CAPACITY,
                "zha_sparse_attend: workspace must be 256-byte aligned with %lld bytes",
                (long long)lay.bytes);
  cudaError_t e = zha::launch_attend(G, d_Q, view, n_tokens, batch, d_chunk_ids, d_n_chunks, max_sel, d_O,
                                     d_lse, static_cast<float*>(d_ws), lay, d_status,
                                     static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "zha_sparse_attend");
  return ZHA_OK;
}

zha_status zha_sparse_attend(const zha_tree* tree, const float* d_Q, const void* d_K,
                             const void* d_V, int64_t ld, int64_t n_tokens, int32_t batch,
                             const int32_t* d_chunk_ids, const int32_t* d_n_chunks,
                             int32_t max_sel, float* d_O, float* d_lse, void* d_ws,
                             size_t ws_bytes, int32_t* d_status, void* stream) {
  if (tree != nullptr && d_K != nullptr && d_V != nullptr && (ld < 1 || n_tokens < 1 || n_tokens > ld))
    return fail(ZHA_ERR_INVALID, "zha_sparse_attend: need 1 <= n_tokens <= ld");
  const zha_kv_cache kv = contiguous(d_K, d_V, ld);
  return zha_sparse_attend_kv(tree, d_Q, &kv, n_tokens, batch, d_chunk_ids, d_n_chunks, max_sel, d_O,
                              d_lse, d_ws, ws_bytes, d_status, stream);
}

}  // extern "C"
