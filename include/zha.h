/*
 * zha.h -- C ABI of the ZHA decode hot path on B200 (sm_100a): tree-summarised
 * KV-cache attention.
 *
 * Citations name a page by its title and a section on it:
 *   [ZHA: <section>]  page "ZHA는 KV 캐시를 트리로 요약해 어텐션 비용을 준(sub)이차로
 *                     낮춘다" (onedev.kr/papers/1556);
 *   [Attention: <section>]  page "Attention"
 *                     (zzong2006.github.io/machine_learning/nlp/attention-function).
 *
 * The method: every contiguous key chunk of C tokens gets, at each of R
 * reference queries q_r, a tangent plane t_r(q) = q.khat_r/sqrt(d) + bhat_r of
 * its log attention mass; level l >= 2 nodes merge C children the same way.
 * At decode time each query head is routed level by level with top-p over the
 * planes' maximum, and exact softmax attention runs over the gathered leaf
 * tokens, the sink (token 0) and the in-progress tail [ZHA: 무엇과 다른가,
 * 전제와 한계]. One tree per KV head serves its GQA query heads.
 *
 * Conventions for every call:
 *  - All pointers named d_* are DEVICE pointers owned by the caller (the library
 *    allocates no device memory). They must be 16-byte aligned.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Calls enqueue work and return; none synchronises the device.
 *  - Return value: ZHA_OK, or a negative zha_status when the host-side checks
 *    reject the arguments (nothing is launched then) or a launch fails
 *    (ZHA_ERR_CUDA). zha_last_error() gives a message for the calling thread.
 *  - Conditions only the device can see are OR-ed into *d_status (int32,
 *    ZHA_DEV_* bits) where the call takes one; the caller zeroes it and reads it
 *    after synchronising.
 *  - Layouts: K and V caches are [n_kv_heads][ld][head_dim] (element type
 *    zha_config.kv_dtype, ld >= tokens used); queries Q are float32
 *    [batch][n_q_heads][head_dim]; query head h uses KV head h / (n_q_heads /
 *    n_kv_heads) [Attention: "Key·value head 를 나눠 쓰거나 압축한다"];
 *    reference queries are float32 [n_kv_heads][n_ref][head_dim].
 *  - No call is thread-safe against another call on the same tree unless the
 *    caller orders them (same stream or events).
 */
#ifndef ZHA_H
#define ZHA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ZHA_ABI_VERSION 3

typedef enum {
    ZHA_OK = 0,
    ZHA_ERR_INVALID = -1,     /* bad argument: null pointer, size, alignment, range */
    ZHA_ERR_CAPACITY = -2,    /* a caller buffer (store, workspace, max_sel) is too small */
    ZHA_ERR_STATE = -3,       /* the tree's built prefix does not match n_tokens */
    ZHA_ERR_CUDA = -4,        /* a CUDA launch or query failed (see zha_last_error) */
    ZHA_ERR_UNSUPPORTED = -6  /* a configuration this build does not implement */
} zha_status;

/* Bits OR-ed into *d_status by device code. */
#define ZHA_DEV_SELECTION_TRUNCATED 1 /* zha_route: a head kept more than max_sel chunks; its list holds the first max_sel (ascending) and d_n_chunks the true count */
#define ZHA_DEV_BAD_SELECTION 2       /* zha_sparse_attend: a chunk list had an id out of range, was not strictly ascending, or a count outside [0, max_sel]; out-of-range ids are never read, and which in-range entries of such a list are attended is unspecified */
#define ZHA_DEV_TIMEOUT 4             /* a kernel's bounded wait for its tensor-core work ran out; its outputs are not valid (it released its resources and returned) */
#define ZHA_DEV_BAD_PAGE 8            /* a paged cache's block table named a page outside the pool (or lacked an entry); those keys were not read (treated as absent) and the outputs that needed them are not valid */

typedef enum { ZHA_F32 = 0, ZHA_BF16 = 1 } zha_dtype;

typedef struct {
    int32_t n_kv_heads;  /* KV heads = trees, >= 1 */
    int32_t n_q_heads;   /* query heads, a multiple of n_kv_heads */
    int32_t head_dim;    /* d: 64 or 128 */
    int32_t chunk;       /* C: tokens per level-1 chunk, 2..128 */
    int32_t levels;      /* L: summary levels, 1..8; level l covers C^l tokens */
    int32_t n_ref;       /* R: reference queries per tree, 1..32 */
    int32_t kv_dtype;    /* zha_dtype of the K and V caches */
    int32_t rope_pairs;  /* rotary positions: 0 = none (position-free keys); else the number
                            of leading element pairs (2i, 2i+1), 1..head_dim/2, that the
                            model turns by position * rope_base^(-2i/head_dim) */
    int64_t max_tokens;  /* tokens the summary store must cover, >= 1 */
    float rope_base;     /* rotation base (> 1) when rope_pairs > 0; ignored otherwise */
    int32_t reserved;    /* must be 0 */
} zha_config;

/* Rotary positions [ZHA: 무엇과 다른가; Attention: "Attention 은 순서를 모르므로 위치
 * 정보를 따로 넣는다"]: with rope_pairs > 0 the caches hold keys as the model
 * rotates them (key of position m turned by m * theta_i per pair i) and decode
 * queries come rotated at their own position. The summaries are then taken at
 * rotated reference queries: node n of level l sits at the position of its
 * first token, p_n = n * C^l, and its reference queries are q_hat_r rotated by
 * p_n. A parent re-evaluates each child c at its own rotated reference query
 * q_hat_{r,P}: u_c = F_c(q_hat_{r,c}) + 1/sqrt(d) <khat_{r,c}, q_hat_{r,P} -
 * q_hat_{r,c}>, which is the child's plane evaluated at q_hat_{r,P}. khat is
 * stored in the keys' (rotated) frame, so routing and attention use the
 * decode queries as they come. */

typedef struct zha_tree zha_tree; /* opaque host handle; holds no device memory */

/* ABI version of the loaded library (ZHA_ABI_VERSION). */
int32_t zha_abi_version(void);

/* Static text for a zha_status. */
const char* zha_status_str(int32_t status);

/* Message describing the last failed call made by the calling thread. */
const char* zha_last_error(void);

/* Number of kernels this library has launched in the process so far. */
uint64_t zha_launch_count(void);

/* Bytes of device memory the summary store of `cfg` needs (0 if cfg is
 * invalid). Layout, level-major: for l = 1..L, float32
 * [n_kv_heads][floor(max_tokens / C^l)][node_floats], each node holding
 * khat [n_ref][head_dim] then bhat [n_ref], padded to node_floats =
 * n_ref*head_dim + round_up(n_ref, 4) [ZHA: 무엇과 다른가]; then, at the next
 * 256-byte boundary, one 256-byte block whose first int32 is the tree's
 * device status word (ZHA_DEV_TIMEOUT set by a build kernel whose bounded wait
 * ran out; zha_build clears it, zha_route passes it on to its d_status).
 * With head_dim 128 and n_ref 16, a second copy of the planes follows, the
 * operand of the tensor-core scoring: for l = 1..L, fp16
 * [n_kv_heads][2][floor(max_tokens / C^l)][n_ref][head_dim], term 0 = khat
 * rounded to fp16 and term 1 = the remainder rounded to fp16. zha_build and
 * zha_append_chunk write it together with the float32 planes; the routing
 * scores from the terms, so a caller that writes planes into the store itself
 * writes their terms as well. */
size_t zha_tree_bytes(const zha_config* cfg);

/* Create a host handle over a caller-owned store (>= zha_tree_bytes bytes,
 * 256-byte aligned) and reference queries d_ref_q [n_kv_heads][n_ref][head_dim]
 * float32, which must stay valid while the tree is used. The tree starts empty
 * (0 tokens built). Returns ZHA_ERR_INVALID / ZHA_ERR_CAPACITY / ZHA_ERR_UNSUPPORTED
 * on bad arguments; *out is set only on success. The learned reference queries
 * are the only trained parameters of the method [ZHA: 어떻게 쓰나]. */
zha_status zha_tree_create(const zha_config* cfg, void* d_store, size_t store_bytes,
                           const float* d_ref_q, zha_tree** out);

/* Release a handle (the store and reference queries stay the caller's). NULL is ignored. */
void zha_tree_destroy(zha_tree* tree);

/* N_b: tokens covered by complete level-1 chunks so far (a multiple of C). */
int64_t zha_tree_built_tokens(const zha_tree* tree);

/* Where level `level` (1..L) lives in the store: float offset of node (g=0,i=0),
 * node capacity per KV head, floats per node. For reading summaries back. */
zha_status zha_tree_level_layout(const zha_tree* tree, int32_t level, int64_t* offset_floats,
                                 int64_t* capacity, int32_t* node_floats);

/* Build every level over the complete chunks of the first n_tokens keys of
 * d_K [n_kv_heads][ld][head_dim] (prefill). Level 1: for chunk i and plane r,
 * s_j = q_r.k_j/sqrt(d) over the chunk, F = LSE_j s_j, khat = sum_j softmax(s)_j k_j,
 * bhat = F - q_r.khat/sqrt(d). Level l >= 2 merges each run of C level-(l-1)
 * nodes: u_c = q_r.khat_{r,c}/sqrt(d) + bhat_{r,c}, F = LSE_c u_c,
 * khat = sum_c softmax(u)_c khat_{r,c}, bhat = F - q_r.khat/sqrt(d)
 * [ZHA: 무엇과 다른가: tangent-plane summary; "parents merge the child summaries
 * in the same way"]. Afterwards N_b = C*floor(n_tokens/C). Requires
 * 0 <= n_tokens <= min(ld, max_tokens). V is not read. The tree's device status
 * word is cleared first; a build kernel whose bounded wait runs out sets
 * ZHA_DEV_TIMEOUT there (its summaries are then not valid), and the next
 * zha_route reports it in its own d_status. */
zha_status zha_build(zha_tree* tree, const void* d_K, int64_t ld, int64_t n_tokens, void* stream);

/* Incremental build while decoding: n_tokens is the cache length after the
 * caller has written the newest keys; the new N_b = C*floor(n_tokens/C) must be
 * >= the tree's N_b (else ZHA_ERR_STATE). Summarises each newly completed chunk
 * and merges every upper-level node the new chunks complete (level 1 every C
 * steps, level 2 every C^2 steps [ZHA: 무엇과 다른가]). One launch when up to
 * 8 chunks are new; a no-op when none is. A time-out of a build kernel is
 * recorded in the tree's device status word as for zha_build. */
zha_status zha_append_chunk(zha_tree* tree, const void* d_K, int64_t ld, int64_t n_tokens,
                            void* stream);

/* Workspace bytes zha_route needs for `batch` queries at n_tokens (grows with
 * n_tokens, so sizing for the largest n_tokens covers smaller ones). */
size_t zha_route_workspace_bytes(const zha_config* cfg, int32_t batch, int64_t n_tokens);

/* uint32 words of the per-level kept bitmaps zha_route can return: level-major
 * for l = 1..L, each [batch][n_q_heads][ceil(n_l / 32)] with n_l =
 * floor(N_b / C^l) nodes at n_tokens; bit i of a head's words = node i kept. */
size_t zha_route_kept_words(const zha_config* cfg, int32_t batch, int64_t n_tokens);

/* Per-level top-p routing of `batch` decode queries d_Q [batch][n_q_heads][d]
 * against the tree at n_tokens (C*floor(n_tokens/C) must equal the tree's N_b,
 * else ZHA_ERR_STATE) [ZHA: 전제와 한계]. For each query head and level L..1:
 * candidates are all level-L nodes at the top, below that the children of the
 * nodes kept one level up plus the level's orphans (nodes whose parent does not
 * exist yet); each candidate n scores sigma_n = max_r (q.khat_{r,n}/sqrt(d) +
 * bhat_{r,n}); pi = softmax(sigma) over the candidates; the kept set is the
 * shortest prefix of the candidates ordered by sigma descending (ties: lower
 * node index first) whose pi sums to >= p; p >= 1 keeps all; 0 < p required.
 * Output: d_chunk_ids [batch][n_q_heads][max_sel] int32, the kept level-1 chunk
 * ids ascending, and d_n_chunks [batch][n_q_heads] their count (the sink and
 * the tail [N_b, n_tokens) are implicit and not listed). d_kept_bits (nullable,
 * zha_route_kept_words words) receives every level's kept bitmap. d_ws:
 * >= zha_route_workspace_bytes bytes. d_status (nullable):
 * ZHA_DEV_SELECTION_TRUNCATED, ZHA_DEV_TIMEOUT (tensor-core scoring, or a
 * build of this tree whose bounded wait ran out, passed on from the tree's
 * status word). */
zha_status zha_route(const zha_tree* tree, const float* d_Q, int32_t batch, int64_t n_tokens,
                     float p, int32_t* d_chunk_ids, int32_t* d_n_chunks, int32_t max_sel,
                     uint32_t* d_kept_bits, void* d_ws, size_t ws_bytes, int32_t* d_status,
                     void* stream);

/* Per-level selection rule of zha_route_ex [ZHA: 전제와 한계]. The pages route
 * with top-p at every level and name its depth scaling: one fixed p per level
 * gives an effective p^L, correcting with p^(1/L) drives p towards 1, so p has
 * to follow depth; they also set top-p against a fixed-budget top-K, which
 * keeps the same number of nodes whether the mass is concentrated or flat. */
typedef enum { ZHA_SELECT_TOP_P = 0, ZHA_SELECT_TOP_K = 1 } zha_select_mode;

typedef struct {
    int32_t mode;      /* zha_select_mode */
    int32_t reserved;  /* must be 0 */
    float p[8];        /* ZHA_SELECT_TOP_P: mass of level l (1..L) at p[l-1]; > 0, finite; >= 1
                          keeps every candidate of that level */
    int32_t k[8];      /* ZHA_SELECT_TOP_K: nodes kept at level l at k[l-1], >= 1: the first
                          min(k, candidates) in the order score descending, node index ascending */
} zha_route_policy;

/* zha_route with a per-level policy: top-p with its own p at each level (for
 * instance p^(1/L) per level), or fixed-budget top-K. Candidates, scores,
 * outputs, workspace and status are as for zha_route; only the cut of each
 * level changes. zha_route(p) is zha_route_ex with mode ZHA_SELECT_TOP_P and p
 * at every level. ZHA_ERR_INVALID for a NULL policy, an unknown mode, reserved
 * != 0, or a p / k of levels 1..L out of range (entries past L are ignored). */
zha_status zha_route_ex(const zha_tree* tree, const float* d_Q, int32_t batch, int64_t n_tokens,
                        const zha_route_policy* policy, int32_t* d_chunk_ids, int32_t* d_n_chunks,
                        int32_t max_sel, uint32_t* d_kept_bits, void* d_ws, size_t ws_bytes,
                        int32_t* d_status, void* stream);

/* Size of the routing scratch built into the library for zha_route_noalloc. */
#define ZHA_ROUTE_NOALLOC_SCRATCH_BYTES (32u << 20) /* 32 MiB per GPU that loads the library */

/* zha_route for callers that cannot allocate device memory. A plugin inside an
 * inference server that owns all device memory may be forbidden to call
 * cudaMalloc; a serving loop with a fixed memory plan cannot allocate per
 * request; a plain C host program may have no device allocator at all. Such
 * callers still pass Q, the outputs, d_kept_bits (nullable) and d_status, as
 * for zha_route, and get the same results, but the scratch zha_route would take
 * as d_ws lives in one fixed device array inside the library
 * (ZHA_ROUTE_NOALLOC_SCRATCH_BYTES, held by every GPU that loads the library
 * until the process exits). This entry point calls no cudaMalloc, cudaFree or
 * other allocating routine.
 *  - A call that needs more scratch than that (zha_route_workspace_bytes, less
 *    the kept bitmaps when d_kept_bits is given) returns ZHA_ERR_CAPACITY and
 *    launches nothing; use zha_route with a workspace then.
 *  - The first call on each device looks up the array's device address (with
 *    that device current) and caches it; make that first call before any
 *    stream capture. With lazy module loading (the CUDA default) that first
 *    lookup is also when the driver loads the library's module on the device
 *    and reserves the array, so a caller whose device memory plan is already
 *    full can see ZHA_ERR_CUDA (out of memory) there: make the first call at
 *    initialisation, before committing the memory plan, or run with eager
 *    module loading (CUDA_MODULE_LOADING=EAGER).
 *  - All calls on a device share the one array and it keeps the last call's
 *    contents (nothing in it needs to start at zero: every call clears or
 *    writes what it reads). Calls whose kernels overlap on the GPU -- on
 *    different streams, or from different threads without ordering -- race on
 *    it; order them.
 * The pages have no counterpart of this call: it only changes where the
 * scratch of zha_route lives. */
zha_status zha_route_noalloc(const zha_tree* tree, const float* d_Q, int32_t batch,
                             int64_t n_tokens, float p, int32_t* d_chunk_ids, int32_t* d_n_chunks,
                             int32_t max_sel, uint32_t* d_kept_bits, int32_t* d_status,
                             void* stream);

/* Workspace bytes zha_sparse_attend needs for `batch` queries at n_tokens. */
size_t zha_attend_workspace_bytes(const zha_config* cfg, int32_t batch, int64_t n_tokens);

/* Exact attention of each query head over S = {0} u tokens(listed chunks) u
 * [N_b, n_tokens), N_b = C*floor(n_tokens/C): o = sum_{j in S} softmax_j(q.k_j/
 * sqrt(d)) v_j, normalised over S only [Attention: "Scaled dot-product attention
 * 의 식"; ZHA: 전제와 한계]. Chunk lists as zha_route writes them (ascending
 * ids < N_b/C, counts <= max_sel); they may also come from elsewhere. The tree
 * supplies only its configuration (its summaries are not read). Output d_O
 * [batch][n_q_heads][d] float32 and, if d_lse is not NULL, d_lse
 * [batch][n_q_heads] = log sum_{j in S} exp(q.k_j/sqrt(d)). d_ws: >=
 * zha_attend_workspace_bytes bytes. d_status (nullable): ZHA_DEV_BAD_SELECTION,
 * ZHA_DEV_TIMEOUT.
 * Requires 1 <= n_tokens <= ld. */
zha_status zha_sparse_attend(const zha_tree* tree, const float* d_Q, const void* d_K,
                             const void* d_V, int64_t ld, int64_t n_tokens, int32_t batch,
                             const int32_t* d_chunk_ids, const int32_t* d_n_chunks,
                             int32_t max_sel, float* d_O, float* d_lse, void* d_ws,
                             size_t ws_bytes, int32_t* d_status, void* stream);

/* ---- Paged K/V caches [Attention: "KV cache 를 담는 방식을 바꾼다: PagedAttention,
 * 양자화"] ---------------------------------------------------------------------
 * A cache held in pages of C tokens (block size = the tree's chunk): a pool
 * [n_pages][C][head_dim] for K and one for V (element type kv_dtype), and a
 * block table: page of chunk c (tokens [cC, (c+1)C)) of KV head g at
 * block_table[g * max_blocks + c]. The in-progress chunk lives in its page too.
 * Summaries, routing and attention are the same as over the contiguous cache
 * holding the same keys and values; only the addresses differ. A table entry
 * outside [0, n_pages) is never dereferenced: ZHA_DEV_BAD_PAGE is set (in the
 * call's d_status, or for builds in the tree's status word, which the next
 * zha_route reports) and those keys count as absent. */
typedef struct {
    const void* k;              /* contiguous: [n_kv_heads][ld][head_dim]; paged: K page pool */
    const void* v;              /* same layout as k; not read by builds (may be NULL there) */
    int64_t ld;                 /* contiguous: token rows per KV head (>= n_tokens); paged: n_pages */
    const int32_t* block_table; /* NULL: contiguous; else [n_kv_heads][max_blocks] int32 page ids */
    int64_t max_blocks;         /* paged: table entries per KV head, >= ceil(n_tokens / C) */
} zha_kv_cache;

/* zha_build / zha_append_chunk / zha_sparse_attend over a zha_kv_cache. The
 * contiguous entry points above are these calls with block_table = NULL. The
 * tensor-core level-1 build serves contiguous caches; paged caches are built
 * by the CUDA-core kernels (same summaries within rounding). */
zha_status zha_build_kv(zha_tree* tree, const zha_kv_cache* kv, int64_t n_tokens, void* stream);
zha_status zha_append_chunk_kv(zha_tree* tree, const zha_kv_cache* kv, int64_t n_tokens, void* stream);
zha_status zha_sparse_attend_kv(const zha_tree* tree, const float* d_Q, const zha_kv_cache* kv,
                                int64_t n_tokens, int32_t batch, const int32_t* d_chunk_ids,
                                const int32_t* d_n_chunks, int32_t max_sel, float* d_O, float* d_lse,
                                void* d_ws, size_t ws_bytes, int32_t* d_status, void* stream);

/* ---- Routing diagnostics [ZHA: 어떻게 쓰나; 전제와 한계] -----------------------
 * How well each level's estimate follows the dense attention mass, for
 * `batch` queries d_Q [batch][n_q_heads][d] against the tree and the keys d_K
 * [n_kv_heads][ld][d] at n_tokens (the tree must cover C*floor(n_tokens/C),
 * else ZHA_ERR_STATE). For every level l and query head:
 *   target p_{l}(n) = the dense softmax weights of q over the keys the level's
 *     complete nodes cover, summed node by node (the reference queries' KL
 *     training target [ZHA: 어떻게 쓰나]; the in-progress tail is in no node);
 *   estimate p_hat_{l}(n) = softmax over the level's nodes of max_r t_r(q);
 *   d_kl[l-1][batch][n_q_heads] = KL(p_l || p_hat_l) (float32, natural log).
 * d_usage (nullable, uint32 [L][n_ref], ACCUMULATED -- the caller zeroes it):
 * for every node of every level and every query head, +1 at the plane r that
 * gives the node's score (lowest r on ties); [ZHA: 전제와 한계] reports that
 * few reference queries serve the upper levels and that their use evens out
 * towards the leaves. Every node of every level is scored and the dense mass of
 * every complete chunk is formed, so this costs a dense pass over the keys: a
 * diagnostic, not part of routing. d_ws: >= zha_diagnostics_workspace_bytes. */
size_t zha_diagnostics_workspace_bytes(const zha_config* cfg, int32_t batch, int64_t n_tokens);
zha_status zha_route_diagnostics(const zha_tree* tree, const float* d_Q, const void* d_K, int64_t ld,
                                 int32_t batch, int64_t n_tokens, float* d_kl, uint32_t* d_usage,
                                 void* d_ws, size_t ws_bytes, void* stream);

/* ---- Test hook (the pages have no counterpart) ------------------------------
 * For tests of the bounded waits of this tree's tensor-core level scoring
 * (head_dim 128, R = 16): wait_polls = polls of each of its mbarrier waits
 * before the wait gives up (0 restores the default, about 2 s; each poll lets
 * the thread sleep up to about 65 us); withhold != 0 makes its producer send
 * nothing, so that the consumers' waits run out with nothing in flight: the
 * kernel releases its tensor memory, returns, and the route reports
 * ZHA_DEV_TIMEOUT (its outputs are then not valid). Not for production use. */
zha_status zha_tree_debug(zha_tree* tree, uint32_t wait_polls, int32_t withhold);

/* ---- Kernel timing (profiling; the pages have no counterpart) ------------
 * While enabled, every kernel the library launches whose name contains
 * `name_filter` (NULL or "" = all) and whose tag equals `tag_filter` (-1 = all;
 * the tag is the tree level for the routing kernels, 0 otherwise) is bracketed
 * by two CUDA events recorded on its stream. Up to `max_records` launches are
 * recorded (later ones are counted as dropped); max_records <= 0 disables
 * tracing. The events are created here (host-side driver objects, no device
 * memory); each enable discards the previous records. Recording events between
 * kernels removes their programmatic overlap, so traced calls run a little
 * slower than untraced ones. Not thread-safe against concurrent launches from
 * other threads while enabled. */
zha_status zha_trace_enable(int32_t max_records, const char* name_filter, int32_t tag_filter);

/* Launches recorded since the last enable or clear, and launches dropped
 * because the records were full. */
int32_t zha_trace_count(void);
int32_t zha_trace_dropped(void);

/* Record i (0 <= i < zha_trace_count()): kernel name (static string), tag and
 * device time in milliseconds. The caller must have synchronised the streams
 * the kernels ran on. */
zha_status zha_trace_read(int32_t i, const char** name, int32_t* tag, float* ms);

/* Forget the records (the events are kept for reuse). */
void zha_trace_clear(void);

#ifdef __cplusplus
}
#endif

#endif /* ZHA_H */
