/*
 * zha.h -- C ABI of libzha, the sm_100a (B200) decode path of Zyphra
 * Hierarchical Attention (ZHA): a tree of key summaries over the KV cache of
 * one GQA attention layer, top-p routing down that tree, and exact attention
 * over the routed tokens.
 *
 * Method (page "Zyphra AI Introduces Zyphra Hierarchical Attention (ZHA)",
 * MarkTechPost article):
 *   - section "Building the tree": the cache is cut into contiguous chunks of c
 *     keys; R learned reference queries each give a chunk a tangent plane of
 *     its log attention mass; c sibling summaries are in turn summarised into
 *     a parent, one level at a time; the largest plane value is the node's
 *     estimate.
 *   - section "How does top-p routing pick tokens": a decode query rates the
 *     nodes of the top level, retains the fewest whose estimated mass adds up
 *     to at least p of the total, rates only the children of those, and goes
 *     on down to the raw KV; token 0 (the attention sink) is attended in
 *     every case.
 *   - explainer widget, step 5: the final attention is exact, over the raw KV
 *     that routing picked plus the sink and the chunk being written; the
 *     whole cache is kept.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller. The library
 *     allocates no device memory; scratch lives in a caller-provided
 *     workspace of zha_workspace_bytes() bytes, the tree in a caller-provided
 *     buffer of zha_tree_bytes() bytes. Pointers must be 16-byte aligned.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as
 *     void*; NULL = legacy default stream) and never synchronises.
 *   - Argument errors are returned synchronously and nothing is enqueued.
 *     Errors the GPU detects (a length beyond max_len, a leaf index out of
 *     range, a capacity overflow) are written to the caller's int32 word
 *     `dev_status` (first error wins; the caller zeroes it and reads it after
 *     a sync); kernels never trap.
 *   - Layouts (row-major, innermost last), dtype = cfg->dtype for
 *     K, V, q, refs, out, k_new, v_new:
 *       K, V   [batch][n_kv_heads][max_len][head_dim]
 *       q      [batch][n_q_heads][head_dim]
 *       refs   [n_kv_heads][n_refs][head_dim]
 *       out    [batch][n_q_heads][head_dim]
 *       lens   [batch] int32: tokens currently in each sequence's cache
 *     Query head h uses KV head h / G, G = n_q_heads / n_kv_heads.
 *   - Supported: head_dim in {64, 128}; chunk a power of two in [2, 256];
 *     1 <= levels <= ZHA_MAX_LEVELS; 1 <= n_refs <= 32; G <= 16;
 *     max_len <= 2^30 and max_len / chunk <= 2^23; dtype BF16 or F32.
 *     Anything else returns ZHA_ERR_UNSUPPORTED.
 */
#ifndef ZHA_H
#define ZHA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ZHA_API __attribute__((visibility("default")))
#else
#define ZHA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum zha_status {
    ZHA_OK = 0,
    ZHA_ERR_INVALID_ARG = 1,
    ZHA_ERR_UNSUPPORTED = 2,
    ZHA_ERR_CAPACITY = 3,
    ZHA_ERR_CUDA = 4,
    ZHA_ERR_TIMEOUT = 5
} zha_status;

enum { ZHA_BF16 = 0, ZHA_F32 = 1 };

/* cfg->flags */
enum {
    /* current chunk = only the incomplete tail [c*floor(N/c), N) instead of the
     * chunk holding the newest token [c*floor((N-1)/c), N) */
    ZHA_FLAG_TAIL_ONLY = 1,
    /* score candidate nodes with the tcgen05 kernel (TMA-fed tensor-core MMAs
     * accumulating in tensor memory) where it applies: bf16, head_dim 128,
     * n_refs 16, G <= 16, batch * n_kv_heads <= 16. The default is the
     * mma.sync kernel, which streams the summaries at a higher fraction of
     * HBM bandwidth on this path */
    ZHA_FLAG_TCGEN05 = 2,
    /* route in one launch: one thread-block cluster (16 CTAs where every
     * group's cluster fits on the GPU at once, else 8) per (sequence, KV
     * head) walks every level -- scoring into the query rows' CTAs through
     * distributed shared memory, a cluster barrier, each row's exact
     * selection by its own CTA, a cluster barrier, the join in every CTA.
     * Same selections, scores and outputs as the default per-level launches,
     * bit for bit. It pays off when few nodes are kept per level (trained
     * references: up to ~1,000 candidates per level and group); a level with
     * more candidates is handled correctly but slowly (one warp per query
     * row selects over the workspace), and there the default is far faster.
     * Applies to bf16 trees with native summaries, n_refs 16, at most 8
     * query heads per KV head and at most 1,024 top-level nodes at max_len
     * (the top level is scored whole), single queries; otherwise the default
     * route runs. */
    ZHA_FLAG_FUSED_ROUTE = 4
};

#define ZHA_MAX_LEVELS 8

/* cfg->summary: how the tree keeps each plane's mu (the bias is always fp32).
 *   ZHA_SUMMARY_NATIVE  mu in the KV dtype.
 *   ZHA_SUMMARY_MXFP8   low-precision router summaries (the MarkTechPost
 *       article's TL;DR box mentions an FP4 router variant without a format;
 *       this library's reading, at 8 bits): mu in blocks of 32 consecutive
 *       coordinates, each block one power-of-two scale 2^e (a biased exponent
 *       byte e + 127) times 32 FP8 E4M3 values, the block layout of the OCP
 *       Microscaling (MX) specification v1.0; e is the smallest exponent with
 *       max|x| <= 448 * 2^e, elements round to nearest even. A node record
 *       shrinks from R*d*2 + 4R bytes to R*d + R*d/32 + 4R. Parents are built
 *       from the stored (rounded) children. Requires dtype ZHA_BF16. Scoring
 *       against these summaries uses warp-level E4M3 MMAs: each query head is
 *       held as 2^e (hi + lo) with hi, lo E4M3 and one power-of-two scale per
 *       head (about 8 significant bits, as bf16). */
enum { ZHA_SUMMARY_NATIVE = 0, ZHA_SUMMARY_MXFP8 = 1 };

typedef struct zha_config {
    int32_t batch;       /* B */
    int32_t n_q_heads;   /* Hq */
    int32_t n_kv_heads;  /* Hkv; one tree per (sequence, KV head) */
    int32_t head_dim;    /* d */
    int32_t chunk;       /* c: keys per leaf, children per parent */
    int32_t levels;      /* L: levels of the tree (1 = leaves only) */
    int32_t n_refs;      /* R: reference queries per KV head */
    int32_t dtype;       /* ZHA_BF16 or ZHA_F32 */
    int64_t max_len;     /* token capacity of K/V per sequence */
    float scale;         /* s; <= 0 selects 1/sqrt(head_dim) */
    int32_t flags;       /* ZHA_FLAG_* */
    int32_t attn_splits; /* split-K CTAs per (sequence, KV head); 0 = auto */
    int32_t summary;     /* ZHA_SUMMARY_NATIVE or ZHA_SUMMARY_MXFP8 */
    int32_t queries;     /* most query positions per sequence in one zha_decode_block
                            call (0 or 1: single-query use only); the workspace is
                            sized for it; queries * (n_q_heads / n_kv_heads) <= 32 */
    int32_t reserved;    /* zero */
} zha_config;

/*
 * Routed selection of every (sequence, KV head) group: the union over the
 * group's G query heads of the kept leaf chunks, ascending, with one bit per
 * query head saying which heads keep each chunk. All device pointers.
 *   leaf_idx  [batch][n_kv_heads][cap1] int32   (cap1 = max_len / chunk)
 *   head_mask [batch][n_kv_heads][cap1] uint32  bit j: query head g*G+j
 *   count     [batch][n_kv_heads]       int32   entries in use
 *   level_kept [batch][n_q_heads][levels] int32 optional (NULL = not written):
 *             nodes kept by each query head at each level (index l-1)
 */
typedef struct zha_selection {
    int32_t *leaf_idx;
    uint32_t *head_mask;
    int32_t *count;
    int32_t *level_kept;
} zha_selection;

/* Byte offsets, inside the workspace, of the per-level routing state of the
 * last zha_route / zha_decode call (valid until the workspace is reused):
 *   cand_idx  [batch][n_kv_heads][cap] int32    candidate node indices, ascending
 *   cand_mask [batch][n_kv_heads][cap] uint32   heads for which it is a candidate
 *                                               (0: padding, a child past the level's end)
 *   scores    [batch][n_kv_heads][G][cap] float estimate max_r(s q.mu_r + b_r)
 *   kept_mask [batch][n_kv_heads][cap] uint32   heads that kept it
 *   count     [batch][n_kv_heads] int32         entries in use
 * cap = nodes at that level for max_len tokens, plus chunk, rounded up to a
 * multiple of 8. */
typedef struct zha_level_view {
    int64_t cap;
    size_t cand_idx, cand_mask, scores, kept_mask, count;
} zha_level_view;

/* Message for a status code (static string). */
ZHA_API const char *zha_status_string(zha_status s);

/* ZHA_OK if the configuration is supported; otherwise why not. */
ZHA_API zha_status zha_check_config(const zha_config *cfg);

/* Nodes at `level` (1 = leaf chunks) for n tokens: n_1 = floor(n / c)
 * (only complete chunks enter the tree), n_l = ceil(n_{l-1} / c). */
ZHA_API int64_t zha_level_nodes(const zha_config *cfg, int64_t n_tokens, int32_t level);

/* Which routing a call with this configuration runs (host only, no GPU
 * work): *fused = 1 if zha_route, zha_decode (T = 1) and zha_decode_block
 * with T query positions score all levels in the one fused launch, 0 if they
 * launch per level. The fused launch needs ZHA_FLAG_FUSED_ROUTE and the
 * configuration that flag's description lists; any other configuration,
 * flag set or not, routes per level. ZHA_ERR_INVALID_ARG for a bad config,
 * T < 1 or a null `fused`. */
ZHA_API zha_status zha_route_fused(const zha_config *cfg, int32_t T, int32_t *fused);

/* Bytes of the tree buffer for cfg->max_len tokens per sequence, and the
 * byte offsets of level l's arrays inside it:
 *   mu   [batch][n_kv_heads][cap_l][n_refs][head_dim]  dtype (summary keys),
 *        or FP8 E4M3 bytes with ZHA_SUMMARY_MXFP8
 *   bias [batch][n_kv_heads][cap_l][n_refs]            float (plane offsets)
 * A node's plane r evaluates to s*q.mu_r + bias_r. */
ZHA_API size_t zha_tree_bytes(const zha_config *cfg);
ZHA_API zha_status zha_tree_level_offsets(const zha_config *cfg, int32_t level, size_t *mu_off,
                                  size_t *bias_off);

/* Byte offset of level l's log-masses inside the tree buffer,
 *   F [batch][n_kv_heads][cap_l][n_refs]  float,
 * F_r = log sum over the node's keys of e^{s r.k}: the node's log attention
 * mass at reference r, where its plane is exact (in exact arithmetic
 * F_r = s r.mu_r + bias_r before mu is rounded for storage). A parent weights
 * child i of reference r by e^{F_{i,r}} (section "Building the tree": a
 * parent summarises its children by the same rule as a chunk its keys). */
ZHA_API zha_status zha_tree_level_logmass(const zha_config *cfg, int32_t level, size_t *lm_off);

/* ZHA_SUMMARY_MXFP8 only: byte offset of level l's block scales,
 *   scale [batch][n_kv_heads][cap_l][n_refs][head_dim / 32]  uint8 = e + 127,
 * mu_r[k] = e4m3(mu byte o(k)) * 2^(scale[k / 32] - 127), where a plane's
 * head_dim bytes are stored permuted so that a scoring lane fetches its bytes
 * of two adjacent blocks with one 16-byte load: with b = k / 32, w = k % 32,
 *   o(k) = 64 (b / 2) + 16 ((w % 16) / 4) + 8 (b % 2) + 4 (w / 16) + w % 4.
 * ZHA_ERR_INVALID_ARG for the native format. */
ZHA_API zha_status zha_tree_level_scales(const zha_config *cfg, int32_t level, size_t *scale_off);

/* Bytes of scratch every call below may use (routing state + split-K
 * partials). Zero it once before its first use: some of its counters and
 * histograms are expected at zero on entry, and every call that returns
 * ZHA_OK with a zero dev_status leaves them at zero again (after a device
 * error, zero it again). One workspace serves one call at a time. */
ZHA_API size_t zha_workspace_bytes(const zha_config *cfg);
ZHA_API zha_status zha_workspace_level_view(const zha_config *cfg, int32_t level, zha_level_view *v);
/* The same for the last zha_decode_block call with T query positions (its
 * scores are [batch][n_kv_heads][T * G][cap], row t * G + head). */
ZHA_API zha_status zha_workspace_level_view_block(const zha_config *cfg, int32_t T, int32_t level,
                                                  zha_level_view *v);

/*
 * zha_tree_build -- summarise the first lens[b] tokens of every sequence
 * from scratch (section "Building the tree").
 * Leaf j, reference r, keys k_t of chunk j:  l_t = s r.k_t,
 * F = log sum_t e^{l_t}, w_t = e^{l_t - F}, mu_r = sum_t w_t k_t,
 * bias_r = F - s r.mu_r. A parent applies the same rule to its existing
 * children, child i entering as the point mu_{i,r} with log-weight F_{i,r},
 * its log-mass at r (see zha_tree_level_logmass); the rightmost node of a
 * level may have fewer than c children. mu is rounded to dtype once
 * computed; parents read the rounded children.
 */
ZHA_API zha_status zha_tree_build(const zha_config *cfg, void *tree, const void *K, const void *refs,
                          const int32_t *lens, int32_t *dev_status, void *stream);

/*
 * zha_tree_append -- the caller has written n_new more tokens into K and
 * lens[b] already counts them: bring the tree from lens[b]-n_new to lens[b]
 * tokens (the chunks that completed, then every ancestor from the first
 * changed node to the right end of each level). Bit-identical to
 * zha_tree_build at the new lengths. Tree depth is fixed by cfg->levels.
 */
ZHA_API zha_status zha_tree_append(const zha_config *cfg, void *tree, const void *K, const void *refs,
                           const int32_t *lens, int32_t n_new, int32_t *dev_status, void *stream);

/*
 * zha_route -- top-p routing of every query head (section "How does top-p
 * routing pick tokens"). Per query head, level L down to 1: the candidates'
 * estimates E = max_r(s q.mu_r + bias_r) are turned into masses e^{E-max};
 * with the candidates ordered by (E descending, node index ascending) the
 * shortest prefix whose running mass reaches p times the total is kept; the
 * existing children of kept nodes are the next level's candidates. Level L's
 * candidates are all its nodes. p_levels[l-1] (host array, L entries) is the
 * fraction at level l; a value >= 1 keeps every candidate; values <= 0 or
 * NaN are ZHA_ERR_INVALID_ARG. Result in *sel (see zha_selection).
 */
ZHA_API zha_status zha_route(const zha_config *cfg, const void *tree, const void *q, const int32_t *lens,
                     const float *p_levels, const zha_selection *sel, void *workspace,
                     int32_t *dev_status, void *stream);

/*
 * zha_sparse_attn -- exact softmax attention of every query head over its
 * token set {0} U {tokens of the leaf chunks of *sel whose head bit is set}
 * U current chunk, with the current chunk [c*floor((N-1)/c), N)
 * (ZHA_FLAG_TAIL_ONLY: [c*floor(N/c), N)), N = lens[b]:
 *   out_h = sum_t softmax_t(s q_h.k_t) v_t   (fp32 accumulation).
 * Leaf indices at or beyond floor(N/c) set ZHA_ERR_INVALID_ARG in dev_status
 * and are skipped. `sel` may come from zha_route or from the caller.
 */
ZHA_API zha_status zha_sparse_attn(const zha_config *cfg, const void *q, const void *K, const void *V,
                           const int32_t *lens, const zha_selection *sel, void *out,
                           void *workspace, int32_t *dev_status, void *stream);

/*
 * zha_decode -- one decode step of the layer: write k_new/v_new
 * ([batch][n_kv_heads][head_dim]) at position lens[b] of K/V, increment
 * lens[b], extend the tree (zha_tree_append with n_new = 1), route the
 * queries q, and attend (zha_sparse_attn). lens is updated on the device.
 * Selection written to *sel.
 */
ZHA_API zha_status zha_decode(const zha_config *cfg, void *tree, void *K, void *V, const void *refs,
                      int32_t *lens, const void *q, const void *k_new, const void *v_new,
                      const float *p_levels, const zha_selection *sel, void *out,
                      void *workspace, int32_t *dev_status, void *stream);

/*
 * zha_decode_block -- T consecutive query positions of every sequence in one
 * call: a multi-query decode or chunked-prefill block. The pages describe
 * routing for one decoding query (section "How does top-p routing pick
 * tokens"); this entry point applies it to T queries that share every
 * summary and KV read. Reading taken here: with N0 = lens[b] tokens cached,
 *   1. the block's keys/values k_new, v_new [batch][T][n_kv_heads][head_dim]
 *      are written at positions N0 .. N0+T-1 and lens[b] becomes N0 + T;
 *   2. every query row (t, head) routes as in zha_route over the tree of the
 *      first N0 tokens (the tree before the block; p_levels as in zha_route);
 *   3. row t attends exactly over {0} U its kept leaf chunks U
 *      [c*floor(N0/c), N0 + t]: the cached tail after the last complete
 *      chunk and the block's tokens up to its own position (causal);
 *   4. the tree is extended by the T new tokens (as zha_tree_append).
 * q and out are [batch][T][n_q_heads][head_dim]. In *sel, a group's head
 * mask bit r is query row r = t * (n_q_heads / n_kv_heads) + head, and
 * level_kept is [batch][n_kv_heads][T][n_q_heads / n_kv_heads][levels].
 * Requires 1 <= T <= max(1, cfg->queries); ZHA_FLAG_TCGEN05 is ignored.
 * With T = 1 the token set equals zha_decode's; the routing differs from it
 * only when the new token completes a chunk (zha_decode routes over the
 * extended tree).
 */
ZHA_API zha_status zha_decode_block(const zha_config *cfg, int32_t T, void *tree, void *K, void *V,
                                    const void *refs, int32_t *lens, const void *q, const void *k_new,
                                    const void *v_new, const float *p_levels, const zha_selection *sel,
                                    void *out, void *workspace, int32_t *dev_status, void *stream);

/*
 * zha_dense_decode -- the comparison kernel: exact softmax attention of every
 * query head over all lens[b] tokens (split-K flash decoding, same numerics
 * as zha_sparse_attn).
 */
ZHA_API zha_status zha_dense_decode(const zha_config *cfg, const void *q, const void *K, const void *V,
                            const int32_t *lens, void *out, void *workspace, int32_t *dev_status,
                            void *stream);

/*
 * zha_dense_decode_noalloc -- zha_dense_decode for callers that cannot
 * allocate device memory (no counterpart on the method's pages). Some callers
 * cannot call cudaMalloc or hand over a workspace: code embedded in a host
 * framework that owns every device allocation through its own arena, or a
 * latency-critical loop that must not pay for cudaMalloc, which can
 * synchronise the device. This entry point takes the same inputs and output
 * as zha_dense_decode and no workspace: its split-K scratch is a fixed 4 MiB
 * array compiled into the library. It takes device memory when the library's
 * module is loaded on a device -- under CUDA's default lazy loading, at the
 * first call into the library on that device, which may be this entry's
 * first call -- and keeps it until the process exits or the context is
 * reset. A caller that hands the rest of device memory to its own arena makes
 * one call (any entry point) first. Configurations whose split-K
 * partials (batch * n_kv_heads * splits * G * (head_dim + 2) floats, each
 * part rounded up to 256 bytes) exceed 4 MiB return ZHA_ERR_CAPACITY.
 * All calls share the array, so calls whose kernels overlap on the GPU (for
 * example on two streams at once) race and must be serialised by the caller.
 * Every call made outside a stream capture looks up the array's device
 * address (with that device current; after a context reset the array may
 * have moved); a call being captured uses the address of the last call
 * outside capture, so make one call before the first capture and again after
 * a reset. It allocates nothing, in the library or in any library it calls.
 */
ZHA_API zha_status zha_dense_decode_noalloc(const zha_config *cfg, const void *q, const void *K,
                                            const void *V, const int32_t *lens, void *out,
                                            int32_t *dev_status, void *stream);

/*
 * zha_topp_select -- one level of the routing selection on given scores,
 * for n_sets independent candidate sets (section "How does top-p routing pick
 * tokens"): set i has counts[i] candidates whose fp32 scores are
 * scores[i*stride .. i*stride+counts[i]) in ascending node order; kept[i*stride+j]
 * (uint8) is set to 1 for the kept ones and 0 otherwise. Same arithmetic as
 * the selection inside zha_route. p as in zha_route. Device pointers.
 */
ZHA_API zha_status zha_topp_select(const float *scores, const int32_t *counts, int32_t n_sets,
                           int64_t stride, float p, uint8_t *kept, int32_t *dev_status,
                           void *stream);


/* schedules of zha_p_schedule */
enum { ZHA_P_FIXED = 0, ZHA_P_DEPTH_ROOT = 1 };

/*
 * zha_p_schedule -- per-level routing fractions for zha_route / zha_decode,
 * written to p_levels[0..levels-1] (index l-1 is level l); host memory, no
 * device work. The caveat cards of the MarkTechPost explainer (tab 5, "Top-p
 * must scale with depth") warn that one p used at every level lets coverage
 * shrink as the tree deepens: where mass is spread evenly, each level keeps
 * about a fraction p of what reaches it, so the kept leaves hold about p^L.
 *   ZHA_P_FIXED       p at every level (the pages' configurations).
 *   ZHA_P_DEPTH_ROOT  p^(1/L) at every level, whose product over the L levels
 *                     is p. The pages name no schedule; this is the plainest
 *                     one that undoes the p^L shrinkage.
 * p >= 1 gives 1 at every level. p <= 0 or NaN, levels outside
 * 1..ZHA_MAX_LEVELS, a null p_levels or an unknown schedule:
 * ZHA_ERR_INVALID_ARG (nothing written).
 */
ZHA_API zha_status zha_p_schedule(float p, int32_t levels, int32_t schedule, float *p_levels);

/* waits of zha_wait_expiry_check */
enum { ZHA_WAIT_ROW_BARRIER = 0, ZHA_WAIT_MBARRIER = 1 };

/*
 * zha_wait_expiry_check -- failure detection (no counterpart on the pages).
 * Every wait inside the library's kernels is bounded: the counter barrier of
 * the selection spread over several CTAs per query row, and the mbarrier
 * waits of the tensor-core kernels, give up after about a second, set
 * ZHA_ERR_TIMEOUT in the call's device status and return (the call's results
 * are then invalid; the context stays usable). This entry runs one of those
 * waits on a condition that nothing satisfies, with a caller-given limit, so
 * that the expiry path can be exercised without a fault:
 *   ZHA_WAIT_ROW_BARRIER  the counter barrier, entered by one of two CTAs
 *                         (the other returns without arriving);
 *   ZHA_WAIT_MBARRIER     an mbarrier wait on a barrier that no copy or
 *                         commit completes.
 * limit_cycles: SM clock cycles before the wait gives up, 1 .. 2^31.
 * dev_status: device int32, required; ZHA_ERR_TIMEOUT is written there when
 * the wait runs out. Asynchronous on `stream`. ZHA_ERR_INVALID_ARG for an
 * unknown kind, a limit outside the range or a null dev_status.
 */
ZHA_API zha_status zha_wait_expiry_check(int32_t kind, int64_t limit_cycles, int32_t *dev_status, void *stream);

/*
 * Instrumentation (no counterpart on the pages; for measurement only).
 * zha_launch_count: kernels this library has launched since it was loaded.
 * zha_profile_enable(1): from now on every kernel launch is bracketed by a
 *   pair of CUDA events recorded on its stream; (0) stops recording.
 * zha_profile_read: waits for the recorded events and returns, per kernel
 *   name (names separated by '\n' in `names`, at most max_kernels entries),
 *   the summed duration in ms and the number of launches; then clears the
 *   record. Returns the number of kernel names written, or -1 on error.
 */
ZHA_API uint64_t zha_launch_count(void);
ZHA_API zha_status zha_profile_enable(int32_t on);
ZHA_API int32_t zha_profile_read(char *names, int32_t names_len, double *ms, int64_t *launches,
                                 int32_t max_kernels);

#ifdef __cplusplus
}
#endif

#endif /* ZHA_H */
