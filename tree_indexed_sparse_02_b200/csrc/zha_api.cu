// zha_api.cu -- the extern "C" entry points of libzha: argument checks, the
// derived geometry (tree and workspace layout), and kernel dispatch.
#include <math.h>
#include <string.h>

#include "zha_common.cuh"

namespace {

using zha::Geo;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

zha_status check_config(const zha_config *c) {
    if (!c) return ZHA_ERR_INVALID_ARG;
    if (c->batch < 1 || c->n_kv_heads < 1 || c->n_q_heads < 1 || c->max_len < 1 || c->levels < 1 ||
        c->n_refs < 1 || c->chunk < 1)
        return ZHA_ERR_INVALID_ARG;
    if (c->n_q_heads % c->n_kv_heads) return ZHA_ERR_INVALID_ARG;
    if (c->n_q_heads / c->n_kv_heads > 16) return ZHA_ERR_UNSUPPORTED;
    if (c->head_dim != 64 && c->head_dim != 128) return ZHA_ERR_UNSUPPORTED;
    if (!pow2(c->chunk) || c->chunk < 2 || c->chunk > 256) return ZHA_ERR_UNSUPPORTED;
    if (c->levels > ZHA_MAX_LEVELS || c->n_refs > 32) return ZHA_ERR_UNSUPPORTED;
    if (c->dtype != ZHA_BF16 && c->dtype != ZHA_F32) return ZHA_ERR_UNSUPPORTED;
    if (c->flags & ~(ZHA_FLAG_TAIL_ONLY | ZHA_FLAG_TCGEN05 | ZHA_FLAG_FUSED_ROUTE)) return ZHA_ERR_UNSUPPORTED;
    // int32 token and leaf indices; fixed-point mass sums need <= 2^23 candidates
    if (c->max_len > (1 << 30) || c->max_len / c->chunk > (1 << 23)) return ZHA_ERR_UNSUPPORTED;
    if (c->attn_splits < 0 || c->attn_splits > 4096) return ZHA_ERR_INVALID_ARG;
    if (!(c->scale == c->scale)) return ZHA_ERR_INVALID_ARG;
    if (c->summary != ZHA_SUMMARY_NATIVE && c->summary != ZHA_SUMMARY_MXFP8) return ZHA_ERR_UNSUPPORTED;
    if (c->summary == ZHA_SUMMARY_MXFP8 && c->dtype != ZHA_BF16) return ZHA_ERR_UNSUPPORTED;
    if (c->queries < 0) return ZHA_ERR_INVALID_ARG;
    if ((c->queries > 1 ? c->queries : 1) * (c->n_q_heads / c->n_kv_heads) > 32) return ZHA_ERR_UNSUPPORTED;
    return ZHA_OK;
}

// Geometry of one call; T query positions per sequence (zha_decode_block),
// 1 for every other entry point. Workspace offsets depend on T; each call
// lays out its own, inside zha_workspace_bytes (sized for the largest T).
Geo make_geo(const zha_config *c, int T = 1) {
    Geo g{};
    g.B = c->batch;
    g.Hq = c->n_q_heads;
    g.Hkv = c->n_kv_heads;
    g.Gq = c->n_q_heads / c->n_kv_heads;
    g.T = T;
    g.G = T * g.Gq;
    g.lag = 0;
    g.d = c->head_dim;
    g.c = c->chunk;
    g.L = c->levels;
    g.R = c->n_refs;
    g.dtype = c->dtype;
    g.flags = c->flags;
    // The fused route scores the top level whole in a cluster's shared memory
    // (up to 1,024 candidates a level); a tree whose top level can outgrow
    // that takes the per-level route, which is the faster one there.
    constexpr int64_t kFusedTopNodes = 1024;
    if (zha::level_nodes(c->max_len, c->chunk, c->levels) > kFusedTopNodes) g.flags &= ~ZHA_FLAG_FUSED_ROUTE;
    g.summary = c->summary;
    g.max_len = c->max_len;
    g.s = c->scale > 0.f ? c->scale : 1.f / sqrtf((float)c->head_dim);
    const size_t groups = (size_t)g.B * g.Hkv;
    const size_t es = g.mu_esize();
    size_t off = 0;
    for (int l = 1; l <= g.L; ++l) {
        g.cap[l] = zha::level_nodes(g.max_len, g.c, l);
        g.mu_off[l] = off;
        off = align256(off + groups * g.cap[l] * g.R * g.d * es);
        g.sc_off[l] = 0;
        if (g.mx()) {
            g.sc_off[l] = off;
            off = align256(off + groups * g.cap[l] * g.R * (g.d / 32));
        }
        g.bias_off[l] = off;
        off = align256(off + groups * g.cap[l] * g.R * sizeof(float));
        g.lm_off[l] = off;
        off = align256(off + groups * g.cap[l] * g.R * sizeof(float));
    }
    g.tree_bytes = off;
    off = 0;
    {
        const size_t rows_max = (size_t)g.Gq * (c->queries > 1 ? c->queries : 1);
        g.ws_ghist = off;
        off = align256(off + groups * rows_max * zha::kSelBuckets * 8);
    }
    for (int l = 1; l <= g.L; ++l) {
        g.capv[l] = (g.cap[l] + g.c + 7) & ~int64_t(7);
        const size_t n = groups * g.capv[l];
        g.ws_cand[l] = off;   off = align256(off + n * 4);
        g.ws_cmask[l] = off;  off = align256(off + n * 4);
        g.ws_kept[l] = off;   off = align256(off + n * 4);
        g.ws_scores[l] = off; off = align256(off + n * g.G * 4);
        g.ws_keptbits[l] = off; off = align256(off + groups * g.G * g.bits_stride(l));
        g.ws_count[l] = off;  off = align256(off + groups * 4);
        const size_t k = groups * g.cap[l];
        g.ws_plist[l] = off;  off = align256(off + k * 4);
        g.ws_pmask[l] = off;  off = align256(off + k * 4);
        g.ws_pcount[l] = off; off = align256(off + groups * 4);
    }
    g.ws_maxkey = off;
    off = align256(off + (size_t)g.L * groups * g.G * 4);
    g.ws_minkey = off;
    off = align256(off + (size_t)g.L * groups * g.G * 4);
    g.ws_done = off;
    off = align256(off + (size_t)g.L * groups * 4);
    g.ws_glidx = off;
    off = align256(off + groups * g.G * zha::kSelList * 4);
    g.ws_glkey = off;
    off = align256(off + groups * g.G * zha::kSelList * 4);
    g.ws_gctr = off;
    off = align256(off + (size_t)g.L * groups * g.G * 4 * 4);
    g.ws_lookback = off;
    for (int l = 1; l <= g.L; ++l) off += groups * ((g.capv[l] + zha::kJoinChunk - 1) / zha::kJoinChunk) * 8;
    off = align256(off);
    g.ws_arrive = off;
    off = align256(off + (size_t)g.B * 4);
    int splits = c->attn_splits;
    if (splits == 0) {
        // one wave of two resident CTAs per SM over all groups, at most one per 64 tokens
        const int64_t want = (148 * 2) / (int64_t)groups;
        const int64_t most = (g.max_len + 63) / 64;
        splits = (int)(want < most ? want : most);
        if (splits < 1) splits = 1;
    }
    g.splits = splits;
    g.ws_part_ml = off;
    off = align256(off + groups * splits * g.G * 2 * 4);
    g.ws_part_o = off;
    off = align256(off + groups * splits * g.G * g.d * 4);
    g.ws_bytes = off;
    return g;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

zha_status cuda_status(cudaError_t e) { return e == cudaSuccess ? ZHA_OK : ZHA_ERR_CUDA; }

zha_status check_p(const zha_config *c, const float *p_levels) {
    if (!p_levels) return ZHA_ERR_INVALID_ARG;
    for (int l = 0; l < c->levels; ++l)
        if (!(p_levels[l] > 0.f)) return ZHA_ERR_INVALID_ARG;  // also rejects NaN
    return ZHA_OK;
}

zha_status check_sel(const zha_selection *sel) {
    if (!sel || !sel->leaf_idx || !sel->head_mask || !sel->count) return ZHA_ERR_INVALID_ARG;
    return ZHA_OK;
}

}  // namespace

namespace zha {
// The geometry of a configuration, for entry points defined in other files.
Geo make_geo_for(const zha_config *c) { return make_geo(c); }
}  // namespace zha

extern "C" {

const char *zha_status_string(zha_status s) {
    switch (s) {
        case ZHA_OK: return "ok";
        case ZHA_ERR_INVALID_ARG: return "invalid argument";
        case ZHA_ERR_UNSUPPORTED: return "unsupported configuration";
        case ZHA_ERR_CAPACITY: return "capacity exceeded (length beyond max_len)";
        case ZHA_ERR_CUDA: return "CUDA error";
        case ZHA_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

zha_status zha_check_config(const zha_config *cfg) { return check_config(cfg); }

int64_t zha_level_nodes(const zha_config *cfg, int64_t n_tokens, int32_t level) {
    if (check_config(cfg) != ZHA_OK || level < 1 || level > cfg->levels || n_tokens < 0) return -1;
    return zha::level_nodes(n_tokens, cfg->chunk, level);
}

zha_status zha_route_fused(const zha_config *cfg, int32_t T, int32_t *fused) {
    zha_status s = check_config(cfg);
    if (s != ZHA_OK) return s;
    if (T < 1 || !fused) return ZHA_ERR_INVALID_ARG;
    const Geo g = make_geo(cfg, T);
    *fused = (g.flags & ZHA_FLAG_FUSED_ROUTE) && zha::fused_route_supported(g) ? 1 : 0;
    return ZHA_OK;
}

size_t zha_tree_bytes(const zha_config *cfg) {
    if (check_config(cfg) != ZHA_OK) return 0;
    return make_geo(cfg).tree_bytes;
}

zha_status zha_tree_level_offsets(const zha_config *cfg, int32_t level, size_t *mu_off,
                                  size_t *bias_off) {
    zha_status s = check_config(cfg);
    if (s != ZHA_OK) return s;
    if (level < 1 || level > cfg->levels || !mu_off || !bias_off) return ZHA_ERR_INVALID_ARG;
    Geo g = make_geo(cfg);
    *mu_off = g.mu_off[level];
    *bias_off = g.bias_off[level];
    return ZHA_OK;
}

zha_status zha_tree_level_logmass(const zha_config *cfg, int32_t level, size_t *lm_off) {
    zha_status s = check_config(cfg);
    if (s != ZHA_OK) return s;
    if (!lm_off || level < 1 || level > cfg->levels) return ZHA_ERR_INVALID_ARG;
    *lm_off = make_geo(cfg).lm_off[level];
    return ZHA_OK;
}

zha_status zha_tree_level_scales(const zha_config *cfg, int32_t level, size_t *scale_off) {
    zha_status s = check_config(cfg);
    if (s != ZHA_OK) return s;
    if (!scale_off || level < 1 || level > cfg->levels || cfg->summary != ZHA_SUMMARY_MXFP8)
        return ZHA_ERR_INVALID_ARG;
    *scale_off = make_geo(cfg).sc_off[level];
    return ZHA_OK;
}

size_t zha_workspace_bytes(const zha_config *cfg) {
    if (check_config(cfg) != ZHA_OK) return 0;
    return make_geo(cfg, cfg->queries > 1 ? cfg->queries : 1).ws_bytes;
}

zha_status zha_workspace_level_view(const zha_config *cfg, int32_t level, zha_level_view *v) {
    return zha_workspace_level_view_block(cfg, 1, level, v);
}

zha_status zha_workspace_level_view_block(const zha_config *cfg, int32_t T, int32_t level,
                                          zha_level_view *v) {
    zha_status s = check_config(cfg);
    if (s != ZHA_OK) return s;
    if (level < 1 || level > cfg->levels || !v) return ZHA_ERR_INVALID_ARG;
    if (T < 1 || T > (cfg->queries > 1 ? cfg->queries : 1)) return ZHA_ERR_INVALID_ARG;
    Geo g = make_geo(cfg, T);
    v->cap = g.capv[level];
    v->cand_idx = g.ws_cand[level];
    v->cand_mask = g.ws_cmask[level];
    v->scores = g.ws_scores[level];
    v->kept_mask = g.ws_kept[level];
    v->count = g.ws_count[level];
    return ZHA_OK;
}

zha_status zha_tree_build(const zha_config *cfg, void *tree, const void *K, const void *refs,
                          const int32_t *lens, int32_t *dev_status, void *stream) {
    zha_status s = check_config(cfg);
    if (s != ZHA_OK) return s;
    if (!tree || !K || !refs || !lens || !aligned16(tree) || !aligned16(K) || !aligned16(refs))
        return ZHA_ERR_INVALID_ARG;
    Geo g = make_geo(cfg);
    return cuda_status(zha::launch_tree_update(g, tree, K, refs, lens, -1, dev_status,
                                               static_cast<cudaStream_t>(stream)));
}

zha_status zha_tree_append(const zha_config *cfg, void *tree, const void *K, const void *refs,
                           const int32_t *lens, int32_t n_new, int32_t *dev_status, void *stream) {
    zha_status s = check_config(cfg);
    if (s != ZHA_OK) return s;
    if (!tree || !K || !refs || !lens || n_new < 0 || !aligned16(tree) || !aligned16(K) ||
        !aligned16(refs))
        return ZHA_ERR_INVALID_ARG;
    if (n_new == 0) return ZHA_OK;
    Geo g = make_geo(cfg);
    return cuda_status(zha::launch_tree_update(g, tree, K, refs, lens, n_new, dev_status,
                                               static_cast<cudaStream_t>(stream)));
}

zha_status zha_route(const zha_config *cfg, const void *tree, const void *q, const int32_t *lens,
                     const float *p_levels, const zha_selection *sel, void *workspace,
                     int32_t *dev_status, void *stream) {
    zha_status s = check_config(cfg);
    if (s != ZHA_OK) return s;
    if ((s = check_p(cfg, p_levels)) != ZHA_OK) return s;
    if ((s = check_sel(sel)) != ZHA_OK) return s;
    if (!tree || !q || !lens || !workspace || !aligned16(tree) || !aligned16(q) ||
        !aligned16(workspace))
        return ZHA_ERR_INVALID_ARG;
    Geo g = make_geo(cfg);
    return cuda_status(zha::launch_route(g, tree, q, lens, p_levels, *sel, workspace, dev_status,
                                         static_cast<cudaStream_t>(stream)));
}

zha_status zha_sparse_attn(const zha_config *cfg, const void *q, const void *K, const void *V,
                           const int32_t *lens, const zha_selection *sel, void *out,
                           void *workspace, int32_t *dev_status, void *stream) {
    zha_status s = check_config(cfg);
    if (s != ZHA_OK) return s;
    if ((s = check_sel(sel)) != ZHA_OK) return s;
    if (!q || !K || !V || !lens || !out || !workspace || !aligned16(q) || !aligned16(K) ||
        !aligned16(V) || !aligned16(out) || !aligned16(workspace))
        return ZHA_ERR_INVALID_ARG;
    Geo g = make_geo(cfg);
    return cuda_status(zha::launch_attention(g, q, K, V, lens, sel, out, workspace, dev_status,
                                             static_cast<cudaStream_t>(stream)));
}

zha_status zha_dense_decode(const zha_config *cfg, const void *q, const void *K, const void *V,
                            const int32_t *lens, void *out, void *workspace, int32_t *dev_status,
                            void *stream) {
    zha_status s = check_config(cfg);
    if (s != ZHA_OK) return s;
    if (!q || !K || !V || !lens || !out || !workspace || !aligned16(q) || !aligned16(K) ||
        !aligned16(V) || !aligned16(out) || !aligned16(workspace))
        return ZHA_ERR_INVALID_ARG;
    Geo g = make_geo(cfg);
    return cuda_status(zha::launch_attention(g, q, K, V, lens, nullptr, out, workspace,
                                             dev_status, static_cast<cudaStream_t>(stream)));
}

zha_status zha_decode(const zha_config *cfg, void *tree, void *K, void *V, const void *refs,
                      int32_t *lens, const void *q, const void *k_new, const void *v_new,
                      const float *p_levels, const zha_selection *sel, void *out,
                      void *workspace, int32_t *dev_status, void *stream) {
    zha_status s = check_config(cfg);
    if (s != ZHA_OK) return s;
    if ((s = check_p(cfg, p_levels)) != ZHA_OK) return s;
    if ((s = check_sel(sel)) != ZHA_OK) return s;
    if (!tree || !K || !V || !refs || !lens || !q || !k_new || !v_new || !out || !workspace ||
        !aligned16(tree) || !aligned16(K) || !aligned16(V) || !aligned16(q) || !aligned16(out) ||
        !aligned16(workspace) || !aligned16(refs))
        return ZHA_ERR_INVALID_ARG;
    Geo g = make_geo(cfg);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = zha::launch_decode_prologue(g, tree, K, V, refs, lens, k_new, v_new, workspace,
                                                dev_status, st);
    if (e == cudaSuccess)
        e = zha::launch_route(g, tree, q, lens, p_levels, *sel, workspace, dev_status, st, false);
    if (e == cudaSuccess)
        e = zha::launch_attention(g, q, K, V, lens, sel, out, workspace, dev_status, st);
    return cuda_status(e);
}

zha_status zha_decode_block(const zha_config *cfg, int32_t T, void *tree, void *K, void *V,
                            const void *refs, int32_t *lens, const void *q, const void *k_new,
                            const void *v_new, const float *p_levels, const zha_selection *sel,
                            void *out, void *workspace, int32_t *dev_status, void *stream) {
    zha_status s = check_config(cfg);
    if (s != ZHA_OK) return s;
    if (T < 1 || T > (cfg->queries > 1 ? cfg->queries : 1)) return ZHA_ERR_INVALID_ARG;
    if ((s = check_p(cfg, p_levels)) != ZHA_OK) return s;
    if ((s = check_sel(sel)) != ZHA_OK) return s;
    if (!tree || !K || !V || !refs || !lens || !q || !k_new || !v_new || !out || !workspace ||
        !aligned16(tree) || !aligned16(K) || !aligned16(V) || !aligned16(q) || !aligned16(out) ||
        !aligned16(workspace) || !aligned16(refs))
        return ZHA_ERR_INVALID_ARG;
    Geo g = make_geo(cfg, T);
    g.flags &= ~ZHA_FLAG_TCGEN05;
    g.block = 1;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // tokens in; route over the tree before the block (lens - T); attend; extend the tree
    cudaError_t e = zha::launch_decode_write(g, K, V, lens, k_new, v_new, dev_status, st);
    if (e == cudaSuccess) {
        Geo gr = g;
        gr.lag = T;
        e = zha::launch_route(gr, tree, q, lens, p_levels, *sel, workspace, dev_status, st);
    }
    if (e == cudaSuccess)
        e = zha::launch_attention(g, q, K, V, lens, sel, out, workspace, dev_status, st);
    if (e == cudaSuccess) e = zha::launch_tree_update(g, tree, K, refs, lens, T, dev_status, st);
    return cuda_status(e);
}

zha_status zha_topp_select(const float *scores, const int32_t *counts, int32_t n_sets,
                           int64_t stride, float p, uint8_t *kept, int32_t *dev_status,
                           void *stream) {
    if (n_sets < 0 || stride < 0 || !(p > 0.f)) return ZHA_ERR_INVALID_ARG;
    if (n_sets == 0) return ZHA_OK;
    if (!scores || !counts || !kept) return ZHA_ERR_INVALID_ARG;
    if (stride > (1 << 23)) return ZHA_ERR_UNSUPPORTED;
    return cuda_status(zha::launch_topp_select(scores, counts, n_sets, stride, p, kept, dev_status,
                                               static_cast<cudaStream_t>(stream)));
}

zha_status zha_wait_expiry_check(int32_t kind, int64_t limit_cycles, int32_t *dev_status, void *stream) {
    if (kind != ZHA_WAIT_ROW_BARRIER && kind != ZHA_WAIT_MBARRIER) return ZHA_ERR_INVALID_ARG;
    if (limit_cycles < 1 || limit_cycles > (int64_t(1) << 31) || !dev_status) return ZHA_ERR_INVALID_ARG;
    return cuda_status(zha::launch_wait_expiry(kind, limit_cycles, dev_status, static_cast<cudaStream_t>(stream)));
}

zha_status zha_p_schedule(float p, int32_t levels, int32_t schedule, float *p_levels) {
    if (!p_levels || !(p > 0.f) || levels < 1 || levels > ZHA_MAX_LEVELS) return ZHA_ERR_INVALID_ARG;
    if (schedule != ZHA_P_FIXED && schedule != ZHA_P_DEPTH_ROOT) return ZHA_ERR_INVALID_ARG;
    float v = p;
    if (p >= 1.f)
        v = 1.f;
    else if (schedule == ZHA_P_DEPTH_ROOT)
        v = static_cast<float>(pow(static_cast<double>(p), 1.0 / levels));
    for (int l = 0; l < levels; ++l) p_levels[l] = v;
    return ZHA_OK;
}

}  // extern "C"
