// zha_common.cuh -- shared device helpers and the derived geometry of one
// configuration (sizes of every tree level, offsets inside the tree buffer and
// the workspace). Internal to libzha.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <utility>

#include "../../include/zha.h"

namespace zha {

constexpr int kMaxLevels = ZHA_MAX_LEVELS;

__host__ __device__ inline int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ inline int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

// Nodes at `level` (1 = leaf chunks) for n tokens: floor(n/c), then ceil(./c).
__host__ __device__ inline int64_t level_nodes(int64_t n, int c, int level) {
    int64_t m = n / c;
    for (int l = 2; l <= level; ++l) m = (m + c - 1) / c;
    return m;
}

constexpr int kSelBuckets = 4096;       // histogram buckets of the top-p selection
constexpr int kSelList = 1024;          // crossing-bucket members ordered in shared memory
constexpr int kJoinChunk = 2048;        // candidates per CTA of the join / compaction

struct Geo {
    // G is the number of query rows a group routes and attends: T query
    // positions x Gq query heads (T = 1 outside zha_decode_block)
    int B, Hq, Hkv, G, d, c, L, R, dtype, flags, splits;
    int T, Gq;
    int lag;                            // block tokens the tree does not hold yet (route reads lens - lag)
    int block;                          // zha_decode_block: causal current span, tree before the block
    int summary;                        // ZHA_SUMMARY_*
    int64_t max_len;
    float s;
    int64_t cap[kMaxLevels + 1];        // nodes per level at max_len (index = level)
    int64_t capv[kMaxLevels + 1];       // candidate slots per level: cap + c (padding children)
    size_t mu_off[kMaxLevels + 1];      // tree buffer offsets
    size_t bias_off[kMaxLevels + 1];
    size_t sc_off[kMaxLevels + 1];      // MX-FP8 block scales (0 for the native format)
    size_t lm_off[kMaxLevels + 1];      // each plane's log-mass at its own reference (fp32)
    size_t tree_bytes;
    // workspace
    size_t ws_cand[kMaxLevels + 1], ws_cmask[kMaxLevels + 1], ws_scores[kMaxLevels + 1],
        ws_kept[kMaxLevels + 1], ws_count[kMaxLevels + 1];     // candidates of a level
    size_t ws_plist[kMaxLevels + 1], ws_pmask[kMaxLevels + 1], ws_pcount[kMaxLevels + 1];  // kept
    size_t ws_keptbits[kMaxLevels + 1];  // [B*Hkv][G][bits_stride] bytes: each row's kept bitmap
    size_t ws_lookback;                 // [L][B*Hkv][join chunks] u64 running counts of the compaction
    size_t ws_arrive;                   // [B] u32 groups of a sequence through the decode prologue
    size_t ws_maxkey, ws_minkey;        // [L][B*Hkv][G] u32 ordered keys of the scores
    size_t ws_done;                     // [L][B*Hkv] u32 finished select CTAs
    size_t ws_part_ml, ws_part_o;       // split-K partials
    // selection spread over several CTAs per query row (same offset for every T:
    // the histograms come first and are left zeroed by every call)
    size_t ws_ghist;                    // [B*Hkv][rows at cfg.queries][kSelBuckets] u64
    size_t ws_glidx, ws_glkey;          // [B*Hkv][G][kSelList] crossing-bucket members
    size_t ws_gctr;                     // [L][B*Hkv][G][4] u32 arrivals, list count, kept count
    size_t ws_bytes;
    __host__ __device__ int groups() const { return B * Hkv; }
    // bytes of one row's kept bitmap at a level (capv / 8, padded to 16 bytes)
    __host__ __device__ int64_t bits_stride(int level) const { return ((capv[level] >> 3) + 15) & ~int64_t(15); }
    // row r of group (b, kvh) -> index of its query vector in q [B][T][Hq][d]
    // (and of its output in out, same layout); rows are ordered (t, head)
    __host__ __device__ int64_t qrow(int b, int kvh, int r) const {
        const int t = r / Gq;
        return ((int64_t)b * T + t) * Hq + kvh * Gq + (r - t * Gq);
    }
    __host__ __device__ int esize() const { return dtype == ZHA_BF16 ? 2 : 4; }
    __host__ __device__ bool mx() const { return summary == ZHA_SUMMARY_MXFP8; }
    __host__ __device__ int mu_esize() const { return mx() ? 1 : esize(); }
};

// ----------------------------------------------------------------- device helpers

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Programmatic dependent launch: kernels on the decode path are launched with
// launch_pdl, so each may be scheduled while the kernel before it on the
// stream finishes. A kernel calls pdl_wait() before it touches memory that
// earlier kernels write (and before any write of its own), and pdl_trigger()
// when its own work is done. Both are no-ops for kernels launched plainly.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// pdl = false launches plainly (full serialisation with the kernel before).
template <typename... P, typename... A>
inline cudaError_t launch_pdl_if(bool pdl, void (*kernel)(P...), dim3 grid, dim3 block, size_t smem,
                                 cudaStream_t st, A &&...args) {
    cudaLaunchConfig_t c{};
    c.gridDim = grid;
    c.blockDim = block;
    c.dynamicSmemBytes = smem;
    c.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    c.attrs = at;
    c.numAttrs = 1;
    return cudaLaunchKernelEx(&c, kernel, std::forward<A>(args)...);
}
template <typename... P, typename... A>
inline cudaError_t launch_pdl(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              A &&...args) {
    return launch_pdl_if(true, kernel, grid, block, smem, st, std::forward<A>(args)...);
}

// First error wins.
__device__ __forceinline__ void set_status(int32_t *status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// Monotone map float -> uint32 (larger float, larger key); 0 is below every
// finite value's key, so it doubles as "no value".
__device__ __forceinline__ uint32_t ordered_key(float f) {
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_to_float(uint32_t k) {
    uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

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

// Load EPL consecutive elements as floats.
template <int EPL>
__device__ __forceinline__ void load_vec(const float *p, float (&v)[EPL]) {
    if constexpr (EPL == 4) {
        float4 t = *reinterpret_cast<const float4 *>(p);
        v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    } else if constexpr (EPL == 2) {
        float2 t = *reinterpret_cast<const float2 *>(p);
        v[0] = t.x; v[1] = t.y;
    } else {
#pragma unroll
        for (int i = 0; i < EPL; ++i) v[i] = p[i];
    }
}
template <int EPL>
__device__ __forceinline__ void load_vec(const __nv_bfloat16 *p, float (&v)[EPL]) {
    if constexpr (EPL == 4) {
        uint2 t = *reinterpret_cast<const uint2 *>(p);
        __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162 *>(&t.x);
        __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&t.y);
        float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
        v[0] = fa.x; v[1] = fa.y; v[2] = fb.x; v[3] = fb.y;
    } else if constexpr (EPL == 2) {
        __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(p);
        float2 fa = __bfloat1622float2(a);
        v[0] = fa.x; v[1] = fa.y;
    } else {
#pragma unroll
        for (int i = 0; i < EPL; ++i) v[i] = __bfloat162float(p[i]);
    }
}
template <int EPL>
__device__ __forceinline__ void store_vec(float *p, const float (&v)[EPL]) {
    if constexpr (EPL == 4) {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    } else if constexpr (EPL == 2) {
        *reinterpret_cast<float2 *>(p) = make_float2(v[0], v[1]);
    } else {
#pragma unroll
        for (int i = 0; i < EPL; ++i) p[i] = v[i];
    }
}
template <int EPL>
__device__ __forceinline__ void store_vec(__nv_bfloat16 *p, const float (&v)[EPL]) {
    if constexpr (EPL == 4) {
        __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
        __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
        uint2 t;
        t.x = *reinterpret_cast<uint32_t *>(&a);
        t.y = *reinterpret_cast<uint32_t *>(&b);
        *reinterpret_cast<uint2 *>(p) = t;
    } else if constexpr (EPL == 2) {
        *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(v[0], v[1]);
    } else {
#pragma unroll
        for (int i = 0; i < EPL; ++i) p[i] = __float2bfloat16_rn(v[i]);
    }
}

// Current chunk start (explainer step 5): the chunk holding the newest token,
// or with ZHA_FLAG_TAIL_ONLY only the incomplete tail.
__host__ __device__ inline int64_t current_chunk_start(int64_t N, int c, int flags) {
    if (N <= 0) return 0;
    return (flags & ZHA_FLAG_TAIL_ONLY) ? (N / c) * c : ((N - 1) / c) * c;
}

}  // namespace zha

// Every kernel launch goes through a ProfScope: it counts the launch and, when
// profiling is on, brackets it with a pair of CUDA events on its stream.
namespace zha {
struct ProfScope {
    ProfScope(const char *name, cudaStream_t st);
    ~ProfScope();
    int slot;
    cudaStream_t st;
};
}  // namespace zha

// Entry points implemented in the kernel files, called by zha_api.cu.
namespace zha {
cudaError_t launch_tree_update(const Geo &g, void *tree, const void *K, const void *refs,
                               const int32_t *lens, int n_new, int32_t *status, cudaStream_t st);
// init = false: the route's state was already reset (by launch_decode_prologue)
cudaError_t launch_route(const Geo &g, const void *tree, const void *q, const int32_t *lens,
                         const float *p_levels, const zha_selection &sel, void *ws,
                         int32_t *status, cudaStream_t st, bool init = true);
cudaError_t launch_attention(const Geo &g, const void *q, const void *K, const void *V,
                             const int32_t *lens, const zha_selection *sel, void *out, void *ws,
                             int32_t *status, cudaStream_t st);
cudaError_t launch_decode_write(const Geo &g, void *K, void *V, int32_t *lens, const void *k_new,
                                const void *v_new, int32_t *status, cudaStream_t st);
// One decode step's prologue in one launch: write the new token, extend the
// tree along its rightmost path, reset the route's state, advance lens.
cudaError_t launch_decode_prologue(const Geo &g, void *tree, void *K, void *V, const void *refs,
                                   int32_t *lens, const void *k_new, const void *v_new, void *ws,
                                   int32_t *status, cudaStream_t st);
Geo make_geo_for(const zha_config *c);
bool score_tc_supported(const Geo &g);
bool fused_route_supported(const Geo &g);
cudaError_t launch_score_tc(const Geo &g, const void *mu_level, const float *bias, const void *q,
                            const int32_t *lens, int level, int32_t *cand, uint32_t *cmask, float *scores,
                            int32_t *count, uint32_t *maxkey, uint32_t *minkey, const int32_t *plist_up,
                            const uint32_t *pmask_up, const int32_t *pcount_up, int32_t *status,
                            cudaStream_t st);
cudaError_t launch_topp_select(const float *scores, const int32_t *counts, int n_sets,
                               int64_t stride, float p, uint8_t *kept, int32_t *status,
                               cudaStream_t st);
cudaError_t launch_wait_expiry(int kind, long long limit, int32_t *status, cudaStream_t st);
}  // namespace zha
