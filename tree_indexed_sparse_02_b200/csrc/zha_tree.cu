// zha_tree.cu -- building and extending the summary tree.
//
// Page "Zyphra AI Introduces Zyphra Hierarchical Attention (ZHA)", section
// "Building the tree": each contiguous chunk of c keys gets, from each of R
// reference queries, a tangent plane of its log attention mass; c sibling
// summaries are then summarised into a parent, one level at a time.
//
// For reference r and points x_i with log-weights a_i (raw keys: a_i = 0;
// children of a parent: x_i = mu_{i,r}, a_i = bias_{i,r}):
//   l_i = s r.x_i + a_i,  F = log sum_i e^{l_i},  w_i = e^{l_i - F},
//   mu_r = sum_i w_i x_i,  bias_r = F - s r.mu_r.
// Since s r.mu_r = sum_i w_i (l_i - a_i), the bias is formed from the same
// per-point dot products, in one online (running-max) pass over the points.
//
// Work split: one warp per (node, reference) pair; each lane owns d/32
// consecutive coordinates, so point loads are coalesced 8/16-byte vectors and
// the dot products end in a warp butterfly (every lane gets bitwise the same
// sum, so all lanes agree on every branch).
#include "zha_common.cuh"
#include "zha_route_state.cuh"

namespace zha {

namespace {

constexpr int kLevelWarps = 8;

// Points of one plane computation, d coordinates each, lane owning EPL of them.
template <typename T, int EPL>
struct RawPoints {        // keys of a leaf chunk, or children kept in the KV dtype
    const T *x0;
    int64_t stride;
    __device__ __forceinline__ void load(int i, int lane, float (&x)[EPL]) const {
        load_vec<EPL>(x0 + (int64_t)i * stride + lane * EPL, x);
    }
};

// 2^(byte - 127) for a biased scale exponent byte in 1..254
__device__ __forceinline__ float mx_scale(uint8_t byte) { return __uint_as_float((uint32_t)byte << 23); }

// Byte offset, within a plane's row of E4M3 bytes, of the EPL coordinates
// a lane owns (coordinates lane*EPL ..). Rows are stored permuted so that a
// scoring lane fetches, with one 16-byte load, its 8 bytes of two adjacent
// 32-coordinate blocks: coordinate k (block b = k / 32, w = k % 32) sits at
// 64 (b / 2) + 16 ((w % 16) / 4) + 8 (b % 2) + 4 (w / 16) + w % 4.
template <int EPL>
__device__ __forceinline__ int mx_lane_offset(int lane) {
    const int k = lane * EPL;
    const int b = k >> 5, w = k & 31;
    return 64 * (b >> 1) + 16 * ((w & 15) >> 2) + 8 * (b & 1) + 4 * (w >> 4) + (w & 3);
}

template <int EPL>
struct Mx8Points {        // children kept as MX-FP8 (E4M3 bytes + one scale per 32)
    const uint8_t *x0;
    const uint8_t *s0;
    int64_t stride, sstride;
    __device__ __forceinline__ void load(int i, int lane, float (&x)[EPL]) const {
        const float sc = mx_scale(s0[(int64_t)i * sstride + (lane * EPL) / 32]);
        const uint8_t *p = x0 + (int64_t)i * stride + mx_lane_offset<EPL>(lane);
#pragma unroll
        for (int e = 0; e < EPL; e += 2) {
            const __nv_fp8x2_storage_t two = *reinterpret_cast<const __nv_fp8x2_storage_t *>(p + e);
            const __half2 h = __half2(__nv_cvt_fp8x2_to_halfraw2(two, __NV_E4M3));
            const float2 f = __half22float2(h);
            x[e] = f.x * sc;
            x[e + 1] = f.y * sc;
        }
    }
};

// mu_out/b_out of one plane from its points (online single pass; see top).
template <class P, int EPL>
__device__ __forceinline__ void warp_plane(const P &pts, const float *a0, int64_t astride, int npts,
                                           const float (&rv)[EPL], float s, float (&acc)[EPL],
                                           float &b_out) {
    float m = -INFINITY, sum = 0.f, wl = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
    const int lane = threadIdx.x & 31;
    for (int i = 0; i < npts; ++i) {
        float x[EPL];
        pts.load(i, lane, x);
        float part = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) part = fmaf(rv[e], x[e], part);
        const float rx = s * warp_sum(part);           // s r.x_i
        const float ai = a0 ? a0[(int64_t)i * astride] : 0.f;
        const float l = rx + ai;
        if (l > m) {
            const float sc = (m == -INFINITY) ? 0.f : expf(m - l);
            sum *= sc;
            wl *= sc;
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[e] *= sc;
            m = l;
        }
        const float w = expf(l - m);
        sum += w;
        wl = fmaf(w, rx, wl);
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = fmaf(w, x[e], acc[e]);
    }
    const float inv = 1.f / sum;
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] *= inv;
    b_out = (m + logf(sum)) - wl * inv;
}

// MX-FP8 store of one plane: the lanes sharing a 32-coordinate block agree on
// its scale exponent e (smallest with max|x| <= 448 * 2^e) and round x / 2^e
// to E4M3, nearest even.
template <int EPL>
__device__ __forceinline__ void mx_store(uint8_t *mu_out, uint8_t *sc_out, const float (&v)[EPL], int lane) {
    constexpr int kLanesPerBlock = 32 / EPL;
    float a = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) a = fmaxf(a, fabsf(v[e]));
#pragma unroll
    for (int o = 1; o < kLanesPerBlock; o <<= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    int ex = 0;
    if (a > 0.f) {
        int k;
        const float f = frexpf(a, &k);                 // a = f 2^k, 448 = 0.875 2^9
        ex = (f <= 0.875f) ? k - 9 : k - 8;
        ex = ex < -126 ? -126 : (ex > 127 ? 127 : ex);
    }
    uint32_t packed = 0;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
        const __nv_fp8_storage_t q = __nv_cvt_float_to_fp8(scalbnf(v[e], -ex), __NV_SATFINITE, __NV_E4M3);
        packed |= (uint32_t)q << (8 * e);
    }
    if constexpr (EPL == 4)
        *reinterpret_cast<uint32_t *>(mu_out + mx_lane_offset<EPL>(lane)) = packed;
    else
        *reinterpret_cast<uint16_t *>(mu_out + mx_lane_offset<EPL>(lane)) = (uint16_t)packed;
    if (lane % kLanesPerBlock == 0) sc_out[lane / kLanesPerBlock] = (uint8_t)(ex + 127);
}

struct TreePtrs {
    void *mu[kMaxLevels + 1];
    uint8_t *sc[kMaxLevels + 1];
    float *bias[kMaxLevels + 1];
};

// Plane r of node `node` at `level` of group `grp`; MX selects the summary format.
template <typename T, int EPL, bool MX>
__device__ __forceinline__ void node_plane(const Geo &g, const TreePtrs &tp, const T *K,
                                           const T *refs, int grp, int level, int64_t node,
                                           int64_t n_below, int r, int lane) {
    const int kvh = grp % g.Hkv;
    float rv[EPL];
    load_vec<EPL>(refs + ((int64_t)kvh * g.R + r) * g.d + lane * EPL, rv);
    const int64_t rec = (grp * g.cap[level] + node) * g.R + r;      // plane record index
    float *bias = tp.bias[level] + rec;
    float acc[EPL];
    float bval;
    if (level == 1) {
        const RawPoints<T, EPL> pts{K + ((int64_t)grp * g.max_len + node * g.c) * g.d, g.d};
        warp_plane(pts, nullptr, 0, g.c, rv, g.s, acc, bval);
    } else {
        const int64_t c0 = node * g.c;
        const int64_t c1 = min(c0 + g.c, n_below);
        const int64_t crec = (grp * g.cap[level - 1] + c0) * g.R + r;
        const float *a0 = tp.bias[level - 1] + crec;
        if constexpr (MX) {
            const Mx8Points<EPL> pts{static_cast<const uint8_t *>(tp.mu[level - 1]) + crec * g.d,
                                     tp.sc[level - 1] + crec * (g.d / 32), (int64_t)g.R * g.d,
                                     (int64_t)g.R * (g.d / 32)};
            warp_plane(pts, a0, g.R, (int)(c1 - c0), rv, g.s, acc, bval);
        } else {
            const RawPoints<T, EPL> pts{static_cast<const T *>(tp.mu[level - 1]) + crec * g.d,
                                        (int64_t)g.R * g.d};
            warp_plane(pts, a0, g.R, (int)(c1 - c0), rv, g.s, acc, bval);
        }
    }
    if constexpr (MX)
        mx_store<EPL>(static_cast<uint8_t *>(tp.mu[level]) + rec * g.d, tp.sc[level] + rec * (g.d / 32), acc,
                      lane);
    else
        store_vec<EPL>(static_cast<T *>(tp.mu[level]) + rec * g.d + lane * EPL, acc);
    if (lane == 0) *bias = bval;
}

// Tokens before/after the update of sequence b; false if nothing changes.
__device__ __forceinline__ bool update_range(const Geo &g, const int32_t *lens, int b, int n_new,
                                             int64_t &n_old, int64_t &n_now, int32_t *status) {
    n_now = lens[b];
    if (n_now < 0 || n_now > g.max_len) {
        set_status(status, ZHA_ERR_CAPACITY);
        return false;
    }
    n_old = (n_new < 0) ? 0 : max64(n_now - n_new, 0);
    return (n_now / g.c) > (n_old / g.c);
}

// One level, many nodes: grid.x covers node slots x references, grid.y groups.
template <typename T, int EPL, bool MX>
__global__ void __launch_bounds__(kLevelWarps * 32)
tree_level_kernel(Geo g, TreePtrs tp, const T *K, const T *refs, const int32_t *lens, int level,
                  int n_new, int64_t slots, int32_t *status) {
    const int grp = blockIdx.y;
    const int b = grp / g.Hkv;
    const int lane = threadIdx.x & 31;
    const int64_t item = (int64_t)blockIdx.x * kLevelWarps + (threadIdx.x >> 5);
    if (item >= slots * g.R) return;
    int64_t n_old, n_now;
    if (!update_range(g, lens, b, n_new, n_old, n_now, status)) return;
    int64_t lo = n_old / g.c;
    for (int l = 2; l <= level; ++l) lo /= g.c;
    const int64_t node = lo + item / g.R;
    const int r = (int)(item % g.R);
    if (node >= level_nodes(n_now, g.c, level)) return;
    const int64_t n_below = level > 1 ? level_nodes(n_now, g.c, level - 1) : 0;
    node_plane<T, EPL, MX>(g, tp, K, refs, grp, level, node, n_below, r, lane);
}

// Few new tokens (a decode step): one block per group walks every level,
// warp r computing plane r of each changed node; levels are separated by a
// block barrier, which also makes the children's global writes visible.
constexpr int kPathWarps = 16;

// The nodes of group grp that change when its cache grows from n_old to
// n_now tokens, level by level (a block barrier between levels also makes
// the children's writes visible).
template <typename T, int EPL, bool MX>
__device__ __forceinline__ void tree_path_levels(const Geo &g, const TreePtrs &tp, const T *K, const T *refs,
                                                 int grp, int64_t n_old, int64_t n_now) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    int64_t lo = n_old / g.c;
    for (int level = 1; level <= g.L; ++level) {
        if (level > 1) lo /= g.c;
        const int64_t hi = level_nodes(n_now, g.c, level);
        const int64_t n_below = level > 1 ? level_nodes(n_now, g.c, level - 1) : 0;
        const int64_t items = (hi - lo) * g.R;
        for (int64_t it = warp; it < items; it += blockDim.x >> 5)
            node_plane<T, EPL, MX>(g, tp, K, refs, grp, level, lo + it / g.R, n_below,
                                   (int)(it % g.R), lane);
        __syncthreads();
    }
}

template <typename T, int EPL, bool MX>
__global__ void __launch_bounds__(kPathWarps * 32) tree_path_kernel(Geo g, TreePtrs tp, const T *K, const T *refs,
                                 const int32_t *lens, int n_new, int32_t *status) {
    const int grp = blockIdx.x;
    const int b = grp / g.Hkv;
    int64_t n_old, n_now;
    const bool any = update_range(g, lens, b, n_new, n_old, n_now, status);
    if (!any) return;  // uniform across the block
    tree_path_levels<T, EPL, MX>(g, tp, K, refs, grp, n_old, n_now);
}

// A decode step's prologue, one block per (sequence, KV head) group: write
// the group's new token at position lens[b], extend the tree along its
// rightmost path if the token completes a chunk, reset the group's routing
// state, and -- in the last of the sequence's groups to get here, after every
// group has read the old length -- advance lens[b].
template <typename T, int EPL, bool MX>
__global__ void __launch_bounds__(kPathWarps * 32)
decode_prologue_kernel(Geo g, TreePtrs tp, T *K, T *V, const T *refs, int32_t *lens, const T *k_new,
                       const T *v_new, uint32_t *arrive, RouteState rs, int32_t *status) {
    __shared__ int64_t s_n;
    const int grp = blockIdx.x;
    const int b = grp / g.Hkv, kvh = grp % g.Hkv;
    pdl_wait();
    if (threadIdx.x == 0) s_n = lens[b];
    __syncthreads();
    const int64_t n = s_n;
    const bool ok = n >= 0 && n + 1 <= g.max_len;
    if (ok) {
        const int64_t dst = ((int64_t)grp * g.max_len + n) * g.d;
        const int64_t src = ((int64_t)b * g.Hkv + kvh) * g.d;
        for (int e = threadIdx.x; e < g.d; e += blockDim.x) {
            K[dst + e] = k_new[src + e];
            V[dst + e] = v_new[src + e];
        }
    }
    route_reset_group(g, rs, grp);
    __syncthreads();
    if (ok && (n + 1) / g.c > n / g.c) tree_path_levels<T, EPL, MX>(g, tp, K, refs, grp, n, n + 1);
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(&arrive[b], 1u) == (uint32_t)(g.Hkv - 1)) {
            arrive[b] = 0u;
            if (ok)
                lens[b] = (int32_t)(n + 1);
            else
                set_status(status, ZHA_ERR_CAPACITY);
        }
    }
    pdl_trigger();
}

template <typename T, int EPL, bool MX>
cudaError_t decode_prologue_t(const Geo &g, const TreePtrs &tp, T *K, T *V, const T *refs, int32_t *lens,
                              const T *k_new, const T *v_new, uint32_t *arrive, const RouteState &rs,
                              int32_t *status, cudaStream_t st) {
    const int warps = g.R < 4 ? 4 : (g.R > kPathWarps ? kPathWarps : g.R);
    ProfScope ps("decode_prologue", st);
    return launch_pdl(decode_prologue_kernel<T, EPL, MX>, dim3(g.groups()), dim3(warps * 32), 0, st, g, tp, K, V,
                      refs, lens, k_new, v_new, arrive, rs, status);
}

template <typename T, int EPL, bool MX>
cudaError_t tree_update_t(const Geo &g, const TreePtrs &tp, const T *K, const T *refs,
                          const int32_t *lens, int n_new, int32_t *status, cudaStream_t st) {
    if (n_new >= 0 && n_new <= g.c) {
        // one warp per plane of a node, up to kPathWarps (more planes: a warp takes several)
        const int warps = g.R < 4 ? 4 : (g.R > kPathWarps ? kPathWarps : g.R);
        ProfScope ps("tree_path", st);
        tree_path_kernel<T, EPL, MX><<<g.groups(), warps * 32, 0, st>>>(g, tp, K, refs, lens, n_new,
                                                                    status);
        return cudaGetLastError();
    }
    int64_t bound = n_new < 0 ? g.cap[1] : (n_new + g.c - 1) / g.c;
    for (int level = 1; level <= g.L; ++level) {
        if (level > 1) bound = n_new < 0 ? g.cap[level] : min64(bound / g.c + 2, g.cap[level]);
        bound = min64(bound, g.cap[level]);
        if (bound <= 0) break;
        const int64_t items = bound * g.R;
        dim3 grid((unsigned)((items + kLevelWarps - 1) / kLevelWarps), g.groups());
        {
            static const char *names[] = {"", "tree_level[l1]", "tree_level[l2]", "tree_level[l3]",
                                          "tree_level[l4]", "tree_level[l5]", "tree_level[l6]",
                                          "tree_level[l7]", "tree_level[l8]"};
            ProfScope ps(names[level], st);
            tree_level_kernel<T, EPL, MX><<<grid, kLevelWarps * 32, 0, st>>>(g, tp, K, refs, lens, level,
                                                                         n_new, bound, status);
        }
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

TreePtrs tree_ptrs(const Geo &g, void *tree) {
    TreePtrs tp{};
    for (int l = 1; l <= g.L; ++l) {
        tp.mu[l] = static_cast<char *>(tree) + g.mu_off[l];
        tp.bias[l] = reinterpret_cast<float *>(static_cast<char *>(tree) + g.bias_off[l]);
        tp.sc[l] = g.mx() ? reinterpret_cast<uint8_t *>(static_cast<char *>(tree) + g.sc_off[l]) : nullptr;
    }
    return tp;
}

cudaError_t launch_decode_prologue(const Geo &g, void *tree, void *K, void *V, const void *refs,
                                   int32_t *lens, const void *k_new, const void *v_new, void *ws,
                                   int32_t *status, cudaStream_t st) {
    const TreePtrs tp = tree_ptrs(g, tree);
    const RouteState rs = route_state(g, ws);
    uint32_t *arrive = reinterpret_cast<uint32_t *>(static_cast<char *>(ws) + g.ws_arrive);
    if (g.dtype == ZHA_BF16) {
        auto k = static_cast<__nv_bfloat16 *>(K);
        auto v = static_cast<__nv_bfloat16 *>(V);
        auto r = static_cast<const __nv_bfloat16 *>(refs);
        auto kn = static_cast<const __nv_bfloat16 *>(k_new);
        auto vn = static_cast<const __nv_bfloat16 *>(v_new);
        if (g.mx())
            return g.d == 128 ? decode_prologue_t<__nv_bfloat16, 4, true>(g, tp, k, v, r, lens, kn, vn, arrive, rs, status, st)
                              : decode_prologue_t<__nv_bfloat16, 2, true>(g, tp, k, v, r, lens, kn, vn, arrive, rs, status, st);
        return g.d == 128 ? decode_prologue_t<__nv_bfloat16, 4, false>(g, tp, k, v, r, lens, kn, vn, arrive, rs, status, st)
                          : decode_prologue_t<__nv_bfloat16, 2, false>(g, tp, k, v, r, lens, kn, vn, arrive, rs, status, st);
    }
    auto k = static_cast<float *>(K);
    auto v = static_cast<float *>(V);
    auto r = static_cast<const float *>(refs);
    auto kn = static_cast<const float *>(k_new);
    auto vn = static_cast<const float *>(v_new);
    return g.d == 128 ? decode_prologue_t<float, 4, false>(g, tp, k, v, r, lens, kn, vn, arrive, rs, status, st)
                      : decode_prologue_t<float, 2, false>(g, tp, k, v, r, lens, kn, vn, arrive, rs, status, st);
}

cudaError_t launch_tree_update(const Geo &g, void *tree, const void *K, const void *refs,
                               const int32_t *lens, int n_new, int32_t *status, cudaStream_t st) {
    TreePtrs tp{};
    for (int l = 1; l <= g.L; ++l) {
        tp.mu[l] = static_cast<char *>(tree) + g.mu_off[l];
        tp.bias[l] = reinterpret_cast<float *>(static_cast<char *>(tree) + g.bias_off[l]);
        tp.sc[l] = g.mx() ? reinterpret_cast<uint8_t *>(static_cast<char *>(tree) + g.sc_off[l]) : nullptr;
    }
    if (g.dtype == ZHA_BF16) {
        auto k = static_cast<const __nv_bfloat16 *>(K);
        auto r = static_cast<const __nv_bfloat16 *>(refs);
        if (g.mx())
            return g.d == 128 ? tree_update_t<__nv_bfloat16, 4, true>(g, tp, k, r, lens, n_new, status, st)
                              : tree_update_t<__nv_bfloat16, 2, true>(g, tp, k, r, lens, n_new, status, st);
        return g.d == 128 ? tree_update_t<__nv_bfloat16, 4, false>(g, tp, k, r, lens, n_new, status, st)
                          : tree_update_t<__nv_bfloat16, 2, false>(g, tp, k, r, lens, n_new, status, st);
    }
    auto k = static_cast<const float *>(K);
    auto r = static_cast<const float *>(refs);
    return g.d == 128 ? tree_update_t<float, 4, false>(g, tp, k, r, lens, n_new, status, st)
                      : tree_update_t<float, 2, false>(g, tp, k, r, lens, n_new, status, st);
}

// Decode step prologue: write the g.T new tokens of every (sequence, KV head)
// (k_new [B][T][Hkv][d]) at positions lens[b] .. lens[b] + T - 1, then advance
// lens[b] by T (one block per sequence, so the increment follows every read
// of the old length in the block).
template <typename T>
__global__ void decode_write_kernel(Geo g, T *K, T *V, int32_t *lens, const T *k_new,
                                    const T *v_new, int32_t *status) {
    const int b = blockIdx.x;
    const int64_t n = lens[b];
    const bool ok = n >= 0 && n + g.T <= g.max_len;
    if (ok) {
        for (int i = threadIdx.x; i < g.T * g.Hkv * g.d; i += blockDim.x) {
            const int t = i / (g.Hkv * g.d), kvh = (i / g.d) % g.Hkv, e = i % g.d;
            const int64_t dst = (((int64_t)b * g.Hkv + kvh) * g.max_len + n + t) * g.d + e;
            const int64_t src = (((int64_t)b * g.T + t) * g.Hkv + kvh) * g.d + e;
            K[dst] = k_new[src];
            V[dst] = v_new[src];
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (ok)
            lens[b] = (int32_t)(n + g.T);
        else
            set_status(status, ZHA_ERR_CAPACITY);
    }
}

cudaError_t launch_decode_write(const Geo &g, void *K, void *V, int32_t *lens, const void *k_new,
                                const void *v_new, int32_t *status, cudaStream_t st) {
    ProfScope ps("decode_write", st);
    if (g.dtype == ZHA_BF16)
        decode_write_kernel<__nv_bfloat16><<<g.B, 256, 0, st>>>(
            g, static_cast<__nv_bfloat16 *>(K), static_cast<__nv_bfloat16 *>(V), lens,
            static_cast<const __nv_bfloat16 *>(k_new), static_cast<const __nv_bfloat16 *>(v_new),
            status);
    else
        decode_write_kernel<float><<<g.B, 256, 0, st>>>(
            g, static_cast<float *>(K), static_cast<float *>(V), lens,
            static_cast<const float *>(k_new), static_cast<const float *>(v_new), status);
    return cudaGetLastError();
}

}  // namespace zha
