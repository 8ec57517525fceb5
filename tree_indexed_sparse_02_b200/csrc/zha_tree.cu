// zha_tree.cu -- building and extending the summary tree.
//
// Page "Zyphra AI Introduces Zyphra Hierarchical Attention (ZHA)", section
// "Building the tree": each contiguous chunk of c keys gets, from each of R
// reference queries, a tangent plane of its log attention mass; c sibling
// summaries are then summarised into a parent, one level at a time.
//
// For reference r over the keys k_t of a chunk: l_t = s r.k_t,
// F = log sum_t e^{l_t}, w_t = e^{l_t - F}, mu_r = sum_t w_t k_t,
// bias_r = F - s r.mu_r (= F - sum_t w_t l_t). A parent applies the same rule
// to its children, child i entering as the point mu_{i,r} (as stored) with
// log-weight F_{i,r}, its log-mass at r (the child's plane value at r, where
// it is exact); every node keeps its F beside its planes.
//
// Leaves of a bf16 cache (tree_leaf_kernel): the dot products of a chunk's
// keys with every reference are a real contraction, S = K R^T. A work item is
// 256 consecutive keys of one (sequence, KV head): TMA brings them into
// shared memory as two 128-row, 128B-swizzled tiles, one thread issues
// tcgen05.mma (M = 128 keys, N = R rounded up to 16, K = head_dim) into
// tensor memory, and the CTA's eight warps read S back (one thread per key),
// take the softmax of each chunk across its threads, and form mu_r as the
// weighted sum of the chunk's keys (read back from the same shared tiles).
// The parents of the item's subtree (every level whose nodes span at most
// 256 keys) follow in the same CTA, reading their just-written children from
// L2. Higher levels, parents on a decode step's rightmost path and every
// level of an fp32 cache use CUDA cores: sixteen lanes per plane, each lane
// owning head_dim / 16 coordinates. A parent reads, for each child, its
// stored summary key and its log-mass at the reference (kept in the tree
// beside each plane: every node's F_r is known when it is built), so
// extending the tree needs no dot products with the children.
//
// Appending reuses the same routines: a decode step's completed chunk is
// computed as a single-leaf item (its keys loaded with plain loads into the
// same tile layout, the same MMAs), so a tree extended token by token equals
// one built at once, bit for bit.
#include "zha_tc.cuh"
#include "zha_route_state.cuh"

namespace zha {

namespace {

constexpr int kItemKeys = 256;            // keys per work item of the leaf kernel
constexpr int kTileRows = 128;            // rows of one MMA tile (M)
constexpr int kLeafWarps = 8;             // one thread per key of an item
constexpr int kLevelWarps = 8;
constexpr int kSub = 8;                   // lanes per plane on the CUDA-core paths
constexpr int kPerWarp = 32 / kSub;       // planes per warp at a time
constexpr long long kTreeWait = 2000000000LL;   // ~1 s at the boost clock: a wait that long is an error

struct TreePtrs {
    void *mu[kMaxLevels + 1];
    uint8_t *sc[kMaxLevels + 1];
    float *bias[kMaxLevels + 1];
    float *lm[kMaxLevels + 1];      // each plane's log-mass F at its reference
};

// Two fp32 values in one 64-bit register pair, for the packed fp32
// instructions of sm_100 (fma.rn.f32x2: two FMAs per instruction).
typedef unsigned long long f2x;
__device__ __forceinline__ f2x pk2(float lo, float hi) {
    f2x r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float2 upk2(f2x v) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}
__device__ __forceinline__ f2x fma2(f2x a, f2x b, f2x c) {
    f2x d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
// bf16 pair (element 0 in the low half) -> packed fp32 pair
__device__ __forceinline__ f2x bf2_to_f2x(uint32_t w) {
    return pk2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// acc[e] = fma(w, x[e], acc[e]) for every pair e.
template <int H>
__device__ __forceinline__ void axpy2(f2x (&acc)[H], float w, const f2x (&x)[H]) {
    const f2x ww = pk2(w, w);
#pragma unroll
    for (int e = 0; e < H; ++e) acc[e] = fma2(ww, x[e], acc[e]);
}
template <int H, int E>
__device__ __forceinline__ void unpack_all(const f2x (&v)[H], float (&out)[E]) {
    static_assert(2 * H == E, "");
#pragma unroll
    for (int e = 0; e < H; ++e) {
        const float2 f = upk2(v[e]);
        out[2 * e] = f.x;
        out[2 * e + 1] = f.y;
    }
}

// ------------------------------------------------------------ loads and stores

// 2^(byte - 127) for a biased scale exponent byte in 1..254
__device__ __forceinline__ float mx_scale(uint8_t byte) { return __uint_as_float((uint32_t)byte << 23); }

// Byte offset, within a plane's row of E4M3 bytes, of coordinate k (for k a
// multiple of 4, the 4 coordinates k .. k+3 are consecutive bytes). Rows are
// stored permuted so that a scoring lane fetches, with one 16-byte load, its
// 8 bytes of two adjacent 32-coordinate blocks: coordinate k (block b = k /
// 32, w = k % 32) sits at 64 (b / 2) + 16 ((w % 16) / 4) + 8 (b % 2) + 4 (w / 16) + w % 4.
__device__ __forceinline__ int mx_offset(int k) {
    const int b = k >> 5, w = k & 31;
    return 64 * (b >> 1) + 16 * ((w & 15) >> 2) + 8 * (b & 1) + 4 * (w >> 4) + (w & 3);
}

// n consecutive elements (n a multiple of 4) as floats.
template <int N>
__device__ __forceinline__ void load_n(const __nv_bfloat16 *p, float (&v)[N]) {
    static_assert(N % 4 == 0, "");
#pragma unroll
    for (int i = 0; i < N; i += 8) {
        if (N - i >= 8) {
            const uint4 t = *reinterpret_cast<const uint4 *>(p + i);
            const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[j]));
                v[i + 2 * j] = f.x;
                v[i + 2 * j + 1] = f.y;
            }
        } else {
            const uint2 t = *reinterpret_cast<const uint2 *>(p + i);
            const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&t.x));
            const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&t.y));
            v[i] = a.x; v[i + 1] = a.y; v[i + 2] = b.x; v[i + 3] = b.y;
        }
    }
}
template <int N>
__device__ __forceinline__ void load_n(const float *p, float (&v)[N]) {
    static_assert(N % 4 == 0, "");
#pragma unroll
    for (int i = 0; i < N; i += 4) {
        const float4 t = *reinterpret_cast<const float4 *>(p + i);
        v[i] = t.x; v[i + 1] = t.y; v[i + 2] = t.z; v[i + 3] = t.w;
    }
}
template <int N>
__device__ __forceinline__ void store_n(__nv_bfloat16 *p, const float (&v)[N]) {
    if constexpr (N == 2) {
        *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(v[0], v[1]);
    } else {
#pragma unroll
        for (int i = 0; i < N; i += 4) {
            __nv_bfloat162 a = __floats2bfloat162_rn(v[i], v[i + 1]);
            __nv_bfloat162 b = __floats2bfloat162_rn(v[i + 2], v[i + 3]);
            uint2 t;
            t.x = *reinterpret_cast<uint32_t *>(&a);
            t.y = *reinterpret_cast<uint32_t *>(&b);
            *reinterpret_cast<uint2 *>(p + i) = t;
        }
    }
}
template <int N>
__device__ __forceinline__ void store_n(float *p, const float (&v)[N]) {
    if constexpr (N == 2) {
        *reinterpret_cast<float2 *>(p) = make_float2(v[0], v[1]);
    } else {
#pragma unroll
        for (int i = 0; i < N; i += 4)
            *reinterpret_cast<float4 *>(p + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
    }
}

// MX-FP8 store of one plane by the lanes that own it, each holding E
// consecutive coordinates (k0 .. k0+E-1); the 32 / E lanes sharing a
// 32-coordinate block (neighbours in lane order) agree on its scale exponent
// e (smallest with max|x| <= 448 * 2^e) and round x / 2^e to E4M3, nearest even.
template <int E>
__device__ __forceinline__ void mx_store(uint8_t *mu_row, uint8_t *sc_row, const float (&v)[E], int k0, bool live) {
    constexpr int kLanesPerBlock = 32 / E;
    float a = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) a = fmaxf(a, fabsf(v[e]));
#pragma unroll
    for (int o = 1; o < kLanesPerBlock; o <<= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    int ex = 0;
    if (a > 0.f) {
        int k;
        const float f = frexpf(a, &k);                 // a = f 2^k, 448 = 0.875 2^9
        ex = (f <= 0.875f) ? k - 9 : k - 8;
        ex = ex < -126 ? -126 : (ex > 127 ? 127 : ex);
    }
    if (!live) return;   // (after the shuffles, which every lane of the warp takes part in)
    uint8_t q[E];
#pragma unroll
    for (int e = 0; e < E; ++e) q[e] = __nv_cvt_float_to_fp8(scalbnf(v[e], -ex), __NV_SATFINITE, __NV_E4M3);
    if constexpr (E == 2) {
        // two coordinates k0, k0+1 (k0 even): adjacent bytes, one 2-byte store
        *reinterpret_cast<uint16_t *>(mu_row + mx_offset(k0)) = (uint16_t)(q[0] | ((uint32_t)q[1] << 8));
    } else {
        static_assert(E % 4 == 0, "coordinates per lane: 2 or a multiple of 4");
#pragma unroll
        for (int e0 = 0; e0 < E; e0 += 4)
            *reinterpret_cast<uint32_t *>(mu_row + mx_offset(k0 + e0)) =
                q[e0] | ((uint32_t)q[e0 + 1] << 8) | ((uint32_t)q[e0 + 2] << 16) | ((uint32_t)q[e0 + 3] << 24);
    }
    if ((k0 & 31) == 0) sc_row[k0 >> 5] = (uint8_t)(ex + 127);
}

// Plane row store: the KV dtype, or MX-FP8. Every lane of the warp calls it
// (the MX block scale is a reduction over neighbouring lanes); only lanes
// with `live` write.
template <typename T, int E, bool MX>
__device__ __forceinline__ void store_plane(const Geo &g, const TreePtrs &tp, int level, int64_t rec,
                                            const float (&v)[E], int k0, bool live) {
    if constexpr (MX)
        mx_store<E>(static_cast<uint8_t *>(tp.mu[level]) + rec * g.d, tp.sc[level] + rec * (g.d / 32), v, k0, live);
    else if (live)
        store_n<E>(static_cast<T *>(tp.mu[level]) + rec * g.d + k0, v);
}

// ------------------------------------------ planes on CUDA cores: 16 lanes per plane

// Points of one plane, lane sl (0 .. kSub-1) of the plane's kSub owning E =
// d/kSub consecutive coordinates.
template <typename T, int E>
struct RawPoints {        // keys of a leaf chunk, or children kept in the KV dtype
    const T *x0;
    int64_t stride;
    __device__ __forceinline__ void load(int i, int sl, float (&x)[E]) const {
        load_n<E>(x0 + (int64_t)i * stride + sl * E, x);
    }
    __device__ __forceinline__ void load2(int i, int sl, f2x (&x)[E / 2]) const {
        const T *p = x0 + (int64_t)i * stride + sl * E;
        if constexpr (sizeof(T) == 2 && E % 8 == 0) {
#pragma unroll
            for (int e = 0; e < E; e += 8) {
                const uint4 t = *reinterpret_cast<const uint4 *>(p + e);
                x[e / 2] = bf2_to_f2x(t.x);
                x[e / 2 + 1] = bf2_to_f2x(t.y);
                x[e / 2 + 2] = bf2_to_f2x(t.z);
                x[e / 2 + 3] = bf2_to_f2x(t.w);
            }
        } else if constexpr (sizeof(T) == 2) {
            static_assert(E == 4, "coordinates per lane: 4 or a multiple of 8");
            const uint2 t = *reinterpret_cast<const uint2 *>(p);   // 8 bytes, 8-byte aligned
            x[0] = bf2_to_f2x(t.x);
            x[1] = bf2_to_f2x(t.y);
        } else {
#pragma unroll
            for (int e = 0; e < E; e += 4) {
                const float4 t = *reinterpret_cast<const float4 *>(p + e);
                x[e / 2] = pk2(t.x, t.y);
                x[e / 2 + 1] = pk2(t.z, t.w);
            }
        }
    }
};

template <int E>
struct Mx8Points {        // children kept as MX-FP8 (E4M3 bytes + one scale per 32)
    const uint8_t *x0;
    const uint8_t *s0;
    int64_t stride, sstride;
    __device__ __forceinline__ void load(int i, int sl, float (&x)[E]) const {
        const int k0 = sl * E;
        const float sc = mx_scale(s0[(int64_t)i * sstride + k0 / 32]);
        const uint8_t *row = x0 + (int64_t)i * stride;
#pragma unroll
        for (int e0 = 0; e0 < E; e0 += 4) {
            const uint32_t four = *reinterpret_cast<const uint32_t *>(row + mx_offset(k0 + e0));
            const float2 lo = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(four & 0xffffu), __NV_E4M3)));
            const float2 hi = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(four >> 16), __NV_E4M3)));
            x[e0] = lo.x * sc;
            x[e0 + 1] = lo.y * sc;
            x[e0 + 2] = hi.x * sc;
            x[e0 + 3] = hi.y * sc;
        }
    }
    __device__ __forceinline__ void load2(int i, int sl, f2x (&x)[E / 2]) const {
        float v[E];
        load(i, sl, v);
#pragma unroll
        for (int e = 0; e < E; e += 2) x[e / 2] = pk2(v[e], v[e + 1]);
    }
};

// One plane from its points (online single pass; see top) by a kSub-lane
// subgroup. All 32 lanes of the warp call this together with the same
// n_max (the largest npts of the warp's four planes); points i >= npts of a
// subgroup are skipped.
template <class P, int E>
__device__ __forceinline__ void sub_plane(const P &pts, const float *a0, int64_t astride, int npts, int n_max,
                                          const float (&rv)[E], float s, float (&acc)[E], float &b_out, float &F_out,
                                          int sl) {
    float m = -INFINITY, sum = 0.f, wl = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    for (int i = 0; i < n_max; ++i) {
        const bool v = i < npts;
        float x[E];
        if (v) {
            pts.load(i, sl, x);
        } else {
#pragma unroll
            for (int e = 0; e < E; ++e) x[e] = 0.f;
        }
        float part = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) part = fmaf(rv[e], x[e], part);
#pragma unroll
        for (int o = 1; o < kSub; o <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (!v) continue;
        const float rx = s * part;                       // s r.x_i
        const float l = rx + (a0 ? a0[(int64_t)i * astride] : 0.f);
        if (l > m) {
            const float sc = (m == -INFINITY) ? 0.f : expf(m - l);
            sum *= sc;
            wl *= sc;
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] *= sc;
            m = l;
        }
        const float w = expf(l - m);
        sum += w;
        wl = fmaf(w, rx, wl);
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = fmaf(w, x[e], acc[e]);
    }
    const float inv = 1.f / sum;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] *= inv;
    F_out = m + logf(sum);
    b_out = F_out - wl * inv;
}

// The same plane from at most NP points, all loaded before any arithmetic
// (one memory round trip instead of one per point), in two passes: the
// largest log-weight first, then the weights and sums. Points i >= npts are
// skipped. All 32 lanes of the warp call this together.
template <int NP, class P, int E>
__device__ __forceinline__ void sub_plane_np(const P &pts, const float *a0, int64_t astride, int npts,
                                             const float (&rv)[E], float s, float (&acc)[E], float &b_out,
                                             float &F_out, int sl) {
    float x[NP][E], a[NP], rx[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i) {
        if (i < npts) {
            pts.load(i, sl, x[i]);
            a[i] = a0 ? a0[(int64_t)i * astride] : 0.f;
        } else {
#pragma unroll
            for (int e = 0; e < E; ++e) x[i][e] = 0.f;
            a[i] = 0.f;
        }
    }
#pragma unroll
    for (int i = 0; i < NP; ++i) {
        float part = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) part = fmaf(rv[e], x[i][e], part);
#pragma unroll
        for (int o = 1; o < kSub; o <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        rx[i] = s * part;                                 // s r.x_i
    }
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < NP; ++i)
        if (i < npts) m = fmaxf(m, rx[i] + a[i]);
    float z = 0.f, wl = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
#pragma unroll
    for (int i = 0; i < NP; ++i) {
        if (i >= npts) continue;
        const float w = expf((rx[i] + a[i]) - m);
        z += w;
        wl = fmaf(w, rx[i], wl);
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = fmaf(w, x[i][e], acc[e]);
    }
    const float inv = 1.f / z;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] *= inv;
    F_out = m + logf(z);
    b_out = F_out - wl * inv;
}

// Plane r of a parent from its npts children's planes r: child i enters as
// its stored summary key x_i with log-weight l_i = F_i, its log-mass at r;
// F = log sum_i e^{l_i}, w_i = e^{l_i - F}, mu = sum_i w_i x_i (the bias,
// F - s r.mu, is left to the caller). The log-masses come first (two passes
// over npts scalars), then the keys stream in with known weights. NP > 0:
// at most NP children (unrolled); NP = 0: any number.
template <int NP, class P, int E>
__device__ __forceinline__ void parent_plane(const P &pts, const float *lm0, int64_t stride, int npts,
                                             float (&out)[E], float &F_out, int sl) {
    constexpr int H = E / 2;
    float l[NP > 0 ? NP : 1];
    float m = -INFINITY, z = 0.f;
    f2x acc[H];
#pragma unroll
    for (int e = 0; e < H; ++e) acc[e] = 0ull;
    if constexpr (NP > 0) {
#pragma unroll
        for (int i = 0; i < NP; ++i)
            if (i < npts) {
                l[i] = lm0[(int64_t)i * stride];
                m = fmaxf(m, l[i]);
            }
#pragma unroll
        for (int i = 0; i < NP; ++i)
            if (i < npts) {
                l[i] = expf(l[i] - m);
                z += l[i];
            }
        const float inv = 1.f / z;
#pragma unroll
        for (int i = 0; i < NP; ++i)
            if (i < npts) {
                f2x x[H];
                pts.load2(i, sl, x);
                axpy2<H>(acc, l[i] * inv, x);
            }
    } else {
        for (int i = 0; i < npts; ++i) m = fmaxf(m, lm0[(int64_t)i * stride]);
        for (int i = 0; i < npts; ++i) z += expf(lm0[(int64_t)i * stride] - m);
        const float inv = 1.f / z;
        for (int i = 0; i < npts; ++i) {
            f2x x[H];
            pts.load2(i, sl, x);
            axpy2<H>(acc, expf(lm0[(int64_t)i * stride] - m) * inv, x);
        }
    }
    unpack_all(acc, out);
    F_out = m + logf(z);
}

// (node, reference) plane p of a range: node offset p / R and reference p % R
// (shifts when R is a power of two).
__device__ __forceinline__ void split_plane(uint32_t p, int R, uint32_t &node_off, int &r) {
    if ((R & (R - 1)) == 0) {
        const int lg = __ffs(R) - 1;
        node_off = p >> lg;
        r = (int)(p & (uint32_t)(R - 1));
    } else {
        node_off = p / (uint32_t)R;
        r = (int)(p - node_off * (uint32_t)R);
    }
}

// Planes of nodes [lo, hi) at `level` of group grp, on CUDA cores: the warp
// takes planes j .. j+3 of the range's (node, reference) list (subgroup
// lane / 8 one each), for j = 4 * job, job = first, first + step, ...
// Level 1 (raw keys) is used for fp32 caches only.
template <typename T, int E, bool MX, int CP>
__device__ __forceinline__ void plane_jobs(const Geo &g, const TreePtrs &tp, const T *K, const T *refs, int grp,
                                           int level, int64_t lo, int64_t hi, int64_t n_below, int64_t first,
                                           int64_t step, int lane) {
    const uint32_t planes = (uint32_t)((hi - lo) * g.R);
    const int sl = lane % kSub;
    const int kvh = grp % g.Hkv;
    for (int64_t job = first; job * kPerWarp < (int64_t)planes; job += step) {
        const uint32_t p = (uint32_t)job * kPerWarp + lane / kSub;
        const bool live = p < planes;
        uint32_t off;
        int r;
        split_plane(live ? p : planes - 1, g.R, off, r);
        const int64_t node = lo + off;
        float rv[E];
        load_n<E>(refs + ((int64_t)kvh * g.R + r) * g.d + sl * E, rv);
        const int64_t rec = (grp * g.cap[level] + node) * g.R + r;
        float acc[E];
        float bval, F;
        if (level == 1) {
            // raw keys (fp32 caches): the dot products with the reference first
            const RawPoints<T, E> pts{K + ((int64_t)grp * g.max_len + node * g.c) * g.d, g.d};
            if constexpr (CP > 0)
                sub_plane_np<CP>(pts, nullptr, 0, g.c, rv, g.s, acc, bval, F, sl);
            else
                sub_plane(pts, nullptr, 0, g.c, g.c, rv, g.s, acc, bval, F, sl);
        } else {
            const int64_t c0 = node * g.c;
            const int npts = (int)(min64(c0 + g.c, n_below) - c0);
            const int64_t crec = (grp * g.cap[level - 1] + c0) * g.R + r;
            const float *lm0 = tp.lm[level - 1] + crec;
            if constexpr (MX) {
                const Mx8Points<E> pts{static_cast<const uint8_t *>(tp.mu[level - 1]) + crec * g.d,
                                       tp.sc[level - 1] + crec * (g.d / 32), (int64_t)g.R * g.d,
                                       (int64_t)g.R * (g.d / 32)};
                parent_plane<CP>(pts, lm0, g.R, npts, acc, F, sl);
            } else {
                const RawPoints<T, E> pts{static_cast<const T *>(tp.mu[level - 1]) + crec * g.d,
                                          (int64_t)g.R * g.d};
                parent_plane<CP>(pts, lm0, g.R, npts, acc, F, sl);
            }
            // bias = F - s r.mu over the subgroup
            float part = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) part = fmaf(rv[e], acc[e], part);
#pragma unroll
            for (int o = 1; o < kSub; o <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
            bval = F - g.s * part;
        }
        store_plane<T, E, MX>(g, tp, level, rec, acc, sl * E, live);
        if (live && sl == 0) {
            tp.bias[level][rec] = bval;
            tp.lm[level][rec] = F;
        }
    }
}

// ------------------------------------------------------ leaves on tensor cores

// Shared-memory layout of a leaf work item of `tiles` 128-row tiles holding
// `leaves` whole chunks (bytes from a 1024-aligned base):
//   A  tiles x [d/64 K-blocks][128 rows][128 B]  keys, swizzled
//   B  [d/64][npad rows][128 B]                   references (rows >= R zero)
//   W  [leaves][R][c] (+ c floats of padding per leaf)  softmax weights
//   X  [8 warps][3]                               cross-warp partials (c > 32)
//   then two mbarriers, the tensor-memory address and an abort flag.
struct LeafLayout {
    int npad, tiles, leaves, wstride;
    uint32_t a, b, w, x, bar, bytes;
};

__host__ __device__ inline LeafLayout leaf_layout(int d, int R, int c, int tiles) {
    LeafLayout L{};
    L.npad = (R + 15) & ~15;
    L.tiles = tiles;
    L.leaves = (tiles * kTileRows) / c > 0 ? (tiles * kTileRows) / c : 1;
    L.wstride = (R + 1) * c;
    L.a = 0;
    L.b = (uint32_t)(tiles * kTileRows * d * 2);
    L.w = L.b + (uint32_t)((d / 64) * L.npad * 128);
    L.x = L.w + (uint32_t)(((L.leaves * L.wstride * 4) + 15) & ~15);
    L.bar = L.x + (uint32_t)(kLeafWarps * 3 * 4);
    L.bar = (L.bar + 15) & ~15u;
    L.bytes = L.bar + 32;
    return L;
}

__host__ __device__ inline uint32_t tmem_cols_for(int npad, int tiles) {
    const int need = npad * tiles;
    return need <= 32 ? 32u : (need <= 64 ? 64u : 128u);
}

// The same key coordinates as packed fp32 pairs.
template <int E>
__device__ __forceinline__ void tile_key2(const uint8_t *A, int d, int row, int k0, f2x (&x)[E / 2]) {
    const int t = row >> 7, rr = row & 127;
    const int byte = k0 * 2;
    const uint8_t *p = A + (size_t)t * kTileRows * d * 2 + swz_offset(rr, byte >> 4, kTileRows) + (byte & 15);
    if constexpr (E == 4) {
        const uint2 v = *reinterpret_cast<const uint2 *>(p);
        x[0] = bf2_to_f2x(v.x);
        x[1] = bf2_to_f2x(v.y);
    } else {
        x[0] = bf2_to_f2x(*reinterpret_cast<const uint32_t *>(p));
    }
}

// Key row `row` (0 .. tiles*128) of an item, coordinates k0 .. k0+E-1 (E = 2 or 4), from the swizzled tiles.
template <int E>
__device__ __forceinline__ void tile_key(const uint8_t *A, int d, int row, int k0, float (&x)[E]) {
    const int t = row >> 7, rr = row & 127;
    const int byte = k0 * 2;                               // logical byte offset in the row
    const uint8_t *p = A + (size_t)t * kTileRows * d * 2 + swz_offset(rr, byte >> 4, kTileRows) + (byte & 15);
    if constexpr (E == 4) {
        const uint2 v = *reinterpret_cast<const uint2 *>(p);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v.y));
        x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
    } else {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
        x[0] = a.x; x[1] = a.y;
    }
}

// References of KV head kvh into the B slab (rows >= R zero), by every thread of the block.
__device__ __forceinline__ void load_refs_tile(uint8_t *B, const __nv_bfloat16 *refs, int kvh, int R, int npad, int d) {
    const int chunks = d / 8;                              // 16-byte chunks per row
    for (int i = threadIdx.x; i < npad * chunks; i += blockDim.x) {
        const int r = i / chunks, j = i % chunks;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (r < R) v = *reinterpret_cast<const uint4 *>(refs + ((int64_t)kvh * R + r) * d + j * 8);
        *reinterpret_cast<uint4 *>(B + swz_offset(r, j, npad)) = v;
    }
}

// S = K R^T of every tile into tensor memory (columns tile * npad ..), issued by one thread.
__device__ __forceinline__ void leaf_mma(uint32_t sA, uint32_t sB, uint32_t tmem, int tiles, int d, int npad,
                                         uint32_t bar) {
    const uint32_t idesc = tc_idesc_bf16((uint32_t)npad);
    for (int t = 0; t < tiles; ++t) {
        for (int kk = 0; kk < d / 16; ++kk) {      // K in steps of 16 elements (32 bytes)
            const uint32_t off = (kk & 3) * 32;
            const uint64_t ad = smem_desc(sA + t * kTileRows * d * 2 + (kk >> 2) * kTileRows * 128 + off);
            const uint64_t bd = smem_desc(sB + (kk >> 2) * npad * 128 + off);
            tc_mma(tmem + t * npad, ad, bd, idesc, kk > 0 ? 1u : 0u);
        }
    }
    tc_commit(bar);
}

// Softmax of every chunk of the item, from S in tensor memory: one thread per
// key row (warp w reads rows 128 (w / 4) + 32 (w % 4) + lane, the tensor-memory
// lanes it may access). Writes the weights w_t of each (leaf, reference) to W
// and, for leaves in [store_lo, store_hi) (item leaf indices), the biases and
// log-masses to global memory. LARGE: chunks span several warps (c > 32). Every thread of
// the block calls this (it holds block barriers).
template <bool LARGE>
__device__ __forceinline__ void leaf_softmax(const Geo &g, const LeafLayout &Ly, uint8_t *smem, uint32_t tmem,
                                             float *bias_out /* bias of item leaf 0, plane 0 */,
                                             float *lm_out /* log-mass of item leaf 0, plane 0 */, int store_lo,
                                             int store_hi, int rows) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = g.c, R = g.R;
    float *W = reinterpret_cast<float *>(smem + Ly.w);
    float *X = reinterpret_cast<float *>(smem + Ly.x);
    const bool active = warp < 4 * Ly.tiles;
    const int row = (warp >> 2) * kTileRows + (warp & 3) * 32 + lane;
    const int leaf = row / c, t = row % c;
    uint32_t S[32];
    if (active) {
        const uint32_t taddr = tmem + ((uint32_t)((warp & 3) * 32) << 16) + (warp >> 2) * Ly.npad;
        uint32_t v[16];
        tc_ld16(taddr, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) S[i] = v[i];
        if (Ly.npad > 16) {
            tc_ld16(taddr + 16, v);
#pragma unroll
            for (int i = 0; i < 16; ++i) S[16 + i] = v[i];
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) S[16 + i] = 0u;
        }
    }
    const bool keep = active && row < rows && leaf >= store_lo && leaf < store_hi;
    if constexpr (!LARGE) {
        if (!active) return;
#pragma unroll
        for (int r = 0; r < 32; ++r) {
            if (r >= R) break;
            const float l = g.s * __uint_as_float(S[r]);
            float m = l;
            for (int o = 1; o < c; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            const float e = expf(l - m);
            float z = e, el = e * l;
            for (int o = 1; o < c; o <<= 1) {
                z += __shfl_xor_sync(0xffffffffu, z, o);
                el += __shfl_xor_sync(0xffffffffu, el, o);
            }
            const float inv = 1.f / z;
            W[leaf * Ly.wstride + r * c + t] = e * inv;
            if (keep && t == 0) {
                const float F = m + logf(z);
                bias_out[(int64_t)leaf * R + r] = F - el * inv;
                lm_out[(int64_t)leaf * R + r] = F;
            }
        }
    } else {
        // chunks of c = 64, 128 or 256 keys: warp partials, combined in warp
        // order, one reference at a time (two block barriers each)
        const int w0 = (leaf * c) >> 5, nw = c >> 5;
        for (int r = 0; r < R; ++r) {
            const float l = active ? g.s * __uint_as_float(S[r]) : 0.f;
            float v = l;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
            if (active && lane == 0) X[warp * 3] = v;
            __syncthreads();
            float m = -INFINITY;
            if (active) {
                m = X[w0 * 3];
                for (int k = 1; k < nw; ++k) m = fmaxf(m, X[(w0 + k) * 3]);
            }
            const float e = active ? expf(l - m) : 0.f;
            float z = e, el = e * l;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                z += __shfl_xor_sync(0xffffffffu, z, o);
                el += __shfl_xor_sync(0xffffffffu, el, o);
            }
            if (active && lane == 0) {
                X[warp * 3 + 1] = z;
                X[warp * 3 + 2] = el;
            }
            __syncthreads();
            if (active) {
                z = X[w0 * 3 + 1];
                el = X[w0 * 3 + 2];
                for (int k = 1; k < nw; ++k) {
                    z += X[(w0 + k) * 3 + 1];
                    el += X[(w0 + k) * 3 + 2];
                }
                const float inv = 1.f / z;
                W[leaf * Ly.wstride + r * c + t] = e * inv;
                if (keep && t == 0) {
                    const float F = m + logf(z);
                    bias_out[(int64_t)leaf * R + r] = F - el * inv;
                    lm_out[(int64_t)leaf * R + r] = F;
                }
            }
        }
    }
}

// mu_r = sum_t w_t k_t of the item's leaves in [store_lo, store_hi): keys from
// the shared tiles, weights from W. Lane owns coordinates lane * E ...
// C > 0: chunks of C keys, held in registers across the references (one
// warp per leaf); C = 0: keys streamed from shared memory, work units of one
// leaf and a block of up to 16 references spread over the warps.
template <typename T, int E, bool MX, int C>
__device__ __forceinline__ void leaf_mu(const Geo &g, const TreePtrs &tp, const LeafLayout &Ly, const uint8_t *smem,
                                        int grp, int64_t leaf0, int store_lo, int store_hi) {
    constexpr int kRB = 16;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    const int c = g.c, R = g.R;
    const float *W = reinterpret_cast<const float *>(smem + Ly.w);
    const uint8_t *A = smem + Ly.a;
    const int k0 = lane * E;
    constexpr int H = E / 2;
    if constexpr (C > 0) {
        for (int j = store_lo + warp; j < store_hi; j += nwarps) {
            f2x k[C][H];
#pragma unroll
            for (int t = 0; t < C; ++t) tile_key2<E>(A, g.d, j * C + t, k0, k[t]);
            const int64_t rec0 = (grp * g.cap[1] + leaf0 + j) * (int64_t)R;
            const float *wj = W + j * Ly.wstride;
            for (int r = 0; r < R; ++r) {
                float w[C];
                if constexpr (C == 4) {
                    const float4 v = *reinterpret_cast<const float4 *>(wj + r * 4);
                    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
                } else {
#pragma unroll
                    for (int t = 0; t < C; ++t) w[t] = wj[r * C + t];
                }
                f2x acc[H];
#pragma unroll
                for (int e = 0; e < H; ++e) acc[e] = 0ull;
#pragma unroll
                for (int t = 0; t < C; ++t) axpy2<H>(acc, w[t], k[t]);
                float v[E];
                unpack_all(acc, v);
                store_plane<T, E, MX>(g, tp, 1, rec0 + r, v, k0, true);
            }
        }
    } else {
        const int leaves = store_hi - store_lo;
        int rb = R < kRB ? R : kRB;
        while (rb > 1 && ((R + rb - 1) / rb) * leaves < nwarps) rb >>= 1;
        const int nrb = (R + rb - 1) / rb;
        for (int u = warp; u < leaves * nrb; u += nwarps) {
            const int j = store_lo + u / nrb, r0 = (u % nrb) * rb;
            f2x acc[kRB][H];
#pragma unroll
            for (int i = 0; i < kRB; ++i)
#pragma unroll
                for (int e = 0; e < H; ++e) acc[i][e] = 0ull;
            for (int t = 0; t < c; ++t) {
                f2x x[H];
                tile_key2<E>(A, g.d, j * c + t, k0, x);
#pragma unroll
                for (int i = 0; i < kRB; ++i) {
                    if (i >= rb || r0 + i >= R) break;
                    axpy2<H>(acc[i], W[j * Ly.wstride + (r0 + i) * c + t], x);
                }
            }
            const int64_t rec0 = (grp * g.cap[1] + leaf0 + j) * (int64_t)R;
#pragma unroll
            for (int i = 0; i < kRB; ++i) {
                if (i >= rb || r0 + i >= R) break;
                float v[E];
                unpack_all(acc[i], v);
                store_plane<T, E, MX>(g, tp, 1, rec0 + r0 + i, v, k0, true);
            }
        }
    }
}

// The leaf work of an item whose key tiles are in shared memory and whose
// MMAs have been issued to `mma_bar`: wait for S, softmax, mu, biases. Every
// thread of the block calls it. Returns false if the MMA wait timed out.
template <typename T, int E, bool MX, int C, bool LARGE>
__device__ __forceinline__ bool leaf_item(const Geo &g, const TreePtrs &tp, const LeafLayout &Ly, uint8_t *smem,
                                          uint32_t tmem, uint32_t mma_bar, volatile int *abort, int grp,
                                          int64_t leaf0, int store_lo, int store_hi, int rows, int32_t *status) {
    if (threadIdx.x == 0) {
        if (!mbar_wait_bounded(mma_bar, 0, kTreeWait, abort, status)) *abort = 1;
    }
    __syncthreads();
    if (*abort) return false;
    tc_fence_after();
    const int64_t rec0 = (grp * g.cap[1] + leaf0) * (int64_t)g.R;
    leaf_softmax<LARGE>(g, Ly, smem, tmem, tp.bias[1] + rec0, tp.lm[1] + rec0, store_lo, store_hi, rows);
    __syncthreads();
    leaf_mu<T, E, MX, C>(g, tp, Ly, smem, grp, leaf0, store_lo, store_hi);
    return true;
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

// Highest level whose nodes span at most one work item of item_keys keys
// (computed inside the leaf kernel's CTA).
__host__ __device__ inline int fused_levels(int c, int L, int item_keys = kItemKeys) {
    int k = 1;
    int64_t span = (int64_t)c * c;
    while (k < L && span <= item_keys) {
        ++k;
        span *= c;
    }
    return k;
}

// Bulk leaves of a bf16 cache (tree build and large appends): one CTA per
// work item of `tiles` 128-key tiles (two; one when a small update's grid
// would leave most SMs idle) (grid.x: items from the one holding the first
// changed leaf; grid.y: groups). Keys come by TMA (3-D tensor map over
// [group][max_len][d], rows past max_len zero-filled), then the leaf work,
// then the item's parents up to fused_levels.
template <typename T, int E, bool MX, int C, bool LARGE>
__global__ void __launch_bounds__(kLeafWarps * 32, 2)
tree_leaf_kernel(const __grid_constant__ CUtensorMap kmap, Geo g, TreePtrs tp, const T *K, const T *refs,
                 const int32_t *lens, int n_new, int tiles, int32_t *status) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int grp = blockIdx.y;
    const int b = grp / g.Hkv, kvh = grp % g.Hkv;
    int64_t n_old, n_now;
    if (!update_range(g, lens, b, n_new, n_old, n_now, status)) return;
    const int64_t lo1 = n_old / g.c, hi1 = n_now / g.c;          // changed leaves
    const int item_keys = tiles * kTileRows;
    const int64_t key0 = ((lo1 * g.c) / item_keys + blockIdx.x) * item_keys;
    if (key0 >= hi1 * g.c) return;
    const int per_item = item_keys / g.c > 0 ? item_keys / g.c : 1;
    const int64_t leaf0 = key0 / g.c;
    const int store_lo = (int)max64(lo1 - leaf0, 0);
    const int store_hi = (int)min64(hi1 - leaf0, per_item);
    const LeafLayout Ly = leaf_layout(g.d, g.R, g.c, tiles);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Ly.bar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const uint32_t full = smem_u32(bars), mma_bar = smem_u32(bars + 1);
    const uint32_t cols = tmem_cols_for(Ly.npad, tiles);
    if (threadIdx.x == 0) {
        mbar_init(full, 1);
        mbar_init(mma_bar, 1);
        *abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncthreads();
    if ((threadIdx.x >> 5) == 0) tc_alloc(tmem_slot, cols);
    if (threadIdx.x == 0) {
        // tiles of 128 rows, d/64 boxes of 64 columns each
        mbar_expect_tx(full, (uint32_t)(tiles * kTileRows * g.d * 2));
        for (int t = 0; t < tiles; ++t)
            for (int kb = 0; kb < g.d / 64; ++kb)
                tma_load_3d(smem_u32(smem + Ly.a + t * kTileRows * g.d * 2 + kb * kTileRows * 128), &kmap,
                            kb * 64, (int)(key0 + t * kTileRows), grp, full);
    }
    load_refs_tile(smem + Ly.b, reinterpret_cast<const __nv_bfloat16 *>(refs), kvh, g.R, Ly.npad, g.d);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (threadIdx.x == 0) {
        if (mbar_wait_bounded(full, 0, kTreeWait, abort, status)) {
            tc_fence_after();
            leaf_mma(smem_u32(smem + Ly.a), smem_u32(smem + Ly.b), tmem, tiles, g.d, Ly.npad, mma_bar);
        }
    }
    const int rows = (int)min64(hi1 * g.c - key0, (int64_t)tiles * kTileRows);
    const bool ok = leaf_item<T, E, MX, C, LARGE>(g, tp, Ly, smem, tmem, mma_bar, abort, grp, leaf0, store_lo,
                                                  store_hi, rows, status);
    tc_fence_before();
    __syncthreads();
    if (!ok) {
        // let the copies already issued land before the shared memory goes away
        const long long t0 = clock64();
        while (clock64() - t0 < 2000000) {
        }
    }
    tc_fence_after();
    if ((threadIdx.x >> 5) == 0) tc_dealloc(tmem, cols);
    if (!ok) return;
    // the item's parents, level by level (children written by this CTA are
    // visible to it after the barrier)
    const int kf = fused_levels(g.c, g.L, item_keys);
    int64_t lo = lo1, first = leaf0, last = leaf0 + per_item;      // item's nodes at the level below
    for (int level = 2; level <= kf; ++level) {
        lo /= g.c;
        first /= g.c;
        last /= g.c;
        const int64_t n_below = level_nodes(n_now, g.c, level - 1);
        const int64_t nlo = max64(first, lo), nhi = min64(last, level_nodes(n_now, g.c, level));
        __syncthreads();   // the level below is written (and visible to this CTA)
        if (nlo < nhi)
            plane_jobs<T, E * 32 / kSub, MX, C>(g, tp, K, refs, grp, level, nlo, nhi, n_below, threadIdx.x >> 5,
                                                blockDim.x >> 5, threadIdx.x & 31);
    }
}

// One level, many nodes, on CUDA cores (levels above fused_levels; every
// level of an fp32 cache): grid.x covers plane quads of the changed nodes,
// grid.y groups.
template <typename T, int E, bool MX, int C>
__global__ void __launch_bounds__(kLevelWarps * 32)
tree_level_kernel(Geo g, TreePtrs tp, const T *K, const T *refs, const int32_t *lens, int level, int n_new,
                  int64_t slots, int32_t *status) {
    const int grp = blockIdx.y;
    const int b = grp / g.Hkv;
    const int lane = threadIdx.x & 31;
    int64_t n_old, n_now;
    if (!update_range(g, lens, b, n_new, n_old, n_now, status)) return;
    int64_t lo = n_old / g.c;
    for (int l = 2; l <= level; ++l) lo /= g.c;
    const int64_t hi = min64(level_nodes(n_now, g.c, level), lo + slots);
    if (lo >= hi) return;
    const int64_t job = (int64_t)blockIdx.x * kLevelWarps + (threadIdx.x >> 5);
    if (job * kPerWarp >= (hi - lo) * g.R) return;
    const int64_t n_below = level > 1 ? level_nodes(n_now, g.c, level - 1) : 0;
    plane_jobs<T, E, MX, C>(g, tp, K, refs, grp, level, lo, hi, n_below, job, (int64_t)1 << 40, lane);
}

// Few new tokens (a decode step; an append of at most c tokens): one block per
// group walks every level -- the leaf that completed (if any), then its
// ancestors -- with a block barrier between levels, which also makes the
// children's global writes visible. A bf16 leaf is a single-leaf item: its
// keys go into the tile with plain loads, then the bulk kernel's MMAs and
// leaf routine (so the result equals the bulk build's bit for bit).
template <typename T, int E, bool MX, int C, bool LARGE>
__device__ __forceinline__ void tree_path_levels(const Geo &g, const TreePtrs &tp, const T *K, const T *refs,
                                                 int grp, int64_t n_old, int64_t n_now, uint8_t *smem,
                                                 int32_t *status) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    int64_t lo = n_old / g.c;
    const int64_t hi1 = n_now / g.c;
    bool ok = true;
    if (hi1 > lo) {
        if constexpr (sizeof(T) == 2) {
            // the one leaf that completed (at most c tokens were added)
            const int64_t leaf = hi1 - 1;
            const int tiles = (g.c + kTileRows - 1) / kTileRows;
            const LeafLayout Ly = leaf_layout(g.d, g.R, g.c, tiles);
            uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Ly.bar);
            uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2);
            volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
            const uint32_t mma_bar = smem_u32(bars + 1);
            const uint32_t cols = tmem_cols_for(Ly.npad, tiles);
            if (threadIdx.x == 0) {
                mbar_init(mma_bar, 1);
                *abort = 0;
                asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
            }
            // keys of the chunk into rows 0 .. c-1 (the MMA's other rows are
            // never read: each row of S depends on its own key row only)
            const int chunks = g.d / 8;
            const T *src = K + ((int64_t)grp * g.max_len + leaf * g.c) * g.d;
            for (int i = threadIdx.x; i < g.c * chunks; i += blockDim.x) {
                const int row = i / chunks, j = i % chunks;
                const uint4 v = *reinterpret_cast<const uint4 *>(src + (int64_t)row * g.d + j * 8);
                *reinterpret_cast<uint4 *>(smem + Ly.a + (row >> 7) * kTileRows * g.d * 2 +
                                           swz_offset(row & 127, j, kTileRows)) = v;
            }
            load_refs_tile(smem + Ly.b, reinterpret_cast<const __nv_bfloat16 *>(refs), grp % g.Hkv, g.R, Ly.npad,
                           g.d);
            if (warp == 0) tc_alloc(tmem_slot, cols);
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            const uint32_t tmem = *tmem_slot;
            if (threadIdx.x == 0) leaf_mma(smem_u32(smem + Ly.a), smem_u32(smem + Ly.b), tmem, tiles, g.d, Ly.npad, mma_bar);
            // one leaf: its planes spread over the warps (C = 0: the same
            // arithmetic as the bulk kernel's register path, plane by plane)
            ok = leaf_item<T, E, MX, 0, LARGE>(g, tp, Ly, smem, tmem, mma_bar, abort, grp, leaf, 0, 1, g.c, status);
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            if (warp == 0) tc_dealloc(tmem, cols);
        } else {
            plane_jobs<T, E * 32 / kSub, MX, C>(g, tp, K, refs, grp, 1, lo, hi1, 0, warp, nwarps, lane);
        }
    }
    if (!ok) return;
    for (int level = 2; level <= g.L; ++level) {
        lo /= g.c;
        const int64_t hi = level_nodes(n_now, g.c, level);
        const int64_t n_below = level_nodes(n_now, g.c, level - 1);
        __syncthreads();
        if (lo < hi)
            plane_jobs<T, E * 32 / kSub, MX, C>(g, tp, K, refs, grp, level, lo, hi, n_below, warp, nwarps, lane);
    }
    __syncthreads();
}

constexpr int kPathMaxThreads = 512;

template <typename T, int E, bool MX, int C, bool LARGE>
__global__ void __launch_bounds__(kPathMaxThreads) tree_path_kernel(Geo g, TreePtrs tp, const T *K, const T *refs, const int32_t *lens, int n_new,
                                 int32_t *status) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int grp = blockIdx.x;
    const int b = grp / g.Hkv;
    int64_t n_old, n_now;
    const bool any = update_range(g, lens, b, n_new, n_old, n_now, status);
    if (!any) return;  // uniform across the block
    tree_path_levels<T, E, MX, C, LARGE>(g, tp, K, refs, grp, n_old, n_now, smem, status);
}

// A decode step's prologue, one block per (sequence, KV head) group: write
// the group's new token at position lens[b], extend the tree along its
// rightmost path if the token completes a chunk, reset the group's routing
// state, and -- in the last of the sequence's groups to get here, after every
// group has read the old length -- advance lens[b].
template <typename T, int E, bool MX, int C, bool LARGE>
__global__ void __launch_bounds__(kPathMaxThreads) decode_prologue_kernel(Geo g, TreePtrs tp, T *K, T *V, const T *refs, int32_t *lens, const T *k_new,
                                       const T *v_new, uint32_t *arrive, RouteState rs, int32_t *status) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
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
    if (ok && (n + 1) / g.c > n / g.c) tree_path_levels<T, E, MX, C, LARGE>(g, tp, K, refs, grp, n, n + 1, smem, status);
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

// ---------------------------------------------------------------------- host

// Dynamic shared memory of the path kernels (a single-leaf item) and of the
// leaf kernel (a 256-key item), with 1 KB of alignment slack.
size_t path_smem(const Geo &g) {
    if (g.dtype != ZHA_BF16) return 0;
    const int tiles = (g.c + kTileRows - 1) / kTileRows;
    return leaf_layout(g.d, g.R, g.c, tiles).bytes + 1024;
}
size_t item_smem(const Geo &g) { return leaf_layout(g.d, g.R, g.c, 2).bytes + 1024; }

int path_threads(const Geo &g) {
    // at least 8 warps (a 256-key chunk's softmax reads 8 warps' worth of
    // tensor-memory lanes); up to one warp per plane otherwise, at most 16
    int warps = g.R > 16 ? 16 : (g.R < 8 ? 8 : g.R);
    return warps * 32;
}

// Opt a kernel in to the dynamic shared memory it needs (once per device and
// size; set whenever it is not small, so that static shared memory and the
// 48 KB default never meet at the limit).
template <auto Kernel>
void set_smem_attr(size_t bytes) {
    static size_t done[64] = {};
    int dev = 0;
    if (bytes <= 16 * 1024 || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64 || done[dev] >= bytes)
        return;
    if (cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) == cudaSuccess)
        done[dev] = bytes;
}

template <typename T, int E, bool MX, int C, bool LARGE>
cudaError_t decode_prologue_t(const Geo &g, const TreePtrs &tp, T *K, T *V, const T *refs, int32_t *lens,
                              const T *k_new, const T *v_new, uint32_t *arrive, const RouteState &rs,
                              int32_t *status, cudaStream_t st) {
    const size_t smem = path_smem(g);
    set_smem_attr<decode_prologue_kernel<T, E, MX, C, LARGE>>(smem);
    ProfScope ps("decode_prologue", st);
    return launch_pdl(decode_prologue_kernel<T, E, MX, C, LARGE>, dim3(g.groups()), dim3(path_threads(g)), smem, st,
                      g, tp, K, V, refs, lens, k_new, v_new, arrive, rs, status);
}

bool make_key_map(const Geo &g, const void *K, CUtensorMap *map) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)g.d, (cuuint64_t)g.max_len, (cuuint64_t)g.groups()};
    const cuuint64_t strides[2] = {(cuuint64_t)g.d * 2, (cuuint64_t)g.max_len * g.d * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)kTileRows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(K), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

const char *level_name(int level) {
    static const char *names[] = {"", "tree_level[l1]", "tree_level[l2]", "tree_level[l3]", "tree_level[l4]",
                                  "tree_level[l5]", "tree_level[l6]", "tree_level[l7]", "tree_level[l8]"};
    return names[level];
}

// Levels first_level .. L on CUDA cores over the nodes an update changes.
template <typename T, int E, bool MX, int C>
cudaError_t level_launches(const Geo &g, const TreePtrs &tp, const T *K, const T *refs, const int32_t *lens,
                           int n_new, int first_level, int32_t *status, cudaStream_t st) {
    int64_t bound = n_new < 0 ? g.cap[1] : (n_new + g.c - 1) / g.c + 1;
    for (int level = 1; level <= g.L; ++level) {
        if (level > 1) bound = n_new < 0 ? g.cap[level] : bound / g.c + 2;
        bound = min64(bound, g.cap[level]);
        if (bound <= 0) break;
        if (level < first_level) continue;
        const int64_t jobs = (bound * g.R + kPerWarp - 1) / kPerWarp;
        dim3 grid((unsigned)((jobs + kLevelWarps - 1) / kLevelWarps), g.groups());
        ProfScope ps(level_name(level), st);
        tree_level_kernel<T, E * 32 / kSub, MX, C><<<grid, kLevelWarps * 32, 0, st>>>(g, tp, K, refs, lens, level,
                                                                                   n_new, bound, status);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

template <typename T, int E, bool MX, int C, bool LARGE>
cudaError_t tree_update_t(const Geo &g, const TreePtrs &tp, const T *K, const T *refs, const int32_t *lens,
                          int n_new, int32_t *status, cudaStream_t st) {
    if (n_new >= 0 && n_new <= g.c) {
        const size_t smem = path_smem(g);
        set_smem_attr<tree_path_kernel<T, E, MX, C, LARGE>>(smem);
        ProfScope ps("tree_path", st);
        tree_path_kernel<T, E, MX, C, LARGE><<<g.groups(), path_threads(g), smem, st>>>(g, tp, K, refs, lens, n_new,
                                                                                      status);
        return cudaGetLastError();
    }
    if constexpr (sizeof(T) == 2) {
        CUtensorMap map;
        if (!make_key_map(g, K, &map)) return cudaErrorNotSupported;
        // items of two tiles; of one where two-tile items would not cover the
        // SMs (an append to a few sequences): twice the CTAs, each half as long
        static const int sms = [] {
            int dev = 0, n = 0;
            if (cudaGetDevice(&dev) != cudaSuccess ||
                cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
                return 0;
            return n;
        }();
        int item_keys = kItemKeys;
        auto items_for = [&](int ik) {
            const int64_t keys = n_new < 0 ? g.cap[1] * g.c : (int64_t)n_new + ik;
            return (keys + ik - 1) / ik + 1;
        };
        if (g.c <= kTileRows && items_for(kItemKeys) * g.groups() <= sms) item_keys = kTileRows;
        const int64_t items = items_for(item_keys);
        const size_t smem = item_smem(g);
        set_smem_attr<tree_leaf_kernel<T, E, MX, C, LARGE>>(smem);
        {
            ProfScope ps("tree_leaf", st);
            tree_leaf_kernel<T, E, MX, C, LARGE><<<dim3((unsigned)items, g.groups()), kLeafWarps * 32, smem, st>>>(
                map, g, tp, K, refs, lens, n_new, item_keys / kTileRows, status);
        }
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        return level_launches<T, E, MX, C>(g, tp, K, refs, lens, n_new, fused_levels(g.c, g.L, item_keys) + 1,
                                           status, st);
    } else {
        return level_launches<T, E, MX, C>(g, tp, K, refs, lens, n_new, 1, status, st);
    }
}

// Dispatch on the chunk size: C = 4 holds a chunk's keys in registers across
// the references (the deep tree); other sizes stream them from shared
// memory; LARGE for chunks spanning several warps (c > 32).
template <typename T, int E, bool MX, class F>
cudaError_t by_chunk(int c, F &&f) {
    if (c == 4) return f.template operator()<T, E, MX, 4, false>();
    if (c <= 32) return f.template operator()<T, E, MX, 0, false>();
    return f.template operator()<T, E, MX, 0, true>();
}

// Dispatch on dtype, head_dim and summary format.
template <class F>
cudaError_t dispatch(const Geo &g, F &&f) {
    if (g.dtype == ZHA_BF16) {
        if (g.mx())
            return g.d == 128 ? by_chunk<__nv_bfloat16, 4, true>(g.c, f) : by_chunk<__nv_bfloat16, 2, true>(g.c, f);
        return g.d == 128 ? by_chunk<__nv_bfloat16, 4, false>(g.c, f) : by_chunk<__nv_bfloat16, 2, false>(g.c, f);
    }
    // fp32 caches: CUDA cores only (C still selects the parents' point loop)
    if (g.c == 4)
        return g.d == 128 ? f.template operator()<float, 4, false, 4, false>()
                          : f.template operator()<float, 2, false, 4, false>();
    return g.d == 128 ? f.template operator()<float, 4, false, 0, false>()
                      : f.template operator()<float, 2, false, 0, false>();
}

}  // namespace

TreePtrs tree_ptrs(const Geo &g, void *tree) {
    TreePtrs tp{};
    for (int l = 1; l <= g.L; ++l) {
        tp.mu[l] = static_cast<char *>(tree) + g.mu_off[l];
        tp.bias[l] = reinterpret_cast<float *>(static_cast<char *>(tree) + g.bias_off[l]);
        tp.sc[l] = g.mx() ? reinterpret_cast<uint8_t *>(static_cast<char *>(tree) + g.sc_off[l]) : nullptr;
        tp.lm[l] = reinterpret_cast<float *>(static_cast<char *>(tree) + g.lm_off[l]);
    }
    return tp;
}

cudaError_t launch_decode_prologue(const Geo &g, void *tree, void *K, void *V, const void *refs,
                                   int32_t *lens, const void *k_new, const void *v_new, void *ws,
                                   int32_t *status, cudaStream_t st) {
    const TreePtrs tp = tree_ptrs(g, tree);
    const RouteState rs = route_state(g, ws);
    uint32_t *arrive = reinterpret_cast<uint32_t *>(static_cast<char *>(ws) + g.ws_arrive);
    return dispatch(g, [&]<typename T, int E, bool MX, int C, bool LARGE>() {
        return decode_prologue_t<T, E, MX, C, LARGE>(g, tp, static_cast<T *>(K), static_cast<T *>(V),
                                                     static_cast<const T *>(refs), lens, static_cast<const T *>(k_new),
                                                     static_cast<const T *>(v_new), arrive, rs, status, st);
    });
}

cudaError_t launch_tree_update(const Geo &g, void *tree, const void *K, const void *refs,
                               const int32_t *lens, int n_new, int32_t *status, cudaStream_t st) {
    const TreePtrs tp = tree_ptrs(g, tree);
    return dispatch(g, [&]<typename T, int E, bool MX, int C, bool LARGE>() {
        return tree_update_t<T, E, MX, C, LARGE>(g, tp, static_cast<const T *>(K), static_cast<const T *>(refs), lens,
                                                 n_new, status, st);
    });
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
