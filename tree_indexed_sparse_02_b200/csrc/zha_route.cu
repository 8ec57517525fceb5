// zha_route.cu -- top-p routing down the summary tree.
//
// Page "Zyphra AI Introduces Zyphra Hierarchical Attention (ZHA)", section
// "How does top-p routing pick tokens": a decode query scores the top-level
// nodes, keeps the smallest set that holds a fraction p of the estimated
// attention mass, expands only their children, and repeats down to the raw
// KV entries. Section "Building the tree": a node's estimate is the max over
// its reference planes, E = max_r (s q.mu_r + bias_r).
//
// Per level, for all (sequence, KV head) groups at once:
//   score  -- every candidate node of a group is read once and scored for all
//             G query heads of the group (mma.sync bf16 tiles: planes x heads);
//   select -- one CTA per (group, query head): exact threshold search for the
//             shortest (score desc, index asc) prefix holding p of the mass,
//             as a 3-pass radix select on the fp32 score bits with masses
//             summed in 2^-40 fixed point (exact, order-independent sums);
//   expand -- one CTA per group: the existing children of the nodes kept by
//             any head become the next level's candidates (ascending), each
//             carrying the bit mask of heads that kept its parent.
#include "zha_common.cuh"

namespace zha {

namespace {

// ------------------------------------------------------------------ level views

struct LevelWs {
    int32_t *cand;
    uint32_t *cmask;
    float *scores;
    uint32_t *kept;
    int32_t *count;
};

__host__ __device__ inline LevelWs level_ws(const Geo &g, void *ws, int l) {
    char *base = static_cast<char *>(ws);
    LevelWs v;
    v.cand = reinterpret_cast<int32_t *>(base + g.ws_cand[l]);
    v.cmask = reinterpret_cast<uint32_t *>(base + g.ws_cmask[l]);
    v.scores = reinterpret_cast<float *>(base + g.ws_scores[l]);
    v.kept = reinterpret_cast<uint32_t *>(base + g.ws_kept[l]);
    v.count = reinterpret_cast<int32_t *>(base + g.ws_count[l]);
    return v;
}

__device__ __forceinline__ uint32_t all_heads(int G) { return G >= 32 ? 0xffffffffu : ((1u << G) - 1u); }

// ----------------------------------------------------------------------- init

__global__ void route_init_kernel(Geo g, LevelWs top, const int32_t *lens, uint32_t *maxkey,
                                  int32_t *status) {
    const int grp = blockIdx.x;
    const int b = grp / g.Hkv;
    int64_t N = lens[b];
    if (N < 0 || N > g.max_len) {
        if (threadIdx.x == 0) set_status(status, ZHA_ERR_CAPACITY);
        N = 0;
    }
    const int64_t nL = level_nodes(N, g.c, g.L);
    const int64_t cap = g.cap[g.L];
    for (int64_t i = threadIdx.x; i < nL; i += blockDim.x) {
        top.cand[grp * cap + i] = (int32_t)i;
        top.cmask[grp * cap + i] = all_heads(g.G);
        top.kept[grp * cap + i] = 0u;
    }
    if (threadIdx.x == 0) top.count[grp] = (int32_t)nL;
    for (int i = threadIdx.x; i < g.L * g.G; i += blockDim.x)
        maxkey[((int64_t)(i / g.G) * g.groups() + grp) * g.G + i % g.G] = 0u;
}

// ---------------------------------------------------------------------- score

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ldg16(const void *p) {
    return __ldg(reinterpret_cast<const uint4 *>(p));
}

constexpr int kScoreWarps = 4;

// bf16 scoring on tensor cores. One warp scores one node per iteration:
// A = the node's planes (16 rows per m-tile, K = head_dim), B = the group's
// query heads (8 columns per n-tile). Coordinates are permuted identically in
// A and B so that each lane fetches 16 contiguous bytes per row and k-pair
// (fully used 32-byte sectors); a dot product is invariant to that.
template <int D, int MT, int NT>
__global__ void __launch_bounds__(kScoreWarps * 32)
score_mma_kernel(Geo g, const __nv_bfloat16 *mu, const float *bias, const __nv_bfloat16 *q,
                 LevelWs lw, int level, uint32_t *maxkey) {
    constexpr int KP = D / 32;
    const int grp = blockIdx.y;
    const int b = grp / g.Hkv, kvh = grp % g.Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gq = lane >> 2, t = lane & 3;
    const int64_t cap = g.cap[level];
    const int n = lw.count[grp];

    uint32_t bq[NT][KP][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int h = nt * 8 + gq;
#pragma unroll
        for (int kp = 0; kp < KP; ++kp) {
            uint4 w = make_uint4(0, 0, 0, 0);
            if (h < g.G) w = ldg16(q + ((int64_t)b * g.Hq + kvh * g.G + h) * D + kp * 32 + t * 8);
            bq[nt][kp][0] = w.x; bq[nt][kp][1] = w.y; bq[nt][kp][2] = w.z; bq[nt][kp][3] = w.w;
        }
    }
    float runmax[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) runmax[nt][0] = runmax[nt][1] = -INFINITY;

    const float s = g.s;
    for (int i = blockIdx.x * kScoreWarps + warp; i < n; i += gridDim.x * kScoreWarps) {
        const int64_t node = lw.cand[grp * cap + i];
        const uint32_t hm = lw.cmask[grp * cap + i];
        const __nv_bfloat16 *base = mu + (grp * cap + node) * (int64_t)g.R * D;
        const float *bb = bias + (grp * cap + node) * (int64_t)g.R;
        uint4 ra[MT][KP], rb[MT][KP];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int r0 = mt * 16 + gq, r1 = r0 + 8;
#pragma unroll
            for (int kp = 0; kp < KP; ++kp) {
                ra[mt][kp] = r0 < g.R ? ldg16(base + (int64_t)r0 * D + kp * 32 + t * 8) : make_uint4(0, 0, 0, 0);
                rb[mt][kp] = r1 < g.R ? ldg16(base + (int64_t)r1 * D + kp * 32 + t * 8) : make_uint4(0, 0, 0, 0);
            }
        }
        float e[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) e[nt][0] = e[nt][1] = -INFINITY;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            float acc[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
            for (int kp = 0; kp < KP; ++kp) {
                const uint32_t a0[4] = {ra[mt][kp].x, rb[mt][kp].x, ra[mt][kp].y, rb[mt][kp].y};
                const uint32_t a1[4] = {ra[mt][kp].z, rb[mt][kp].z, ra[mt][kp].w, rb[mt][kp].w};
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    mma_bf16_16816(acc[nt], a0, bq[nt][kp][0], bq[nt][kp][1]);
                    mma_bf16_16816(acc[nt], a1, bq[nt][kp][2], bq[nt][kp][3]);
                }
            }
            const int r0 = mt * 16 + gq, r1 = r0 + 8;
            const float b0 = r0 < g.R ? bb[r0] : -INFINITY;
            const float b1 = r1 < g.R ? bb[r1] : -INFINITY;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                e[nt][0] = fmaxf(e[nt][0], fmaxf(fmaf(s, acc[nt][0], b0), fmaf(s, acc[nt][2], b1)));
                e[nt][1] = fmaxf(e[nt][1], fmaxf(fmaf(s, acc[nt][1], b0), fmaf(s, acc[nt][3], b1)));
            }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                float v = e[nt][j];
                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
                v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
                e[nt][j] = v;
            }
        if (gq == 0) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int h = nt * 8 + 2 * t + j;
                    if (h < g.G) {
                        lw.scores[(grp * g.G + h) * cap + i] = e[nt][j];
                        if ((hm >> h) & 1u) runmax[nt][j] = fmaxf(runmax[nt][j], e[nt][j]);
                    }
                }
        }
    }
    if (gq == 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int h = nt * 8 + 2 * t + j;
                if (h < g.G && runmax[nt][j] > -INFINITY)
                    atomicMax(&maxkey[(int64_t)grp * g.G + h], ordered_key(runmax[nt][j]));
            }
    }
}

// fp32 scoring on CUDA cores: one block per node per iteration, one thread
// per (plane, head) dot product.
template <int D>
__global__ void score_f32_kernel(Geo g, const float *mu, const float *bias, const float *q,
                                 LevelWs lw, int level, uint32_t *maxkey) {
    __shared__ float qs[16][D];
    __shared__ float es[32][16];
    const int grp = blockIdx.y;
    const int b = grp / g.Hkv, kvh = grp % g.Hkv;
    const int64_t cap = g.cap[level];
    const int n = lw.count[grp];
    for (int i = threadIdx.x; i < g.G * D; i += blockDim.x)
        qs[i / D][i % D] = q[((int64_t)b * g.Hq + kvh * g.G + i / D) * D + i % D];
    float runmax = -INFINITY;
    __syncthreads();
    for (int i = blockIdx.x; i < n; i += gridDim.x) {
        const int64_t node = lw.cand[grp * cap + i];
        const uint32_t hm = lw.cmask[grp * cap + i];
        const float *base = mu + (grp * cap + node) * (int64_t)g.R * D;
        const float *bb = bias + (grp * cap + node) * (int64_t)g.R;
        for (int pr = threadIdx.x; pr < g.R * g.G; pr += blockDim.x) {
            const int r = pr / g.G, h = pr % g.G;
            float acc = 0.f;
            for (int k = 0; k < D; ++k) acc = fmaf(base[(int64_t)r * D + k], qs[h][k], acc);
            es[r][h] = fmaf(g.s, acc, bb[r]);
        }
        __syncthreads();
        if (threadIdx.x < g.G) {
            const int h = threadIdx.x;
            float e = -INFINITY;
            for (int r = 0; r < g.R; ++r) e = fmaxf(e, es[r][h]);
            lw.scores[(grp * g.G + h) * cap + i] = e;
            if ((hm >> h) & 1u) runmax = fmaxf(runmax, e);
        }
        __syncthreads();
    }
    if (threadIdx.x < g.G && runmax > -INFINITY)
        atomicMax(&maxkey[(int64_t)grp * g.G + threadIdx.x], ordered_key(runmax));
}

// --------------------------------------------------------------------- select

constexpr int kSelThreads = 512;
constexpr int kBuckets = 2048;
constexpr int kMaxTies = 1024;
// masses e^{E - max} in (0, 1] are summed as integers in units of 2^-40
constexpr float kMassScale = 1099511627776.0f;

__device__ __forceinline__ unsigned long long fixed_mass(float e, float m) {
    return __float2ull_rn(expf(e - m) * kMassScale);
}

template <typename V>
__device__ __forceinline__ V block_sum(V v, V *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    V tot = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += red[w];
    __syncthreads();
    return tot;
}

// Exclusive prefix sum over the block (thread order); *total gets the sum.
template <typename V>
__device__ __forceinline__ V block_exclusive_scan(V v, V *red, V *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nw = blockDim.x >> 5;
    V x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        V y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    __syncthreads();
    if (lane == 31) red[warp] = x;
    __syncthreads();
    V before = 0, tot = 0;
    for (int w = 0; w < nw; ++w) {
        if (w < warp) before += red[w];
        tot += red[w];
    }
    __syncthreads();
    *total = tot;
    return before + x - v;
}

struct SelShared {
    unsigned long long hist[kBuckets];
    unsigned long long red[kSelThreads / 32];
    int32_t ties[kMaxTies];
    int32_t sorted_ties[kMaxTies];
    unsigned long long above, target;
    uint32_t digit;
    uint32_t maxkey;
    int ntie;
};

// Exact top-p over the members of one candidate set:
//   member(i)  -- candidate i belongs to this head's set
//   score(i)   -- its fp32 estimate
//   emit(i)    -- called once for every kept candidate
// Returns (in every thread) the number kept.
template <class Member, class Score, class Emit>
__device__ int topp_core(SelShared &sh, int64_t n, float p, uint32_t maxkey_in, Member member,
                         Score score, Emit emit) {
    const int tid = threadIdx.x;
    // max over the members (passed in when the scorer already has it)
    if (tid == 0) sh.maxkey = maxkey_in;
    __syncthreads();
    if (maxkey_in == 0u) {
        uint32_t mk = 0u;
        for (int64_t i = tid; i < n; i += blockDim.x)
            if (member(i)) mk = max(mk, ordered_key(score(i)));
        if (mk) atomicMax(&sh.maxkey, mk);
        __syncthreads();
    }
    const uint32_t mk = sh.maxkey;
    if (mk == 0u) return 0;  // no member
    int kept = 0;
    if (p >= 1.f) {
        for (int64_t i = tid; i < n; i += blockDim.x)
            if (member(i)) {
                emit(i);
                ++kept;
            }
        return (int)block_sum<unsigned long long>((unsigned long long)kept, sh.red);
    }
    const float m = key_to_float(mk);
    // three radix passes (11, 11, 10 bits) find tau, the key of the crossing
    // candidate, and `above`, the mass of all candidates with larger keys.
    uint32_t prefix = 0u;
    int hi_shift = 32;
    if (tid == 0) sh.above = 0ull;
    for (int pass = 0; pass < 3; ++pass) {
        const int bits = pass < 2 ? 11 : 10;
        const int shift = hi_shift - bits;
        for (int i = tid; i < kBuckets; i += blockDim.x) sh.hist[i] = 0ull;
        __syncthreads();
        for (int64_t i = tid; i < n; i += blockDim.x) {
            if (!member(i)) continue;
            const float e = score(i);
            const uint32_t k = ordered_key(e);
            if (hi_shift < 32 && (k >> hi_shift) != (prefix >> hi_shift)) continue;
            atomicAdd(&sh.hist[(k >> shift) & ((1u << bits) - 1u)], fixed_mass(e, m));
        }
        __syncthreads();
        if (pass == 0) {
            unsigned long long z = 0ull;
            for (int i = tid; i < kBuckets; i += blockDim.x) z += sh.hist[i];
            z = block_sum<unsigned long long>(z, sh.red);
            if (tid == 0) sh.target = (unsigned long long)ceil((double)p * (double)z);
            __syncthreads();
        }
        // crossing bucket: running mass from the top bucket down first reaches target
        constexpr int per = kBuckets / kSelThreads;
        unsigned long long mine = 0ull;
#pragma unroll
        for (int j = 0; j < per; ++j) mine += sh.hist[tid * per + j];
        // suffix sum over threads of higher index = total - inclusive prefix
        unsigned long long tot;
        const unsigned long long excl = block_exclusive_scan<unsigned long long>(mine, sh.red, &tot);
        unsigned long long run = sh.above + (tot - excl - mine);
        const unsigned long long target = sh.target;
        __syncthreads();
#pragma unroll
        for (int j = per - 1; j >= 0; --j) {
            const int dgt = tid * per + j;
            const unsigned long long hgt = sh.hist[dgt];
            if (hgt && run < target && run + hgt >= target) {
                sh.digit = (uint32_t)dgt;
                sh.above = run;  // mass strictly above this bucket
            }
            run += hgt;
        }
        __syncthreads();
        prefix |= sh.digit << shift;
        hi_shift = shift;
    }
    const uint32_t tau = prefix;
    const unsigned long long above = sh.above, target = sh.target;
    if (tid == 0) sh.ntie = 0;
    __syncthreads();
    // keys above tau are kept; ties at tau are resolved in index order
    for (int64_t i = tid; i < n; i += blockDim.x) {
        if (!member(i)) continue;
        const uint32_t k = ordered_key(score(i));
        if (k > tau) {
            emit(i);
            ++kept;
        } else if (k == tau) {
            const int slot = atomicAdd(&sh.ntie, 1);
            if (slot < kMaxTies) sh.ties[slot] = (int32_t)i;
        }
    }
    __syncthreads();
    const int ntie = sh.ntie;
    if (ntie <= kMaxTies) {
        for (int j = tid; j < ntie; j += blockDim.x) {
            int rank = 0;
            const int32_t v = sh.ties[j];
            for (int u = 0; u < ntie; ++u) rank += sh.ties[u] < v;
            sh.sorted_ties[rank] = v;
        }
        __syncthreads();
        if (tid == 0) {
            unsigned long long cum = above;
            for (int j = 0; j < ntie && cum < target; ++j) {
                const int32_t i = sh.sorted_ties[j];
                emit(i);
                ++kept;
                cum += fixed_mass(score(i), m);
            }
        }
    } else if (tid == 0) {
        // more exact ties than fit: walk the whole set in index order
        unsigned long long cum = above;
        for (int64_t i = 0; i < n && cum < target; ++i) {
            if (!member(i) || ordered_key(score(i)) != tau) continue;
            emit(i);
            ++kept;
            cum += fixed_mass(score(i), m);
        }
    }
    return (int)block_sum<unsigned long long>((unsigned long long)kept, sh.red);
}

__global__ void __launch_bounds__(kSelThreads)
select_kernel(Geo g, LevelWs lw, int level, float p, const uint32_t *maxkey, int32_t *level_kept) {
    __shared__ SelShared sh;
    const int h = blockIdx.x, grp = blockIdx.y;
    const int64_t cap = g.cap[level];
    const int64_t n = lw.count[grp];
    const uint32_t bit = 1u << h;
    const uint32_t *cmask = lw.cmask + grp * cap;
    const float *sc = lw.scores + (grp * g.G + h) * cap;
    uint32_t *kept = lw.kept + grp * cap;
    const uint32_t mk = maxkey[(int64_t)grp * g.G + h];
    const int nk = topp_core(
        sh, n, p, mk, [&](int64_t i) { return (cmask[i] & bit) != 0u; },
        [&](int64_t i) { return sc[i]; }, [&](int64_t i) { atomicOr(&kept[i], bit); });
    if (level_kept && threadIdx.x == 0) {
        const int b = grp / g.Hkv, kvh = grp % g.Hkv;
        level_kept[((int64_t)b * g.Hq + kvh * g.G + h) * g.L + (level - 1)] = mk ? nk : 0;
    }
}

__global__ void __launch_bounds__(kSelThreads)
select_sets_kernel(const float *scores, const int32_t *counts, int64_t stride, float p,
                   uint8_t *kept, int32_t *status) {
    __shared__ SelShared sh;
    const int set = blockIdx.x;
    int64_t n = counts[set];
    if (n < 0 || n > stride) {
        if (threadIdx.x == 0) set_status(status, ZHA_ERR_INVALID_ARG);
        n = 0;
    }
    const float *sc = scores + set * stride;
    uint8_t *kp = kept + set * stride;
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) kp[i] = 0;
    __syncthreads();
    topp_core(
        sh, n, p, 0u, [&](int64_t) { return true; }, [&](int64_t i) { return sc[i]; },
        [&](int64_t i) { kp[i] = 1; });
}

// --------------------------------------------------------------------- expand

constexpr int kExpThreads = 1024;

__global__ void __launch_bounds__(kExpThreads)
expand_kernel(Geo g, LevelWs cur, LevelWs nxt, int level, const int32_t *lens,
              zha_selection sel) {
    __shared__ int64_t red[kExpThreads / 32];
    const int grp = blockIdx.x;
    const int b = grp / g.Hkv;
    int64_t N = lens[b];
    if (N < 0 || N > g.max_len) N = 0;
    const int64_t cap = g.cap[level];
    const int64_t n = cur.count[grp];
    const int64_t n_below = level > 1 ? level_nodes(N, g.c, level - 1) : 0;
    const int64_t cap_next = level > 1 ? g.cap[level - 1] : g.cap[1];
    int64_t run = 0;
    for (int64_t base = 0; base < n; base += blockDim.x) {
        const int64_t i = base + threadIdx.x;
        uint32_t km = 0u;
        int64_t node = 0;
        if (i < n) {
            km = cur.kept[grp * cap + i];
            node = cur.cand[grp * cap + i];
        }
        int64_t nch = 0;
        if (km) nch = level > 1 ? min64(g.c, n_below - node * g.c) : 1;
        int64_t tot;
        const int64_t off = run + block_exclusive_scan<int64_t>(nch, red, &tot);
        if (level > 1) {
            for (int64_t j = 0; j < nch; ++j) {
                nxt.cand[grp * cap_next + off + j] = (int32_t)(node * g.c + j);
                nxt.cmask[grp * cap_next + off + j] = km;
                nxt.kept[grp * cap_next + off + j] = 0u;
            }
        } else if (nch) {
            sel.leaf_idx[grp * cap_next + off] = (int32_t)node;
            sel.head_mask[grp * cap_next + off] = km;
        }
        run += tot;
    }
    if (threadIdx.x == 0) {
        if (level > 1)
            nxt.count[grp] = (int32_t)run;
        else
            sel.count[grp] = (int32_t)run;
    }
}

}  // namespace

cudaError_t launch_route(const Geo &g, const void *tree, const void *q, const int32_t *lens,
                         const float *p_levels, const zha_selection &sel, void *ws,
                         int32_t *status, cudaStream_t st) {
    uint32_t *maxkey = reinterpret_cast<uint32_t *>(static_cast<char *>(ws) + g.ws_maxkey);
    const int groups = g.groups();
    static const char *score_names[] = {"", "score[l1]", "score[l2]", "score[l3]", "score[l4]",
                                        "score[l5]", "score[l6]", "score[l7]", "score[l8]"};
    static const char *select_names[] = {"", "select[l1]", "select[l2]", "select[l3]", "select[l4]",
                                         "select[l5]", "select[l6]", "select[l7]", "select[l8]"};
    static const char *expand_names[] = {"", "expand[l1]", "expand[l2]", "expand[l3]", "expand[l4]",
                                         "expand[l5]", "expand[l6]", "expand[l7]", "expand[l8]"};
    {
        ProfScope ps("route_init", st);
        route_init_kernel<<<groups, 256, 0, st>>>(g, level_ws(g, ws, g.L), lens, maxkey, status);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    for (int level = g.L; level >= 1; --level) {
        LevelWs lw = level_ws(g, ws, level);
        uint32_t *mk = maxkey + (int64_t)(level - 1) * groups * g.G;
        const char *tb = static_cast<const char *>(tree);
        const int64_t cap = g.cap[level];
        if (g.dtype == ZHA_BF16) {
            ProfScope ps(score_names[level], st);
            const auto *mu = reinterpret_cast<const __nv_bfloat16 *>(tb + g.mu_off[level]);
            const auto *bias = reinterpret_cast<const float *>(tb + g.bias_off[level]);
            const auto *qq = static_cast<const __nv_bfloat16 *>(q);
            const int64_t want = (cap + kScoreWarps - 1) / kScoreWarps;
            const int per_group = (int)max64(1, min64(want, (148 * 8 + groups - 1) / groups));
            dim3 grid(per_group, groups);
            const int mt = g.R > 16 ? 2 : 1, nt = g.G > 8 ? 2 : 1;
#define ZHA_SCORE(D, MT, NT) score_mma_kernel<D, MT, NT><<<grid, kScoreWarps * 32, 0, st>>>(g, mu, bias, qq, lw, level, mk)
            if (g.d == 128) {
                if (mt == 1 && nt == 1) ZHA_SCORE(128, 1, 1);
                else if (mt == 1) ZHA_SCORE(128, 1, 2);
                else if (nt == 1) ZHA_SCORE(128, 2, 1);
                else ZHA_SCORE(128, 2, 2);
            } else {
                if (mt == 1 && nt == 1) ZHA_SCORE(64, 1, 1);
                else if (mt == 1) ZHA_SCORE(64, 1, 2);
                else if (nt == 1) ZHA_SCORE(64, 2, 1);
                else ZHA_SCORE(64, 2, 2);
            }
#undef ZHA_SCORE
        } else {
            ProfScope ps(score_names[level], st);
            const auto *mu = reinterpret_cast<const float *>(tb + g.mu_off[level]);
            const auto *bias = reinterpret_cast<const float *>(tb + g.bias_off[level]);
            const auto *qq = static_cast<const float *>(q);
            const int per_group = (int)max64(1, min64(cap, (148 * 8 + groups - 1) / groups));
            dim3 grid(per_group, groups);
            if (g.d == 128)
                score_f32_kernel<128><<<grid, 128, 0, st>>>(g, mu, bias, qq, lw, level, mk);
            else
                score_f32_kernel<64><<<grid, 128, 0, st>>>(g, mu, bias, qq, lw, level, mk);
        }
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        {
            ProfScope ps(select_names[level], st);
            select_kernel<<<dim3(g.G, groups), kSelThreads, 0, st>>>(g, lw, level, p_levels[level - 1],
                                                                     mk, sel.level_kept);
        }
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        LevelWs nx = level > 1 ? level_ws(g, ws, level - 1) : lw;
        {
            ProfScope ps(expand_names[level], st);
            expand_kernel<<<groups, kExpThreads, 0, st>>>(g, lw, nx, level, lens, sel);
        }
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_topp_select(const float *scores, const int32_t *counts, int n_sets,
                               int64_t stride, float p, uint8_t *kept, int32_t *status,
                               cudaStream_t st) {
    if (n_sets <= 0) return cudaSuccess;
    ProfScope ps("select_sets", st);
    select_sets_kernel<<<n_sets, kSelThreads, 0, st>>>(scores, counts, stride, p, kept, status);
    return cudaGetLastError();
}

}  // namespace zha
