// zha_route.cu -- top-p routing down the summary tree.
//
// Page "Zyphra AI Introduces Zyphra Hierarchical Attention (ZHA)", section
// "How does top-p routing pick tokens": a decode query rates the top level's
// nodes, retains the fewest whose estimated attention mass reaches p of the
// total, rates only their children next, and so on down to raw keys. Section
// "Building the tree": a node's estimate is its largest reference-plane
// value, E = max_r (s q.mu_r + bias_r).
//
// Per level, for all (sequence, KV head) groups at once, two launches (three
// on the largest levels):
//   score  -- candidate i of a group is child i % c of the (i / c)-th node
//             the group kept one level up (all nodes at the top level); each
//             candidate's summary is read once and scored for all G query
//             heads of the group on tensor cores (mma.sync bf16: planes x
//             heads), and the per-head max and min score are kept;
//   select -- exact threshold search for the shortest (score desc, index
//             asc) prefix holding p of the mass, with masses summed in 2^-31
//             fixed point (exact and order-independent): a histogram of the
//             masses over the score's distance below the max finds the bucket
//             where the running mass crosses p, whose members are then
//             ordered exactly (a radix search over the ordered score keys
//             when too many share it). Levels with at most 512 candidate
//             slots per group: one CTA per group, a warp per query row, and
//             the join in the same CTA. Larger levels: one CTA per (group,
//             query head), or several per head on levels with many
//             candidates; each head writes a kept bitmap;
//   join   -- the G bitmaps become per-candidate head masks and the
//             candidates some head kept are compacted into the next level's
//             parent list (or, at level 1, into the selection): by the last
//             of a group's select CTAs to finish, or, on the largest levels,
//             by a launch of its own.
#include "zha_common.cuh"
#include "zha_route_state.cuh"
#include "zha_tc.cuh"

namespace zha {

namespace {

// ------------------------------------------------------------------ level views

struct LevelWs {
    int32_t *cand;      // [groups][capv] node index of candidate i
    uint32_t *cmask;    // [groups][capv] heads that have it as a candidate (0 = padding)
    float *scores;      // [groups][G][capv]
    uint32_t *kept;     // [groups][capv] heads that kept it
    int32_t *count;     // [groups] candidate entries in use
    int32_t *plist;     // [groups][cap] nodes kept by some head, ascending
    uint32_t *pmask;    // [groups][cap] heads that kept them
    int32_t *pcount;    // [groups]
    uint32_t *maxkey;   // [groups][G]
    uint32_t *minkey;   // [groups][G]
    uint32_t *done;     // [groups]
};

inline LevelWs level_ws(const Geo &g, void *ws, int l) {
    char *base = static_cast<char *>(ws);
    const size_t lg = (size_t)(l - 1) * g.groups();
    LevelWs v;
    v.cand = reinterpret_cast<int32_t *>(base + g.ws_cand[l]);
    v.cmask = reinterpret_cast<uint32_t *>(base + g.ws_cmask[l]);
    v.scores = reinterpret_cast<float *>(base + g.ws_scores[l]);
    v.kept = reinterpret_cast<uint32_t *>(base + g.ws_kept[l]);
    v.count = reinterpret_cast<int32_t *>(base + g.ws_count[l]);
    v.plist = reinterpret_cast<int32_t *>(base + g.ws_plist[l]);
    v.pmask = reinterpret_cast<uint32_t *>(base + g.ws_pmask[l]);
    v.pcount = reinterpret_cast<int32_t *>(base + g.ws_pcount[l]);
    v.maxkey = reinterpret_cast<uint32_t *>(base + g.ws_maxkey) + lg * g.G;
    v.minkey = reinterpret_cast<uint32_t *>(base + g.ws_minkey) + lg * g.G;
    v.done = reinterpret_cast<uint32_t *>(base + g.ws_done) + lg;
    return v;
}

__device__ __forceinline__ uint32_t all_heads(int G) { return G >= 32 ? 0xffffffffu : ((1u << G) - 1u); }

// Candidate i of a group at a level: its node and the heads it is a candidate for.
// Loads of workspace data: through the read-only path where the kernel only
// reads it; plain (coherent) loads where other CTAs of the same launch write
// it between cluster barriers.
template <bool NC, typename T>
__device__ __forceinline__ T ld_ws(const T *p) {
    if constexpr (NC)
        return __ldg(p);
    else
        return *p;
}

struct CandSource {
    int lc;                   // log2(c)
    int top;                  // top level: candidate i is node i, for every head
    int n_here;               // nodes at this level
    const int32_t *plist;     // nodes kept one level up
    const uint32_t *pmask;
    template <bool NC = true>
    __device__ __forceinline__ void at(int i, int &node, uint32_t &mask, uint32_t all) const {
        if (top) {
            node = i;
            mask = all;
            return;
        }
        const int j = i >> lc;
        node = (ld_ws<NC>(&plist[j]) << lc) | (i & ((1 << lc) - 1));
        mask = node < n_here ? ld_ws<NC>(&pmask[j]) : 0u;
    }
};

// tokens the tree of group grp holds (a block call routes over the tree before its block)
__device__ __forceinline__ int64_t group_len(const Geo &g, const int32_t *lens, int grp) {
    const int64_t N = (int64_t)lens[grp / g.Hkv] - g.lag;
    return (N < 0 || N > g.max_len) ? 0 : N;
}

// ----------------------------------------------------------------------- init

__global__ void route_init_kernel(Geo g, RouteState rs, const int32_t *lens, int32_t *status) {
    const int grp = blockIdx.x;
    pdl_wait();
    if (threadIdx.x == 0) {
        const int64_t N = (int64_t)lens[grp / g.Hkv] - g.lag;
        if (N < 0 || N > g.max_len) set_status(status, ZHA_ERR_CAPACITY);
    }
    route_reset_group(g, rs, grp);
    pdl_trigger();
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

__device__ __forceinline__ CandSource cand_source(const Geo &g, const LevelWs &up, int level,
                                                  int grp, int64_t N) {
    const int64_t cap_up = level < g.L ? g.cap[level + 1] : 0;
    return CandSource{__ffs(g.c) - 1, level == g.L, (int)level_nodes(N, g.c, level),
                      up.plist + grp * cap_up, up.pmask + grp * cap_up};
}

__device__ __forceinline__ int64_t cand_count(const Geo &g, const LevelWs &up, int level, int grp,
                                              int64_t n_here) {
    return level == g.L ? n_here : (int64_t)up.pcount[grp] * g.c;
}

// bf16 scoring on tensor cores. One warp scores one candidate per iteration:
// A = the node's planes (16 rows per m-tile, K = head_dim), B = the group's
// query heads (8 columns per n-tile). Coordinates are permuted identically in
// A and B so that each lane fetches 16 contiguous bytes per row and k-pair
// (fully used 32-byte sectors); a dot product is invariant to that.
template <int D, int MT, int NT>
__global__ void __launch_bounds__(kScoreWarps * 32)
score_mma_kernel(Geo g, const __nv_bfloat16 *mu, const float *bias, const __nv_bfloat16 *q,
                 const int32_t *lens, LevelWs lw, LevelWs up, int level) {
    constexpr int KP = D / 32;
    const int grp = blockIdx.y;
    const int b = grp / g.Hkv, kvh = grp % g.Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gq = lane >> 2, t = lane & 3;
    const int64_t cap = g.cap[level], capv = g.capv[level];

    // B fragments (query rows): in registers, or -- with 4 n-tiles, where
    // registers run out -- in shared memory, one 16-byte fragment per lane
    constexpr bool QS = NT >= 4;
    __shared__ uint4 qsm[QS ? NT * KP * 32 : 1];
    uint32_t bq[QS ? 1 : NT][KP][4];
    if constexpr (QS) {
        for (int i = threadIdx.x; i < NT * KP * 32; i += blockDim.x) {
            const int ln = i & 31, kp = (i >> 5) % KP, nt = (i >> 5) / KP;
            const int h = nt * 8 + (ln >> 2);
            uint4 w = make_uint4(0, 0, 0, 0);
            if (h < g.G) w = ldg16(q + g.qrow(b, kvh, h) * D + kp * 32 + (ln & 3) * 8);
            qsm[i] = w;
        }
        __syncthreads();
    } else {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int h = nt * 8 + gq;
#pragma unroll
            for (int kp = 0; kp < KP; ++kp) {
                uint4 w = make_uint4(0, 0, 0, 0);
                if (h < g.G) w = ldg16(q + g.qrow(b, kvh, h) * D + kp * 32 + t * 8);
                bq[nt][kp][0] = w.x; bq[nt][kp][1] = w.y; bq[nt][kp][2] = w.z; bq[nt][kp][3] = w.w;
            }
        }
    }
    // the queries are the call's input; everything below depends on earlier kernels
    pdl_wait();
    const CandSource src = cand_source(g, up, level, grp, group_len(g, lens, grp));
    const int n = (int)cand_count(g, up, level, grp, src.n_here);
    if (blockIdx.x == 0 && threadIdx.x == 0) lw.count[grp] = n;
    const uint32_t all = all_heads(g.G);
    float runmax[NT][2], runmin[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        runmax[nt][0] = runmax[nt][1] = -INFINITY;
        runmin[nt][0] = runmin[nt][1] = INFINITY;
    }

    const float s = g.s;
    // U candidates per warp and iteration, their loads issued together
    constexpr int U = QS ? 1 : 2;
    const int stride = gridDim.x * kScoreWarps * U;
    // a warp's candidates are looked up an iteration ahead, while the
    // previous ones' summaries load: one round trip per iteration, not two
    int nnode[U];
    uint32_t nhm[U];
    auto lookup = [&](int j0) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            nnode[u] = 0;
            nhm[u] = 0u;
            if (j0 + u < n) src.at(j0 + u, nnode[u], nhm[u], all);
        }
    };
    lookup((blockIdx.x * kScoreWarps + warp) * U);
    for (int i0 = (blockIdx.x * kScoreWarps + warp) * U; i0 < n; i0 += stride) {
        int node[U];
        uint32_t hm[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u;
            node[u] = nnode[u];
            hm[u] = nhm[u];
            if (i < n && lane == 0) {
                lw.cand[grp * capv + i] = node[u];
                lw.cmask[grp * capv + i] = hm[u];
            }
        }
        uint4 ra[U][MT][KP], rb[U][MT][KP];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const __nv_bfloat16 *base = mu + (grp * cap + node[u]) * (int64_t)g.R * D;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const int r0 = mt * 16 + gq, r1 = r0 + 8;
#pragma unroll
                for (int kp = 0; kp < KP; ++kp) {
                    ra[u][mt][kp] = (hm[u] && r0 < g.R) ? ldg16(base + (int64_t)r0 * D + kp * 32 + t * 8)
                                                        : make_uint4(0, 0, 0, 0);
                    rb[u][mt][kp] = (hm[u] && r1 < g.R) ? ldg16(base + (int64_t)r1 * D + kp * 32 + t * 8)
                                                        : make_uint4(0, 0, 0, 0);
                }
            }
        }
        lookup(i0 + stride);
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u;
            if (i >= n) break;
            if (hm[u] == 0u) {
                if (lane < g.G) lw.scores[(grp * g.G + lane) * capv + i] = -INFINITY;
                continue;
            }
            const float *bb = bias + (grp * cap + node[u]) * (int64_t)g.R;
            float e[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) e[nt][0] = e[nt][1] = -INFINITY;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                // two accumulation chains (first and second k16 half of each
                // 32-wide k step), added at the end: half the dependent depth
                float acc[NT][4], acc2[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int v = 0; v < 4; ++v) acc[nt][v] = acc2[nt][v] = 0.f;
#pragma unroll
                for (int kp = 0; kp < KP; ++kp) {
                    const uint4 &xa = ra[u][mt][kp], &xb = rb[u][mt][kp];
                    const uint32_t a0[4] = {xa.x, xb.x, xa.y, xb.y};
                    const uint32_t a1[4] = {xa.z, xb.z, xa.w, xb.w};
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        if constexpr (QS) {
                            const uint4 f = qsm[(nt * KP + kp) * 32 + lane];
                            mma_bf16_16816(acc[nt], a0, f.x, f.y);
                            mma_bf16_16816(acc2[nt], a1, f.z, f.w);
                        } else {
                            mma_bf16_16816(acc[nt], a0, bq[nt][kp][0], bq[nt][kp][1]);
                            mma_bf16_16816(acc2[nt], a1, bq[nt][kp][2], bq[nt][kp][3]);
                        }
                    }
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int v = 0; v < 4; ++v) acc[nt][v] += acc2[nt][v];
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
                            lw.scores[(grp * g.G + h) * capv + i] = e[nt][j];
                            if ((hm[u] >> h) & 1u) {
                                runmax[nt][j] = fmaxf(runmax[nt][j], e[nt][j]);
                                runmin[nt][j] = fminf(runmin[nt][j], e[nt][j]);
                            }
                        }
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
                if (h < g.G && runmax[nt][j] > -INFINITY) {
                    atomicMax(&lw.maxkey[(int64_t)grp * g.G + h], ordered_key(runmax[nt][j]));
                    atomicMin(&lw.minkey[(int64_t)grp * g.G + h], ordered_key(runmin[nt][j]));
                }
            }
    }
    pdl_trigger();
}

// bf16 scoring for R = 2^RL < 16 planes per node: the 16 rows of an MMA tile
// are (candidate, plane) pairs, 16/R candidates per tile, so no row is idle.
// Lane (gq, t) holds rows gq and gq + 8, i.e. planes of candidates gq >> RL
// and (gq + 8) >> RL; a candidate's estimate is the max over its R rows,
// reduced across the lanes that share it. Same coordinate permutation and
// outputs as score_mma_kernel.
template <int D, int NT, int RL, int U>
__global__ void __launch_bounds__(kScoreWarps * 32)
score_pack_kernel(Geo g, const __nv_bfloat16 *mu, const float *bias, const __nv_bfloat16 *q,
                  const int32_t *lens, LevelWs lw, LevelWs up, int level) {
    constexpr int KP = D / 32;
    constexpr int R = 1 << RL;
    constexpr int CPT = 16 / R;          // candidates per tile
    const int grp = blockIdx.y;
    const int b = grp / g.Hkv, kvh = grp % g.Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gq = lane >> 2, t = lane & 3;
    const int64_t cap = g.cap[level], capv = g.capv[level];

    uint32_t bq[NT][KP][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int h = nt * 8 + gq;
#pragma unroll
        for (int kp = 0; kp < KP; ++kp) {
            uint4 w = make_uint4(0, 0, 0, 0);
            if (h < g.G) w = ldg16(q + g.qrow(b, kvh, h) * D + kp * 32 + t * 8);
            bq[nt][kp][0] = w.x; bq[nt][kp][1] = w.y; bq[nt][kp][2] = w.z; bq[nt][kp][3] = w.w;
        }
    }
    pdl_wait();
    const CandSource src = cand_source(g, up, level, grp, group_len(g, lens, grp));
    const int n = (int)cand_count(g, up, level, grp, src.n_here);
    if (blockIdx.x == 0 && threadIdx.x == 0) lw.count[grp] = n;
    const uint32_t all = all_heads(g.G);
    float runmax[NT][2], runmin[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        runmax[nt][0] = runmax[nt][1] = -INFINITY;
        runmin[nt][0] = runmin[nt][1] = INFINITY;
    }
    const float s = g.s;
    const int pa = gq & (R - 1), pb = (gq + 8) & (R - 1);   // planes of rows gq, gq + 8
    const int ca = gq >> RL, cb = (gq + 8) >> RL;           // their candidates in the tile
    const int stride = gridDim.x * kScoreWarps * U * CPT;
    for (int i0 = (blockIdx.x * kScoreWarps + warp) * U * CPT; i0 < n; i0 += stride) {
        int na[U], nb[U];
        uint32_t ma[U], mb[U];
        uint4 ra[U][KP], rb[U][KP];
        float ba[U], bb[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int ia = i0 + u * CPT + ca, ib = i0 + u * CPT + cb;
            na[u] = nb[u] = 0;
            ma[u] = mb[u] = 0u;
            if (ia < n) src.at(ia, na[u], ma[u], all);
            if (ib < n) src.at(ib, nb[u], mb[u], all);
            const __nv_bfloat16 *rowa = mu + ((grp * cap + na[u]) * (int64_t)R + pa) * D;
            const __nv_bfloat16 *rowb = mu + ((grp * cap + nb[u]) * (int64_t)R + pb) * D;
#pragma unroll
            for (int kp = 0; kp < KP; ++kp) {
                ra[u][kp] = ma[u] ? ldg16(rowa + kp * 32 + t * 8) : make_uint4(0, 0, 0, 0);
                rb[u][kp] = mb[u] ? ldg16(rowb + kp * 32 + t * 8) : make_uint4(0, 0, 0, 0);
            }
            ba[u] = ma[u] ? __ldg(bias + (grp * cap + na[u]) * (int64_t)R + pa) : -INFINITY;
            bb[u] = mb[u] ? __ldg(bias + (grp * cap + nb[u]) * (int64_t)R + pb) : -INFINITY;
            // candidate bookkeeping: one lane per candidate of the tile
            if (t == 0 && pa == 0 && ia < n) {
                lw.cand[grp * capv + ia] = na[u];
                lw.cmask[grp * capv + ia] = ma[u];
            }
            if (t == 0 && pb == 0 && ib < n) {
                lw.cand[grp * capv + ib] = nb[u];
                lw.cmask[grp * capv + ib] = mb[u];
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (i0 + u * CPT >= n) break;
            float acc[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
            for (int kp = 0; kp < KP; ++kp) {
                const uint4 &xa = ra[u][kp], &xb = rb[u][kp];
                const uint32_t a0[4] = {xa.x, xb.x, xa.y, xb.y};
                const uint32_t a1[4] = {xa.z, xb.z, xa.w, xb.w};
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    mma_bf16_16816(acc[nt], a0, bq[nt][kp][0], bq[nt][kp][1]);
                    mma_bf16_16816(acc[nt], a1, bq[nt][kp][2], bq[nt][kp][3]);
                }
            }
            float ea[NT][2], eb[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    float va = fmaf(s, acc[nt][j], ba[u]);
                    float vb = fmaf(s, acc[nt][2 + j], bb[u]);
#pragma unroll
                    for (int o = 4; o < 4 * R; o <<= 1) {       // max over the candidate's R rows
                        va = fmaxf(va, __shfl_xor_sync(0xffffffffu, va, o));
                        vb = fmaxf(vb, __shfl_xor_sync(0xffffffffu, vb, o));
                    }
                    ea[nt][j] = va;
                    eb[nt][j] = vb;
                }
            if (pa == 0) {   // pb == 0 as well: 8 is a multiple of R
                const int ia = i0 + u * CPT + ca, ib = i0 + u * CPT + cb;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int h = nt * 8 + 2 * t + j;
                        if (h >= g.G) continue;
                        if (ia < n) {
                            const float e = ma[u] ? ea[nt][j] : -INFINITY;
                            lw.scores[(grp * g.G + h) * capv + ia] = e;
                            if ((ma[u] >> h) & 1u) {
                                runmax[nt][j] = fmaxf(runmax[nt][j], e);
                                runmin[nt][j] = fminf(runmin[nt][j], e);
                            }
                        }
                        if (ib < n) {
                            const float e = mb[u] ? eb[nt][j] : -INFINITY;
                            lw.scores[(grp * g.G + h) * capv + ib] = e;
                            if ((mb[u] >> h) & 1u) {
                                runmax[nt][j] = fmaxf(runmax[nt][j], e);
                                runmin[nt][j] = fminf(runmin[nt][j], e);
                            }
                        }
                    }
            }
        }
    }
    // per-head max/min over the lanes that saw each head (columns 2t, 2t + 1)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            float mx = runmax[nt][j], mn = runmin[nt][j];
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            }
            const int h = nt * 8 + 2 * t + j;
            if (gq == 0 && h < g.G && mx > -INFINITY) {
                atomicMax(&lw.maxkey[(int64_t)grp * g.G + h], ordered_key(mx));
                atomicMin(&lw.minkey[(int64_t)grp * g.G + h], ordered_key(mn));
            }
        }
    pdl_trigger();
}

__device__ __forceinline__ void mma_e4m3_16832(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t e4m3_rn(float x) {
    return (uint32_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ float e4m3_value(uint32_t byte) {
    return __half2float(__half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)byte, __NV_E4M3)));
}

// Scoring against MX-FP8 summaries (E4M3 bytes, one power-of-two scale per 32
// coordinates of a plane) with warp-level E4M3 MMAs: mma.sync m16n8k32
// (A = planes, B = query heads, one MMA per 32-coordinate block and query
// term; the stored rows are permuted so that one 16-byte load brings a lane's
// bytes of two blocks). On sm_100a this warp-level FP8 form is not a native
// tensor-core instruction: the compiler expands each into conversions and
// fp16 MMAs (ncu per-opcode counts per candidate: 66 F2FP, 33 FADD, 16 HMMA),
// which makes this kernel instruction-bound at about half the HBM bandwidth;
// native FP8 (and hardware block scaling) is tcgen05's kind::mxf8f6f4.
// Each query head is held as two
// E4M3 terms with one power-of-two scale per head: q ~ 2^e (hi + lo), hi the
// nearest E4M3 of q / 2^e (e the smallest with max|q| <= 448 * 2^e), lo that
// of the remainder -- about 8 significant bits, the precision of bf16.
// Each lane reads 8 contiguous bytes of a row per block, so an MMA sees one
// plane scale per row; the block's two MMAs (hi, then lo into the same
// accumulator) are scaled into the plane sums, and the head scale is applied
// once at the end.
template <int D, int MT, int NT, int U>
__global__ void __launch_bounds__(kScoreWarps * 32)
score_mx8_kernel(Geo g, const uint8_t *mu, const uint8_t *scl, const float *bias, const __nv_bfloat16 *q,
                 const int32_t *lens, LevelWs lw, LevelWs up, int level) {
    constexpr int KP = D / 32;          // blocks per plane
    const int grp = blockIdx.y;
    const int b = grp / g.Hkv, kvh = grp % g.Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gq = lane >> 2, t = lane & 3;
    const int64_t cap = g.cap[level], capv = g.capv[level];

    // B fragments: head nt*8 + gq, block kp, bytes [32 kp + 8 t, +8) as two words,
    // for the hi and lo terms; hscale[nt][j]: 2^e of the head in C column 2t + j
    uint32_t bhi[NT][KP][2], blo[NT][KP][2];
    float hscale[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int h = nt * 8 + gq;
        float v[KP][8];
        float amax = 0.f;
#pragma unroll
        for (int kp = 0; kp < KP; ++kp) {
            // coordinates 32 kp + 4 t + (0..3) and 32 kp + 16 + 4 t + (0..3): the
            // k-slots of this lane in an m16n8k32 fragment
            uint2 lo = make_uint2(0, 0), hi = make_uint2(0, 0);
            if (h < g.G) {
                const __nv_bfloat16 *qh = q + g.qrow(b, kvh, h) * D + kp * 32 + t * 4;
                lo = __ldg(reinterpret_cast<const uint2 *>(qh));
                hi = __ldg(reinterpret_cast<const uint2 *>(qh + 16));
            }
            const uint32_t in[4] = {lo.x, lo.y, hi.x, hi.y};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&in[j]));
                v[kp][2 * j] = f.x;
                v[kp][2 * j + 1] = f.y;
                amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
            }
        }
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        int ex = 0;
        if (amax > 0.f) {
            int k;
            const float f = frexpf(amax, &k);          // amax = f 2^k, 448 = 0.875 2^9
            ex = (f <= 0.875f) ? k - 9 : k - 8;
        }
#pragma unroll
        for (int kp = 0; kp < KP; ++kp)
#pragma unroll
            for (int w2 = 0; w2 < 2; ++w2) {
                uint32_t hi = 0u, lo = 0u;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float x = scalbnf(v[kp][4 * w2 + e], -ex);
                    const uint32_t bh = e4m3_rn(x);
                    const uint32_t bl = e4m3_rn(x - e4m3_value(bh));
                    hi |= bh << (8 * e);
                    lo |= bl << (8 * e);
                }
                bhi[nt][kp][w2] = hi;
                blo[nt][kp][w2] = lo;
            }
        const float myscale = scalbnf(1.f, ex);
        hscale[nt][0] = __shfl_sync(0xffffffffu, myscale, (2 * t) * 4);
        hscale[nt][1] = __shfl_sync(0xffffffffu, myscale, (2 * t + 1) * 4);
    }
    pdl_wait();
    const CandSource src = cand_source(g, up, level, grp, group_len(g, lens, grp));
    const int n = (int)cand_count(g, up, level, grp, src.n_here);
    if (blockIdx.x == 0 && threadIdx.x == 0) lw.count[grp] = n;
    const uint32_t all = all_heads(g.G);
    float runmax[NT][2], runmin[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        runmax[nt][0] = runmax[nt][1] = -INFINITY;
        runmin[nt][0] = runmin[nt][1] = INFINITY;
    }

    const float s = g.s;
    const int stride = gridDim.x * kScoreWarps * U;
    // a warp's candidates are looked up an iteration ahead, while the
    // previous ones' summaries load: one round trip per iteration, not two
    int nnode[U];
    uint32_t nhm[U];
    auto lookup = [&](int j0) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            nnode[u] = 0;
            nhm[u] = 0u;
            if (j0 + u < n) src.at(j0 + u, nnode[u], nhm[u], all);
        }
    };
    lookup((blockIdx.x * kScoreWarps + warp) * U);
    for (int i0 = (blockIdx.x * kScoreWarps + warp) * U; i0 < n; i0 += stride) {
        int node[U];
        uint32_t hm[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u;
            node[u] = nnode[u];
            hm[u] = nhm[u];
            if (i < n && lane == 0) {
                lw.cand[grp * capv + i] = node[u];
                lw.cmask[grp * capv + i] = hm[u];
            }
        }
        // all loads of the U candidates first: E4M3 rows (one 16-byte load covers
        // this lane's bytes of two blocks), block scales, biases
        uint4 ra[U][MT][KP / 2], rb[U][MT][KP / 2];
        uint32_t sa[U][MT], sb[U][MT];
        float ba[U][MT], bb[U][MT];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t rec = (grp * cap + node[u]) * (int64_t)g.R;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const int r0 = mt * 16 + gq, r1 = r0 + 8;
                const bool v0 = hm[u] && r0 < g.R, v1 = hm[u] && r1 < g.R;
#pragma unroll
                for (int pp = 0; pp < KP / 2; ++pp) {
                    ra[u][mt][pp] = v0 ? ldg16(mu + (rec + r0) * D + pp * 64 + t * 16) : make_uint4(0, 0, 0, 0);
                    rb[u][mt][pp] = v1 ? ldg16(mu + (rec + r1) * D + pp * 64 + t * 16) : make_uint4(0, 0, 0, 0);
                }
                if constexpr (KP == 4) {
                    sa[u][mt] = v0 ? __ldg(reinterpret_cast<const uint32_t *>(scl + (rec + r0) * KP)) : 0u;
                    sb[u][mt] = v1 ? __ldg(reinterpret_cast<const uint32_t *>(scl + (rec + r1) * KP)) : 0u;
                } else {
                    sa[u][mt] = v0 ? __ldg(reinterpret_cast<const uint16_t *>(scl + (rec + r0) * KP)) : 0u;
                    sb[u][mt] = v1 ? __ldg(reinterpret_cast<const uint16_t *>(scl + (rec + r1) * KP)) : 0u;
                }
                ba[u][mt] = v0 ? __ldg(bias + rec + r0) : -INFINITY;
                bb[u][mt] = v1 ? __ldg(bias + rec + r1) : -INFINITY;
            }
        }
        lookup(i0 + stride);
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u;
            if (i >= n) break;
            if (hm[u] == 0u) {
                if (lane < g.G) lw.scores[(grp * g.G + lane) * capv + i] = -INFINITY;
                continue;
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
                    const uint4 &pa = ra[u][mt][kp >> 1], &pb = rb[u][mt][kp >> 1];
                    const uint2 xa = (kp & 1) ? make_uint2(pa.z, pa.w) : make_uint2(pa.x, pa.y);
                    const uint2 xb = (kp & 1) ? make_uint2(pb.z, pb.w) : make_uint2(pb.x, pb.y);
                    // 2^(byte - 127) of this block for rows r0 and r1
                    const float s0 = __uint_as_float(__byte_perm(sa[u][mt], 0u, 0x4440u + kp) << 23);
                    const float s1 = __uint_as_float(__byte_perm(sb[u][mt], 0u, 0x4440u + kp) << 23);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        float tq[4] = {0.f, 0.f, 0.f, 0.f};
                        mma_e4m3_16832(tq, xa.x, xb.x, xa.y, xb.y, bhi[nt][kp][0], bhi[nt][kp][1]);
                        mma_e4m3_16832(tq, xa.x, xb.x, xa.y, xb.y, blo[nt][kp][0], blo[nt][kp][1]);
                        acc[nt][0] = fmaf(s0, tq[0], acc[nt][0]);
                        acc[nt][1] = fmaf(s0, tq[1], acc[nt][1]);
                        acc[nt][2] = fmaf(s1, tq[2], acc[nt][2]);
                        acc[nt][3] = fmaf(s1, tq[3], acc[nt][3]);
                    }
                }
                const float b0 = ba[u][mt], b1 = bb[u][mt];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const float c0 = s * hscale[nt][0], c1 = s * hscale[nt][1];
                    e[nt][0] = fmaxf(e[nt][0], fmaxf(fmaf(c0, acc[nt][0], b0), fmaf(c0, acc[nt][2], b1)));
                    e[nt][1] = fmaxf(e[nt][1], fmaxf(fmaf(c1, acc[nt][1], b0), fmaf(c1, acc[nt][3], b1)));
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
                            lw.scores[(grp * g.G + h) * capv + i] = e[nt][j];
                            if ((hm[u] >> h) & 1u) {
                                runmax[nt][j] = fmaxf(runmax[nt][j], e[nt][j]);
                                runmin[nt][j] = fminf(runmin[nt][j], e[nt][j]);
                            }
                        }
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
                if (h < g.G && runmax[nt][j] > -INFINITY) {
                    atomicMax(&lw.maxkey[(int64_t)grp * g.G + h], ordered_key(runmax[nt][j]));
                    atomicMin(&lw.minkey[(int64_t)grp * g.G + h], ordered_key(runmin[nt][j]));
                }
            }
    }
    pdl_trigger();
}

// fp32 scoring on CUDA cores: one block per candidate per iteration, one
// thread per (plane, head) dot product.
template <int D>
__global__ void score_f32_kernel(Geo g, const float *mu, const float *bias, const float *q,
                                 const int32_t *lens, LevelWs lw, LevelWs up, int level) {
    __shared__ float qs[32][D];
    __shared__ float es[32][32];
    const int grp = blockIdx.y;
    const int b = grp / g.Hkv, kvh = grp % g.Hkv;
    const int64_t cap = g.cap[level], capv = g.capv[level];
    for (int i = threadIdx.x; i < g.G * D; i += blockDim.x)
        qs[i / D][i % D] = q[g.qrow(b, kvh, i / D) * D + i % D];
    pdl_wait();
    const CandSource src = cand_source(g, up, level, grp, group_len(g, lens, grp));
    const int n = (int)cand_count(g, up, level, grp, src.n_here);
    if (blockIdx.x == 0 && threadIdx.x == 0) lw.count[grp] = n;
    const uint32_t all = all_heads(g.G);
    float runmax = -INFINITY, runmin = INFINITY;
    __syncthreads();
    for (int i = blockIdx.x; i < n; i += gridDim.x) {
        int node;
        uint32_t hm;
        src.at(i, node, hm, all);
        if (threadIdx.x == 0) {
            lw.cand[grp * capv + i] = (int32_t)node;
            lw.cmask[grp * capv + i] = hm;
        }
        if (hm == 0u) {
            if (threadIdx.x < g.G) lw.scores[(grp * g.G + threadIdx.x) * capv + i] = -INFINITY;
            continue;  // uniform across the block
        }
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
            lw.scores[(grp * g.G + h) * capv + i] = e;
            if ((hm >> h) & 1u) {
                runmax = fmaxf(runmax, e);
                runmin = fminf(runmin, e);
            }
        }
        __syncthreads();
    }
    if (threadIdx.x < g.G && runmax > -INFINITY) {
        atomicMax(&lw.maxkey[(int64_t)grp * g.G + threadIdx.x], ordered_key(runmax));
        atomicMin(&lw.minkey[(int64_t)grp * g.G + threadIdx.x], ordered_key(runmin));
    }
    pdl_trigger();
}

// --------------------------------------------------------------------- select

constexpr int kSelThreads = 1024;
constexpr int kDigitBits = 12;
constexpr int kBuckets = 1 << kDigitBits;
constexpr int kMaxTies = kSelList;
static_assert(kBuckets == kSelBuckets, "select histogram size");
// masses e^{E - max} in (0, 1] are summed exactly as integers in units of
// 2^-31 (per-candidate rounding error <= 2^-32)
constexpr float kMassScale = 2147483648.0f;

__device__ __forceinline__ uint32_t fixed_mass(float e, float m) {
    return __float2uint_rn(expf(e - m) * kMassScale);
}

// 64-bit histogram bucket from native 32-bit shared atomics: the low word
// accumulates, and the one addition that wraps it bumps the carry word.
__device__ __forceinline__ void hist_add(uint32_t *lo, uint32_t *carry, int b, uint32_t w) {
    const uint32_t old = atomicAdd(&lo[b], w);
    if (old > 0xffffffffu - w) atomicAdd(&carry[b], 1u);
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

// masses below e^-23 of the maximum round to 0 in 2^-31 fixed point
constexpr float kMassRange = 23.f;

struct SelShared {
    uint32_t hist_lo[kBuckets];
    uint32_t hist_hi[kBuckets];
    unsigned long long red[kSelThreads / 32];
    int32_t ties[kMaxTies];
    int32_t sorted_ties[kMaxTies];
    uint32_t tkey[kMaxTies];
    unsigned long long above, target;
    uint32_t digit, kmax, kmin;
    int ntie;
    int last;
};

// Exact top-p over the members of one candidate set, visited in blocks of 8
// consecutive candidates (two blocks in flight per thread):
//   load8(blk, e)    -- fills e[0..8) with the scores of candidates 8 blk ..
//                       8 blk + 7 and returns the bit mask of those that are
//                       members (and < n)
//   store8(blk, m)   -- records the kept bits m of block blk (called once for
//                       every block)
//   add_kept(i)      -- marks one more candidate kept (thread 0 only, after
//                       every store8)
// kmax_in / kmin_in: ordered keys of the members' max / min score (kmax_in = 0:
// unknown, found here). Returns (in every thread) the number kept.
template <class Load8, class Store8, class AddKept>
__device__ int topp_core(SelShared &sh, int64_t n, float p, uint32_t kmax_in, uint32_t kmin_in,
                         Load8 load8, Store8 store8, AddKept add_kept) {
    const int tid = threadIdx.x;
    const int64_t nblk = (n + 7) >> 3;
    const int64_t step = blockDim.x;
    if (tid == 0) {
        sh.kmax = kmax_in;
        sh.kmin = kmax_in ? kmin_in : 0xffffffffu;
    }
    __syncthreads();
    if (kmax_in == 0u) {
        uint32_t mx = 0u, mn = 0xffffffffu;
        for (int64_t blk = tid; blk < nblk; blk += step) {
            float e[8];
            const uint32_t mb = load8(blk, e);
#pragma unroll
            for (int v = 0; v < 8; ++v)
                if ((mb >> v) & 1u) {
                    const uint32_t k = ordered_key(e[v]);
                    mx = max(mx, k);
                    mn = min(mn, k);
                }
        }
        if (mx) {
            atomicMax(&sh.kmax, mx);
            atomicMin(&sh.kmin, mn);
        }
        __syncthreads();
    }
    const uint32_t kmax = sh.kmax, kmin = sh.kmin;
    int kept = 0;
    if (kmax == 0u || p >= 1.f) {  // no member, or keep every member (uniform)
        for (int64_t blk = tid; blk < nblk; blk += step) {
            float e[8];
            const uint32_t mb = kmax ? load8(blk, e) : 0u;
            store8(blk, mb);
            kept += __popc(mb);
        }
        return (int)block_sum<unsigned long long>((unsigned long long)kept, sh.red);
    }
    const float m = key_to_float(kmax);
    // Common case, two passes: a histogram of the masses over the score's
    // distance below the max, in nvb equal steps of at most kMassRange
    // nats (monotone in the score, so the buckets are contiguous in the
    // (score desc) order), finds the bucket where the running mass crosses
    // p; the members of that bucket are then ordered exactly by (score desc,
    // index asc) in shared memory. If that bucket holds more than kMaxTies
    // members (near-equal scores), the radix search below decides instead.
    {
        const float span = m - key_to_float(kmin);
        // buckets: about one per candidate (a power of two), at least one per thread, at most kBuckets
        int nvb = (int)blockDim.x;
        while (nvb < kBuckets && nvb < n) nvb <<= 1;
        const float W = (float)nvb / fminf(span, kMassRange);
        if (kmax != kmin && W < 1e30f) {
            auto bucket = [&](float e) -> int {
                const float x = (m - e) * W;
                return x < (float)(nvb - 1) ? (int)x : nvb - 1;
            };
            for (int i = tid; i < nvb; i += blockDim.x) sh.hist_lo[i] = sh.hist_hi[i] = 0u;
            if (tid == 0) {
                sh.above = 0ull;
                sh.ntie = 0;
            }
            __syncthreads();
            auto add_block = [&](uint32_t mb, const float (&e)[8]) {
#pragma unroll
                for (int v = 0; v < 8; ++v)
                    if ((mb >> v) & 1u) hist_add(sh.hist_lo, sh.hist_hi, bucket(e[v]), fixed_mass(e[v], m));
            };
            for (int64_t blk = tid; blk < nblk; blk += 2 * step) {
                float e0[8], e1[8];
                const uint32_t m0 = load8(blk, e0);
                const uint32_t m1 = blk + step < nblk ? load8(blk + step, e1) : 0u;
                add_block(m0, e0);
                add_block(m1, e1);
            }
            __syncthreads();
            const int per = nvb / (int)blockDim.x;
            unsigned long long mine = 0ull;
            for (int j = 0; j < per; ++j)
                mine += ((unsigned long long)sh.hist_hi[tid * per + j] << 32) | sh.hist_lo[tid * per + j];
            unsigned long long z;
            const unsigned long long excl = block_exclusive_scan<unsigned long long>(mine, sh.red, &z);
            const unsigned long long target = (unsigned long long)ceil((double)p * (double)z);
            unsigned long long run = excl;
            for (int j = 0; j < per; ++j) {
                const int bk = tid * per + j;
                const unsigned long long hgt = ((unsigned long long)sh.hist_hi[bk] << 32) | sh.hist_lo[bk];
                if (hgt && run < target && run + hgt >= target) {
                    sh.digit = (uint32_t)bk;
                    sh.above = run;
                }
                run += hgt;
            }
            __syncthreads();
            const int bstar = (int)sh.digit;
            const unsigned long long above = sh.above;
            for (int64_t blk = tid; blk < nblk; blk += step) {
                float e[8];
                const uint32_t mb = load8(blk, e);
                uint32_t kb = 0u;
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    if (!((mb >> v) & 1u)) continue;
                    const int bk = bucket(e[v]);
                    if (bk < bstar) {
                        kb |= 1u << v;
                    } else if (bk == bstar) {
                        const int slot = atomicAdd(&sh.ntie, 1);
                        if (slot < kMaxTies) {
                            sh.ties[slot] = (int32_t)((blk << 3) + v);
                            sh.tkey[slot] = ordered_key(e[v]);
                        }
                    }
                }
                store8(blk, kb);
                kept += __popc(kb);
            }
            __syncthreads();
            const int nl = sh.ntie;
            if (nl <= kMaxTies) {
                for (int j = tid; j < nl; j += blockDim.x) {
                    const uint32_t kj = sh.tkey[j];
                    const int32_t ij = sh.ties[j];
                    int rank = 0;
                    for (int w = 0; w < nl; ++w) {
                        const uint32_t kw = sh.tkey[w];
                        rank += (kw > kj) || (kw == kj && sh.ties[w] < ij);
                    }
                    sh.sorted_ties[rank] = j;
                }
                __syncthreads();
                if (tid == 0) {
                    unsigned long long cum = above;
                    for (int r = 0; r < nl && cum < target; ++r) {
                        const int j = sh.sorted_ties[r];
                        add_kept(sh.ties[j]);
                        ++kept;
                        cum += fixed_mass(key_to_float(sh.tkey[j]), m);
                    }
                }
                return (int)block_sum<unsigned long long>((unsigned long long)kept, sh.red);
            }
            kept = 0;   // too many near-equal scores: the radix search rewrites every block
            __syncthreads();
        }
    }
    // u = kmax - key: 0 for the best candidate, growing as the score falls.
    const uint32_t span = kmax - kmin;
    int hi = span ? 32 - __clz(span) : 0;  // bits of u that can be non-zero
    uint32_t prefix = 0u;                   // known bits of the crossing u (bits >= hi)
    if (tid == 0) sh.above = 0ull;
    bool first = true;
    do {
        const int bits = hi < kDigitBits ? hi : kDigitBits;
        const int shift = hi - bits;
        for (int i = tid; i < kBuckets; i += blockDim.x) sh.hist_lo[i] = sh.hist_hi[i] = 0u;
        __syncthreads();
        auto add_block = [&](uint32_t mb, const float (&e)[8]) {
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                if (!((mb >> v) & 1u)) continue;
                const uint32_t u = kmax - ordered_key(e[v]);
                if (hi < 32 && (u >> hi) != (prefix >> hi)) continue;
                hist_add(sh.hist_lo, sh.hist_hi, (int)((u >> shift) & ((1u << bits) - 1u)),
                         fixed_mass(e[v], m));
            }
        };
        for (int64_t blk = tid; blk < nblk; blk += 2 * step) {
            float e0[8], e1[8];
            const uint32_t m0 = load8(blk, e0);
            const uint32_t m1 = blk + step < nblk ? load8(blk + step, e1) : 0u;
            add_block(m0, e0);
            add_block(m1, e1);
        }
        __syncthreads();
        if (first) {
            unsigned long long z = 0ull;
            for (int i = tid; i < kBuckets; i += blockDim.x)
                z += ((unsigned long long)sh.hist_hi[i] << 32) | sh.hist_lo[i];
            z = block_sum<unsigned long long>(z, sh.red);
            if (tid == 0) sh.target = (unsigned long long)ceil((double)p * (double)z);
            __syncthreads();
            first = false;
        }
        // crossing digit: running mass from digit 0 (best) upward first reaches target
        const int per = kBuckets / (int)blockDim.x;
        unsigned long long mine = 0ull;
        for (int j = 0; j < per; ++j)
            mine += ((unsigned long long)sh.hist_hi[tid * per + j] << 32) | sh.hist_lo[tid * per + j];
        unsigned long long tot;
        const unsigned long long excl = block_exclusive_scan<unsigned long long>(mine, sh.red, &tot);
        unsigned long long run = sh.above + excl;
        const unsigned long long target = sh.target;
        __syncthreads();
        for (int j = 0; j < per; ++j) {
            const int dgt = tid * per + j;
            const unsigned long long hgt = ((unsigned long long)sh.hist_hi[dgt] << 32) | sh.hist_lo[dgt];
            if (hgt && run < target && run + hgt >= target) {
                sh.digit = (uint32_t)dgt;
                sh.above = run;  // mass of the candidates with smaller u
            }
            run += hgt;
        }
        __syncthreads();
        prefix |= sh.digit << shift;
        hi = shift;
    } while (hi > 0);
    const uint32_t tau = prefix;
    const unsigned long long above = sh.above, target = sh.target;
    if (tid == 0) sh.ntie = 0;
    __syncthreads();
    // smaller u kept; ties at tau resolved in index order below
    for (int64_t blk = tid; blk < nblk; blk += step) {
        float e[8];
        const uint32_t mb = load8(blk, e);
        uint32_t kb = 0u;
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            if (!((mb >> v) & 1u)) continue;
            const uint32_t u = kmax - ordered_key(e[v]);
            if (u < tau) {
                kb |= 1u << v;
            } else if (u == tau) {
                const int slot = atomicAdd(&sh.ntie, 1);
                if (slot < kMaxTies) sh.ties[slot] = (int32_t)((blk << 3) + v);
            }
        }
        store8(blk, kb);
        kept += __popc(kb);
    }
    __syncthreads();
    const int ntie = sh.ntie;
    if (ntie <= kMaxTies) {
        for (int j = tid; j < ntie; j += blockDim.x) {
            int rank = 0;
            const int32_t v = sh.ties[j];
            for (int w = 0; w < ntie; ++w) rank += sh.ties[w] < v;
            sh.sorted_ties[rank] = v;
        }
        __syncthreads();
        if (tid == 0) {
            unsigned long long cum = above;
            for (int j = 0; j < ntie && cum < target; ++j) {
                const int32_t i = sh.sorted_ties[j];
                float e[8];
                load8((int64_t)i >> 3, e);
                add_kept(i);
                ++kept;
                cum += fixed_mass(e[i & 7], m);
            }
        }
    } else if (tid == 0) {
        // more exact ties than fit: walk the whole set in index order
        unsigned long long cum = above;
        for (int64_t blk = 0; blk < nblk && cum < target; ++blk) {
            float e[8];
            const uint32_t mb = load8(blk, e);
            for (int v = 0; v < 8 && cum < target; ++v) {
                if (!((mb >> v) & 1u) || kmax - ordered_key(e[v]) != tau) continue;
                add_kept((blk << 3) + v);
                ++kept;
                cum += fixed_mass(e[v], m);
            }
        }
    }
    return (int)block_sum<unsigned long long>((unsigned long long)kept, sh.red);
}

// Join of a small level (at most blockDim.x blocks of 8 candidates, bitmaps of
// at most 32 KB) in one CTA: the rows' bitmaps staged in shared memory, row
// masks, one block scan, the kept candidates written in order.
__device__ void small_join(const Geo &g, const LevelWs &lw, const uint8_t *keptbits, int level, int grp,
                           int64_t n, const zha_selection &sel, SelShared &sh) {
    const int tid = threadIdx.x;
    const int64_t capv = g.capv[level];
    const int64_t bstride = g.bits_stride(level);
    const int64_t nblk = (n + 7) >> 3;
    uint8_t *sb = reinterpret_cast<uint8_t *>(&sh.hist_lo[0]);
    const uint4 *src = reinterpret_cast<const uint4 *>(keptbits + (int64_t)grp * g.G * bstride);
    for (int64_t i = tid; i < g.G * bstride / 16; i += blockDim.x)
        reinterpret_cast<uint4 *>(sb)[i] = __ldcg(src + i);
    __syncthreads();
    uint32_t km[8];
#pragma unroll
    for (int v = 0; v < 8; ++v) km[v] = 0u;
    const bool mine = tid < nblk;
    if (mine) {
        for (int h = 0; h < g.G; ++h) {
            const uint32_t b = sb[h * bstride + tid];
#pragma unroll
            for (int v = 0; v < 8; ++v) km[v] |= ((b >> v) & 1u) << h;
        }
        uint4 *kp = reinterpret_cast<uint4 *>(lw.kept + grp * capv + ((int64_t)tid << 3));
        kp[0] = make_uint4(km[0], km[1], km[2], km[3]);
        kp[1] = make_uint4(km[4], km[5], km[6], km[7]);
    }
    int cnt = 0;
#pragma unroll
    for (int v = 0; v < 8; ++v) cnt += km[v] != 0u;
    unsigned long long total;
    int64_t o = (int64_t)block_exclusive_scan<unsigned long long>((unsigned long long)cnt, sh.red, &total);
    int32_t *out_idx = level > 1 ? lw.plist + grp * g.cap[level] : sel.leaf_idx + grp * g.cap[1];
    uint32_t *out_mask = level > 1 ? lw.pmask + grp * g.cap[level] : sel.head_mask + grp * g.cap[1];
    if (mine && cnt) {
        const int32_t *cand = lw.cand + grp * capv + ((int64_t)tid << 3);
        const int4 c0 = *reinterpret_cast<const int4 *>(cand);
        const int4 c1 = *reinterpret_cast<const int4 *>(cand + 4);
        const int32_t cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int v = 0; v < 8; ++v)
            if (km[v]) {
                out_idx[o] = cv[v];
                out_mask[o] = km[v];
                ++o;
            }
    }
    if (tid == 0) {
        if (level > 1)
            lw.pcount[grp] = (int32_t)total;
        else
            sel.count[grp] = (int32_t)total;
    }
}

__global__ void __launch_bounds__(kSelThreads)
select_kernel(Geo g, LevelWs lw, uint8_t *keptbits, int level, float p, int32_t *level_kept, int fuse_join,
              zha_selection sel) {
    __shared__ SelShared sh;
    pdl_wait();
    const int h = blockIdx.x, grp = blockIdx.y;
    const int64_t capv = g.capv[level];
    const int64_t bstride = g.bits_stride(level);  // bytes of one row's bitmap
    const int64_t n = lw.count[grp];
    const uint32_t bit = 1u << h;
    const uint32_t *cmask = lw.cmask + grp * capv;
    const float *sc = lw.scores + (grp * g.G + h) * capv;
    uint8_t *mybits = keptbits + ((int64_t)grp * g.G + h) * bstride;
    const uint32_t kmax = lw.maxkey[(int64_t)grp * g.G + h];
    const uint32_t kmin = lw.minkey[(int64_t)grp * g.G + h];
    // rows are padded to a multiple of 8 entries, so 8-wide loads stay in bounds
    const int nk = topp_core(
        sh, n, p, kmax, kmin,
        [&](int64_t blk, float (&e)[8]) {
            const int64_t i0 = blk << 3;
            const float4 e0 = __ldg(reinterpret_cast<const float4 *>(sc + i0));
            const float4 e1 = __ldg(reinterpret_cast<const float4 *>(sc + i0) + 1);
            const uint4 m0 = __ldg(reinterpret_cast<const uint4 *>(cmask + i0));
            const uint4 m1 = __ldg(reinterpret_cast<const uint4 *>(cmask + i0) + 1);
            e[0] = e0.x; e[1] = e0.y; e[2] = e0.z; e[3] = e0.w;
            e[4] = e1.x; e[5] = e1.y; e[6] = e1.z; e[7] = e1.w;
            const uint32_t mm[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
            uint32_t mb = 0u;
#pragma unroll
            for (int v = 0; v < 8; ++v) mb |= ((mm[v] & bit) != 0u && i0 + v < n) ? (1u << v) : 0u;
            return mb;
        },
        [&](int64_t blk, uint32_t kb) { mybits[blk] = (uint8_t)kb; },
        [&](int64_t i) { mybits[i >> 3] |= (uint8_t)(1u << (i & 7)); });
    if (level_kept && threadIdx.x == 0) level_kept[((int64_t)grp * g.G + h) * g.L + (level - 1)] = nk;
    if (!fuse_join) {
        pdl_trigger();
        return;
    }
    // small level: the last of the group's G rows to finish joins them here
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) sh.last = atomicAdd(&lw.done[grp], 1u) == (uint32_t)(g.G - 1);
    __syncthreads();
    if (!sh.last) return;
    __threadfence();
    small_join(g, lw, keptbits, level, grp, n, sel, sh);
    if (threadIdx.x == 0) lw.done[grp] = 0u;
    pdl_trigger();
}

// ------------------------------------------------------ small levels: one CTA per group
//
// Levels with at most kSmallMax candidate slots per group: one CTA per group,
// one warp per query row (rows w, w + kSmallWarps, ...). The same exact
// selection as topp_core, every step warp-synchronous: a 256-bucket mass
// histogram over the score's distance below the max finds the crossing
// bucket; its members, listed in index order, are ordered by (score desc,
// index asc) in shared memory, or -- when more than kSmallList of them share
// it -- a radix search over the ordered key inside that bucket finds the
// crossing key, whose equal-score members are taken in index order. Kept
// candidates are OR-ed into a per-candidate head mask, and after one barrier
// the CTA joins the rows into the compacted candidate list itself.

constexpr int kSmallWarps = 8;
constexpr int kSmallThreads = kSmallWarps * 32;
constexpr int kSmallMax = 512;
constexpr int kSmallBuckets = 256;
constexpr int kSmallList = 128;

struct SmallShared {
    uint32_t kmask[kSmallMax];                      // heads that kept candidate i
    uint32_t hlo[kSmallWarps][kSmallBuckets];       // each warp's mass histogram: low words ...
    uint32_t hhi[kSmallWarps][kSmallBuckets];       // ... and carry words
    int32_t lidx[kSmallWarps][kSmallList];          // crossing-bucket members, index order
    uint32_t lkey[kSmallWarps][kSmallList];         // their ordered keys
    int32_t lord[kSmallWarps][kSmallList];          // list positions in (score desc, index asc) order
    unsigned long long red[kSmallWarps];
};

__device__ __forceinline__ unsigned long long warp_incl_scan64(unsigned long long x, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    return x;
}

__device__ __forceinline__ int warp_sum_int(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// One warp's histogram: lane l owns buckets [8 l, 8 l + 8).
struct WarpHist {
    static constexpr int kPer = kSmallBuckets / 32;
    unsigned long long h[kPer];
    unsigned long long excl;    // mass of the buckets before this lane's
    unsigned long long total;   // mass of all buckets
};

__device__ __forceinline__ void warp_hist_scan(const uint32_t *lo, const uint32_t *hi, int lane, WarpHist &wh) {
    unsigned long long mine = 0ull;
#pragma unroll
    for (int j = 0; j < WarpHist::kPer; ++j) {
        const int b = lane * WarpHist::kPer + j;
        wh.h[j] = ((unsigned long long)hi[b] << 32) | lo[b];
        mine += wh.h[j];
    }
    const unsigned long long incl = warp_incl_scan64(mine, lane);
    wh.excl = incl - mine;
    wh.total = __shfl_sync(0xffffffffu, incl, 31);
}

// First bucket at which the running mass, starting from run0 before bucket 0,
// reaches target (-1 if none); *above gets the running mass before it.
__device__ __forceinline__ int warp_hist_cross(const WarpHist &wh, int lane, unsigned long long run0,
                                               unsigned long long target, unsigned long long *above) {
    unsigned long long run = run0 + wh.excl, ab = 0ull;
    int found = -1;
#pragma unroll
    for (int j = 0; j < WarpHist::kPer; ++j) {
        if (found < 0 && wh.h[j] && run < target && run + wh.h[j] >= target) {
            found = lane * WarpHist::kPer + j;
            ab = run;
        }
        run += wh.h[j];
    }
    const unsigned ball = __ballot_sync(0xffffffffu, found >= 0);
    if (!ball) return -1;
    const int src = __ffs(ball) - 1;
    *above = __shfl_sync(0xffffffffu, ab, src);
    return __shfl_sync(0xffffffffu, found, src);
}

// Exact top-p of one query row by one warp: members are candidates i < n with
// (cmask[i] & bit); their kept bits are OR-ed into kmask[i] (shared or global
// memory). Returns (in every lane) the number kept.
template <bool NC = true>
__device__ __forceinline__ int small_row_topp(SmallShared &sh, uint32_t *kmask, int w, const float *sc,
                                              const uint32_t *cmask, int n, uint32_t bit, float p, uint32_t kmax,
                                              uint32_t kmin) {
    const int lane = threadIdx.x & 31;
    const unsigned lt = (1u << lane) - 1u;
    if (kmax == 0u) return 0;  // no member
    int kept = 0;
    if (p >= 1.f) {
        for (int i = lane; i < n; i += 32)
            if (ld_ws<NC>(cmask + i) & bit) {
                atomicOr(&kmask[i], bit);
                ++kept;
            }
        return warp_sum_int(kept);
    }
    uint32_t *lo = sh.hlo[w], *hi = sh.hhi[w];
    const float m = key_to_float(kmax);
    float W = (float)kSmallBuckets / fminf(m - key_to_float(kmin), kMassRange);
    if (kmax == kmin || !(W < 1e30f)) W = 0.f;  // one score value (or a sub-denormal span): one bucket
    auto bucket = [&](float e) -> int {
        const float x = (m - e) * W;
        return x < (float)(kSmallBuckets - 1) ? (int)x : kSmallBuckets - 1;
    };
    for (int j = lane; j < kSmallBuckets; j += 32) lo[j] = hi[j] = 0u;
    __syncwarp();
    constexpr int kU = 4;
    for (int i0 = 0; i0 < n; i0 += 32 * kU) {
        float e[kU];
        uint32_t c[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int i = i0 + u * 32 + lane;
            c[u] = i < n ? ld_ws<NC>(cmask + i) : 0u;
            e[u] = i < n ? ld_ws<NC>(sc + i) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kU; ++u)
            if (c[u] & bit) hist_add(lo, hi, bucket(e[u]), fixed_mass(e[u], m));
    }
    __syncwarp();
    WarpHist wh;
    warp_hist_scan(lo, hi, lane, wh);
    const unsigned long long target = (unsigned long long)ceil((double)p * (double)wh.total);
    unsigned long long above = 0ull;
    int bstar = warp_hist_cross(wh, lane, 0ull, target, &above);
    if (bstar < 0) bstar = kSmallBuckets;  // unreachable (target <= total): keep every member
    __syncwarp();

    // buckets before bstar are kept; bstar's members are listed in index order
    int ntie = 0;
    for (int i0 = 0; i0 < n; i0 += 32 * kU) {
        float e[kU];
        uint32_t c[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int i = i0 + u * 32 + lane;
            c[u] = i < n ? ld_ws<NC>(cmask + i) : 0u;
            e[u] = i < n ? ld_ws<NC>(sc + i) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int i = i0 + u * 32 + lane;
            const int bk = (c[u] & bit) ? bucket(e[u]) : kSmallBuckets + 1;
            if (bk < bstar) {
                atomicOr(&kmask[i], bit);
                ++kept;
            }
            const unsigned tb = __ballot_sync(0xffffffffu, bk == bstar);
            if (bk == bstar) {
                const int slot = ntie + __popc(tb & lt);
                if (slot < kSmallList) {
                    sh.lidx[w][slot] = i;
                    sh.lkey[w][slot] = ordered_key(e[u]);
                }
            }
            ntie += __popc(tb);
        }
    }
    __syncwarp();
    if (ntie <= kSmallList) {
        // order the list by (key desc, index asc): it is in index order already
        for (int j = lane; j < ntie; j += 32) {
            const uint32_t kj = sh.lkey[w][j];
            int rank = 0;
            for (int v = 0; v < ntie; ++v) {
                const uint32_t kv = sh.lkey[w][v];
                rank += (kv > kj) || (kv == kj && v < j);
            }
            sh.lord[w][rank] = j;
        }
        __syncwarp();
        unsigned long long cum = above;
        for (int r0 = 0; r0 < ntie && cum < target; r0 += 32) {
            const int r = r0 + lane;
            const int j = r < ntie ? sh.lord[w][r] : 0;
            const unsigned long long ms = r < ntie ? fixed_mass(key_to_float(sh.lkey[w][j]), m) : 0ull;
            const unsigned long long incl = warp_incl_scan64(ms, lane);
            if (r < ntie && cum + (incl - ms) < target) {
                atomicOr(&kmask[sh.lidx[w][j]], bit);
                ++kept;
            }
            cum += __shfl_sync(0xffffffffu, incl, 31);
        }
    } else {
        // many members in the crossing bucket: radix search over u = kmax - key
        // among them (8-bit digits), then equal-score members in index order
        const uint32_t uspan = kmax - kmin;
        int hb = uspan ? 32 - __clz(uspan) : 0;
        uint32_t prefix = 0u;
        unsigned long long ab = above;
        while (hb > 0) {
            const int bits = hb < 8 ? hb : 8;
            const int shift = hb - bits;
            for (int j = lane; j < kSmallBuckets; j += 32) lo[j] = hi[j] = 0u;
            __syncwarp();
            for (int i = lane; i < n; i += 32) {
                if (!(ld_ws<NC>(cmask + i) & bit)) continue;
                const float e = ld_ws<NC>(sc + i);
                if (bucket(e) != bstar) continue;
                const uint32_t u = kmax - ordered_key(e);
                if (hb < 32 && (u >> hb) != (prefix >> hb)) continue;
                hist_add(lo, hi, (int)((u >> shift) & ((1u << bits) - 1u)), fixed_mass(e, m));
            }
            __syncwarp();
            WarpHist rh;
            warp_hist_scan(lo, hi, lane, rh);
            unsigned long long a2 = ab;
            const int dg = warp_hist_cross(rh, lane, ab, target, &a2);
            __syncwarp();
            if (dg < 0) break;  // unreachable: the bucket's mass crosses target
            prefix |= (uint32_t)dg << shift;
            ab = a2;
            hb = shift;
        }
        const uint32_t tau = prefix;
        unsigned long long cum = ab;
        for (int i0 = 0; i0 < n; i0 += 32) {
            const int i = i0 + lane;
            const bool mem = i < n && (ld_ws<NC>(cmask + i) & bit);
            const float e = mem ? ld_ws<NC>(sc + i) : 0.f;
            const bool inb = mem && bucket(e) == bstar;
            const uint32_t u = inb ? kmax - ordered_key(e) : 0u;
            if (inb && u < tau) {
                atomicOr(&kmask[i], bit);
                ++kept;
            }
            const bool tie = inb && u == tau;
            const unsigned long long ms = (tie && cum < target) ? (unsigned long long)fixed_mass(e, m) : 0ull;
            const unsigned long long incl = warp_incl_scan64(ms, lane);
            if (tie && cum + (incl - ms) < target) {
                atomicOr(&kmask[i], bit);
                ++kept;
            }
            cum += __shfl_sync(0xffffffffu, incl, 31);
        }
    }
    __syncwarp();
    return warp_sum_int(kept);
}

__global__ void __launch_bounds__(kSmallThreads)
select_small_kernel(Geo g, LevelWs lw, int level, float p, int32_t *level_kept, zha_selection sel) {
    __shared__ SmallShared sh;
    const int grp = blockIdx.x, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int64_t capv = g.capv[level];
    pdl_wait();
    const int n = (int)min64((int64_t)lw.count[grp], min64(capv, kSmallMax));
    for (int i = tid; i < n; i += kSmallThreads) sh.kmask[i] = 0u;
    __syncthreads();
    const uint32_t *cmask = lw.cmask + grp * capv;
    for (int h = w; h < g.G; h += kSmallWarps) {
        const uint32_t kmax = lw.maxkey[(int64_t)grp * g.G + h];
        const uint32_t kmin = lw.minkey[(int64_t)grp * g.G + h];
        const int nk = small_row_topp(sh, sh.kmask, w, lw.scores + (grp * g.G + h) * capv, cmask, n, 1u << h, p,
                                      kmax, kmin);
        if (level_kept && lane == 0) level_kept[((int64_t)grp * g.G + h) * g.L + (level - 1)] = nk;
    }
    __syncthreads();
    // join: the candidates some row kept, in index order, each thread a run of consecutive slots
    const int per = (n + kSmallThreads - 1) / kSmallThreads;
    const int i0 = tid * per;
    int cnt = 0;
    for (int k = 0; k < per; ++k) {
        const int i = i0 + k;
        cnt += (i < n && sh.kmask[i] != 0u);
    }
    unsigned long long total;
    int64_t o = (int64_t)block_exclusive_scan<unsigned long long>((unsigned long long)cnt, sh.red, &total);
    int32_t *out_idx = level > 1 ? lw.plist + grp * g.cap[level] : sel.leaf_idx + grp * g.cap[1];
    uint32_t *out_mask = level > 1 ? lw.pmask + grp * g.cap[level] : sel.head_mask + grp * g.cap[1];
    for (int k = 0; k < per; ++k) {
        const int i = i0 + k;
        if (i >= n) break;
        const uint32_t km = sh.kmask[i];
        lw.kept[grp * capv + i] = km;
        if (km) {
            out_idx[o] = lw.cand[grp * capv + i];
            out_mask[o] = km;
            ++o;
        }
    }
    if (tid == 0) {
        if (level > 1)
            lw.pcount[grp] = (int32_t)total;
        else
            sel.count[grp] = (int32_t)total;
    }
    pdl_trigger();
}

// ------------------------------------------------------ fused route: one launch
//
// The whole route in one launch, for trees where few nodes are kept per level
// (trained references): one thread-block cluster per (sequence, KV head)
// group walks the levels top-down, CTA r owning query row r (16 CTAs per
// cluster where all the groups' clusters fit on the GPU at once, else 8).
// Per level:
//   1. the cluster's CTAs score the group's candidates (each warp two
//      candidates at a time, on the mma.sync scheme of score_mma_kernel, so
//      the scores are the same bits) and deliver row h's scores and extremes
//      to CTA h through distributed shared memory; a cluster barrier;
//   2. CTA r selects row r with all its threads (the exact selection of the
//      per-level kernels) and ORs its kept bits into every CTA's kept masks;
//      a cluster barrier;
//   3. every CTA joins the rows into the next level's candidates by itself,
//      so the next level starts without another barrier.
// The level's candidates and scores are copied out to the workspace views
// that the per-level launches fill -- by the CTAs that own no row while the
// rows select (16-CTA clusters), else after the join. A level with more than
// kFusedSm candidates goes through the workspace instead (correct at any
// size, but one warp per row then selects over all of them: the per-level
// launches are the faster route there). Cluster barriers are hardware
// barriers that every CTA takes the same number of times, so nothing waits
// unboundedly.

constexpr int kFusedSm = 1024;     // candidates per level that a level keeps in shared memory
constexpr int kFusedPer = kFusedSm / kSmallThreads;
static_assert(kSmallThreads == kSmallBuckets, "one histogram bucket per thread");

struct FusedArgs {
    LevelWs lw[kMaxLevels + 1];
    float p[kMaxLevels + 1];
    const __nv_bfloat16 *mu[kMaxLevels + 1];
    const float *bias[kMaxLevels + 1];
};

// Per-CTA shared state. CTA r < G of a cluster owns query row r of its group:
// the other CTAs deliver that row's scores and extremes to it through
// distributed shared memory, and each row's CTA ORs its kept bits into every
// CTA's km, so that each CTA joins the level by itself.
struct FusedShared {
    float sc[2][kFusedSm];          // this CTA's row: scores of the level's candidates (by level parity)
    uint32_t km[kFusedSm];          // kept head masks of the level's candidates
    uint32_t rk[kFusedSm];          // this CTA's row: candidate kept (1) or not (0)
    uint32_t mb[kFusedSm];          // this CTA's row: candidate is a member (for the warp selection)
    int32_t pl[2][kFusedSm];        // nodes kept one level up and their head masks, when they fit
    uint32_t pm[2][kFusedSm];       // (by level parity: a join writes one half while the other is read)
    uint32_t hlo[kSmallBuckets];    // the row's mass histogram (64-bit buckets from native 32-bit
    uint32_t hhi[kSmallBuckets];    // shared atomics: low words and carry words)
    unsigned long long above, target;
    int32_t tidx[kSmallList];       // crossing-bucket members: index, ordered key, rank order
    uint32_t tkey[kSmallList];
    int32_t tord[kSmallList];
    int32_t wsum[kSmallWarps];      // per-warp kept counts of the join
    uint32_t maxk, mink;            // ordered keys of this row's largest and smallest member score
    int32_t bstar, ntie, nkept;
    SmallShared sh;                 // the warp selection: rows with many equal-bucket members
};

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;\n" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
    return r;
}

// shared::cluster address of the same shared variable in CTA `rank` of the cluster
template <typename T>
__device__ __forceinline__ uint32_t cluster_addr(T *p, uint32_t rank) {
    uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p)), r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(a), "r"(rank));
    return r;
}

// reductions into another CTA's shared memory that return nothing (no round trip)
__device__ __forceinline__ void red_max_cluster(uint32_t addr, uint32_t v) {
    asm volatile("red.relaxed.cluster.shared::cluster.max.u32 [%0], %1;\n" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void red_min_cluster(uint32_t addr, uint32_t v) {
    asm volatile("red.relaxed.cluster.shared::cluster.min.u32 [%0], %1;\n" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void red_or_cluster(uint32_t addr, uint32_t v) {
    asm volatile("red.relaxed.cluster.shared::cluster.or.b32 [%0], %1;\n" ::"r"(addr), "r"(v) : "memory");
}

// generic address of the same shared variable in CTA `rank` of the cluster
template <typename T>
__device__ __forceinline__ T *cluster_peer(T *p, uint32_t rank) {
    uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p)), r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(a), "r"(rank));
    uint64_t gen;
    asm volatile("cvta.shared::cluster.u64 %0, %1;\n" : "=l"(gen) : "l"((uint64_t)r));
    return reinterpret_cast<T *>(gen);
}

// Exact top-p of this CTA's row over the level's n <= kFusedSm candidates, in
// shared memory, by the whole CTA: the same definition as small_row_topp (and
// topp_core) -- members by (score desc, index asc), each kept while the mass
// before it is below ceil(p * total), masses in 2^-31 fixed point relative to
// the row's maximum -- found with one mass histogram over the same buckets
// (scanned by one warp), and the crossing bucket's members ranked by one
// warp. A crossing bucket with more than kSmallList members goes to
// small_row_topp. Sets fs.rk[i] for the kept candidates and returns (in every
// thread) how many were kept. The histogram is all zero on entry and on return.
template <class Member>
__device__ int cta_row_topp(FusedShared &fs, const float *sc, int n, float p, Member member) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t kmax = fs.maxk, kmin = fs.mink;
    if (kmax == 0u) {   // no member
#pragma unroll
        for (int k = 0; k < kFusedPer; ++k)
            if (tid + k * kSmallThreads < n) fs.rk[tid + k * kSmallThreads] = 0u;
        __syncthreads();
        return 0;
    }
    float e[kFusedPer];
    bool mem[kFusedPer];
#pragma unroll
    for (int k = 0; k < kFusedPer; ++k) {
        const int i = tid + k * kSmallThreads;
        mem[k] = i < n && member(i);
        e[k] = mem[k] ? sc[i] : 0.f;
        if (i < n) fs.rk[i] = 0u;
    }
    int kept = 0;
    if (p >= 1.f) {
#pragma unroll
        for (int k = 0; k < kFusedPer; ++k)
            if (mem[k]) {
                fs.rk[tid + k * kSmallThreads] = 1u;
                ++kept;
            }
        return (int)block_sum<unsigned long long>((unsigned long long)kept, fs.sh.red);
    }
    const float m = key_to_float(kmax);
    float W = (float)kSmallBuckets / fminf(m - key_to_float(kmin), kMassRange);
    if (kmax == kmin || !(W < 1e30f)) W = 0.f;  // one score value (or a sub-denormal span): one bucket
    auto bucket = [&](float x) -> int {
        const float y = (m - x) * W;
        return y < (float)(kSmallBuckets - 1) ? (int)y : kSmallBuckets - 1;
    };
#pragma unroll
    for (int k = 0; k < kFusedPer; ++k)
        if (mem[k]) {
            const uint32_t w = fixed_mass(e[k], m);
            if (w) hist_add(fs.hlo, fs.hhi, bucket(e[k]), w);
        }
    __syncthreads();
    if (warp == 0) {
        // lane l scans buckets [8 l, 8 l + 8) (and zeroes them for the next use)
        constexpr int kPer = kSmallBuckets / 32;
        unsigned long long hb[kPer], mine = 0ull;
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int bk = lane * kPer + j;
            hb[j] = ((unsigned long long)fs.hhi[bk] << 32) | fs.hlo[bk];
            fs.hlo[bk] = fs.hhi[bk] = 0u;
            mine += hb[j];
        }
        const unsigned long long incl = warp_incl_scan64(mine, lane);
        const unsigned long long total = __shfl_sync(0xffffffffu, incl, 31);
        const unsigned long long target = (unsigned long long)ceil((double)p * (double)total);
        unsigned long long run = incl - mine, ab = 0ull;
        int found = -1;
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            if (found < 0 && hb[j] && run < target && run + hb[j] >= target) {
                found = lane * kPer + j;
                ab = run;
            }
            run += hb[j];
        }
        const unsigned ball = __ballot_sync(0xffffffffu, found >= 0);
        if (lane == 0) {
            fs.bstar = kSmallBuckets;   // unreachable (target <= total): keep every member
            fs.ntie = 0;
            fs.nkept = 0;
            fs.target = target;
        }
        if (ball && lane == __ffs(ball) - 1) {
            fs.bstar = found;
            fs.above = ab;
        }
    }
    __syncthreads();
    const int bstar = fs.bstar;
#pragma unroll
    for (int k = 0; k < kFusedPer; ++k) {
        if (!mem[k]) continue;
        const int i = tid + k * kSmallThreads;
        const int b = bucket(e[k]);
        if (b < bstar) {
            fs.rk[i] = 1u;
            ++kept;
        } else if (b == bstar) {
            const int slot = atomicAdd(&fs.ntie, 1);
            if (slot < kSmallList) {
                fs.tidx[slot] = i;
                fs.tkey[slot] = ordered_key(e[k]);
            }
        }
    }
    __syncthreads();
    const int ntie = fs.ntie;
    if (ntie == 1) {
        // a lone member of the crossing bucket: the mass before it (that of
        // the buckets before) is below the target, so it is kept
        if (tid == 0) {
            fs.rk[fs.tidx[0]] = 1u;
            ++kept;
        }
    } else if (ntie <= kSmallList) {
        if (warp == 0) {
            const unsigned long long target = fs.target;
            // rank the crossing bucket's members by (key desc, index asc)
            for (int j = lane; j < ntie; j += 32) {
                const uint32_t kj = fs.tkey[j];
                const int ij = fs.tidx[j];
                int r = 0;
                for (int v = 0; v < ntie; ++v) {
                    const uint32_t kv = fs.tkey[v];
                    r += (kv > kj) || (kv == kj && fs.tidx[v] < ij);
                }
                fs.tord[r] = j;
            }
            __syncwarp();
            unsigned long long cum = fs.above;
            for (int r0 = 0; r0 < ntie && cum < target; r0 += 32) {
                const int r = r0 + lane;
                const int j = r < ntie ? fs.tord[r] : 0;
                const unsigned long long ms = r < ntie ? fixed_mass(key_to_float(fs.tkey[j]), m) : 0ull;
                const unsigned long long incl = warp_incl_scan64(ms, lane);
                if (r < ntie && cum + (incl - ms) < target) {
                    fs.rk[fs.tidx[j]] = 1u;
                    ++kept;
                }
                cum += __shfl_sync(0xffffffffu, incl, 31);
            }
        }
    }
    if (ntie <= kSmallList) {
        const int wk = __reduce_add_sync(0xffffffffu, kept);
        if (lane == 0 && wk) atomicAdd(&fs.nkept, wk);
        __syncthreads();
        return fs.nkept;
    }
    // many members in the crossing bucket: warp 0 runs the warp selection over
    // the whole row (it marks a superset of the candidates marked above:
    // exactly the kept ones)
#pragma unroll
    for (int k = 0; k < kFusedPer; ++k) {
        const int i = tid + k * kSmallThreads;
        if (i < n) fs.mb[i] = mem[k] ? 1u : 0u;
    }
    __syncthreads();
    if (warp == 0) small_row_topp<false>(fs.sh, fs.rk, 0, sc, fs.mb, n, 1u, p, kmax, kmin);
    __syncthreads();
    kept = 0;
#pragma unroll
    for (int k = 0; k < kFusedPer; ++k) {
        const int i = tid + k * kSmallThreads;
        kept += (i < n && fs.rk[i] != 0u);
    }
    return (int)block_sum<unsigned long long>((unsigned long long)kept, fs.sh.red);
}

template <int D, int CL>
__global__ void __launch_bounds__(kSmallThreads, 2)
route_fused_kernel(Geo g, FusedArgs a, const __nv_bfloat16 *q, const int32_t *lens, zha_selection sel) {
    extern __shared__ __align__(16) unsigned char fused_raw[];
    FusedShared &fs = *reinterpret_cast<FusedShared *>(fused_raw);
    constexpr int KP = D / 32;
    const int grp = blockIdx.y;
    const int b = grp / g.Hkv, kvh = grp % g.Hkv;
    const int rank = (int)cluster_ctarank();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gq = lane >> 2, t = lane & 3;
    // the group's query rows (G <= 8: one n-tile), as B fragments
    uint32_t bq[KP][4];
#pragma unroll
    for (int kp = 0; kp < KP; ++kp) {
        uint4 w = make_uint4(0, 0, 0, 0);
        if (gq < g.G) w = ldg16(q + g.qrow(b, kvh, gq) * D + kp * 32 + t * 8);
        bq[kp][0] = w.x; bq[kp][1] = w.y; bq[kp][2] = w.z; bq[kp][3] = w.w;
    }
    for (int i = tid; i < kFusedSm; i += kSmallThreads) fs.km[i] = 0u;
    fs.hlo[tid] = fs.hhi[tid] = 0u;
    if (tid == 0) {
        fs.maxk = 0u;
        fs.mink = 0xffffffffu;
    }
    pdl_wait();
    const int64_t N = group_len(g, lens, grp);
    const uint32_t all = all_heads(g.G);
    const float s = g.s;
    const int lc = __ffs(g.c) - 1;
    // nodes of each level (c is a power of two: shifts, not divisions)
    auto nodes_at = [&](int level) -> int {
        int64_t m = N >> lc;
        for (int l = 2; l <= level; ++l) m = (m + g.c - 1) >> lc;
        return (int)m;
    };
    // scores and extremes of row h go to CTA h (lanes with gq == 0 hold rows 2t, 2t + 1)
    float *sc_row[2][2];
    uint32_t mx_row[2], mn_row[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const uint32_t h = (uint32_t)min(2 * t + j, CL - 1);
        sc_row[0][j] = cluster_peer(&fs.sc[0][0], h);
        sc_row[1][j] = cluster_peer(&fs.sc[1][0], h);
        mx_row[j] = cluster_addr(&fs.maxk, h);
        mn_row[j] = cluster_addr(&fs.mink, h);
    }
    cluster_sync();   // every CTA has started (its shared memory exists) and reset its state
    bool pl_local = false;  // the nodes kept one level up are in fs.pl[par] (else in the workspace)
    int par = 0, n_up = 0;
    int n_here = nodes_at(g.L);
    for (int level = g.L; level >= 1; --level) {
        const LevelWs &lw = a.lw[level];
        const LevelWs &up = a.lw[level < g.L ? level + 1 : level];
        const bool top = level == g.L;
        const int n = top ? n_here : n_up * g.c;
        const int n_below = level > 1 ? nodes_at(level - 1) : 0;
        const bool sm = n <= kFusedSm;
        const int64_t cap = g.cap[level], capv = g.capv[level];
        const int64_t cap_up = top ? 0 : g.cap[level + 1];
        // candidate i: its node and the heads that route to it
        auto cand_at = [&](int i, int &node, uint32_t &hm) {
            if (top) {
                node = i;
                hm = all;
                return;
            }
            const int j = i >> lc;
            const int pn = pl_local ? fs.pl[par][j] : up.plist[grp * cap_up + j];
            node = (pn << lc) | (i & (g.c - 1));
            hm = node < n_here ? (pl_local ? fs.pm[par][j] : up.pmask[grp * cap_up + j]) : 0u;
        };
        // the level's candidates and scores, out to the workspace views (a
        // level held in shared memory). With CTAs that own no row, those copy
        // while the rows select (before the level's last cluster barrier: the
        // rows' scores are read from their CTAs' shared memory). Otherwise
        // every CTA copies after the join, its own row's scores and a share of
        // the candidates: no CTA reads another's shared memory after the last
        // barrier, when that CTA may have finished.
        auto copy_out = [&]() {
            if (CL > g.G) {
                const int nc = CL - g.G, rc = rank - g.G;
                for (int x = rc * kSmallThreads + tid; x < n * (g.G + 1); x += nc * kSmallThreads) {
                    const int h = x / n, i = x - h * n;
                    if (h < g.G) {
                        lw.scores[(grp * g.G + h) * capv + i] = cluster_peer(&fs.sc[par][0], (uint32_t)h)[i];
                    } else {
                        int node;
                        uint32_t hm;
                        cand_at(i, node, hm);
                        lw.cand[grp * capv + i] = node;
                        lw.cmask[grp * capv + i] = hm;
                    }
                }
            } else {
                for (int i = tid; i < n; i += kSmallThreads) lw.scores[(grp * g.G + rank) * capv + i] = fs.sc[par][i];
                for (int i = rank * kSmallThreads + tid; i < n; i += CL * kSmallThreads) {
                    int node;
                    uint32_t hm;
                    cand_at(i, node, hm);
                    lw.cand[grp * capv + i] = node;
                    lw.cmask[grp * capv + i] = hm;
                }
            }
        };
        if (!sm && rank == 0)
            for (int i = tid; i < n; i += kSmallThreads) lw.kept[grp * capv + i] = 0u;
        // 1. scores of every candidate for every query row, each warp two
        //    candidates at a time: to the row's CTA, or (a level with more
        //    candidates than fit) to the workspace
        constexpr int U = 2;
        float runmax[2] = {-INFINITY, -INFINITY}, runmin[2] = {INFINITY, INFINITY};
        for (int i0 = (rank * kSmallWarps + warp) * U; i0 < n; i0 += CL * kSmallWarps * U) {
            int node[U];
            uint32_t hm[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                node[u] = 0;
                hm[u] = 0u;
                if (i0 + u < n) {
                    cand_at(i0 + u, node[u], hm[u]);
                    if (!sm && lane == 0) {
                        lw.cand[grp * capv + i0 + u] = node[u];
                        lw.cmask[grp * capv + i0 + u] = hm[u];
                    }
                }
            }
            uint4 ra[U][KP], rb[U][KP];
            float b0[U], b1[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const __nv_bfloat16 *base = a.mu[level] + (grp * cap + node[u]) * (int64_t)g.R * D;
                const float *bb = a.bias[level] + (grp * cap + node[u]) * (int64_t)g.R;
#pragma unroll
                for (int kp = 0; kp < KP; ++kp) {
                    ra[u][kp] = hm[u] ? ldg16(base + (int64_t)gq * D + kp * 32 + t * 8) : make_uint4(0, 0, 0, 0);
                    rb[u][kp] = hm[u] ? ldg16(base + (int64_t)(gq + 8) * D + kp * 32 + t * 8) : make_uint4(0, 0, 0, 0);
                }
                b0[u] = hm[u] ? bb[gq] : 0.f;
                b1[u] = hm[u] ? bb[gq + 8] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = i0 + u;
                if (i >= n) break;
                float e[2] = {-INFINITY, -INFINITY};
                if (hm[u]) {
                    float acc[4] = {0.f, 0.f, 0.f, 0.f}, acc2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int kp = 0; kp < KP; ++kp) {
                        const uint4 &xa = ra[u][kp], &xb = rb[u][kp];
                        const uint32_t a0[4] = {xa.x, xb.x, xa.y, xb.y};
                        const uint32_t a1[4] = {xa.z, xb.z, xa.w, xb.w};
                        mma_bf16_16816(acc, a0, bq[kp][0], bq[kp][1]);
                        mma_bf16_16816(acc2, a1, bq[kp][2], bq[kp][3]);
                    }
#pragma unroll
                    for (int v = 0; v < 4; ++v) acc[v] += acc2[v];
                    e[0] = fmaxf(-INFINITY, fmaxf(fmaf(s, acc[0], b0[u]), fmaf(s, acc[2], b1[u])));
                    e[1] = fmaxf(-INFINITY, fmaxf(fmaf(s, acc[1], b0[u]), fmaf(s, acc[3], b1[u])));
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        float v = e[j];
                        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
                        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
                        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
                        e[j] = v;
                    }
                }
                if (gq == 0) {
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int h = 2 * t + j;
                        if (h < g.G) {
                            if (sm)
                                (par ? sc_row[1][j] : sc_row[0][j])[i] = e[j];
                            else
                                lw.scores[(grp * g.G + h) * capv + i] = e[j];
                            if ((hm[u] >> h) & 1u) {
                                runmax[j] = fmaxf(runmax[j], e[j]);
                                runmin[j] = fminf(runmin[j], e[j]);
                            }
                        }
                    }
                }
            }
        }
        if (gq == 0) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int h = 2 * t + j;
                if (h < g.G && runmax[j] > -INFINITY) {
                    red_max_cluster(mx_row[j], ordered_key(runmax[j]));
                    red_min_cluster(mn_row[j], ordered_key(runmin[j]));
                }
            }
        }
        if (!sm) __threadfence();   // workspace scores and kept masks reach the other CTAs through L2
        cluster_sync();
        // 2. CTA r selects row r, and ORs its kept bits into every CTA's km
        //    (CTAs without a row copy the level out meanwhile)
        if (sm && CL > g.G && rank >= g.G) copy_out();
        if (rank < g.G) {
            const uint32_t bit = 1u << rank;
            int nk;
            if (sm) {
                nk = cta_row_topp(fs, fs.sc[par], n, a.p[level], [&](int i) {
                    int node;
                    uint32_t hm;
                    cand_at(i, node, hm);
                    return (hm & bit) != 0u;
                });
                for (int i = tid; i < n; i += kSmallThreads)
                    if (fs.rk[i])
#pragma unroll
                        for (int r = 0; r < CL; ++r) red_or_cluster(cluster_addr(&fs.km[i], (uint32_t)r), bit);
            } else {
                nk = 0;
                if (warp == 0)
                    nk = small_row_topp<false>(fs.sh, lw.kept + grp * capv, 0, lw.scores + (grp * g.G + rank) * capv,
                                               lw.cmask + grp * capv, n, bit, a.p[level], fs.maxk, fs.mink);
                __syncthreads();
            }
            if (sel.level_kept && tid == 0) sel.level_kept[((int64_t)grp * g.G + rank) * g.L + (level - 1)] = nk;
            if (tid == 0) {
                fs.maxk = 0u;
                fs.mink = 0xffffffffu;
            }
        }
        if (!sm) __threadfence();
        cluster_sync();
        // 3. every CTA joins the rows into the next level's candidates (the
        //    first CTA also writes them to the workspace and the selection):
        //    thread-contiguous runs, compacted in order
        const int per = (n + kSmallThreads - 1) / kSmallThreads;
        const int i0 = tid * per;
        const uint32_t *kmv = sm ? fs.km : lw.kept + grp * capv;
        int cnt = 0;
        for (int k = 0; k < per; ++k) {
            const int i = i0 + k;
            cnt += (i < n && kmv[i] != 0u);
        }
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) fs.wsum[warp] = incl;
        __syncthreads();
        int o = incl - cnt, total = 0;
#pragma unroll
        for (int w = 0; w < kSmallWarps; ++w) {
            const int v = fs.wsum[w];
            o += w < warp ? v : 0;
            total += v;
        }
        const bool fits = total <= kFusedSm;
        int32_t *out_idx = level > 1 ? lw.plist + grp * cap : sel.leaf_idx + grp * g.cap[1];
        uint32_t *out_mask = level > 1 ? lw.pmask + grp * cap : sel.head_mask + grp * g.cap[1];
        for (int k = 0; k < per; ++k) {
            const int i = i0 + k;
            if (i >= n) break;
            const uint32_t m = kmv[i];
            if (sm && rank == 0) lw.kept[grp * capv + i] = m;
            if (m) {
                int node;
                if (sm) {
                    uint32_t hm;
                    cand_at(i, node, hm);
                } else {
                    node = lw.cand[grp * capv + i];
                }
                if (fits) {
                    fs.pl[par ^ 1][o] = node;
                    fs.pm[par ^ 1][o] = m;
                }
                if (rank == 0) {
                    out_idx[o] = node;
                    out_mask[o] = m;
                }
                ++o;
            }
        }
        if (rank == 0 && tid == 0) {
            lw.count[grp] = n;
            if (level > 1)
                lw.pcount[grp] = total;
            else
                sel.count[grp] = total;
        }
        __syncthreads();
        if (sm) {
            for (int i = tid; i < n; i += kSmallThreads) fs.km[i] = 0u;
            if (CL == g.G) copy_out();
        }
        if (!fits) {
            // the next level reads the kept nodes from the workspace
            __threadfence();
            cluster_sync();
        }
        pl_local = fits;
        n_up = total;
        n_here = n_below;
        par ^= 1;
    }
    pdl_trigger();
}

// ------------------------------------------------- selection over several CTAs per row

constexpr int kSplitThreads = 256;
constexpr int kSplitMinBuckets = 1024;                // buckets of a row's histogram summed across its CTAs:
constexpr int kSplitPerBucket = 64;                   // about n / 64 (a power of two), from 1024 to kBuckets
constexpr int kSplitMinSlice = 4096;                  // candidates per CTA, at least
constexpr long long kSpinCycles = 2000000000LL;       // about a second: a wait that long is an error

struct SplitWs {
    unsigned long long *hist;   // [rows][kSelBuckets], left zeroed
    int32_t *lidx;              // [rows][kSelList]
    uint32_t *lkey;
    uint32_t *ctr;              // [L][rows][4]: arrivals, list count, kept count
};

// Arrive at a counter shared by the CTAs of one row and wait, bounded, until
// it reaches target. On timeout the status is set and false returned (the
// results of the call are then invalid; nothing waits forever).
__device__ bool row_barrier(uint32_t *ctr, uint32_t target, int32_t *status, int *ok_sh,
                            long long limit = kSpinCycles) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(ctr, 1u);
        const long long t0 = clock64();
        int ok = 1;
        while (*reinterpret_cast<volatile uint32_t *>(ctr) < target) {
            if (clock64() - t0 > limit) {
                set_status(status, ZHA_ERR_TIMEOUT);
                ok = 0;
                break;
            }
            __nanosleep(64);
        }
        __threadfence();
        *ok_sh = ok;
    }
    __syncthreads();
    return *ok_sh != 0;
}

// The selection of select_kernel with one row's candidates spread over the
// gridDim.x CTAs of (blockIdx.y = row, blockIdx.z = group): each CTA builds
// the mass histogram of its slice and adds it to the row's global histogram;
// after a barrier every CTA finds the same crossing bucket, keeps its slice's
// members below it and lists the crossing bucket's members; after a second
// barrier the row's first CTA orders that list and finalises the row. The
// grid is sized on the host so that all its CTAs can be resident at once,
// and the row's CTAs are consecutive in launch order.
__global__ void __launch_bounds__(kSplitThreads, 4)
select_split_kernel(Geo g, LevelWs lw, uint8_t *keptbits, int level, float p, int32_t *level_kept,
                    SplitWs sw, int32_t *status) {
    __shared__ SelShared sh;
    pdl_wait();
    __shared__ int ok_sh;
    const int sidx = blockIdx.x, S = gridDim.x, h = blockIdx.y, grp = blockIdx.z;
    const int tid = threadIdx.x;
    const int64_t step = blockDim.x;
    const int64_t capv = g.capv[level];
    const int64_t bstride = g.bits_stride(level);
    const int64_t n = lw.count[grp];
    const int64_t nblk = (n + 7) >> 3;
    const int64_t blo = nblk * sidx / S, bhi = nblk * (sidx + 1) / S;
    const int64_t row = (int64_t)grp * g.G + h;
    const uint32_t bit = 1u << h;
    const uint32_t *cmask = lw.cmask + grp * capv;
    const float *sc = lw.scores + row * capv;
    uint8_t *mybits = keptbits + row * bstride;
    const uint32_t kmax = lw.maxkey[row], kmin = lw.minkey[row];
    uint32_t *ctr = sw.ctr + (((int64_t)(level - 1) * g.groups() + grp) * g.G + h) * 4;
    unsigned long long *gh = sw.hist + row * kBuckets;
    auto load8 = [&](int64_t blk, float (&e)[8]) -> uint32_t {
        const int64_t i0 = blk << 3;
        const float4 e0 = __ldg(reinterpret_cast<const float4 *>(sc + i0));
        const float4 e1 = __ldg(reinterpret_cast<const float4 *>(sc + i0) + 1);
        const uint4 m0 = __ldg(reinterpret_cast<const uint4 *>(cmask + i0));
        const uint4 m1 = __ldg(reinterpret_cast<const uint4 *>(cmask + i0) + 1);
        e[0] = e0.x; e[1] = e0.y; e[2] = e0.z; e[3] = e0.w;
        e[4] = e1.x; e[5] = e1.y; e[6] = e1.z; e[7] = e1.w;
        const uint32_t mm[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
        uint32_t mb = 0u;
#pragma unroll
        for (int v = 0; v < 8; ++v) mb |= ((mm[v] & bit) != 0u && i0 + v < n) ? (1u << v) : 0u;
        return mb;
    };
    auto store8 = [&](int64_t blk, uint32_t kb) { mybits[blk] = (uint8_t)kb; };
    auto add_kept = [&](int64_t i) { mybits[i >> 3] |= (uint8_t)(1u << (i & 7)); };
    auto finalise = [&](int nk) {
        if (level_kept && tid == 0) level_kept[row * g.L + (level - 1)] = nk;
    };

    const float m = key_to_float(kmax);
    int nb = kSplitMinBuckets;
    while (nb < kBuckets && (int64_t)nb * kSplitPerBucket < n) nb <<= 1;
    const float W = (float)nb / fminf(m - key_to_float(kmin), kMassRange);
    if (kmax == 0u || p >= 1.f) {
        // no member, or every member kept: each slice stores its membership
        int kept = 0;
        for (int64_t blk = blo + tid; blk < bhi; blk += step) {
            float e[8];
            const uint32_t mb = kmax ? load8(blk, e) : 0u;
            store8(blk, mb);
            kept += __popc(mb);
        }
        kept = (int)block_sum<unsigned long long>((unsigned long long)kept, sh.red);
        if (tid == 0 && kept) atomicAdd(&ctr[2], (uint32_t)kept);
        if (!row_barrier(&ctr[0], (uint32_t)S, status, &ok_sh)) return;
        if (sidx == 0) finalise((int)*reinterpret_cast<volatile uint32_t *>(&ctr[2]));
        return;
    }
    if (kmax == kmin || !(W < 1e30f)) {
        // equal scores (or a range too narrow to bucket): the row on one CTA
        if (sidx != 0) return;
        const int nk = topp_core(sh, n, p, kmax, kmin, load8, store8, add_kept);
        finalise(nk);
        return;
    }
    auto bucket = [&](float e) -> int {
        const float x = (m - e) * W;
        return x < (float)(nb - 1) ? (int)x : nb - 1;
    };
    // 1. this slice's mass histogram into the row's global histogram
    for (int i = tid; i < nb; i += blockDim.x) sh.hist_lo[i] = sh.hist_hi[i] = 0u;
    __syncthreads();
    auto add_block = [&](uint32_t mb, const float (&e)[8]) {
#pragma unroll
        for (int v = 0; v < 8; ++v)
            if ((mb >> v) & 1u) hist_add(sh.hist_lo, sh.hist_hi, bucket(e[v]), fixed_mass(e[v], m));
    };
    for (int64_t blk = blo + tid; blk < bhi; blk += 2 * step) {
        float e0[8], e1[8];
        const uint32_t m0 = load8(blk, e0);
        const uint32_t m1 = blk + step < bhi ? load8(blk + step, e1) : 0u;
        add_block(m0, e0);
        add_block(m1, e1);
    }
    __syncthreads();
    for (int i = tid; i < nb; i += blockDim.x) {
        const unsigned long long v = ((unsigned long long)sh.hist_hi[i] << 32) | sh.hist_lo[i];
        if (v) atomicAdd(&gh[i], v);
    }
    if (!row_barrier(&ctr[0], (uint32_t)S, status, &ok_sh)) return;
    // 2. the crossing bucket (every CTA of the row computes the same); the row's
    // histogram comes in with all loads in flight at once
    constexpr int kMaxPer = kBuckets / kSplitThreads;
    const int per = nb / kSplitThreads;
    unsigned long long hv[kMaxPer];
#pragma unroll
    for (int j = 0; j < kMaxPer; ++j) hv[j] = j < per ? __ldcg(&gh[tid * per + j]) : 0ull;
    unsigned long long mine = 0ull;
#pragma unroll
    for (int j = 0; j < kMaxPer; ++j) mine += hv[j];
    unsigned long long z;
    if (tid == 0) {
        sh.digit = nb - 1;
        sh.above = 0ull;
    }
    const unsigned long long excl = block_exclusive_scan<unsigned long long>(mine, sh.red, &z);
    const unsigned long long target = (unsigned long long)ceil((double)p * (double)z);
    unsigned long long run = excl;
#pragma unroll
    for (int j = 0; j < kMaxPer; ++j) {
        const int bk = tid * per + j;
        const unsigned long long hgt = hv[j];
        if (hgt && run < target && run + hgt >= target) {
            sh.digit = (uint32_t)bk;
            sh.above = run;
        }
        run += hgt;
    }
    __syncthreads();
    const int bstar = (int)sh.digit;
    const unsigned long long above = sh.above;
    // 3. keep this slice's members below the crossing bucket; list the bucket's members
    int kept = 0;
    for (int64_t blk = blo + tid; blk < bhi; blk += step) {
        float e[8];
        const uint32_t mb = load8(blk, e);
        uint32_t kb = 0u;
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            if (!((mb >> v) & 1u)) continue;
            const int bk = bucket(e[v]);
            if (bk < bstar) {
                kb |= 1u << v;
            } else if (bk == bstar) {
                const uint32_t slot = atomicAdd(&ctr[1], 1u);
                if (slot < (uint32_t)kSelList) {
                    sw.lidx[row * kSelList + slot] = (int32_t)((blk << 3) + v);
                    sw.lkey[row * kSelList + slot] = ordered_key(e[v]);
                }
            }
        }
        store8(blk, kb);
        kept += __popc(kb);
    }
    kept = (int)block_sum<unsigned long long>((unsigned long long)kept, sh.red);
    if (tid == 0 && kept) atomicAdd(&ctr[2], (uint32_t)kept);
    if (!row_barrier(&ctr[0], 2u * (uint32_t)S, status, &ok_sh)) return;
    // 4. every CTA has read the histogram: clear this CTA's share for the next use
    for (int i = (int)((int64_t)nb * sidx / S) + tid; i < (int)((int64_t)nb * (sidx + 1) / S);
         i += blockDim.x)
        gh[i] = 0ull;
    if (sidx != 0) return;
    // 5. the row's first CTA: the crossing bucket in (score desc, index asc) order
    const uint32_t nl = *reinterpret_cast<volatile uint32_t *>(&ctr[1]);
    if (nl <= (uint32_t)kSelList) {
        for (uint32_t j = tid; j < nl; j += blockDim.x) {
            sh.ties[j] = __ldcg(&sw.lidx[row * kSelList + j]);
            sh.tkey[j] = __ldcg(&sw.lkey[row * kSelList + j]);
        }
        __syncthreads();
        for (uint32_t j = tid; j < nl; j += blockDim.x) {
            const uint32_t kj = sh.tkey[j];
            const int32_t ij = sh.ties[j];
            int rank = 0;
            for (uint32_t w = 0; w < nl; ++w) {
                const uint32_t kw = sh.tkey[w];
                rank += (kw > kj) || (kw == kj && sh.ties[w] < ij);
            }
            sh.sorted_ties[rank] = (int)j;
        }
        __syncthreads();
        // the ordered list, a block of members at a time: a member is kept
        // while the running mass before it is below target
        int added = 0;
        unsigned long long cum = above;
        for (uint32_t r0 = 0; r0 < nl && cum < target; r0 += blockDim.x) {
            const uint32_t r = r0 + tid;
            const int j = r < nl ? sh.sorted_ties[r] : 0;
            const unsigned long long ms = r < nl ? fixed_mass(key_to_float(sh.tkey[j]), m) : 0ull;
            unsigned long long tot;
            const unsigned long long excl = block_exclusive_scan<unsigned long long>(ms, sh.red, &tot);
            if (r < nl && cum + excl < target) {
                const int64_t i = sh.ties[j];
                // other CTAs wrote neighbouring bytes: set the bit with a word atomic
                const uintptr_t a = reinterpret_cast<uintptr_t>(mybits + (i >> 3));
                atomicOr(reinterpret_cast<uint32_t *>(a & ~uintptr_t(3)), 1u << (((a & 3u) << 3) + (i & 7)));
                ++added;
            }
            cum += tot;
        }
        added = (int)block_sum<unsigned long long>((unsigned long long)added, sh.red);
        finalise((int)*reinterpret_cast<volatile uint32_t *>(&ctr[2]) + added);
        return;
    }
    // too many members in the crossing bucket (near-equal scores): the row on this CTA
    const int nk = topp_core(sh, n, p, kmax, kmin, load8, store8, add_kept);
    finalise(nk);
}

// ------------------------------------------------------------------ join

constexpr int kJoinThreads = kJoinChunk / 8;       // 8 candidates per thread
constexpr unsigned long long kLbAggregate = 1ull << 62, kLbInclusive = 2ull << 62;
constexpr unsigned long long kLbValue = (1ull << 62) - 1;

// The G rows' kept bitmaps of a group joined into per-candidate row masks
// (written to kept[]), and the candidates some row kept compacted, in order,
// into the next level's parent list (or, at level 1, the selection). One CTA
// per chunk of kJoinChunk candidates; the output offset of a chunk is the
// number kept by the chunks before it, found by looking back over their
// published counts (each chunk publishes its own count at once and its
// running total once known; every wait is bounded).
__global__ void __launch_bounds__(kJoinThreads)
join_kernel(Geo g, LevelWs lw, const uint8_t *keptbits, int level, zha_selection sel,
            unsigned long long *lb, int32_t *status) {
    __shared__ __align__(16) uint8_t sbits[32][kJoinChunk / 8];
    pdl_wait();
    __shared__ unsigned long long red[kJoinThreads / 32];
    __shared__ unsigned long long s_excl;
    const int chunk = blockIdx.x, grp = blockIdx.y;
    const int tid = threadIdx.x;
    const int64_t capv = g.capv[level];
    const int64_t bstride = g.bits_stride(level);
    const int64_t n = lw.count[grp];
    const int64_t nchunks = (n + kJoinChunk - 1) / kJoinChunk;
    if (n <= 0) {
        if (chunk == 0 && tid == 0) {
            if (level > 1)
                lw.pcount[grp] = 0;
            else
                sel.count[grp] = 0;
        }
        return;
    }
    if (chunk >= nchunks) return;
    unsigned long long *mylb = lb + (int64_t)grp * gridDim.x;
    const int64_t blk0 = (int64_t)chunk * (kJoinChunk / 8);
    const int nb = (int)min64(kJoinChunk / 8, ((n + 7) >> 3) - blk0);
    // 1. the rows' bitmap bytes of this chunk, 16 bytes per load
    const uint8_t *gbits = keptbits + (int64_t)grp * g.G * bstride + blk0;
    constexpr int kVec = kJoinChunk / 8 / 16;         // 16-byte words per row and chunk
    for (int i = tid; i < g.G * kVec; i += blockDim.x) {
        const int h = i / kVec, j = i % kVec;
        uint4 w = make_uint4(0, 0, 0, 0);
        if (j * 16 < nb && blk0 + j * 16 + 16 <= bstride)
            w = __ldcg(reinterpret_cast<const uint4 *>(gbits + h * bstride) + j);
        else if (j * 16 < nb) {
            uint8_t tmp[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) tmp[k] = (blk0 + j * 16 + k < bstride) ? __ldcg(gbits + h * bstride + j * 16 + k) : 0;
            w = *reinterpret_cast<const uint4 *>(tmp);
        }
        *reinterpret_cast<uint4 *>(&sbits[h][j * 16]) = w;
    }
    __syncthreads();
    // 2. row masks of this thread's 8 candidates
    uint32_t km[8];
#pragma unroll
    for (int v = 0; v < 8; ++v) km[v] = 0u;
    const bool mine = tid < nb;
    if (mine) {
        for (int h = 0; h < g.G; ++h) {
            const uint32_t b = sbits[h][tid];
#pragma unroll
            for (int v = 0; v < 8; ++v) km[v] |= ((b >> v) & 1u) << h;
        }
        uint4 *kp = reinterpret_cast<uint4 *>(lw.kept + grp * capv + ((blk0 + tid) << 3));
        kp[0] = make_uint4(km[0], km[1], km[2], km[3]);
        kp[1] = make_uint4(km[4], km[5], km[6], km[7]);
    }
    int cnt = 0;
#pragma unroll
    for (int v = 0; v < 8; ++v) cnt += km[v] != 0u;
    unsigned long long total;
    const unsigned long long local = block_exclusive_scan<unsigned long long>((unsigned long long)cnt, red, &total);
    // 3. running total of the chunks before this one: warp 0 reads the
    // published words of 32 predecessors at once, adds the counts up to the
    // nearest running total, and moves on by 32 if there is none yet
    if (tid < 32) {
        if (tid == 0) {
            __threadfence();
            atomicExch(&mylb[chunk], (chunk == 0 ? kLbInclusive : kLbAggregate) | total);
        }
        unsigned long long excl = 0ull;
        int64_t end_pc = chunk;                   // predecessors [.., end_pc) still to add
        const long long t0 = clock64();
        while (end_pc > 0) {
            const int64_t pc = end_pc - 1 - tid;  // lane 0: nearest predecessor
            const unsigned long long w =
                pc >= 0 ? *reinterpret_cast<volatile unsigned long long *>(&mylb[pc]) : (2ull << 62);
            const uint32_t st = (uint32_t)(w >> 62);
            // the nearest lane holding a running total (lanes past the first chunk count as one)
            const uint32_t incl = __ballot_sync(0xffffffffu, st == 2u);
            const int stop = incl ? __ffs(incl) - 1 : 31;
            const uint32_t missing = __ballot_sync(0xffffffffu, st == 0u) & (stop == 31 ? 0xffffffffu : ((2u << stop) - 1u));
            if (missing) {
                if (__any_sync(0xffffffffu, clock64() - t0 > kSpinCycles)) {   // same decision in every lane
                    if (tid == 0) set_status(status, ZHA_ERR_TIMEOUT);
                    break;
                }
                __nanosleep(32);
                continue;
            }
            unsigned long long v = (tid <= stop && pc >= 0) ? (w & kLbValue) : 0ull;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            excl += v;
            if (incl) break;
            end_pc -= 32;
        }
        if (tid == 0) {
            if (chunk > 0) {
                __threadfence();
                atomicExch(&mylb[chunk], kLbInclusive | (excl + total));
            }
            s_excl = excl;
        }
    }
    __syncthreads();
    // 4. the kept candidates, in order
    const int64_t base = (int64_t)s_excl + (int64_t)local;
    int32_t *out_idx;
    uint32_t *out_mask;
    if (level > 1) {
        out_idx = lw.plist + grp * g.cap[level];
        out_mask = lw.pmask + grp * g.cap[level];
    } else {
        out_idx = sel.leaf_idx + grp * g.cap[1];
        out_mask = sel.head_mask + grp * g.cap[1];
    }
    if (mine && cnt) {
        const int32_t *cand = lw.cand + grp * capv + ((blk0 + tid) << 3);
        const int4 c0 = *reinterpret_cast<const int4 *>(cand);
        const int4 c1 = *reinterpret_cast<const int4 *>(cand + 4);
        const int32_t cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        int64_t o = base;
#pragma unroll
        for (int v = 0; v < 8; ++v)
            if (km[v]) {
                out_idx[o] = cv[v];
                out_mask[o] = km[v];
                ++o;
            }
    }
    if (chunk == nchunks - 1 && tid == 0) {
        const int32_t m = (int32_t)(s_excl + total);
        if (level > 1)
            lw.pcount[grp] = m;
        else
            sel.count[grp] = m;
    }
    pdl_trigger();
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
    topp_core(
        sh, n, p, 0u, 0xffffffffu,
        [&](int64_t blk, float (&e)[8]) {
            uint32_t mb = 0u;
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const int64_t i = (blk << 3) + v;
                const bool in = i < n;
                e[v] = in ? sc[i] : 0.f;
                mb |= in ? (1u << v) : 0u;
            }
            return mb;
        },
        [&](int64_t blk, uint32_t kb) {
#pragma unroll
            for (int v = 0; v < 8; ++v)
                if ((blk << 3) + v < n) kp[(blk << 3) + v] = (uint8_t)((kb >> v) & 1u);
        },
        [&](int64_t i) { kp[i] = 1; });
}

// Scoring CTAs (128 threads, up to ~170 registers) resident on the current
// device at once: three per SM.
int64_t score_wave() {
    static int64_t wave[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (wave[dev] == 0) {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        wave[dev] = (int64_t)sms * 3;
    }
    return wave[dev];
}

// CTAs of select_split_kernel that fit on the current device at once (0: none known)
int64_t split_slots() {
    static int64_t slots[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (slots[dev] == 0) {
        int sms = 0, per_sm = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, select_split_kernel, kSplitThreads, 0) !=
                cudaSuccess)
            return 0;
        slots[dev] = (int64_t)sms * per_sm;
    }
    return slots[dev];
}

}  // namespace

// The fused route covers bf16 trees with native summaries, 16 reference
// planes per node and at most 8 query rows per group (single queries).
bool fused_route_supported(const Geo &g) {
    return g.dtype == ZHA_BF16 && !g.mx() && g.R == 16 && g.G <= 8 && g.T == 1 && g.lag == 0 &&
           (g.d == 64 || g.d == 128);
}

#define ZHA_TRY(call)                         \
    do {                                      \
        const cudaError_t le_ = (call);       \
        if (le_ != cudaSuccess) return le_;   \
    } while (0)

cudaError_t launch_route(const Geo &g, const void *tree, const void *q, const int32_t *lens,
                         const float *p_levels, const zha_selection &sel, void *ws,
                         int32_t *status, cudaStream_t st, bool init) {
    static const char *score_names[] = {"", "score[l1]", "score[l2]", "score[l3]", "score[l4]",
                                        "score[l5]", "score[l6]", "score[l7]", "score[l8]"};
    static const char *select_names[] = {"", "select[l1]", "select[l2]", "select[l3]", "select[l4]",
                                         "select[l5]", "select[l6]", "select[l7]", "select[l8]"};
    static const char *join_names[] = {"", "join[l1]", "join[l2]", "join[l3]", "join[l4]",
                                       "join[l5]", "join[l6]", "join[l7]", "join[l8]"};
    // look-back words of each level's join: [groups][chunks of that level]
    int64_t lb_off[kMaxLevels + 2] = {};
    for (int l = 1; l <= g.L; ++l)
        lb_off[l + 1] = lb_off[l] + (int64_t)g.groups() * ((g.capv[l] + kJoinChunk - 1) / kJoinChunk);
    const int groups = g.groups();
    cudaError_t e = cudaSuccess;
    if (init) {
        ProfScope ps("route_init", st);
        e = launch_pdl(route_init_kernel, dim3(groups), dim3(64), 0, st, g, route_state(g, ws), lens, status);
        if (e != cudaSuccess) return e;
    }
    const char *tb = static_cast<const char *>(tree);
    if ((g.flags & ZHA_FLAG_FUSED_ROUTE) && fused_route_supported(g)) {
        FusedArgs a{};
        for (int l = 1; l <= g.L; ++l) {
            a.lw[l] = level_ws(g, ws, l);
            a.p[l] = p_levels[l - 1];
            a.mu[l] = reinterpret_cast<const __nv_bfloat16 *>(tb + g.mu_off[l]);
            a.bias[l] = reinterpret_cast<const float *>(tb + g.bias_off[l]);
        }
        // clusters of 16 where every group's cluster is resident at once, else 8
        static const int max16 = [] {
            const int bytes = (int)sizeof(FusedShared);
            for (auto k : {route_fused_kernel<128, 8>, route_fused_kernel<64, 8>, route_fused_kernel<128, 16>,
                           route_fused_kernel<64, 16>})
                if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
                    return -1;
            for (auto k : {route_fused_kernel<128, 16>, route_fused_kernel<64, 16>})
                if (cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
                    return 0;
            cudaLaunchConfig_t c{};
            c.gridDim = dim3(16, 1);
            c.blockDim = dim3(kSmallThreads);
            c.dynamicSmemBytes = bytes;
            cudaLaunchAttribute at;
            at.id = cudaLaunchAttributeClusterDimension;
            at.val.clusterDim.x = 16;
            at.val.clusterDim.y = 1;
            at.val.clusterDim.z = 1;
            c.attrs = &at;
            c.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, route_fused_kernel<128, 16>, &c) != cudaSuccess) {
                (void)cudaGetLastError();
                return 0;
            }
            return n;
        }();
        if (max16 < 0) return cudaErrorInvalidConfiguration;
        const int cl = max16 >= groups ? 16 : 8;
        cudaLaunchConfig_t c{};
        c.gridDim = dim3(cl, groups);
        c.blockDim = dim3(kSmallThreads);
        c.dynamicSmemBytes = sizeof(FusedShared);
        c.stream = st;
        cudaLaunchAttribute at[2];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = cl;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at[1].val.programmaticStreamSerializationAllowed = 1;
        c.attrs = at;
        c.numAttrs = 2;
        ProfScope ps("route_fused", st);
        const auto *qq = static_cast<const __nv_bfloat16 *>(q);
        if (g.d == 128)
            e = cl == 16 ? cudaLaunchKernelEx(&c, route_fused_kernel<128, 16>, g, a, qq, lens, sel)
                         : cudaLaunchKernelEx(&c, route_fused_kernel<128, 8>, g, a, qq, lens, sel);
        else
            e = cl == 16 ? cudaLaunchKernelEx(&c, route_fused_kernel<64, 16>, g, a, qq, lens, sel)
                         : cudaLaunchKernelEx(&c, route_fused_kernel<64, 8>, g, a, qq, lens, sel);
        return e;
    }
    for (int level = g.L; level >= 1; --level) {
        LevelWs lw = level_ws(g, ws, level);
        LevelWs up = level < g.L ? level_ws(g, ws, level + 1) : lw;
        const int64_t capv = g.capv[level];
        int fuse_join = 0;
        {
            ProfScope ps(score_names[level], st);
            // a scoring grid of several waves starts plainly: launched early
            // behind the kernel before it, such grids made the 256K B=4 step
            // 29 us slower (most likely their first wave starts unevenly on
            // the SMs that kernel still holds), while one-wave grids gain
            bool one_wave = true;
            if (g.mx()) {
                const auto *mu = reinterpret_cast<const uint8_t *>(tb + g.mu_off[level]);
                const auto *scl = reinterpret_cast<const uint8_t *>(tb + g.sc_off[level]);
                const auto *bias = reinterpret_cast<const float *>(tb + g.bias_off[level]);
                const auto *qq = static_cast<const __nv_bfloat16 *>(q);
                const int64_t want = (capv + kScoreWarps - 1) / kScoreWarps;
                const int per_group = (int)max64(1, min64(want, (148 * 8 + groups - 1) / groups));
                dim3 grid(per_group, groups);
                one_wave = (int64_t)per_group * groups <= score_wave();
                const int mt = g.R > 16 ? 2 : 1, nt = g.G > 16 ? 4 : (g.G > 8 ? 2 : 1);
#define ZHA_SCORE_MX(D, MT, NT, U) \
    ZHA_TRY(launch_pdl_if(one_wave, score_mx8_kernel<D, MT, NT, U>, grid, dim3(kScoreWarps * 32), 0, st, g, mu, scl, bias, qq, \
                       lens, lw, up, level))
#define ZHA_SCORE_MX_N(D, MT, U1) \
    do { if (nt == 1) ZHA_SCORE_MX(D, MT, 1, U1); else if (nt == 2) ZHA_SCORE_MX(D, MT, 2, 2); \
         else ZHA_SCORE_MX(D, MT, 4, 1); } while (0)
                if (g.d == 128) {
                    if (mt == 1) ZHA_SCORE_MX_N(128, 1, 2); else ZHA_SCORE_MX_N(128, 2, 2);
                } else {
                    if (mt == 1) ZHA_SCORE_MX_N(64, 1, 2); else ZHA_SCORE_MX_N(64, 2, 2);
                }
#undef ZHA_SCORE_MX_N
#undef ZHA_SCORE_MX
            } else if (g.dtype == ZHA_BF16 && (g.flags & ZHA_FLAG_TCGEN05) && score_tc_supported(g)) {
                e = launch_score_tc(g, tb + g.mu_off[level], reinterpret_cast<const float *>(tb + g.bias_off[level]),
                                    q, lens, level, lw.cand, lw.cmask, lw.scores, lw.count, lw.maxkey, lw.minkey,
                                    up.plist, up.pmask, up.pcount, status, st);
                if (e != cudaSuccess) return e;
            } else if (g.dtype == ZHA_BF16 && g.R < 16 && (g.R & (g.R - 1)) == 0) {
                const auto *mu = reinterpret_cast<const __nv_bfloat16 *>(tb + g.mu_off[level]);
                const auto *bias = reinterpret_cast<const float *>(tb + g.bias_off[level]);
                const auto *qq = static_cast<const __nv_bfloat16 *>(q);
                const int cpt = 16 / g.R;
                const int64_t want = (capv + kScoreWarps * cpt - 1) / (kScoreWarps * cpt);
                const int per_group = (int)max64(1, min64(want, (148 * 8 + groups - 1) / groups));
                dim3 grid(per_group, groups);
                one_wave = (int64_t)per_group * groups <= score_wave();
                const int rl = __builtin_ctz(g.R);
#define ZHA_SCORE_PACK(D, NT, RL) \
    ZHA_TRY(launch_pdl_if(one_wave, score_pack_kernel<D, NT, RL, 2>, grid, dim3(kScoreWarps * 32), 0, st, g, mu, bias, qq, lens, \
                       lw, up, level))
#define ZHA_SCORE_PACK_R(D, NT) \
    do { if (rl == 0) ZHA_SCORE_PACK(D, NT, 0); else if (rl == 1) ZHA_SCORE_PACK(D, NT, 1); \
         else if (rl == 2) ZHA_SCORE_PACK(D, NT, 2); else ZHA_SCORE_PACK(D, NT, 3); } while (0)
                if (g.d == 128) {
                    if (g.G > 16) ZHA_SCORE_PACK_R(128, 4);
                    else if (g.G > 8) ZHA_SCORE_PACK_R(128, 2);
                    else ZHA_SCORE_PACK_R(128, 1);
                } else {
                    if (g.G > 16) ZHA_SCORE_PACK_R(64, 4);
                    else if (g.G > 8) ZHA_SCORE_PACK_R(64, 2);
                    else ZHA_SCORE_PACK_R(64, 1);
                }
#undef ZHA_SCORE_PACK_R
#undef ZHA_SCORE_PACK
            } else if (g.dtype == ZHA_BF16) {
                const auto *mu = reinterpret_cast<const __nv_bfloat16 *>(tb + g.mu_off[level]);
                const auto *bias = reinterpret_cast<const float *>(tb + g.bias_off[level]);
                const auto *qq = static_cast<const __nv_bfloat16 *>(q);
                const int64_t want = (capv + kScoreWarps - 1) / kScoreWarps;
                const int per_group = (int)max64(1, min64(want, (148 * 8 + groups - 1) / groups));
                dim3 grid(per_group, groups);
                one_wave = (int64_t)per_group * groups <= score_wave();
                const int mt = g.R > 16 ? 2 : 1, nt = g.G > 16 ? 4 : (g.G > 8 ? 2 : 1);
#define ZHA_SCORE(D, MT, NT) \
    ZHA_TRY(launch_pdl_if(one_wave, score_mma_kernel<D, MT, NT>, grid, dim3(kScoreWarps * 32), 0, st, g, mu, bias, qq, lens, lw, \
                       up, level))
#define ZHA_SCORE_N(D, MT) \
    do { if (nt == 1) ZHA_SCORE(D, MT, 1); else if (nt == 2) ZHA_SCORE(D, MT, 2); else ZHA_SCORE(D, MT, 4); } while (0)
                if (g.d == 128) {
                    if (mt == 1) ZHA_SCORE_N(128, 1); else ZHA_SCORE_N(128, 2);
                } else {
                    if (mt == 1) ZHA_SCORE_N(64, 1); else ZHA_SCORE_N(64, 2);
                }
#undef ZHA_SCORE_N
#undef ZHA_SCORE
            } else {
                const auto *mu = reinterpret_cast<const float *>(tb + g.mu_off[level]);
                const auto *bias = reinterpret_cast<const float *>(tb + g.bias_off[level]);
                const auto *qq = static_cast<const float *>(q);
                const int per_group = (int)max64(1, min64(capv, (148 * 8 + groups - 1) / groups));
                dim3 grid(per_group, groups);
                one_wave = (int64_t)per_group * groups <= score_wave();
                if (g.d == 128)
                    ZHA_TRY(launch_pdl_if(one_wave, score_f32_kernel<128>, grid, dim3(128), 0, st, g, mu, bias, qq, lens, lw, up,
                                       level));
                else
                    ZHA_TRY(launch_pdl_if(one_wave, score_f32_kernel<64>, grid, dim3(128), 0, st, g, mu, bias, qq, lens, lw, up,
                                       level));
            }
        }
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        {
            ProfScope ps(select_names[level], st);
            uint8_t *keptbits = reinterpret_cast<uint8_t *>(static_cast<char *>(ws) + g.ws_keptbits[level]);
            // rows with many candidates: several CTAs per row, as many as can be resident together
            const int64_t rows = (int64_t)g.G * groups;
            const int S = (int)min64(capv / kSplitMinSlice, split_slots() / rows);
            // mid-size levels: the join runs in the last select CTA of each group, and
            // the CTAs are smaller (fewer warps at each of the selection's barriers)
            const int sel_threads = capv <= 8 * 256 ? 256 : kSelThreads;
            fuse_join = S < 2 && (capv >> 3) <= sel_threads && g.G * g.bits_stride(level) <= 32768;
            if (S < 2 && capv <= kSmallMax) {
                fuse_join = 1;
                ZHA_TRY(launch_pdl(select_small_kernel, dim3(groups), dim3(kSmallThreads), 0, st, g, lw, level,
                                   p_levels[level - 1], sel.level_kept, sel));
            } else if (S >= 2) {
                char *base = static_cast<char *>(ws);
                const SplitWs sw{reinterpret_cast<unsigned long long *>(base + g.ws_ghist),
                                 reinterpret_cast<int32_t *>(base + g.ws_glidx),
                                 reinterpret_cast<uint32_t *>(base + g.ws_glkey),
                                 reinterpret_cast<uint32_t *>(base + g.ws_gctr)};
                ZHA_TRY(launch_pdl(select_split_kernel, dim3(S, g.G, groups), dim3(kSplitThreads), 0, st, g, lw,
                                   keptbits, level, p_levels[level - 1], sel.level_kept, sw, status));
            } else {
                ZHA_TRY(launch_pdl(select_kernel, dim3(g.G, groups), dim3(sel_threads), 0, st, g, lw, keptbits, level,
                                   p_levels[level - 1], sel.level_kept, fuse_join, sel));
            }
        }
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        if (!fuse_join) {
            ProfScope ps(join_names[level], st);
            const uint8_t *keptbits = reinterpret_cast<const uint8_t *>(static_cast<char *>(ws) + g.ws_keptbits[level]);
            const int64_t chunks = (capv + kJoinChunk - 1) / kJoinChunk;
            unsigned long long *lb = reinterpret_cast<unsigned long long *>(static_cast<char *>(ws) + g.ws_lookback) +
                                     lb_off[level];
            ZHA_TRY(launch_pdl(join_kernel, dim3((unsigned)chunks, groups), dim3(kJoinThreads), 0, st, g, lw,
                               keptbits, level, sel, lb, status));
        }
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// ------------------------------------------------------- bounded-wait expiry
//
// The library's bounded device waits, run on conditions that nothing
// satisfies, with a caller-given limit: the counter barrier of the multi-CTA
// selection entered by one of two CTAs (the other returns without arriving,
// as a lost arrival would), and an mbarrier wait on a barrier that no copy or
// commit completes. Each must give up after its limit, set ZHA_ERR_TIMEOUT and
// return, leaving the context usable.

__device__ uint32_t g_expiry_ctr;

__global__ void wait_expiry_kernel(int kind, long long limit, int32_t *status) {
    __shared__ int ok_sh;
    __shared__ __align__(8) uint64_t bar;
    if (kind == ZHA_WAIT_ROW_BARRIER) {
        if (blockIdx.x == 1) return;   // the CTA that never arrives
        if (threadIdx.x == 0) g_expiry_ctr = 0u;
        row_barrier(&g_expiry_ctr, 2u, status, &ok_sh, limit);
    } else {
        if (blockIdx.x != 0) return;
        if (threadIdx.x == 0) mbar_init(smem_u32(&bar), 1u);
        __syncthreads();
        if (threadIdx.x == 0) mbar_wait_bounded(smem_u32(&bar), 0u, limit, nullptr, status);
        __syncthreads();
    }
}

cudaError_t launch_wait_expiry(int kind, long long limit, int32_t *status, cudaStream_t st) {
    ProfScope ps("wait_expiry", st);
    wait_expiry_kernel<<<2, 64, 0, st>>>(kind, limit, status);
    return cudaGetLastError();
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
