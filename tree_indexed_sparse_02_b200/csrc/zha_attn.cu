// zha_attn.cu -- exact attention over the routed tokens (and the dense
// comparison kernel), split-K flash decoding with a log-sum-exp merge.
//
// Page "Zyphra AI Introduces Zyphra Hierarchical Attention (ZHA)", explainer
// widget step 5: the final attention is exact, over the routed raw KV plus
// token 0 (the sink, section "How does top-p routing pick tokens") and the
// chunk being written.
//
// Every (sequence, KV head) group streams the union of its heads' tokens
// once; each token carries the bit mask of query heads that attend to it, so
// one K/V read serves all G heads of the group. The token stream of a group
// is: the kept leaf chunks (ascending), then the sink if no kept chunk holds
// it, then the current chunk if no kept chunk is it.
//
// bf16: per warp, 16 tokens at a time on tensor cores (mma.sync m16n8k16):
// S = Q K^T with the heads as the 16 rows, online softmax in registers in
// base 2, then O += P V with P taken straight from the S accumulators. K and V
// rows go global -> registers in fully used 32-byte sectors (coordinates of
// the QK product are permuted identically in Q and K; the value coordinates
// each lane owns are a contiguous block).
// fp32: one token per lane on CUDA cores, same partial format.
#include "zha_common.cuh"

namespace zha {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kAttnWarps = 4;

// Which cache position virtual token v of a group is, and which heads see it.
// All token counts fit in int32 (max_len <= 2^30).
struct TokenPlan {
    int N, cur_start, n1;
    int nsel, sel_tokens;  // kept leaf chunks, their tokens
    int a_len;             // sink span [0, a_len)
    int b_start, b_len;    // current-chunk span
    int nv;                // stream length
    int lc;                // log2(c)
    int blk_start;         // zha_decode_block: first block position (INT_MAX otherwise)
    int gq;                // query heads per position: row r is position r / gq of the block
    uint32_t all;
    const int32_t *leaf;
    const uint32_t *hmask;

    // rows that see position pos of the always-attended spans: all of them,
    // except for a block token, which the block's earlier positions do not see
    __device__ __forceinline__ uint32_t span_mask(int pos) const {
        if (pos < blk_start) return all;
        const int k = (pos - blk_start) * gq;
        return k >= 32 ? 0u : (all & ~((1u << k) - 1u));
    }

    __device__ __forceinline__ void at(int v, int &pos, uint32_t &mask, int32_t *status) const {
        if (v < sel_tokens) {
            const int e = v >> lc;
            const int lf = __ldg(&leaf[e]);
            if ((unsigned)lf >= (unsigned)n1) {
                set_status(status, ZHA_ERR_INVALID_ARG);
                pos = 0;
                mask = 0u;
                return;
            }
            pos = (lf << lc) | (v & ((1 << lc) - 1));
            mask = __ldg(&hmask[e]) | ((pos == 0 || pos >= cur_start) ? span_mask(pos) : 0u);
            return;
        }
        v -= sel_tokens;
        if (v < a_len) {
            pos = 0;
            mask = all;
            return;
        }
        v -= a_len;
        if (v < b_len) {
            pos = b_start + v;
            mask = span_mask(pos);
            return;
        }
        pos = 0;
        mask = 0u;
    }
};

__device__ __forceinline__ TokenPlan make_plan(const Geo &g, const int32_t *lens, int grp,
                                               const zha_selection *sel, bool dense,
                                               int32_t *status) {
    TokenPlan tp{};
    const int b = grp / g.Hkv;
    int N = lens[b];
    if (N < 0 || N > g.max_len) {
        set_status(status, ZHA_ERR_CAPACITY);
        N = 0;
    }
    tp.N = N;
    tp.lc = __ffs(g.c) - 1;
    tp.all = g.G >= 32 ? 0xffffffffu : ((1u << g.G) - 1u);
    tp.n1 = N >> tp.lc;
    tp.blk_start = 0x7fffffff;
    tp.gq = g.Gq;
    if (dense || N == 0) {
        tp.b_start = 0;
        tp.b_len = N;
        tp.cur_start = 0;
        tp.nv = N;
        return tp;
    }
    if (g.block) {
        // the tree holds the first N - T tokens; the rest is the cached tail
        // after its last complete chunk plus the block, attended causally
        int n_tree = N - g.T;
        if (n_tree < 0) {
            set_status(status, ZHA_ERR_INVALID_ARG);
            n_tree = 0;
        }
        tp.blk_start = n_tree;
        tp.n1 = n_tree >> tp.lc;
        tp.cur_start = tp.n1 << tp.lc;
    } else {
        tp.cur_start = (int)current_chunk_start(N, g.c, g.flags);
    }
    int ns = sel->count[grp];
    if (ns < 0 || ns > g.cap[1]) {
        set_status(status, ZHA_ERR_INVALID_ARG);
        ns = 0;
    }
    tp.leaf = sel->leaf_idx + grp * g.cap[1];
    tp.hmask = sel->head_mask + grp * g.cap[1];
    tp.nsel = ns;
    tp.sel_tokens = ns << tp.lc;
    const bool has_leaf0 = ns > 0 && tp.leaf[0] == 0;
    const bool cur_complete = tp.cur_start + g.c <= N;
    const bool cur_covered = cur_complete && ns > 0 && (tp.leaf[ns - 1] << tp.lc) == tp.cur_start;
    tp.a_len = (!has_leaf0 && tp.cur_start > 0) ? 1 : 0;
    tp.b_start = tp.cur_start;
    tp.b_len = cur_covered ? 0 : N - tp.cur_start;
    tp.nv = tp.sel_tokens + tp.a_len + tp.b_len;
    return tp;
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Partials: ml[((grp*S + s)*G + h)*2 + {0,1}] = (max in log2 units, sum),
// o[((grp*S + s)*G + h)*D + dim] (unnormalised).

constexpr int kTile = 64;    // tokens per pipeline stage (16 per warp)
constexpr int kStages = 3;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
                 "r"(valid ? 16 : 0));
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(dst), "l"(src));
}
__device__ __forceinline__ uint32_t sbase_of(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                          uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

template <int D>
__host__ __device__ constexpr int attn_smem_bytes() {
    return kStages * 2 * kTile * D * 2;
}

// bf16 split-K attention. The CTA's 128 threads stream 64-token tiles of the
// group's token list (K and V rows, gathered by position) into a 3-stage
// shared-memory ring with cp.async; rows are stored with their 16-byte
// chunks XOR-swizzled by (row & 7) so that ldmatrix reads of 8 rows at one
// column are bank-conflict free. Each warp then computes its 16 tokens for
// MT tiles of 16 query rows (MT = 2 for groups of more than 16 rows: a
// block of several query positions), so each K/V fragment read from shared
// memory serves all of them and the group's K/V cross DRAM once.
template <int D, int MT>
__global__ void __launch_bounds__(kAttnWarps * 32)
attn_mma_kernel(Geo g, const __nv_bfloat16 *q, const __nv_bfloat16 *K, const __nv_bfloat16 *V,
                const int32_t *lens, zha_selection sel, int dense, float *part_ml, float *part_o,
                int32_t *status) {
    constexpr int ROWB = D * 2;            // bytes per token row
    constexpr int CH = ROWB / 16;          // 16-byte chunks per row
    constexpr int TILE_B = kTile * ROWB;
    constexpr int STAGE_B = 2 * TILE_B;    // K tile then V tile
    constexpr int NJ = D / 8;              // n-tiles of the PV product
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(smem);

    constexpr int RB = 16 * MT;            // query rows per CTA
    const int grp = blockIdx.z, split = blockIdx.y, S = gridDim.y;
    const int rbase = blockIdx.x * RB;     // this CTA's query rows of the group
    const int b = grp / g.Hkv, kvh = grp % g.Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gq = lane >> 2, t = lane & 3;
    const __nv_bfloat16 *Kg = K + (int64_t)grp * g.max_len * D;
    const __nv_bfloat16 *Vg = V + (int64_t)grp * g.max_len * D;

    // Q as the A operand: in m-tile mt, rows gq and gq+8 are query rows
    // rbase + 16 mt + gq (+8) of this group (rows >= G are zero)
    uint32_t qf[MT][D / 16][4];
    uint32_t mrow[MT][2];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const int h0 = rbase + 16 * mt + gq, h1 = h0 + 8;
        const uint32_t *q0 = reinterpret_cast<const uint32_t *>(q + g.qrow(b, kvh, h0 < g.G ? h0 : 0) * D);
        const uint32_t *q1 = reinterpret_cast<const uint32_t *>(q + g.qrow(b, kvh, h1 < g.G ? h1 : 0) * D);
#pragma unroll
        for (int st = 0; st < D / 16; ++st) {
            qf[mt][st][0] = h0 < g.G ? q0[st * 8 + t] : 0u;
            qf[mt][st][1] = h1 < g.G ? q1[st * 8 + t] : 0u;
            qf[mt][st][2] = h0 < g.G ? q0[st * 8 + 4 + t] : 0u;
            qf[mt][st][3] = h1 < g.G ? q1[st * 8 + 4 + t] : 0u;
        }
        mrow[mt][0] = h0 < g.G ? (1u << h0) : 0u;
        mrow[mt][1] = h1 < g.G ? (1u << h1) : 0u;
    }
    // the queries are the call's input; the cache, lengths and selection come from earlier kernels
    pdl_wait();
    const TokenPlan tp = make_plan(g, lens, grp, &sel, dense != 0, status);

    const int ntiles = (tp.nv + kTile - 1) / kTile;
    const int t_lo = (int)((int64_t)ntiles * split / S), t_hi = (int)((int64_t)ntiles * (split + 1) / S);

    // Each warp owns rows 16 w .. 16 w + 15 of every tile: it copies their
    // selection entries (kept leaf, head mask) into a shared-memory ring
    // kAhead tiles ahead of their compute, with cp.async in the same commit
    // groups as the K/V copies (so waiting on them costs nothing extra),
    // turns them into cache positions and masks when it issues the tile's K/V
    // copies, and computes on the tile, so the pipeline needs no block-wide
    // barrier.
    constexpr int kAhead = kStages + 1;         // lookups copied this many tiles ahead
    constexpr int kLook = kAhead;               // lookup ring slots (tile x: slot x % kLook)
    constexpr int kSlots = kStages + 1;         // position/mask slots (tile x: slot x % kSlots)
    __shared__ int spos[kSlots][kTile];
    __shared__ uint32_t smask[kSlots][kTile];
    __shared__ int32_t lk_leaf[kLook][kTile];
    __shared__ uint32_t lk_hm[kLook][kTile];
    const int lrow = warp * 16 + (lane & 15);
    // selection entries of the warp's rows of tile `tile` (lanes 0..15, one row each)
    auto look = [&](int tile) {
        const int v = tile * kTile + lrow;
        if (lane < 16 && tile < t_hi && v < tp.sel_tokens) {
            const int slot = (tile - t_lo) % kLook;
            cp_async4(sbase_of(&lk_leaf[slot][lrow]), tp.leaf + (v >> tp.lc));
            cp_async4(sbase_of(&lk_hm[slot][lrow]), tp.hmask + (v >> tp.lc));
        }
    };
    // positions and masks of the warp's rows of `tile` from its (completed) entries
    auto resolve = [&](int tile) {
        if (lane < 16) {
            const int v = tile * kTile + lrow;
            int pos = 0;
            uint32_t m = 0u;
            if (v < tp.sel_tokens) {
                const int slot = (tile - t_lo) % kLook;
                const int lf = lk_leaf[slot][lrow];
                if ((unsigned)lf >= (unsigned)tp.n1) {
                    set_status(status, ZHA_ERR_INVALID_ARG);
                } else {
                    pos = (lf << tp.lc) | (v & ((1 << tp.lc) - 1));
                    m = lk_hm[slot][lrow] | ((pos == 0 || pos >= tp.cur_start) ? tp.span_mask(pos) : 0u);
                }
            } else if (v < tp.nv) {
                tp.at(v, pos, m, status);
            }
            spos[(tile - t_lo) % kSlots][lrow] = pos;
            smask[(tile - t_lo) % kSlots][lrow] = m;
        }
    };
    // the warp's 16 rows, one 16-byte chunk of K and of V per lane and step
    auto issue = [&](int tile, int stage) {
        const uint32_t kb = sbase + stage * STAGE_B, vb = kb + TILE_B;
        const int slot = (tile - t_lo) % kSlots;
#pragma unroll
        for (int k = 0; k < 16 * CH / 32; ++k) {
            const int c = lane + k * 32;
            const int row = warp * 16 + c / CH, ch = c % CH;
            const int pos = spos[slot][row];
            const bool valid = tile * kTile + row < tp.nv;
            const uint32_t off = row * ROWB + ((ch ^ (row & 7)) << 4);
            cp_async16(kb + off, Kg + (int64_t)pos * D + ch * 8, valid);
            cp_async16(vb + off, Vg + (int64_t)pos * D + ch * 8, valid);
        }
    };

    const float sl2 = g.s * kLog2e;
    float m_run[MT][2], l_run[MT][2];
    float o[MT][NJ][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        m_run[mt][0] = m_run[mt][1] = -INFINITY;
        l_run[mt][0] = l_run[mt][1] = 0.f;
#pragma unroll
        for (int j = 0; j < NJ; ++j) o[mt][j][0] = o[mt][j][1] = o[mt][j][2] = o[mt][j][3] = 0.f;
    }

    // Commit groups: the prologue's lookups of tiles t_lo .. t_lo + kAhead - 1
    // (waited for at once), then one group per tile of the first kStages - 1
    // tiles' K/V, then, in iteration it, the K/V of tile it + kStages - 1 with
    // the lookups of tile it + kAhead. The wait at the top of iteration it
    // leaves only the newest group pending, so the K/V of tile it and the
    // lookups of tile it + kStages - 1 (committed kStages - 1 groups earlier
    // or in the prologue) are complete.
#pragma unroll
    for (int st = 0; st < kAhead; ++st) look(t_lo + st);
    cp_async_commit();
    cp_async_wait<0>();
    __syncwarp();
#pragma unroll
    for (int st = 0; st < kStages - 1; ++st) {
        if (t_lo + st < t_hi) resolve(t_lo + st);
        __syncwarp();
        if (t_lo + st < t_hi) issue(t_lo + st, st);
        cp_async_commit();
    }
    for (int it = 0; t_lo + it < t_hi; ++it) {
        cp_async_wait<kStages - 2>();
        // contiguous (dense) streams keep the warps in step, so that the CTA's
        // copies of a tile hit the same DRAM pages together
        if (dense) __syncthreads();
        else __syncwarp();
        {
            const int nt = t_lo + it + kStages - 1;
            if (nt < t_hi) resolve(nt);
            __syncwarp();
            if (nt < t_hi) issue(nt, (it + kStages - 1) % kStages);
            look(t_lo + it + kAhead);
            cp_async_commit();
        }
        const int stage = it % kStages;
        const uint32_t kb = sbase + stage * STAGE_B, vb = kb + TILE_B;
        const int row0 = warp * 16;
        // heads that see this lane's S columns / V rows: tokens 2t, 2t+1, 8+2t, 9+2t
        uint32_t mv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) mv[u] = smask[it % kSlots][row0 + (u >> 1) * 8 + 2 * t + (u & 1)];
        float s0[MT][4], s1[MT][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int u = 0; u < 4; ++u) s0[mt][u] = s1[mt][u] = 0.f;
#pragma unroll
        for (int kp = 0; kp < D / 32; ++kp) {
            uint32_t b0, b1, b2, b3;
            const int ch = 4 * kp + (lane >> 3);
            int row = row0 + (lane & 7);
            ldsm_x4(kb + row * ROWB + ((ch ^ (row & 7)) << 4), b0, b1, b2, b3);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const uint32_t(&qa)[4] = qf[mt][2 * kp];
                const uint32_t(&qb)[4] = qf[mt][2 * kp + 1];
                mma16816(s0[mt], qa[0], qa[1], qa[2], qa[3], b0, b1);
                mma16816(s0[mt], qb[0], qb[1], qb[2], qb[3], b2, b3);
            }
            row += 8;
            ldsm_x4(kb + row * ROWB + ((ch ^ (row & 7)) << 4), b0, b1, b2, b3);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const uint32_t(&qa)[4] = qf[mt][2 * kp];
                const uint32_t(&qb)[4] = qf[mt][2 * kp + 1];
                mma16816(s1[mt], qa[0], qa[1], qa[2], qa[3], b0, b1);
                mma16816(s1[mt], qb[0], qb[1], qb[2], qb[3], b2, b3);
            }
        }
        uint32_t pa[MT][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            float x[2][4];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                x[r][0] = (mv[0] & mrow[mt][r]) ? s0[mt][2 * r + 0] * sl2 : -INFINITY;
                x[r][1] = (mv[1] & mrow[mt][r]) ? s0[mt][2 * r + 1] * sl2 : -INFINITY;
                x[r][2] = (mv[2] & mrow[mt][r]) ? s1[mt][2 * r + 0] * sl2 : -INFINITY;
                x[r][3] = (mv[3] & mrow[mt][r]) ? s1[mt][2 * r + 1] * sl2 : -INFINITY;
            }
            float p[2][4];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                float mx = fmaxf(fmaxf(x[r][0], x[r][1]), fmaxf(x[r][2], x[r][3]));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                const float m_new = fmaxf(m_run[mt][r], mx);
                const float corr = (m_run[mt][r] == -INFINITY) ? 0.f : exp2f(m_run[mt][r] - m_new);
                float ls = 0.f;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    p[r][u] = (x[r][u] == -INFINITY) ? 0.f : exp2f(x[r][u] - m_new);
                    ls += p[r][u];
                }
                l_run[mt][r] = l_run[mt][r] * corr + ls;
                m_run[mt][r] = m_new;
#pragma unroll
                for (int j = 0; j < NJ; ++j) {
                    o[mt][j][2 * r] *= corr;
                    o[mt][j][2 * r + 1] *= corr;
                }
            }
            pa[mt][0] = pack_bf16(p[0][0], p[0][1]);
            pa[mt][1] = pack_bf16(p[1][0], p[1][1]);
            pa[mt][2] = pack_bf16(p[0][2], p[0][3]);
            pa[mt][3] = pack_bf16(p[1][2], p[1][3]);
        }
#pragma unroll
        for (int jp = 0; jp < NJ / 2; ++jp) {
            uint32_t b0, b1, b2, b3;
            const int row = row0 + (lane & 7) + ((lane >> 3) & 1) * 8;
            const int ch = 2 * jp + (lane >> 4);
            ldsm_x4_t(vb + row * ROWB + ((ch ^ (row & 7)) << 4), b0, b1, b2, b3);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                mma16816(o[mt][2 * jp], pa[mt][0], pa[mt][1], pa[mt][2], pa[mt][3], b0, b1);
                mma16816(o[mt][2 * jp + 1], pa[mt][0], pa[mt][1], pa[mt][2], pa[mt][3], b2, b3);
            }
        }
    }
    cp_async_wait<0>();
    __syncthreads();
    // row sums across the 4 lanes of a row, then the 4 warps' partials via
    // shared memory (in the ring's space: [warps][RB] maxima and sums, then
    // [warps][RB][D + 4] outputs)
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            l_run[mt][r] += __shfl_xor_sync(0xffffffffu, l_run[mt][r], 1);
            l_run[mt][r] += __shfl_xor_sync(0xffffffffu, l_run[mt][r], 2);
        }
    float *sm_m = reinterpret_cast<float *>(smem);                 // [warps][RB]
    float *sm_l = sm_m + kAttnWarps * RB;                           // [warps][RB]
    float *sm_o = sm_l + kAttnWarps * RB;                           // [warps][RB][D + 4]
    constexpr int OS = D + 4;
    static_assert((2 * kAttnWarps * RB + kAttnWarps * RB * OS) * 4 <= attn_smem_bytes<D>(),
                  "the epilogue fits in the ring");
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const int r0 = warp * RB + 16 * mt + gq;
        if (t == 0) {
            sm_m[r0] = m_run[mt][0];
            sm_m[r0 + 8] = m_run[mt][1];
            sm_l[r0] = l_run[mt][0];
            sm_l[r0 + 8] = l_run[mt][1];
        }
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
            sm_o[r0 * OS + 8 * j + 2 * t] = o[mt][j][0];
            sm_o[r0 * OS + 8 * j + 2 * t + 1] = o[mt][j][1];
            sm_o[(r0 + 8) * OS + 8 * j + 2 * t] = o[mt][j][2];
            sm_o[(r0 + 8) * OS + 8 * j + 2 * t + 1] = o[mt][j][3];
        }
    }
    __syncthreads();
    const int64_t pbase = ((int64_t)grp * S + split) * g.G + rbase;
    const int rows = min(RB, g.G - rbase);
    for (int i = threadIdx.x; i < rows * D; i += blockDim.x) {
        const int h = i / D, dim = i % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, sm_m[w * RB + h]);
        float L = 0.f, acc = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kAttnWarps; ++w) {
                const float mw = sm_m[w * RB + h];
                if (mw == -INFINITY) continue;
                const float f = exp2f(mw - M);
                L += sm_l[w * RB + h] * f;
                acc += sm_o[(w * RB + h) * OS + dim] * f;
            }
        }
        part_o[(pbase + h) * D + dim] = acc;
        if (dim == 0) {
            part_ml[(pbase + h) * 2 + 0] = M;
            part_ml[(pbase + h) * 2 + 1] = L;
        }
    }
    pdl_trigger();
}

// CUDA-core variant (fp32 inputs, or any dtype for checking): one token per lane.
template <typename T, int D>
__global__ void __launch_bounds__(kAttnWarps * 32)
attn_simt_kernel(Geo g, const T *q, const T *K, const T *V, const int32_t *lens,
                 zha_selection sel, int dense, float *part_ml, float *part_o, int32_t *status) {
    constexpr int DL = D / 32;
    __shared__ float qs[16][D];
    __shared__ float sm_m[kAttnWarps][16], sm_l[kAttnWarps][16];
    __shared__ float sm_o[kAttnWarps][16][D];
    // the 16-row tiles of a (group, split) are adjacent in launch order, so
    // with more than 16 rows their CTAs stream the same K/V at about the same
    // time and the second read comes from L2
    const int grp = blockIdx.z, split = blockIdx.y, S = gridDim.y;
    const int rbase = blockIdx.x * 16;     // this CTA's 16 query rows of the group
    const int b = grp / g.Hkv, kvh = grp % g.Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int G = min(16, g.G - rbase);
    for (int i = threadIdx.x; i < G * D; i += blockDim.x)
        qs[i / D][i % D] = to_f32(q[g.qrow(b, kvh, rbase + i / D) * D + i % D]);
    pdl_wait();
    const TokenPlan tp = make_plan(g, lens, grp, &sel, dense != 0, status);
    __syncthreads();
    const T *Kg = K + (int64_t)grp * g.max_len * D;
    const T *Vg = V + (int64_t)grp * g.max_len * D;
    const float sl2 = g.s * kLog2e;
    float m_run[16], l_run[16], o[16][DL];
#pragma unroll
    for (int h = 0; h < 16; ++h) {
        m_run[h] = -INFINITY;
        l_run[h] = 0.f;
#pragma unroll
        for (int e = 0; e < DL; ++e) o[h][e] = 0.f;
    }
    const int W = (tp.nv + 31) / 32;
    const int w_lo = (int)((int64_t)W * split / S), w_hi = (int)((int64_t)W * (split + 1) / S);
    for (int wt = w_lo + warp; wt < w_hi; wt += kAttnWarps) {
        const int v = wt * 32 + lane;
        int pos;
        uint32_t mask;
        tp.at(v, pos, mask, status);
        if (v >= tp.nv) mask = 0u;
        float sc[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) sc[h] = 0.f;
        const T *kr = Kg + (int64_t)pos * D;
        for (int k = 0; k < D; ++k) {
            const float kv = to_f32(kr[k]);
#pragma unroll
            for (int h = 0; h < 16; ++h)
                if (h < G) sc[h] = fmaf(qs[h][k], kv, sc[h]);
        }
#pragma unroll
        for (int h = 0; h < 16; ++h) {
            if (h >= G) continue;
            const float x = ((mask >> (rbase + h)) & 1u) ? sc[h] * sl2 : -INFINITY;
            const float mx = warp_max(x);
            const float m_new = fmaxf(m_run[h], mx);
            const float corr = (m_run[h] == -INFINITY) ? 0.f : exp2f(m_run[h] - m_new);
            const float pw = (x == -INFINITY) ? 0.f : exp2f(x - m_new);
            l_run[h] = l_run[h] * corr + warp_sum(pw);
            m_run[h] = m_new;
#pragma unroll
            for (int e = 0; e < DL; ++e) o[h][e] *= corr;
            sc[h] = pw;
        }
        for (int j = 0; j < 32; ++j) {
            const int64_t pj = __shfl_sync(0xffffffffu, pos, j);
            float vv[DL];
#pragma unroll
            for (int e = 0; e < DL; ++e) vv[e] = to_f32(Vg[pj * D + lane + 32 * e]);
#pragma unroll
            for (int h = 0; h < 16; ++h) {
                if (h >= G) continue;
                const float pj_h = __shfl_sync(0xffffffffu, sc[h], j);
#pragma unroll
                for (int e = 0; e < DL; ++e) o[h][e] = fmaf(pj_h, vv[e], o[h][e]);
            }
        }
    }
    if (lane == 0)
        for (int h = 0; h < G; ++h) {
            sm_m[warp][h] = m_run[h];
            sm_l[warp][h] = l_run[h];
        }
#pragma unroll
    for (int h = 0; h < 16; ++h)
        if (h < G)
#pragma unroll
            for (int e = 0; e < DL; ++e) sm_o[warp][h][lane + 32 * e] = o[h][e];
    __syncthreads();
    const int64_t pbase = ((int64_t)grp * S + split) * g.G + rbase;
    for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
        const int h = i / D, dim = i % D;
        float M = -INFINITY;
        for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, sm_m[w][h]);
        float L = 0.f, acc = 0.f;
        if (M != -INFINITY)
            for (int w = 0; w < kAttnWarps; ++w) {
                if (sm_m[w][h] == -INFINITY) continue;
                const float f = exp2f(sm_m[w][h] - M);
                L += sm_l[w][h] * f;
                acc += sm_o[w][h][dim] * f;
            }
        part_o[(pbase + h) * D + dim] = acc;
        if (dim == 0) {
            part_ml[(pbase + h) * 2 + 0] = M;
            part_ml[(pbase + h) * 2 + 1] = L;
        }
    }
    pdl_trigger();
}

// Log-sum-exp merge of the split-K partials: one block per (group, head).
constexpr int kMergeLanes = 4;     // threads per output coordinate, each summing every 4th split

template <typename T>
__global__ void attn_merge_kernel(Geo g, int S, const float *part_ml, const float *part_o,
                                  T *out) {
    // One block per (group, row), kMergeLanes x head_dim threads: the splits'
    // weights 2^(m_s - M) are formed in parallel (shared memory), then each
    // coordinate's weighted sum is split over kMergeLanes threads, with
    // independent loads in flight, and combined through shared memory.
    extern __shared__ float wsplit[];                 // [S] weights, then [kMergeLanes][D] partial sums
    __shared__ float red[32];
    const int grp = blockIdx.x / g.G, h = blockIdx.x % g.G;
    const int b = grp / g.Hkv, kvh = grp % g.Hkv;
    const int D = g.d;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const int64_t base = (int64_t)grp * S;
    pdl_wait();
    float mx = -INFINITY;
    for (int s = tid; s < S; s += blockDim.x) mx = fmaxf(mx, part_ml[((base + s) * g.G + h) * 2]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    float M = -INFINITY;
    for (int w = 0; w < nw; ++w) M = fmaxf(M, red[w]);
    __syncthreads();
    float ls = 0.f;
    for (int s = tid; s < S; s += blockDim.x) {
        const int64_t idx = (base + s) * g.G + h;
        const float ms = part_ml[idx * 2];
        const float f = (ms == -INFINITY) ? 0.f : exp2f(ms - M);
        wsplit[s] = f;
        ls += f == 0.f ? 0.f : part_ml[idx * 2 + 1] * f;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
    if (lane == 0) red[warp] = ls;
    __syncthreads();
    float L = 0.f;
    for (int w = 0; w < nw; ++w) L += red[w];
    const int q = tid / D, dim = tid % D;
    float acc = 0.f;
    if (M != -INFINITY && q < kMergeLanes) {
#pragma unroll 4
        for (int s = q; s < S; s += kMergeLanes) {
            const float f = wsplit[s];
            if (f != 0.f) acc = fmaf(part_o[((base + s) * g.G + h) * D + dim], f, acc);
        }
    }
    float *psum = wsplit + S;
    if (q < kMergeLanes) psum[q * D + dim] = acc;
    __syncthreads();
    if (q == 0) {
        float tot = 0.f;
#pragma unroll
        for (int k = 0; k < kMergeLanes; ++k) tot += psum[k * D + dim];
        out[g.qrow(b, kvh, h) * D + dim] = from_f32<T>(L > 0.f ? tot / L : 0.f);
    }
    pdl_trigger();
}

}  // namespace

cudaError_t launch_attention(const Geo &g, const void *q, const void *K, const void *V,
                             const int32_t *lens, const zha_selection *sel, void *out, void *ws,
                             int32_t *status, cudaStream_t st) {
    float *part_ml = reinterpret_cast<float *>(static_cast<char *>(ws) + g.ws_part_ml);
    float *part_o = reinterpret_cast<float *>(static_cast<char *>(ws) + g.ws_part_o);
    const int S = g.splits;
    const int dense = sel == nullptr;
    zha_selection sv{};
    if (sel) sv = *sel;
    // bf16: one CTA per 32 query rows when a group has more than 16 (two
    // m-tiles sharing each K/V fragment), else per 16; fp32: per 16 rows
    const bool two_tiles = g.dtype == ZHA_BF16 && g.G > 16;
    dim3 grid(two_tiles ? (g.G + 31) / 32 : (g.G + 15) / 16, S, g.groups());
    const char *attn_name = dense ? "attn_dense" : "attn_sparse";
    if (g.dtype == ZHA_BF16) {
        auto qq = static_cast<const __nv_bfloat16 *>(q);
        auto kk = static_cast<const __nv_bfloat16 *>(K);
        auto vv = static_cast<const __nv_bfloat16 *>(V);
        {
            // the shared-memory opt-in is a per-device function attribute
            static bool attr_set[64] = {};
            int dev = 0;
            cudaGetDevice(&dev);
            if (dev >= 0 && dev < 64 && !attr_set[dev]) {
                cudaFuncSetAttribute(attn_mma_kernel<128, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     attn_smem_bytes<128>());
                cudaFuncSetAttribute(attn_mma_kernel<64, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     attn_smem_bytes<64>());
                cudaFuncSetAttribute(attn_mma_kernel<128, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     attn_smem_bytes<128>());
                cudaFuncSetAttribute(attn_mma_kernel<64, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     attn_smem_bytes<64>());
                attr_set[dev] = true;
            }
            ProfScope ps(attn_name, st);
            const dim3 blk(kAttnWarps * 32);
            const cudaError_t e = g.d == 128
                ? (two_tiles ? launch_pdl(attn_mma_kernel<128, 2>, grid, blk, attn_smem_bytes<128>(), st,
                                          g, qq, kk, vv, lens, sv, dense, part_ml, part_o, status)
                             : launch_pdl(attn_mma_kernel<128, 1>, grid, blk, attn_smem_bytes<128>(), st,
                                          g, qq, kk, vv, lens, sv, dense, part_ml, part_o, status))
                : (two_tiles ? launch_pdl(attn_mma_kernel<64, 2>, grid, blk, attn_smem_bytes<64>(), st,
                                          g, qq, kk, vv, lens, sv, dense, part_ml, part_o, status)
                             : launch_pdl(attn_mma_kernel<64, 1>, grid, blk, attn_smem_bytes<64>(), st,
                                          g, qq, kk, vv, lens, sv, dense, part_ml, part_o, status));
            if (e != cudaSuccess) return e;
        }
        ProfScope pm("attn_merge", st);
        const cudaError_t e = launch_pdl(attn_merge_kernel<__nv_bfloat16>, dim3(g.groups() * g.G),
                                         dim3(kMergeLanes * g.d), (S + kMergeLanes * g.d) * sizeof(float), st,
                                         g, S, part_ml, part_o, static_cast<__nv_bfloat16 *>(out));
        if (e != cudaSuccess) return e;
    } else {
        auto qq = static_cast<const float *>(q);
        auto kk = static_cast<const float *>(K);
        auto vv = static_cast<const float *>(V);
        {
        ProfScope ps(attn_name, st);
        const cudaError_t e = g.d == 128
            ? launch_pdl(attn_simt_kernel<float, 128>, grid, dim3(kAttnWarps * 32), 0, st,
                         g, qq, kk, vv, lens, sv, dense, part_ml, part_o, status)
            : launch_pdl(attn_simt_kernel<float, 64>, grid, dim3(kAttnWarps * 32), 0, st,
                         g, qq, kk, vv, lens, sv, dense, part_ml, part_o, status);
        if (e != cudaSuccess) return e;
        }
        ProfScope pm("attn_merge", st);
        const cudaError_t e = launch_pdl(attn_merge_kernel<float>, dim3(g.groups() * g.G), dim3(kMergeLanes * g.d),
                                         (S + kMergeLanes * g.d) * sizeof(float), st,
                                         g, S, part_ml, part_o, static_cast<float *>(out));
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace zha
