// zha_score_tc.cu -- node scoring on the 5th-generation tensor cores.
//
// Page "Zyphra AI Introduces Zyphra Hierarchical Attention (ZHA)", sections
// "Building the tree" and "How does top-p routing pick tokens": a candidate
// node's estimate for query head h is E = max_r (s q_h.mu_r + bias_r).
//
// For bf16, head_dim 128, 16 reference planes per node and at most 16 query
// heads per KV head, a tile of 8 candidate nodes is a 128 x 128 (planes x
// head_dim) bf16 matrix; times the group's queries (16 x 128, zero-padded
// heads) it is one M=128, N=16, K=128 tcgen05.mma (8 instructions of K=16),
// accumulated in fp32 in tensor memory. Per CTA (one per SM, persistent over
// the tiles of one group):
//   warp 0      -- TMA producer: a tile's nodes are 1-4 runs of
//                  consecutive nodes (looked up 32 runs at a time by the
//                  lanes); one tiled load per run and half of head_dim into a
//                  4-stage ring of 128B-swizzled shared-memory tiles, plus a
//                  bulk copy of the runs' biases;
//   warp 1      -- allocates 32 TMEM columns and, from one lane, issues the
//                  MMAs into one of two 16-column accumulators, committing to
//                  mbarriers that free the smem stage and publish the result;
//   warps 2..5  -- epilogue: tcgen05.ld of the accumulator (one TMEM lane per
//                  plane), bias, max over each node's 16 planes, scores out.
// An A stage is freed by the MMA's commit; each tile's biases and node
// metadata sit in a deeper ring that the epilogue frees after reading them.
// Every mbarrier wait is bounded; on expiry the kernel records
// ZHA_ERR_TIMEOUT, stops issuing work, lets copies in flight land, frees its
// tensor memory and returns.
#include "zha_tc.cuh"

namespace zha {

namespace {

constexpr int kTcStages = 4;
constexpr int kTcThreads = 192;            // 6 warps
constexpr int kTileNodes = 8;              // 8 nodes x 16 planes = 128 rows
constexpr int kRows = 128;
constexpr int kHalfBytes = kRows * 128;    // one 64-column half of a tile: 16 KB
constexpr int kABytes = 2 * kHalfBytes;    // the tile's two halves
constexpr int kBiasBytes = kTileNodes * 16 * 4;
constexpr int kStageBytes = kABytes;       // A stages, freed as soon as the MMAs have read them
constexpr int kMetaSlots = 8;              // biases (512 B) + node/mask metadata (64 B) per tile,
constexpr int kMetaBytes = 1024;           // a deeper ring freed by the epilogue
constexpr int kQBytes = 2 * 16 * 128;      // one group's queries: 16 rows x 128 columns, two halves
constexpr int kMaxGroups = 16;             // queries of every group stay in shared memory
constexpr int kTcSmem = kTcStages * kStageBytes + kMetaSlots * kMetaBytes + kMaxGroups * kQBytes + 1024 + 1024;
constexpr uint32_t kTmemCols = 32;
constexpr long long kWaitCycles = 4000000000ll;  // ~2 s at the boost clock

constexpr uint32_t kIdesc = tc_idesc_bf16(16);

// Bounded wait: false if the barrier did not complete in time or the CTA is
// aborting (then also raises the abort flag and the status).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort,
                                          int32_t *status) {
    return mbar_wait_bounded(bar, parity, kWaitCycles, abort, status);
}

struct TcArgs {
    const __nv_bfloat16 *q;
    const float *bias;
    const int32_t *lens;
    int32_t *cand;
    uint32_t *cmask;
    float *scores;
    int32_t *count;
    uint32_t *maxkey, *minkey;
    const int32_t *plist_up;    // kept nodes one level up ([groups][cap_up]); unused at the top
    const uint32_t *pmask_up;
    const int32_t *pcount_up;
    int64_t cap, capv, cap_up;
    int level;
    int runs;                   // node runs per tile: 1 (top level or c >= 8), else 8 / c
    int32_t *status;
};

// Per-group tile bookkeeping: the tiles of all groups form one index space that
// the persistent CTAs split evenly (a group may hold most of a level's work).
struct GroupTiles {
    int n[kMaxGroups];        // candidate entries
    int n_here[kMaxGroups];   // nodes at this level
    int first[kMaxGroups + 1];  // first global tile of each group
};

__device__ __forceinline__ int tile_group(const GroupTiles &gt, int groups, int tau) {
    int g = 0;
    while (g + 1 < groups && gt.first[g + 1] <= tau) ++g;
    return g;
}

__global__ void __launch_bounds__(kTcThreads, 1)
score_tc_kernel(const __grid_constant__ CUtensorMap mu_map, Geo g, TcArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t mbase = sbase + kTcStages * kStageBytes;
    uint8_t *metas = smem + kTcStages * kStageBytes;
    const uint32_t qbase = mbase + kMetaSlots * kMetaBytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kTcStages * kStageBytes + kMetaSlots * kMetaBytes +
                                                  kMaxGroups * kQBytes);
    // bars: full[S], empty[S], tfull[2], tempty[2], mfull[8], mempty[8]; then tmem address, abort flag
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * kTcStages + 4 + 2 * kMetaSlots);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + kTcStages);
    const uint32_t tfull0 = smem_u32(bars + 2 * kTcStages), tempty0 = smem_u32(bars + 2 * kTcStages + 2);
    const uint32_t mfull0 = smem_u32(bars + 2 * kTcStages + 4), mempty0 = smem_u32(bars + 2 * kTcStages + 4 + kMetaSlots);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int groups = g.groups();
    const int lc = __ffs(g.c) - 1;
    const bool top = a.level == g.L;
    __shared__ GroupTiles gt;
    if (threadIdx.x < groups) {
        const int grp = threadIdx.x;
        int64_t N = a.lens[grp / g.Hkv];
        if (N < 0 || N > g.max_len) N = 0;
        gt.n_here[grp] = (int)level_nodes(N, g.c, a.level);
        gt.n[grp] = top ? gt.n_here[grp] : a.pcount_up[grp] << lc;
        if (blockIdx.x == 0) a.count[grp] = gt.n[grp];
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int grp = 0; grp < groups; ++grp) {
            gt.first[grp] = acc;
            acc += (gt.n[grp] + kTileNodes - 1) / kTileNodes;
        }
        gt.first[groups] = acc;
    }
    __syncthreads();
    const int ntiles = gt.first[groups];
    const int per_cta = (ntiles + gridDim.x - 1) / gridDim.x;
    const int t_begin = blockIdx.x * per_cta, t_end = min(ntiles, t_begin + per_cta);
    const uint32_t all = g.G >= 32 ? 0xffffffffu : ((1u << g.G) - 1u);
    const int P = a.runs;                  // runs per tile
    const int run_nodes = kTileNodes / P;  // consecutive nodes per run

    // every group's queries -> shared memory, canonical K-major 128B-swizzled layout
    for (int e = threadIdx.x; e < groups * 16 * 16; e += blockDim.x) {   // rows x 16-byte chunks
        const int grp = e >> 8, row = (e >> 4) & 15, chunk = e & 15;
        const int b = grp / g.Hkv, kvh = grp % g.Hkv;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (row < g.G)
            v = *reinterpret_cast<const uint4 *>(a.q + g.qrow(b, kvh, row) * 128 + chunk * 8);
        const int half = chunk >> 3, c8 = chunk & 7;
        *reinterpret_cast<uint4 *>(smem + kTcStages * kStageBytes + kMetaSlots * kMetaBytes + grp * kQBytes +
                                   half * 2048 + row * 128 +
                                   ((c8 ^ (row & 7)) << 4)) = v;
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        for (int m = 0; m < kMetaSlots; ++m) {
            mbar_init(mfull0 + 8 * m, 1);
            mbar_init(mempty0 + 8 * m, 128);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(tfull0 + 8 * s, 1);
            mbar_init(tempty0 + 8 * s, 128);
        }
        *abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    fence_proxy_async_smem();  // q stores -> async proxy
    if (warp == 1) tc_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        // Lanes look up the first node of 32 runs at a time (the next batch is
        // fetched while this one is issued); then, per tile: metadata to the
        // stage, arm the barrier, one TMA box per run and half, one bulk copy of
        // the run's biases.
        // (one producer: every stage's barrier phases are then waited on in order)
        const int tiles_per_batch = 32 / P;
        auto tile_of = [&](int j) { return t_begin + j; };
        auto lookup = [&](int jb, int &node0, uint32_t &hm, int &valid) {
            const int tau = tile_of(jb + lane / P), r = lane % P;
            node0 = 0;
            hm = 0u;
            valid = 0;
            if (tau < t_end) {
                const int grp = tile_group(gt, groups, tau);
                const int n = gt.n[grp];
                const int i0 = (tau - gt.first[grp]) * kTileNodes + r * run_nodes;   // first candidate of the run
                if (i0 < n) {
                    if (top) {
                        node0 = i0;
                        hm = all;
                        valid = min(run_nodes, n - i0);
                    } else {
                        const int j = i0 >> lc;
                        node0 = (__ldg(&a.plist_up[grp * a.cap_up + j]) << lc) + (i0 & (g.c - 1));
                        hm = __ldg(&a.pmask_up[grp * a.cap_up + j]);
                        valid = max(0, min(run_nodes, gt.n_here[grp] - node0));
                    }
                }
            }
        };
        int nx0 = 0, nv = 0;
        uint32_t nhm = 0u;
        lookup(0, nx0, nhm, nv);
        bool ok = true;
        for (int jb = 0; tile_of(jb) < t_end && ok; jb += tiles_per_batch) {
            const int c_node0 = nx0, c_valid = nv;
            const uint32_t c_hm = nhm;
            lookup(jb + tiles_per_batch, nx0, nhm, nv);   // next batch, in flight meanwhile
            for (int tt = 0; tt < tiles_per_batch && tile_of(jb + tt) < t_end; ++tt) {
                const int k = tile_of(jb + tt) - t_begin;   // tile ordinal within the CTA
                const int s = k % kTcStages, mslot = k % kMetaSlots;
                int w_ok = 1;
                if (lane == 0)
                    w_ok = mbar_wait(mempty0 + 8 * mslot, ((k / kMetaSlots) & 1) ^ 1, abort, a.status) &&
                           mbar_wait(empty0 + 8 * s, ((k / kTcStages) & 1) ^ 1, abort, a.status);
                if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
                    ok = false;
                    break;
                }
                const uint32_t stage = sbase + s * kStageBytes;
                uint8_t *meta = metas + mslot * kMetaBytes + kBiasBytes;
                // runs of this tile live in lanes tt*P .. tt*P+P-1
                int r0[4], rv[4];
                uint32_t rh[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int src = (tt * P + (r < P ? r : 0)) & 31;
                    r0[r] = __shfl_sync(0xffffffffu, c_node0, src);
                    rv[r] = __shfl_sync(0xffffffffu, c_valid, src);
                    rh[r] = __shfl_sync(0xffffffffu, c_hm, src);
                }
                if (lane < kTileNodes) {   // slot metadata: node and head mask (0 = padding)
                    const int r = lane / run_nodes, m = lane % run_nodes;
                    reinterpret_cast<int *>(meta)[lane] = r0[r] + m;
                    reinterpret_cast<uint32_t *>(meta)[kTileNodes + lane] = m < rv[r] ? rh[r] : 0u;
                }
                uint32_t bias_bytes = 0;
#pragma unroll
                for (int r = 0; r < 4; ++r)
                    if (r < P) bias_bytes += (uint32_t)(rv[r] > 0 ? rv[r] : 0) * 64u;
                __syncwarp();
                if (lane == 0) {
                    mbar_expect_tx(mfull0 + 8 * mslot, bias_bytes);
                    mbar_expect_tx(full0 + 8 * s, (uint32_t)kABytes);
                }
                __syncwarp();
                if (lane < P) {
                    const int grp = tile_group(gt, groups, tile_of(jb + tt));
                    const int y = (int)((grp * a.cap + r0[lane]) * 16);
                    const uint32_t rows_off = lane * run_nodes * 16 * 128;
                    tma_load_2d(stage + rows_off, &mu_map, 0, y, full0 + 8 * s);
                    tma_load_2d(stage + kHalfBytes + rows_off, &mu_map, 64, y, full0 + 8 * s);
                    if (rv[lane] > 0)
                        bulk_load(mbase + mslot * kMetaBytes + lane * run_nodes * 64,
                                  a.bias + (grp * a.cap + r0[lane]) * 16, (uint32_t)rv[lane] * 64u,
                                  mfull0 + 8 * mslot);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int k = 0;
            for (int t = t_begin; t < t_end; ++t, ++k) {
                const int s = k % kTcStages, acc = k & 1;
                if (!mbar_wait(tempty0 + 8 * acc, ((k >> 1) & 1) ^ 1, abort, a.status)) break;
                if (!mbar_wait(full0 + 8 * s, (k / kTcStages) & 1, abort, a.status)) break;
                tc_fence_after();
                const int grp = tile_group(gt, groups, t);
                const uint32_t abase = sbase + s * kStageBytes;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {   // K = 128 in steps of 16 (32 bytes)
                    const uint32_t off = (kk & 3) * 32;
                    const uint64_t ad = smem_desc(abase + (kk >> 2) * kHalfBytes + off);
                    const uint64_t bd = smem_desc(qbase + grp * kQBytes + (kk >> 2) * 2048 + off);
                    tc_mma(tmem + acc * 16, ad, bd, kIdesc, kk > 0 ? 1u : 0u);
                }
                tc_commit(empty0 + 8 * s);     // A stage free once these MMAs have read it
                tc_commit(tfull0 + 8 * acc);
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        const int quarter = warp & 3;            // TMEM lanes this warp may read
        const int row = quarter * 32 + lane;     // plane row of the tile
        const int slot = row >> 4, r = row & 15;
        float runmax[16], runmin[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) {
            runmax[h] = -INFINITY;
            runmin[h] = INFINITY;
        }
        int cur = -1;   // group whose running max/min are held
        auto flush = [&]() {
            if (r != 0 || cur < 0) return;
#pragma unroll
            for (int h = 0; h < 16; ++h) {
                if (h >= g.G) break;
                if (runmax[h] > -INFINITY) {
                    atomicMax(&a.maxkey[(int64_t)cur * g.G + h], ordered_key(runmax[h]));
                    atomicMin(&a.minkey[(int64_t)cur * g.G + h], ordered_key(runmin[h]));
                }
                runmax[h] = -INFINITY;
                runmin[h] = INFINITY;
            }
        };
        int k = 0;
        for (int t = t_begin; t < t_end; ++t, ++k) {
            const int mslot = k % kMetaSlots, acc = k & 1;
            const int grp = tile_group(gt, groups, t);
            if (grp != cur) {
                flush();
                cur = grp;
            }
            if (!mbar_wait(tfull0 + 8 * acc, (k >> 1) & 1, abort, a.status)) break;
            if (!mbar_wait(mfull0 + 8 * mslot, (k / kMetaSlots) & 1, abort, a.status)) break;
            tc_fence_after();
            uint32_t v[16];
            tc_ld16(tmem + ((uint32_t)(quarter * 32) << 16) + acc * 16, v);
            tc_fence_before();
            mbar_arrive(tempty0 + 8 * acc);
            const uint8_t *st = metas + mslot * kMetaBytes;
            const int node = reinterpret_cast<const int *>(st + kBiasBytes)[slot];
            const uint32_t hm = reinterpret_cast<const uint32_t *>(st + kBiasBytes)[kTileNodes + slot];
            const float bs = hm ? reinterpret_cast<const float *>(st)[slot * 16 + r] : 0.f;
            mbar_arrive(mempty0 + 8 * mslot);   // metadata slot free for the producer
            const int i = (t - gt.first[grp]) * kTileNodes + slot;
            float e[16];
#pragma unroll
            for (int h = 0; h < 16; ++h) {
                float x = fmaf(g.s, __uint_as_float(v[h]), bs);
                x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
                x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
                x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 4));
                x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 8));
                e[h] = x;
            }
            if (r == 0 && i < gt.n[grp]) {
                a.cand[grp * a.capv + i] = node;
                a.cmask[grp * a.capv + i] = hm;
#pragma unroll
                for (int h = 0; h < 16; ++h) {
                    if (h >= g.G) break;
                    a.scores[(grp * g.G + h) * a.capv + i] = hm ? e[h] : -INFINITY;
                    if ((hm >> h) & 1u) {
                        runmax[h] = fmaxf(runmax[h], e[h]);
                        runmin[h] = fminf(runmin[h], e[h]);
                    }
                }
            }
        }
        flush();
    }
    tc_fence_before();
    __syncthreads();
    if (*abort) {
        // let copies already issued land before the shared memory goes away
        const long long t0 = clock64();
        while (clock64() - t0 < 2000000) {
        }
    }
    tc_fence_after();
    if (warp == 1) tc_dealloc(tmem, kTmemCols);
}

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}


bool score_tc_supported(const Geo &g) {
    return g.dtype == ZHA_BF16 && !g.mx() && g.T == 1 && g.lag == 0 && g.d == 128 && g.R == 16 && g.G <= 16 && g.groups() <= kMaxGroups &&
           tensor_map_encoder() != nullptr;
}

// One level of scoring on tcgen05; the layout of the inputs and outputs is
// that of the mma.sync kernel in zha_route.cu.
cudaError_t launch_score_tc(const Geo &g, const void *mu_level, const float *bias, const void *q,
                            const int32_t *lens, int level, int32_t *cand, uint32_t *cmask, float *scores,
                            int32_t *count, uint32_t *maxkey, uint32_t *minkey, const int32_t *plist_up,
                            const uint32_t *pmask_up, const int32_t *pcount_up, int32_t *status,
                            cudaStream_t st) {
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        cudaFuncSetAttribute(score_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmem);
        attr_set[dev] = true;
    }
    // a tile of 8 candidates is 1, 2 or 4 runs of consecutive nodes: one run at
    // the top level (consecutive nodes) and for c >= 8, else the 8/c parents'
    // children; one TMA box covers a run (16 rows per node)
    const int runs = (level == g.L || g.c >= kTileNodes) ? 1 : kTileNodes / g.c;
    CUtensorMap map;
    const cuuint64_t dims[2] = {128, (cuuint64_t)g.groups() * (cuuint64_t)g.cap[level] * 16};
    const cuuint64_t strides[1] = {128 * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)(kRows / runs)};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = tensor_map_encoder()(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(mu_level), dims, strides,
                             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    TcArgs a{};
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.bias = bias;
    a.lens = lens;
    a.cand = cand;
    a.cmask = cmask;
    a.scores = scores;
    a.count = count;
    a.maxkey = maxkey;
    a.minkey = minkey;
    a.plist_up = plist_up;
    a.pmask_up = pmask_up;
    a.pcount_up = pcount_up;
    a.cap = g.cap[level];
    a.capv = g.capv[level];
    a.cap_up = level < g.L ? g.cap[level + 1] : 0;
    a.level = level;
    a.runs = runs;
    a.status = status;
    // one persistent CTA per SM; each takes a contiguous range of all groups' tiles
    dim3 grid(148, 1);
    score_tc_kernel<<<grid, kTcThreads, kTcSmem, st>>>(map, g, a);
    return cudaGetLastError();
}

}  // namespace zha
