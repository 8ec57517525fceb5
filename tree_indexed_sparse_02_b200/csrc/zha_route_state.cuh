// zha_route_state.cuh -- the per-route scratch state that a route resets
// before its first level, shared by the route's own reset kernel and by the
// fused decode-step prologue.
#pragma once
#include "zha_common.cuh"

namespace zha {

struct RouteState {
    uint32_t *maxkey;              // [L][groups][G] ordered keys of each row's largest score
    uint32_t *minkey;              // [L][groups][G] and smallest
    uint32_t *done;                // [L][groups] finished select CTAs
    uint32_t *gctr;                // [L][groups][G][4] counters of the multi-CTA selection
    unsigned long long *lookback;  // the joins' look-back words, every level
};

inline RouteState route_state(const Geo &g, void *ws) {
    char *base = static_cast<char *>(ws);
    return RouteState{reinterpret_cast<uint32_t *>(base + g.ws_maxkey),
                      reinterpret_cast<uint32_t *>(base + g.ws_minkey),
                      reinterpret_cast<uint32_t *>(base + g.ws_done),
                      reinterpret_cast<uint32_t *>(base + g.ws_gctr),
                      reinterpret_cast<unsigned long long *>(base + g.ws_lookback)};
}

// Reset one group's state (all threads of the calling block take part).
__device__ __forceinline__ void route_reset_group(const Geo &g, const RouteState &rs, int grp) {
    for (int i = threadIdx.x; i < g.L * g.G; i += blockDim.x) {
        const int64_t at = ((int64_t)(i / g.G) * g.groups() + grp) * g.G + i % g.G;
        rs.maxkey[at] = 0u;
        rs.minkey[at] = 0xffffffffu;
#pragma unroll
        for (int k = 0; k < 4; ++k) rs.gctr[at * 4 + k] = 0u;
    }
    for (int l = threadIdx.x; l < g.L; l += blockDim.x) rs.done[(int64_t)l * g.groups() + grp] = 0u;
    int64_t off = 0;
    for (int l = 1; l <= g.L; ++l) {
        const int64_t chunks = (g.capv[l] + kJoinChunk - 1) / kJoinChunk;
        for (int64_t i = threadIdx.x; i < chunks; i += blockDim.x) rs.lookback[off + grp * chunks + i] = 0ull;
        off += (int64_t)g.groups() * chunks;
    }
}

}  // namespace zha
