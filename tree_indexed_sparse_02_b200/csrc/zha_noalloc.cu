// zha_noalloc.cu -- dense decode for callers that cannot allocate device
// memory: the split-K partials live in a fixed array compiled into the
// library instead of a caller workspace.
#include <mutex>

#include "zha_common.cuh"

namespace {

// 4 MiB of split-K scratch, placed in a device's memory when the library's
// module is loaded there (on first use under CUDA's lazy loading) and kept
// until the process exits or the context is reset. Calls share it and it
// keeps the last call's partials; every partial a call reads it first
// writes, so nothing needs clearing between calls.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void *g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// The device address of the scratch array on the current device. The name of
// a __device__ variable is only a host-side handle, so the address is asked
// for with the device current. It is asked for again on every call made
// outside a stream capture (a reset context reloads the module, and the array
// may move); a call being captured, where a lookup that loads the module is
// not allowed, uses the address of the last call outside capture.
zha_status scratch_address(cudaStream_t stream, void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ZHA_ERR_CUDA;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) {
        (void)cudaGetLastError();
        cs = cudaStreamCaptureStatusActive;   // unknown: do not look up
    }
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (cs == cudaStreamCaptureStatusNone || !g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            (void)cudaGetLastError();
            return ZHA_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return ZHA_OK;
}

}  // namespace

extern "C" zha_status zha_dense_decode_noalloc(const zha_config *cfg, const void *q, const void *K,
                                               const void *V, const int32_t *lens, void *out,
                                               int32_t *dev_status, void *stream) {
    const size_t ws = zha_workspace_bytes(cfg);
    if (ws == 0) return zha_check_config(cfg) == ZHA_OK ? ZHA_ERR_INVALID_ARG : zha_check_config(cfg);
    if (!q || !K || !V || !lens || !out) return ZHA_ERR_INVALID_ARG;
    if (((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(K) |
          reinterpret_cast<uintptr_t>(V) | reinterpret_cast<uintptr_t>(out)) & 15u) != 0)
        return ZHA_ERR_INVALID_ARG;
    // the layout of the ordinary workspace, with only the split-K partials kept
    // and placed at the start of the scratch array
    zha::Geo g = zha::make_geo_for(cfg);
    const size_t groups = (size_t)g.B * g.Hkv;
    const size_t ml_bytes = align256(groups * g.splits * g.G * 2 * sizeof(float));
    const size_t o_bytes = align256(groups * g.splits * g.G * g.d * sizeof(float));
    if (ml_bytes + o_bytes > kNoAllocScratchBytes) return ZHA_ERR_CAPACITY;
    g.ws_part_ml = 0;
    g.ws_part_o = ml_bytes;
    void *scratch = nullptr;
    zha_status s = scratch_address(static_cast<cudaStream_t>(stream), &scratch);
    if (s != ZHA_OK) return s;
    cudaError_t e = zha::launch_attention(g, q, K, V, lens, nullptr, out, scratch, dev_status,
                                          static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ZHA_OK : ZHA_ERR_CUDA;
}
