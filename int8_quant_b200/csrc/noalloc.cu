// noalloc.cu — ssd_scan_fwd_bf16_static: the bf16 scan for callers that cannot
// allocate device memory.
//
// Some callers have no way to hand the library a workspace: code running inside a
// memory pool or arena that owns every device allocation, plugins and embedded
// runtimes that are not allowed to call cudaMalloc, or hosts that must not take
// allocation locks on a latency-critical thread.  For them this entry point keeps
// the scan's scratch (per-chunk cumulative decays, chunk states, passed states and
// the status word) in a fixed array in the library's own device memory, sized at
// compile time.  Every GPU that loads the library holds that array until the
// process exits, so it is kept modest: SSD_STATIC_SCRATCH_BYTES (32 MiB).
#include <mutex>

#include "../../include/ssd.h"
#include "kernels.h"

namespace {

static __device__ __align__(256) unsigned char g_static_scratch[SSD_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device, looked up once per
// device.  In host code the symbol name is only a host-side handle, so the address
// the kernels need must come from cudaGetSymbolAddress with that device current.
ssd_status scratch_for_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SSD_ERR_CUDA;
    std::lock_guard<std::mutex> g(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return SSD_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return SSD_OK;
}

}  // namespace

extern "C" ssd_status ssd_scan_fwd_bf16_static(const ssd_shape* shape, const uint16_t* x,
                                               const float* dt, const float* A,
                                               const uint16_t* B, const uint16_t* C,
                                               const float* D, uint16_t* y, float* final_state,
                                               cudaStream_t stream) {
    const size_t need = ssd_workspace_bytes(shape, 0);
    if (need == 0) {
        // invalid or unsupported shape: let the regular entry point report which
        return ssd_scan_fwd_bf16(shape, x, dt, A, B, C, D, y, final_state, nullptr, 0, stream);
    }
    if (need > (size_t)SSD_STATIC_SCRATCH_BYTES) return SSD_ERR_WORKSPACE;
    void* scratch = nullptr;
    const ssd_status st = scratch_for_current_device(&scratch);
    if (st != SSD_OK) return st;
    // The kernels clear the status word at the start of the call and write every
    // other scratch region before reading it, so stale contents of a previous call
    // are never seen.
    return ssd_scan_fwd_bf16(shape, x, dt, A, B, C, D, y, final_state, scratch,
                             (size_t)SSD_STATIC_SCRATCH_BYTES, stream);
}
