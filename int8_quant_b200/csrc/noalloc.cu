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
#include "../../include/ssd.h"
#include "kernels.h"

namespace {

static __device__ __align__(256) unsigned char g_static_scratch[SSD_STATIC_SCRATCH_BYTES];

// Device address of g_static_scratch in the current device's current context.  In host
// code the symbol name is only a host-side handle, so the address the kernels need must
// come from cudaGetSymbolAddress with that device current.  It is looked up on every
// call (cheap once the module is loaded), so that no cached address can outlive a
// cudaDeviceReset or belong to another context.  Under lazy module loading the first
// lookup on a device loads the module and with it the array.
ssd_status scratch_for_current_device(void** out) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return SSD_ERR_CUDA;
    *out = p;
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

extern "C" ssd_status ssd_static_scratch_status(cudaStream_t stream) {
    // the first int of the scratch is the status word that the scan's kernels set
    void* p = nullptr;
    const ssd_status st = scratch_for_current_device(&p);
    if (st != SSD_OK) return st;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return SSD_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SSD_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return SSD_ERR_CUDA;
    }
    return v == 0 ? SSD_OK : (ssd_status)v;
}
