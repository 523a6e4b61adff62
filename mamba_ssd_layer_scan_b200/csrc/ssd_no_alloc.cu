// ssd_chunk_scan_fwd_static: the chunked scan for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at the point where they run the scan:
// code that runs inside a framework's memory-planning pass where the allocator is locked, code
// embedded in a runtime that owns all device memory and hands out only the tensors it planned,
// or hosts that forbid allocation after start-up so memory use stays fixed.  They can still pass
// their inputs and outputs, but not a workspace.  This entry point gives them one: a fixed
// scratch array that lives in this library's device image, declared below.
//
// How it works: the array is a file-scope __device__ variable, so every GPU that loads the
// library holds kStaticScratchBytes of device memory for it until the process exits.  In host
// code its name is only a host-side stand-in, never a device address, so the first call on each
// device (with that device current) asks the runtime for the real address with
// cudaGetSymbolAddress, checks the result, and remembers it; later calls reuse it.  That first
// call therefore does a little setup work and should happen before any stream capture.  The
// address is then handed to the same kernels ssd_chunk_scan_fwd runs, as their workspace.
//
// The scratch address is cached per device ordinal, for the device's primary context (the one
// the CUDA runtime uses); a caller that runs the scan in a context of its own making, or that
// resets the device after the first call, is not supported.
//
// Nothing here allocates: no cudaMalloc, no cudaFree, no allocating library call.  Nothing in
// the array needs to start at zero: the scan's first kernel clears the status word and every
// other byte it reads was written earlier in the same call.  The array keeps whatever the last
// call left in it.  All calls on a device share the one array, so calls whose kernels overlap
// on the GPU (different streams, or several host threads on the same device) race and corrupt
// each other's results; issue them on one stream, one after the other.
#include <atomic>
#include <cstdio>
#include <mutex>

#include "../../include/ssd.h"
#include "common.cuh"

namespace {

// 32 MiB: enough for the scan at, e.g., batch 2 x 2048 tokens x 24 heads (P 64, N 128, Q 256,
// about 19.3 MB of workspace).  Larger problems are rejected with SSD_ERR_UNSUPPORTED.
constexpr size_t kStaticScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

__device__ __align__(256) static unsigned char g_ssd_static_scratch[kStaticScratchBytes];

std::mutex g_setup_mutex;
std::atomic<void *> g_scratch_addr[kMaxDevices];

// The device address of the scratch array on the current device (set up once per device).
cudaError_t scratch_address(void **out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    void *p = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lock(g_setup_mutex);
        p = g_scratch_addr[dev].load(std::memory_order_relaxed);
        if (!p) {
            e = cudaGetSymbolAddress(&p, g_ssd_static_scratch);
            if (e != cudaSuccess) return e;
            if (!p) return cudaErrorInvalidSymbol;
            g_scratch_addr[dev].store(p, std::memory_order_release);
        }
    }
    *out = p;
    return cudaSuccess;
}

}  // namespace

extern "C" {

ssd_status ssd_chunk_scan_fwd_static(const ssd_shape *shape, const void *x, const float *dt,
                                     const float *A, const void *B, const void *C,
                                     const float *D, int chunk_size, const float *init_state,
                                     void *y, float *final_state, void *stream)
{
    const size_t need = ssd_chunk_scan_workspace_size(shape, chunk_size);
    if (need == 0)  // invalid shape or chunk size: report the reason through the normal path
        return ssd_chunk_scan_fwd(shape, x, dt, A, B, C, D, chunk_size, init_state, y,
                                  final_state, nullptr, 0, stream);
    char msg[256];
    if (need > kStaticScratchBytes) {
        snprintf(msg, sizeof(msg),
                 "ssd_chunk_scan_fwd_static: this problem needs %zu bytes of scratch but the "
                 "built-in array holds %zu; call ssd_chunk_scan_fwd with a caller workspace",
                 need, kStaticScratchBytes);
        ssd::set_last_error(msg);
        return SSD_ERR_UNSUPPORTED;
    }
    void *scratch = nullptr;
    const cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess) {
        snprintf(msg, sizeof(msg),
                 "ssd_chunk_scan_fwd_static: cannot get the scratch array's device address: %s",
                 cudaGetErrorString(e));
        ssd::set_last_error(msg);
        return SSD_ERR_CUDA;
    }
    return ssd_chunk_scan_fwd(shape, x, dt, A, B, C, D, chunk_size, init_state, y, final_state,
                              scratch, kStaticScratchBytes, stream);
}

ssd_status ssd_chunk_scan_fwd_static_status(void *stream)
{
    void *scratch = nullptr;
    const cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof(msg),
                 "ssd_chunk_scan_fwd_static_status: cannot get the scratch array's device "
                 "address: %s", cudaGetErrorString(e));
        ssd::set_last_error(msg);
        return SSD_ERR_CUDA;
    }
    return ssd_workspace_status(scratch, kStaticScratchBytes, stream);
}

}  // extern "C"
