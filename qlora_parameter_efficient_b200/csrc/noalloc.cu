// noalloc.cu -- a forward entry point that needs no caller workspace and allocates nothing.
//
// qlora_linear_fwd takes its scratch (zero-padded adapters, the scaled projection sU and the
// split-K partials of U = X A^T) from a caller-provided workspace.  Some callers have no
// device memory to lend and may not call cudaMalloc themselves: code running inside an
// engine that owns every byte of device memory through its own pool, or a latency-critical
// path that must not take the allocator's locks and implicit synchronisation.  For them this
// file holds the scratch in a fixed device array that is part of the library's module image.
//
// Costs and limits:
//  - Every GPU that loads the library holds kNoAllocScratchBytes (16 MiB) of device memory
//    until the process exits.
//  - A call whose workspace need exceeds that size is rejected with QLORA_ERR_UNSUPPORTED
//    before anything is launched.
//  - All calls share the one array and it keeps the previous call's contents; the forward
//    kernels overwrite every scratch byte they read, so nothing needs clearing.  Calls whose
//    work overlaps on the GPU (two streams, or two host threads) race on the array.
//  - The array's device address is looked up (cudaGetSymbolAddress, with the device current)
//    on every call made outside stream capture, so a context re-created after cudaDeviceReset
//    is followed; while the stream is being captured the address cached by the last such call
//    on that device is used, so the first call on a device must come before any capture.
//  - Arguments are checked exactly as qlora_linear_fwd checks them, and give the same status.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/qlora.h"

namespace {

constexpr size_t kNoAllocScratchBytes = QLORA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// In host code this name is only a host-side stand-in; kernels get the device address below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device: looked up on every call outside
// stream capture, from the cache of the last such call while `stream` is being captured.
qlora_status scratch_address(cudaStream_t stream, void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QLORA_ERR_CUDA;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    const bool capturing = cudaStreamIsCapturing(stream, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone;
    if (capturing) cudaGetLastError();
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!capturing || !g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return QLORA_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return QLORA_OK;
}

}  // namespace

// The argument checks of qlora_linear_fwd (defined beside it; not exported).
extern "C" qlora_status qlora_fwd_check_args(const qlora_nf4* w, const void* X, int64_t T, const void* A,
                                  const void* B, int32_t r, qlora_dtype dtype, const void* H,
                                  const void* U_save);

extern "C" qlora_status qlora_linear_fwd_noalloc(const qlora_nf4* w, const void* X, int64_t T,
                                                 const void* A, const void* B, int32_t r,
                                                 float alpha, qlora_dtype dtype, void* H,
                                                 void* U_save, cudaStream_t stream) {
    const qlora_status v = qlora_fwd_check_args(w, X, T, A, B, r, dtype, H, U_save);
    if (v != QLORA_OK) return v;
    const size_t need = qlora_workspace_bytes(QLORA_OP_FWD, dtype, T, w->d_out, w->d_in, r);
    if (need == 0 || need > kNoAllocScratchBytes) return QLORA_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    const qlora_status s = scratch_address(stream, &scratch);
    if (s != QLORA_OK) return s;
    return qlora_linear_fwd(w, X, T, A, B, r, alpha, dtype, H, U_save, scratch,
                            kNoAllocScratchBytes, stream);
}
