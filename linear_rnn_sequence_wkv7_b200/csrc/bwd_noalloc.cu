// wkv7_backward_noalloc: the backward without any caller-provided or
// library-allocated workspace.
//
// Some callers cannot allocate device memory at the point where they need the
// backward: an inference/training engine plugin whose enqueue path must not
// call the allocator, or a framework whose memory pool has already reserved
// the device's memory (an extra cudaMalloc would fail, or stall the stream
// while the driver synchronizes).  For them this entry point takes its scratch
// (state checkpoints and the recompute history) from a fixed array in device
// global memory that is part of the library image.
//
// Limits and rules:
//  - The array holds kNoAllocScratchBytes (32 MiB).  Every GPU that loads the
//    library keeps it resident until the process exits.  A problem whose
//    minimum scratch (wkv7_backward_workspace_size without the chunks'
//    transition images) exceeds it is rejected with WKV7_ERR_TOO_LARGE before
//    anything is launched; one whose full size fits also takes the transition
//    chain for dS.
//  - Host code cannot pass the array's name to a kernel (on the host it is
//    only a stand-in symbol).  The first call on each device looks up the
//    array's device address with cudaGetSymbolAddress, with that device
//    current, and caches it; make that first call before any stream capture.
//  - All calls share the one array and it keeps the previous call's contents.
//    The backward writes every scratch byte it reads before reading it, so no
//    clearing is needed.  Calls whose work overlaps on the GPU (other streams,
//    other host threads) race on the array; serialize them.
//  - Nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include <mutex>

#include "common.cuh"

namespace wkv7 {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 128;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mutex;
void *g_noalloc_ptr[kMaxDevices] = {};

// Device address of the static scratch on the current device (looked up once
// per device, with that device current).
wkv7_status noalloc_scratch(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return WKV7_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return WKV7_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return WKV7_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return WKV7_OK;
}

}  // namespace
}  // namespace wkv7

extern "C" wkv7_status wkv7_backward_noalloc(int B, int T, int H, int N, wkv7_dtype in_dtype,
                                             wkv7_dtype grad_dtype, const void *r, const void *w, const void *k,
                                             const void *v, const void *a, const void *b, const float *s0,
                                             const void *dy, const float *dsT, void *dr, void *dw, void *dk,
                                             void *dv, void *da, void *db, float *ds0, cudaStream_t stream) {
    using namespace wkv7;
    if (B > 0 && T > 0 && H > 0 && N == kN && bwd_workspace_min(B, T, H) > kNoAllocScratchBytes)
        return WKV7_ERR_TOO_LARGE;
    void *scratch = nullptr;
    const wkv7_status s = noalloc_scratch(&scratch);
    if (s != WKV7_OK) return s;
    return wkv7_backward(B, T, H, N, in_dtype, grad_dtype, r, w, k, v, a, b, s0, dy, dsT, dr, dw, dk, dv, da, db,
                         ds0, scratch, kNoAllocScratchBytes, stream);
}
