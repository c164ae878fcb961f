// wkv7_noalloc.cu — wkv7_backward_noalloc: the backward with a fixed scratch
// owned by the library, for callers that cannot allocate device memory at the
// point of the call.
//
// Such callers include code that runs under a device-memory budget which
// forbids new allocations, runtimes that hand kernels only preallocated
// buffers, and latency-critical paths that must not call cudaMalloc (which can
// synchronise the device).  The scratch is a file-scope __device__ array, so
// it is allocated once, when this module is loaded, and never again.
//
// Limit: WKV7_NOALLOC_SCRATCH_BYTES (16 MiB), i.e.
// wkv7_backward_workspace_bytes(B, T, H, 64, packed) <= 16 MiB; larger
// problems get WKV7_ERR_SCRATCH_LIMIT and must use wkv7_backward with a
// caller-provided workspace.
//
// Nothing in the scratch has to start at zero: the backward writes every
// checkpoint and every recomputed state before it reads it, so no clearing is
// done.  There is one scratch per device: calls whose kernels may overlap on a
// device (different streams without ordering, or several host threads) race on
// it and must be serialised by the caller.
#include <cuda_runtime.h>

#include "wkv7.h"

namespace {

constexpr size_t kScratchBytes = WKV7_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) float g_bwd_scratch[kScratchBytes / sizeof(float)];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};

// Address of this device's scratch, looked up once per device with that device
// current (the first call on a device does this; it may load the module).
int scratch_for_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return WKV7_ERR_CUDA;
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || !p) return WKV7_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return WKV7_OK;
}

}  // namespace

extern "C" int wkv7_backward_noalloc(const void* r, const void* w_log, const void* k, const void* v, const void* a,
                                     const void* b, const float* s0, const void* dy, const float* dsT, void* dr,
                                     void* dw_log, void* dk, void* dv, void* da, void* db, float* ds0, int B, int T,
                                     int H, int D, const int32_t* seq_offsets, int io_dtype, int w_dtype,
                                     void* stream) {
    // decided before any CUDA call; the remaining checks are wkv7_backward's own
    if (B <= 0 || T < 0 || H <= 0 || D <= 0) return WKV7_ERR_INVALID_ARG;
    if (D != 64) return WKV7_ERR_UNSUPPORTED;
    if (wkv7_backward_workspace_bytes(B, T, H, D, seq_offsets ? 1 : 0) > kScratchBytes) return WKV7_ERR_SCRATCH_LIMIT;
    void* ws = nullptr;
    const int st = scratch_for_current_device(&ws);
    if (st != WKV7_OK) return st;
    return wkv7_backward(r, w_log, k, v, a, b, s0, dy, dsT, dr, dw_log, dk, dv, da, db, ds0, ws, kScratchBytes, B, T,
                         H, D, seq_offsets, io_dtype, w_dtype, stream);
}
