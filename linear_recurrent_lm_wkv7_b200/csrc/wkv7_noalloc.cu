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

// Address of the scratch on the current device.  cudaGetSymbolAddress
// allocates nothing and is cheap, so it runs on every call: no cached address
// can outlive a device reset, and host threads share no mutable state here.
// The first call on a device may load the library's module there (which is
// why that first call should come before any stream capture).
int scratch_for_current_device(void** out) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || !p) return WKV7_ERR_CUDA;
    *out = p;
    return WKV7_OK;
}

}  // namespace

extern "C" int wkv7_backward_noalloc(const void* r, const void* w_log, const void* k, const void* v, const void* a,
                                     const void* b, const float* s0, const void* dy, const float* dsT, void* dr,
                                     void* dw_log, void* dk, void* dv, void* da, void* db, float* ds0, int B, int T,
                                     int H, int D, const int32_t* seq_offsets, int io_dtype, int w_dtype,
                                     void* stream) {
    // The argument checks that come before the scratch limit, in wkv7_backward's
    // order, so that both entry points return the same code for the same bad
    // arguments; the remaining checks are wkv7_backward's own.
    if (B <= 0 || T < 0 || H <= 0 || D <= 0) return WKV7_ERR_INVALID_ARG;
    const bool dt_ok = (io_dtype == WKV7_F32 || io_dtype == WKV7_BF16) && (w_dtype == WKV7_F32 || w_dtype == WKV7_BF16);
    if (!dt_ok) return WKV7_ERR_INVALID_ARG;
    if (D != 64) return WKV7_ERR_UNSUPPORTED;
    if (!ds0) return WKV7_ERR_INVALID_ARG;
    if (wkv7_backward_workspace_bytes(B, T, H, D, seq_offsets ? 1 : 0) > kScratchBytes) return WKV7_ERR_SCRATCH_LIMIT;
    void* ws = nullptr;
    const int st = scratch_for_current_device(&ws);
    if (st != WKV7_OK) return st;
    return wkv7_backward(r, w_log, k, v, a, b, s0, dy, dsT, dr, dw_log, dk, dv, da, db, ds0, ws, kScratchBytes, B, T,
                         H, D, seq_offsets, io_dtype, w_dtype, stream);
}
