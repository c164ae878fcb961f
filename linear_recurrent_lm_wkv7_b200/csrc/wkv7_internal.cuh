// wkv7_internal.cuh — launch interface between the C-ABI layer (wkv7_api.cu)
// and the kernels (wkv7_decode.cu, wkv7_prefill*.cu, wkv7_gate.cu).  Not part of the ABI.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "wkv7.h"

namespace wkv7 {

constexpr int kHead = 64;  // D: head size supported by every kernel
// Smallest decay a 64-token chunk of the prefill may accumulate in one key
// channel (Gamma_64 = prod of w over the chunk): the chunked algebra scales
// operands by 1 / Gamma_t, which must stay far from the fp32 / bf16 overflow
// at 3.4e38.  Smaller values are reported as WKV7_ERR_DECAY_RANGE.
constexpr float kMinGammaL = 1e-30f;

struct PrefillArgs {
    const void* r;
    const void* w_log;
    const void* k;
    const void* v;
    const void* a;
    const void* b;
    const float* s0;
    void* y;
    float* sT;
    int B, T, H;
    const int32_t* seq_offsets;
    int* status;  // device status word of the current device
    // gated read-out (wkv7_forward_gated): y then holds z; both null otherwise
    const float* rk = nullptr;  // [H][D] fp32
    const void* g = nullptr;    // gate, same layout and dtype as r
    // fused prologue (wkv7_forward_fused): a holds a_lr, b is unused, k and v
    // have H_kv heads; the kernels form kk, a, b and the scaled key themselves
    bool prologue = false;
    int H_kv = 0;
    // state map (wkv7_state_map): v is treated as zero (v may be any valid pointer),
    // the initial state is the identity (s0 ignored); y == nullptr writes no y rows
    bool zero_v = false;
    bool s0_identity = false;
    // two-phase prefill (wkv7_forward_long), first phase: each chunk's
    // state-independent results go to the workspace arrays below (layouts in
    // wkv7_prefill_pipe.cu)
    uint8_t* ex_as = nullptr;
    float* ex_out = nullptr;
    float* ex_gam = nullptr;
};

struct DecodeArgs {
    const void* r;
    const void* w_log;
    const void* k;
    const void* v;
    const void* a;
    const void* b;
    const float* s_in;
    void* y;
    float* s_out;
    int B, H;
    // fused prologue (wkv7_decode_step_fused): a holds a_lr, b is unused, k and v
    // have H_kv heads; rk and g (both or neither) add the gated read-out
    bool prologue = false;
    int H_kv = 0;
    const float* rk = nullptr;
    const void* g = nullptr;
};

struct BackwardArgs {
    const void* r;
    const void* w_log;
    const void* k;
    const void* v;
    const void* a;
    const void* b;
    const float* s0;   // null: zero initial state
    const void* dy;
    const float* dsT;  // null: no gradient on the final state
    void* dr;
    void* dw_log;
    void* dk;
    void* dv;
    void* da;
    void* db;
    float* ds0;
    float* ws;  // workspace (layout owned by the kernel that uses it)
    int B, T, H;
    const int32_t* seq_offsets;
    long ckpt_chunks;  // checkpoint slots per head in the workspace
    int* status;
};

cudaError_t launch_prefill(const PrefillArgs& p, int io_dtype, int w_dtype, cudaStream_t stream);
// warp-specialised kernel for bf16 inputs (wkv7_prefill_pipe.cu)
cudaError_t launch_prefill_pipe(const PrefillArgs& p, int w_dtype, cudaStream_t stream);
// its export mode: the first phase of the two-phase prefill (dense bf16 batches)
cudaError_t launch_prefill_pipe_export(const PrefillArgs& p, int w_dtype, cudaStream_t stream);
// two-phase prefill (wkv7_prefill_long.cu): workspace bytes, and both phases
size_t prefill_long_workspace_bytes(int B, int T, int H);
cudaError_t launch_prefill_long(const PrefillArgs& p, int w_dtype, void* ws, cudaStream_t stream);
cudaError_t launch_decode(const DecodeArgs& p, int io_dtype, int w_dtype, int* status, cudaStream_t stream);
// z <- (z / sqrt(D) + (sum_d r k rk) v) * g in place over ntok x H rows (wkv7_gate.cu).
// With a_lr non-null (after the fused prologue) the key is k (1 - w + a_lr) with
// w = exp(-exp(w_log)), and k, v are rows of kv head h / (H / H_kv).
cudaError_t launch_gate(void* z, const void* r, const void* k, const void* v, const float* rk, const void* g,
                        long ntok, int H, int io_dtype, cudaStream_t stream, const void* w_log = nullptr,
                        const void* a_lr = nullptr, int H_kv = 0, int w_dtype = WKV7_F32);
cudaError_t launch_expire_wait(int spins, int* status, cudaStream_t stream);
// S_out = S_in M + Q for n (sequence, head) units (S_in null: zero), fp32 (wkv7_state.cu)
cudaError_t launch_state_apply(const float* S_in, const float* M, const float* Q, float* S_out, long n,
                               cudaStream_t stream);
// M <- identity, Q <- 0 for n units (the map of an empty token range); either may be null
cudaError_t launch_state_identity(float* M, float* Q, long n, cudaStream_t stream);
// backward of the recurrence in chunked form (wkv7_backward.cu)
long backward_ckpt_chunks(int B, int T, int packed);
size_t backward_workspace_floats(int B, int T, int H, int packed);
cudaError_t launch_backward(const BackwardArgs& p, int io_dtype, int w_dtype, cudaStream_t stream);

// Raises `kern`'s dynamic shared-memory limit to `bytes` the first time it is
// launched on the current device.  `configured` holds one bit per device
// ordinal below 64 (ordinals from 64 up set the attribute on every call).  Two
// threads that launch first at the same time may both set it, which is
// harmless: the call is idempotent.
template <typename K>
cudaError_t configure_smem_once(K kern, int bytes, std::atomic<unsigned long long>& configured) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = dev < 64 ? 1ull << dev : 0ull;
    if (bit && (configured.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit, std::memory_order_release);
    return cudaSuccess;
}

// Records the first device-side error of a call sequence (first writer wins).
__device__ __forceinline__ void report_status(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f32(float x) { return x; }
template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

}  // namespace wkv7
