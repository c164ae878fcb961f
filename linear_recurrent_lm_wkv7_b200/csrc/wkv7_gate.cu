// wkv7_gate.cu — gated read-out of the WKV output as a separate pass, used for
// fp32 inputs (the bf16 prefill kernel applies it to its output rows directly):
//
//   u = sum_d r_d k_d rk[h][d],   z_i = (y_i / sqrt(D) + u v_i) g_i
//
// the steps the forward listing of "RWKV hxa07D architecture explainer"
// applies to the WKV result before its output projection (scaling, the r-k-v
// term with the per-head weights r_k, the output gate; section 9 of that page).
// One warp per (token, head) row: lane l holds elements 2l and 2l + 1.
// PRO (after wkv7_forward_fused): the key of the r-k-v term is the prologue's
// scaled key k (1 - w + a_lr), and k and v are rows of kv head h / (H / H_kv).
#include "wkv7_internal.cuh"

namespace wkv7 {
namespace {

template <typename T, typename WT, bool PRO>
__global__ void __launch_bounds__(256) wkv7_gate_kernel(T* __restrict__ z, const T* __restrict__ r,
                                                        const T* __restrict__ k, const T* __restrict__ v,
                                                        const float* __restrict__ rk, const T* __restrict__ g,
                                                        long rows, int H, const WT* __restrict__ wl,
                                                        const T* __restrict__ a_lr, int H_kv) {
    const long row = static_cast<long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int lane = threadIdx.x & 31, h = static_cast<int>(row % H);
    const long e = row * kHead + 2 * lane;
    // k and v element of this lane (kv head under the prologue)
    const long ekv = PRO ? ((row / H) * H_kv + h / (H / H_kv)) * kHead + 2 * lane : e;
    const float* rkh = rk + static_cast<long>(h) * kHead + 2 * lane;
    float k0 = to_f32(k[ekv]), k1 = to_f32(k[ekv + 1]);
    if constexpr (PRO) {
        k0 *= 1.f - expf(-expf(to_f32(wl[e]))) + to_f32(a_lr[e]);
        k1 *= 1.f - expf(-expf(to_f32(wl[e + 1]))) + to_f32(a_lr[e + 1]);
    }
    float u = to_f32(r[e]) * k0 * rkh[0] + to_f32(r[e + 1]) * k1 * rkh[1];
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) u += __shfl_xor_sync(0xffffffffu, u, m);
    constexpr float scale = 0.125f;  // 1 / sqrt(64)
#pragma unroll
    for (int i = 0; i < 2; ++i)
        z[e + i] = from_f32<T>((to_f32(z[e + i]) * scale + u * to_f32(v[ekv + i])) * to_f32(g[e + i]));
}

template <typename T, typename WT, bool PRO>
void launch_gate_typed(void* z, const void* r, const void* k, const void* v, const float* rk, const void* g, long rows,
                       int H, const void* w_log, const void* a_lr, int H_kv, cudaStream_t stream) {
    const unsigned blocks = static_cast<unsigned>((rows + 7) / 8);
    wkv7_gate_kernel<T, WT, PRO><<<blocks, 256, 0, stream>>>(
        static_cast<T*>(z), static_cast<const T*>(r), static_cast<const T*>(k), static_cast<const T*>(v), rk,
        static_cast<const T*>(g), rows, H, static_cast<const WT*>(w_log), static_cast<const T*>(a_lr), H_kv);
}

}  // namespace

cudaError_t launch_gate(void* z, const void* r, const void* k, const void* v, const float* rk, const void* g,
                        long ntok, int H, int io_dtype, cudaStream_t stream, const void* w_log, const void* a_lr,
                        int H_kv, int w_dtype) {
    const long rows = ntok * H;
    if (rows <= 0) return cudaSuccess;
    const bool pro = a_lr != nullptr;
    if (io_dtype == WKV7_F32) {
        if (!pro)
            launch_gate_typed<float, float, false>(z, r, k, v, rk, g, rows, H, nullptr, nullptr, H, stream);
        else if (w_dtype == WKV7_BF16)
            launch_gate_typed<float, __nv_bfloat16, true>(z, r, k, v, rk, g, rows, H, w_log, a_lr, H_kv, stream);
        else
            launch_gate_typed<float, float, true>(z, r, k, v, rk, g, rows, H, w_log, a_lr, H_kv, stream);
    } else {
        if (pro) return cudaErrorInvalidValue;  // the bf16 kernel fuses both itself
        launch_gate_typed<__nv_bfloat16, float, false>(z, r, k, v, rk, g, rows, H, nullptr, nullptr, H, stream);
    }
    return cudaGetLastError();
}

}  // namespace wkv7
