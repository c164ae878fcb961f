// wkv7_gate.cu — gated read-out of the WKV output as a separate pass, used for
// fp32 inputs (the bf16 prefill kernel applies it to its output rows directly):
//
//   u = sum_d r_d k_d rk[h][d],   z_i = (y_i / sqrt(D) + u v_i) g_i
//
// the steps the forward listing of "RWKV hxa07D architecture explainer"
// applies to the WKV result before its output projection (scaling, the r-k-v
// term with the per-head weights r_k, the output gate; section 9 of that page).
// One warp per (token, head) row: lane l holds elements 2l and 2l + 1.
#include "wkv7_internal.cuh"

namespace wkv7 {
namespace {

template <typename T>
__global__ void __launch_bounds__(256) wkv7_gate_kernel(T* __restrict__ z, const T* __restrict__ r,
                                                        const T* __restrict__ k, const T* __restrict__ v,
                                                        const float* __restrict__ rk, const T* __restrict__ g,
                                                        long rows, int H) {
    const long row = static_cast<long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int lane = threadIdx.x & 31, h = static_cast<int>(row % H);
    const long e = row * kHead + 2 * lane;
    const float* rkh = rk + static_cast<long>(h) * kHead + 2 * lane;
    float u = to_f32(r[e]) * to_f32(k[e]) * rkh[0] + to_f32(r[e + 1]) * to_f32(k[e + 1]) * rkh[1];
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) u += __shfl_xor_sync(0xffffffffu, u, m);
    constexpr float scale = 0.125f;  // 1 / sqrt(64)
#pragma unroll
    for (int i = 0; i < 2; ++i)
        z[e + i] = from_f32<T>((to_f32(z[e + i]) * scale + u * to_f32(v[e + i])) * to_f32(g[e + i]));
}

}  // namespace

cudaError_t launch_gate(void* z, const void* r, const void* k, const void* v, const float* rk, const void* g,
                        long ntok, int H, int io_dtype, cudaStream_t stream) {
    const long rows = ntok * H;
    if (rows <= 0) return cudaSuccess;
    const unsigned blocks = static_cast<unsigned>((rows + 7) / 8);
    if (io_dtype == WKV7_F32)
        wkv7_gate_kernel<float><<<blocks, 256, 0, stream>>>(
            static_cast<float*>(z), static_cast<const float*>(r), static_cast<const float*>(k),
            static_cast<const float*>(v), rk, static_cast<const float*>(g), rows, H);
    else
        wkv7_gate_kernel<__nv_bfloat16><<<blocks, 256, 0, stream>>>(
            static_cast<__nv_bfloat16*>(z), static_cast<const __nv_bfloat16*>(r),
            static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), rk,
            static_cast<const __nv_bfloat16*>(g), rows, H);
    return cudaGetLastError();
}

}  // namespace wkv7
