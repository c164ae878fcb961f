// wkv7_state.cu — the affine maps of token ranges: S_out = S_in M + Q per
// (sequence, head) unit, and the identity map of an empty range.
//
// Over a token range the recurrence is affine in its start state, since each
// step maps S to S (diag(w_t) + a_t b_t^T) + v_t k_t^T (the generalized delta rule
// of "RWKV-7 Goose: Expressive Dynamic State Evolution", section "Generalized
// Delta rule").  With M = prod_t (diag(w_t) + a_t b_t^T) (key x key) and Q the
// end state from S = 0, the end state from any S is S M + Q.  Splitting a long
// sequence into ranges therefore needs only these maps to hand each range its
// start state.
#include "wkv7_internal.cuh"

namespace wkv7 {
namespace {

constexpr int D = kHead;

// One block of 256 threads per unit: thread t computes row i = t / 4 of the
// output, columns 16 (t % 4) .. 16 (t % 4) + 15, in fp32 from S_in and M staged
// in shared memory (S_in is read before any output is written, so S_out may be
// S_in).
__global__ void __launch_bounds__(256) state_apply_kernel(const float* __restrict__ S_in, const float* __restrict__ M,
                                                          const float* __restrict__ Q, float* S_out) {
    __shared__ float sS[D * D];
    __shared__ __align__(16) float sM[D * D];
    const long base = static_cast<long>(blockIdx.x) * D * D;
    const int t = threadIdx.x;
    for (int e = t; e < D * D / 4; e += 256) {
        const float4 m4 = reinterpret_cast<const float4*>(M + base)[e];
        reinterpret_cast<float4*>(sM)[e] = m4;
        const float4 s4 = S_in ? reinterpret_cast<const float4*>(S_in + base)[e] : make_float4(0.f, 0.f, 0.f, 0.f);
        reinterpret_cast<float4*>(sS)[e] = s4;
    }
    __syncthreads();
    const int i = t >> 2, j0 = 16 * (t & 3);
    float acc[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) acc[c] = Q[base + i * D + j0 + c];
    if (S_in) {
#pragma unroll 4
        for (int jp = 0; jp < D; ++jp) {
            const float s = sS[i * D + jp];
            const float4* mrow = reinterpret_cast<const float4*>(sM + jp * D + j0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 m4 = mrow[q];
                acc[4 * q + 0] = fmaf(s, m4.x, acc[4 * q + 0]);
                acc[4 * q + 1] = fmaf(s, m4.y, acc[4 * q + 1]);
                acc[4 * q + 2] = fmaf(s, m4.z, acc[4 * q + 2]);
                acc[4 * q + 3] = fmaf(s, m4.w, acc[4 * q + 3]);
            }
        }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q)
        reinterpret_cast<float4*>(S_out + base + i * D + j0)[q] =
            make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
}

__global__ void state_identity_kernel(float* M, float* Q, long n) {
    const long total = n * D * D;
    for (long e = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
         e += static_cast<long>(gridDim.x) * blockDim.x) {
        const int rc = static_cast<int>(e % (D * D));
        if (M) M[e] = (rc / D == rc % D) ? 1.f : 0.f;
        if (Q) Q[e] = 0.f;
    }
}

}  // namespace

cudaError_t launch_state_apply(const float* S_in, const float* M, const float* Q, float* S_out, long n,
                               cudaStream_t stream) {
    if (n <= 0) return cudaSuccess;
    state_apply_kernel<<<static_cast<unsigned>(n), 256, 0, stream>>>(S_in, M, Q, S_out);
    return cudaGetLastError();
}

cudaError_t launch_state_identity(float* M, float* Q, long n, cudaStream_t stream) {
    if (n <= 0) return cudaSuccess;
    const long total = n * D * D;
    const int blocks = static_cast<int>((total + 255) / 256 < 1184 ? (total + 255) / 256 : 1184);
    state_identity_kernel<<<blocks, 256, 0, stream>>>(M, Q, n);
    return cudaGetLastError();
}

}  // namespace wkv7
