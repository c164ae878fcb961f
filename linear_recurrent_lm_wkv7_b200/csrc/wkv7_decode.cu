// wkv7_decode.cu — one recurrent step per sequence (RNN-mode decoding).
//
// Per (sequence, head) unit the step reads the D x D fp32 state once and writes
// it once, which is where all the time goes (the recurrent mode of "RWKV-7 Goose
// architecture analysis", youngju.dev: constant memory and time per token).
// Per value row i:
//   sa_i = sum_j S_ij a_j                 (previous state)
//   S_ij <- S_ij w_j + sa_i b_j + v_i k_j (w_j = exp(-exp(w_log_j)))
//   y_i  = sum_j S_ij r_j                 (updated state)
//
// Mapping: one 256-thread block per unit.  A thread owns 4 consecutive key
// columns (one 16-byte vector) of 4 value rows spaced 16 apart; 16 threads
// cover one row, so both row reductions are 4 xor-shuffles inside a 16-lane
// group.  All four 16-byte state loads are issued before any arithmetic, the
// state is read and written with streaming (evict-first) accesses, and a block
// moves 32 KB of state, so an SM keeps ~128 KB of loads in flight.
#include "wkv7_internal.cuh"

namespace wkv7 {
namespace {

template <typename T>
__device__ __forceinline__ void load4(const T* p, float (&o)[4]);
template <>
__device__ __forceinline__ void load4<float>(const float* p, float (&o)[4]) {
    const float4 x = __ldg(reinterpret_cast<const float4*>(p));
    o[0] = x.x; o[1] = x.y; o[2] = x.z; o[3] = x.w;
}
template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16* p, float (&o)[4]) {
    const uint2 x = __ldg(reinterpret_cast<const uint2*>(p));
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&x.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&x.y);
    const float2 fl = __bfloat1622float2(lo), fh = __bfloat1622float2(hi);
    o[0] = fl.x; o[1] = fl.y; o[2] = fh.x; o[3] = fh.y;
}

__device__ __forceinline__ float sum16(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 8);
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    return x;
}

template <typename IO, typename WT>
__global__ void __launch_bounds__(256) wkv7_decode_kernel(const IO* __restrict__ r, const WT* __restrict__ wl,
                                                          const IO* __restrict__ k, const IO* __restrict__ v,
                                                          const IO* __restrict__ a, const IO* __restrict__ b,
                                                          const float* s_in, IO* __restrict__ y, float* s_out) {
    const long unit = blockIdx.x;
    const int tid = threadIdx.x;
    const int cg = tid & 15;  // key columns 4*cg .. 4*cg+3
    const int rg = tid >> 4;  // value rows rg, rg+16, rg+32, rg+48
    const long vbase = unit * kHead;
    const long sbase = unit * kHead * kHead;

    float4 s[4];
    if (s_in) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
            s[q] = __ldcs(reinterpret_cast<const float4*>(s_in + sbase + (rg + 16 * q) * kHead + 4 * cg));
    } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) s[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float wv[4], av[4], bv[4], kv[4], rv[4];
    load4(wl + vbase + 4 * cg, wv);
    load4(a + vbase + 4 * cg, av);
    load4(b + vbase + 4 * cg, bv);
    load4(k + vbase + 4 * cg, kv);
    load4(r + vbase + 4 * cg, rv);
#pragma unroll
    for (int c = 0; c < 4; ++c) wv[c] = expf(-expf(wv[c]));
    float vrow[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) vrow[q] = to_f32(v[vbase + rg + 16 * q]);

#pragma unroll
    for (int q = 0; q < 4; ++q) {
        float4 x = s[q];
        const float sa = sum16(x.x * av[0] + x.y * av[1] + x.z * av[2] + x.w * av[3]);
        const float vi = vrow[q];
        x.x = fmaf(x.x, wv[0], fmaf(sa, bv[0], vi * kv[0]));
        x.y = fmaf(x.y, wv[1], fmaf(sa, bv[1], vi * kv[1]));
        x.z = fmaf(x.z, wv[2], fmaf(sa, bv[2], vi * kv[2]));
        x.w = fmaf(x.w, wv[3], fmaf(sa, bv[3], vi * kv[3]));
        const float yi = sum16(x.x * rv[0] + x.y * rv[1] + x.z * rv[2] + x.w * rv[3]);
        __stcs(reinterpret_cast<float4*>(s_out + sbase + (rg + 16 * q) * kHead + 4 * cg), x);
        if (cg == 0) y[vbase + rg + 16 * q] = from_f32<IO>(yi);
    }
}

template <typename IO, typename WT>
cudaError_t launch_typed(const DecodeArgs& p, cudaStream_t stream) {
    const long units = static_cast<long>(p.B) * p.H;
    wkv7_decode_kernel<IO, WT><<<static_cast<unsigned>(units), 256, 0, stream>>>(
        static_cast<const IO*>(p.r), static_cast<const WT*>(p.w_log), static_cast<const IO*>(p.k),
        static_cast<const IO*>(p.v), static_cast<const IO*>(p.a), static_cast<const IO*>(p.b), p.s_in,
        static_cast<IO*>(p.y), p.s_out);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& p, int io_dtype, int w_dtype, cudaStream_t stream) {
    if (io_dtype == WKV7_BF16) {
        return w_dtype == WKV7_BF16 ? launch_typed<__nv_bfloat16, __nv_bfloat16>(p, stream)
                                    : launch_typed<__nv_bfloat16, float>(p, stream);
    }
    return w_dtype == WKV7_BF16 ? launch_typed<float, __nv_bfloat16>(p, stream) : launch_typed<float, float>(p, stream);
}

}  // namespace wkv7
