// prefill_common.cuh — operand-tile helpers shared by the two chunked
// prefill kernels: element and row accessors of 128-byte swizzled bf16 / tf32
// tiles, matrix descriptors, TMEM stores and group barriers.
#pragma once
#include <cuda_bf16.h>

#include <cstdint>

#include "sm100_ptx.cuh"

namespace wkv7 {

// bf16 pair <-> 32-bit word without taking addresses (keeps values in registers)
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ float bf16lo_to_f32(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

template <bool TF32>
struct OpType {
    static constexpr uint32_t EB = TF32 ? 4 : 2;       // bytes per operand element
    static constexpr uint32_t FMT = TF32 ? 2 : 1;      // instruction-descriptor format
    static constexpr uint32_t KSTEP = TF32 ? 8 : 16;   // K per tcgen05.mma
    static constexpr uint32_t KSTEPS = 64 / KSTEP;     // MMAs per K = 64
    static constexpr uint32_t TILE64 = 64 * 64 * EB;   // 64 rows x 64 elements
    static constexpr uint32_t TILE128 = 128 * 64 * EB; // 128 rows x 64 elements
};

__device__ __forceinline__ float round_tf32(float x) {
    uint32_t u;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(u) : "f"(x));
    return __uint_as_float(u);
}

// element (row, col) of a swizzled operand tile with R rows
template <bool TF32>
__device__ __forceinline__ void st_op(uint8_t* tile, uint32_t R, uint32_t row, uint32_t col, float x) {
    if constexpr (TF32) {
        *reinterpret_cast<float*>(tile + swz(row, col * 4, R)) = round_tf32(x);
    } else {
        *reinterpret_cast<__nv_bfloat16*>(tile + swz(row, col * 2, R)) = __float2bfloat16_rn(x);
    }
}
template <bool TF32>
__device__ __forceinline__ float ld_op(const uint8_t* tile, uint32_t R, uint32_t row, uint32_t col) {
    if constexpr (TF32) {
        return *reinterpret_cast<const float*>(tile + swz(row, col * 4, R));
    } else {
        return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(tile + swz(row, col * 2, R)));
    }
}
// 32 consecutive elements [c0, c0+32) of one row, written with 16-byte stores
template <bool TF32>
__device__ __forceinline__ void st_op_row32(uint8_t* tile, uint32_t R, uint32_t row, uint32_t c0, const float* x) {
    if constexpr (TF32) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            float4 v = make_float4(round_tf32(x[4 * q]), round_tf32(x[4 * q + 1]), round_tf32(x[4 * q + 2]),
                                   round_tf32(x[4 * q + 3]));
            *reinterpret_cast<float4*>(tile + swz(row, (c0 + 4 * q) * 4, R)) = v;
        }
    } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 v = make_uint4(pack_bf16x2(x[8 * q], x[8 * q + 1]), pack_bf16x2(x[8 * q + 2], x[8 * q + 3]),
                                       pack_bf16x2(x[8 * q + 4], x[8 * q + 5]),
                                       pack_bf16x2(x[8 * q + 6], x[8 * q + 7]));
            *reinterpret_cast<uint4*>(tile + swz(row, (c0 + 8 * q) * 2, R)) = v;
        }
    }
}
template <bool TF32>
__device__ __forceinline__ void ld_op_row32(const uint8_t* tile, uint32_t R, uint32_t row, uint32_t c0, float* x) {
    if constexpr (TF32) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 v = *reinterpret_cast<const float4*>(tile + swz(row, (c0 + 4 * q) * 4, R));
            x[4 * q] = v.x; x[4 * q + 1] = v.y; x[4 * q + 2] = v.z; x[4 * q + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 v = *reinterpret_cast<const uint4*>(tile + swz(row, (c0 + 8 * q) * 2, R));
            x[8 * q + 0] = bf16lo_to_f32(v.x); x[8 * q + 1] = bf16hi_to_f32(v.x);
            x[8 * q + 2] = bf16lo_to_f32(v.y); x[8 * q + 3] = bf16hi_to_f32(v.y);
            x[8 * q + 4] = bf16lo_to_f32(v.z); x[8 * q + 5] = bf16hi_to_f32(v.z);
            x[8 * q + 6] = bf16lo_to_f32(v.w); x[8 * q + 7] = bf16hi_to_f32(v.w);
        }
    }
}

// Descriptor of K-step s of a K-major operand tile with R rows (K = 64 elements).
template <bool TF32>
__device__ __forceinline__ uint64_t kmajor_desc(const uint8_t* tile, uint32_t R, uint32_t s) {
    const uint32_t kbyte = s * 32u;  // 16 bf16 or 8 tf32 per step
    const uint32_t addr = smem_u32(tile) + (kbyte >> 7) * (R << 7) + (kbyte & 127u);
    return sdesc_sw128(addr, 16, 1024);
}
// Descriptor of K-step s of an MN-major operand tile whose rows are K (R rows).
template <bool TF32>
__device__ __forceinline__ uint64_t mnmajor_desc(const uint8_t* tile, uint32_t R, uint32_t s) {
    const uint32_t addr = smem_u32(tile) + s * OpType<TF32>::KSTEP * 128u;
    return sdesc_sw128(addr, R * 128u, 1024);
}


// Barrier over the `nthreads` threads of one warp group (named barrier `id`),
// returning the AND of `pred` over them.
// The warp is reconverged first (the callers come out of divergent bounded
// waits), and the non-aligned barrier form is used.
__device__ __forceinline__ bool group_sync_and(uint32_t id, uint32_t nthreads, bool pred) {
    uint32_t r;
    __syncwarp();
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"(pred ? 1u : 0u), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void group_sync(uint32_t id, uint32_t nthreads) {
    __syncwarp();
    asm volatile("barrier.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Plain arrive (release) on an mbarrier.
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Hint: fetch the cache line holding global address p into L2.
__device__ __forceinline__ void prefetch_line_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

}  // namespace wkv7
