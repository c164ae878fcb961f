// tma_host.cuh — host-side construction of the TMA descriptors the prefill
// kernels use: every token-major input viewed as [tokens][H][64] with a box of
// 64 tokens x 1 head x 64 channels (one chunk of one head).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace wkv7 {

struct TmaMaps {
    CUtensorMap r, k, a, b, wl, v;
};

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
inline EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    }
    return fn;
}

// [ntok][H][64] tensor of `esize`-byte elements, box 64 x 1 x 64; rows beyond
// ntok read as zeros.
inline bool make_token_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t esize, uint64_t H,
                           uint64_t ntok, CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {64, H, ntok};
    const cuuint64_t strides[2] = {64 * esize, H * 64 * esize};
    const cuuint32_t box[3] = {64, 1, 64};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Maps for bf16 r, a, b over H heads, bf16 k over H_kv heads (no swizzle), w_log of
// `wbytes`-byte elements over H heads (no swizzle) and bf16 v over H_kv heads
// (128-byte swizzle: the MN-major operand layout).  b may be null (no map).
inline bool make_prefill_maps(TmaMaps* m, const void* r, const void* wl, const void* k, const void* v, const void* a,
                              const void* b, uint64_t H, uint64_t H_kv, uint64_t ntok, uint32_t wbytes) {
    const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const CUtensorMapDataType wdt = wbytes == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const CUtensorMapSwizzle none = CU_TENSOR_MAP_SWIZZLE_NONE;
    return make_token_map(&m->r, r, bf, 2, H, ntok, none) && make_token_map(&m->k, k, bf, 2, H_kv, ntok, none) &&
           make_token_map(&m->a, a, bf, 2, H, ntok, none) &&
           (b == nullptr || make_token_map(&m->b, b, bf, 2, H, ntok, none)) &&
           make_token_map(&m->wl, wl, wdt, wbytes, H, ntok, none) &&
           make_token_map(&m->v, v, bf, 2, H_kv, ntok, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace wkv7
