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
// Streaming: a persistent grid of two blocks per SM, each eight compute warps
// and one producer warp.  A block walks over units u = blockIdx.x,
// blockIdx.x + gridDim.x, ... through a ring of four shared-memory stages.  The
// producer's lane 0 fills each stage with one unit's 16 KB state and its input
// rows by untiled bulk copies (mbarrier `full` per stage); the compute warps
// update the state in place and arrive on the stage's `done` mbarrier; the
// producer then writes the state back with one bulk store and, once the store
// of the unit before has finished reading its stage, refills that stage.  The
// compute warps never wait for a copy to be issued, only for its data.
//
// Thread mapping inside a unit: a thread owns 4 consecutive key columns (one
// 16-byte vector) of 4 value rows spaced 16 apart; 16 threads cover one row,
// so both row reductions are 4 xor-shuffles inside a 16-lane group.
//
// PRO (wkv7_decode_step_fused): the prologue of the WKV call on the raw inputs
// ("RWKV hxa07D architecture explainer", forward listing before the WKV call):
// k and v are rows of kv head h / (H / H_kv), the `a` row carries a_lr, and
//   kk = k / max(||k||, 1e-12),  a = -kk,  b = kk a_lr,  k <- k (1 - w + a_lr)
// (the norm is one more 16-lane reduction); `b` is not read.  GATED: the output
// row is z = (y / sqrt(D) + u v) (.) g with u = sum_d r k rk (k the scaled key),
// the read-out the same listing applies after the call; r_k and g rows join the
// stage's inputs.
#include "prefill_common.cuh"
#include "sm100_ptx.cuh"
#include "wkv7_internal.cuh"

namespace wkv7 {
namespace {

constexpr int NST = 4;                        // pipeline stages per block
constexpr int BLOCKS_PER_SM = 2;              // measured: 3 per SM streams slower (66 vs 58 us per B256 H40 step)
constexpr uint32_t ST_STATE = kHead * kHead * 4;  // 16 KB fp32 state
constexpr uint32_t ST_BYTES = ST_STATE + 2048;    // + input rows (at most 8 x 256 B)
constexpr uint32_t SMEM_BYTES = NST * ST_BYTES + 2 * NST * 8;  // stages, then full[NST], done[NST]
constexpr int NCONS = 256;                                      // compute threads
constexpr int NTHR = NCONS + 32;                                // + the producer warp
constexpr uint64_t WAIT_NS = 1000000000ull;  // 1 s

template <typename T>
__device__ __forceinline__ void lds4(const uint8_t* p, float (&o)[4]);
template <>
__device__ __forceinline__ void lds4<float>(const uint8_t* p, float (&o)[4]) {
    const float4 x = *reinterpret_cast<const float4*>(p);
    o[0] = x.x; o[1] = x.y; o[2] = x.z; o[3] = x.w;
}
template <>
__device__ __forceinline__ void lds4<__nv_bfloat16>(const uint8_t* p, float (&o)[4]) {
    const uint2 x = *reinterpret_cast<const uint2*>(p);
    o[0] = __uint_as_float(x.x << 16); o[1] = __uint_as_float(x.x & 0xFFFF0000u);
    o[2] = __uint_as_float(x.y << 16); o[3] = __uint_as_float(x.y & 0xFFFF0000u);
}
template <typename T>
__device__ __forceinline__ float lds1(const uint8_t* p, int i) {
    return to_f32(reinterpret_cast<const T*>(p)[i]);
}

__device__ __forceinline__ float sum16(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 8);
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    return x;
}

template <typename IO, typename WT, bool PRO, bool GATED>
__global__ void __launch_bounds__(NTHR, BLOCKS_PER_SM)
    wkv7_decode_kernel(const IO* __restrict__ r, const WT* __restrict__ wl, const IO* __restrict__ k,
                       const IO* __restrict__ v, const IO* __restrict__ a, const IO* __restrict__ b,
                       const float* s_in, IO* __restrict__ y, float* s_out, long units, int* status, int H,
                       int H_kv, const float* __restrict__ rk, const IO* __restrict__ gte) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + NST * ST_BYTES);
    uint64_t* done = full + NST;
    const int tid = threadIdx.x;
    constexpr uint32_t IOB = sizeof(IO) * kHead, WB = sizeof(WT) * kHead;
    constexpr uint32_t O_R = ST_STATE, O_K = O_R + IOB, O_V = O_K + IOB, O_A = O_V + IOB, O_B = O_A + IOB,
                       O_W = O_B + IOB, O_RK = O_W + WB, O_G = O_RK + kHead * 4;
    static_assert(O_G + IOB <= ST_BYTES, "stage inputs overflow");

    if (tid == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&done[i], NCONS);
        }
        fence_mbar_init();
    }
    __syncthreads();

    const long first = blockIdx.x, stride = gridDim.x;
    const long nmine = first < units ? (units - first + stride - 1) / stride : 0;

    if (tid >= NCONS) {
        // ------------------------------------------------------------ producer
        if (tid != NCONS) return;
        const uint32_t tx = (s_in ? ST_STATE : 0u) + (PRO ? 4u : 5u) * IOB + WB + (GATED ? kHead * 4u + IOB : 0u);
        long n_issued = 0;
        // sequence and head of the next unit to issue: units are issued in order, so they
        // advance by the grid stride with one carry (no division per unit)
        long in_n = first / H;
        int in_h = static_cast<int>(first % H);
        const long step_n = stride / H;
        const int step_h = static_cast<int>(stride % H);
        const int rep = PRO ? H / H_kv : 1;  // heads per kv head
        auto issue = [&](long j) {
            const long u = first + j * stride;
            uint8_t* base = smem + (j % NST) * ST_BYTES;
            uint64_t* bar = &full[j % NST];
            mbar_arrive_expect_tx(bar, tx);
            // row of k and v: the unit's own, or its kv head's
            const long ukv = PRO ? in_n * H_kv + in_h / rep : u;
            if (s_in) bulk_load(base, s_in + u * (kHead * kHead), ST_STATE, bar);
            bulk_load(base + O_R, r + u * kHead, IOB, bar);
            bulk_load(base + O_K, k + ukv * kHead, IOB, bar);
            bulk_load(base + O_V, v + ukv * kHead, IOB, bar);
            bulk_load(base + O_A, a + u * kHead, IOB, bar);
            if constexpr (!PRO) bulk_load(base + O_B, b + u * kHead, IOB, bar);
            bulk_load(base + O_W, wl + u * kHead, WB, bar);
            if constexpr (GATED) {
                bulk_load(base + O_RK, rk + static_cast<long>(in_h) * kHead, kHead * 4, bar);
                bulk_load(base + O_G, gte + u * kHead, IOB, bar);
            }
            in_n += step_n;
            in_h += step_h;
            if (in_h >= H) {
                in_h -= H;
                ++in_n;
            }
            ++n_issued;
        };
        for (long j = 0; j < NST && j < nmine; ++j) issue(j);
        long j = 0;
        bool ok = true;
        for (; j < nmine; ++j) {
            // unit j updated in its stage (the compute threads fenced their writes for the async proxy)
            if (!mbar_wait(&done[j % NST], static_cast<uint32_t>(j / NST) & 1u, WAIT_NS)) {
                ok = false;
                break;
            }
            const long u = first + j * stride;
            bulk_store(s_out + u * (kHead * kHead), smem + (j % NST) * ST_BYTES, ST_STATE);
            bulk_commit();
            if (j >= 1) {
                bulk_wait_read<1>();  // unit j-1's store has finished reading its stage
                if (j - 1 + NST < nmine) issue(j - 1 + NST);
            }
        }
        if (!ok) {
            report_status(status, WKV7_ERR_DEVICE_TIMEOUT);
            for (long m = j; m < n_issued; ++m)  // copies still landing in shared memory
                mbar_wait(&full[m % NST], static_cast<uint32_t>(m / NST) & 1u, WAIT_NS);
        }
        bulk_wait_all();  // every state store has completed
        return;
    }

    // ---------------------------------------------------------------- compute warps
    const int cg = tid & 15;  // key columns 4*cg .. 4*cg+3
    const int rg = tid >> 4;  // value rows rg, rg+16, rg+32, rg+48
    for (long j = 0; j < nmine; ++j) {
        const long u = first + j * stride;
        uint8_t* base = smem + (j % NST) * ST_BYTES;
        const bool w_ok = tid == 0 ? mbar_wait(&full[j % NST], static_cast<uint32_t>(j / NST) & 1u, WAIT_NS) : true;
        if (!group_sync_and(1, NCONS, w_ok)) {
            if (tid == 0) report_status(status, WKV7_ERR_DEVICE_TIMEOUT);
            break;
        }
        float wv[4], av[4], bv[4], kv[4], rv[4], vrow[4];
        lds4<WT>(base + O_W + 4 * cg * sizeof(WT), wv);
        lds4<IO>(base + O_A + 4 * cg * sizeof(IO), av);
        if constexpr (!PRO) lds4<IO>(base + O_B + 4 * cg * sizeof(IO), bv);
        lds4<IO>(base + O_K + 4 * cg * sizeof(IO), kv);
        lds4<IO>(base + O_R + 4 * cg * sizeof(IO), rv);
#pragma unroll
        for (int q = 0; q < 4; ++q) vrow[q] = lds1<IO>(base + O_V, rg + 16 * q);
#pragma unroll
        for (int c = 0; c < 4; ++c) wv[c] = expf(-expf(wv[c]));
        if constexpr (PRO) {
            // av holds a_lr: form kk, a, b and the scaled key
            const float inv =
                1.f / fmaxf(sqrtf(sum16(kv[0] * kv[0] + kv[1] * kv[1] + kv[2] * kv[2] + kv[3] * kv[3])), 1e-12f);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float kn = kv[c] * inv, alr = av[c];
                bv[c] = kn * alr;
                av[c] = -kn;
                kv[c] *= 1.f - wv[c] + alr;
            }
        }
        float uu = 0.f;  // gated read-out: u = sum_d r k rk
        if constexpr (GATED) {
            float rkv[4];
            lds4<float>(base + O_RK + 16 * cg, rkv);
            uu = sum16(rv[0] * kv[0] * rkv[0] + rv[1] * kv[1] * rkv[1] + rv[2] * kv[2] * rkv[2] +
                       rv[3] * kv[3] * rkv[3]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float4* sp = reinterpret_cast<float4*>(base + ((rg + 16 * q) * kHead + 4 * cg) * 4);
            float4 x = s_in ? *sp : make_float4(0.f, 0.f, 0.f, 0.f);
            const float sa = sum16(x.x * av[0] + x.y * av[1] + x.z * av[2] + x.w * av[3]);
            const float vi = vrow[q];
            x.x = fmaf(x.x, wv[0], fmaf(sa, bv[0], vi * kv[0]));
            x.y = fmaf(x.y, wv[1], fmaf(sa, bv[1], vi * kv[1]));
            x.z = fmaf(x.z, wv[2], fmaf(sa, bv[2], vi * kv[2]));
            x.w = fmaf(x.w, wv[3], fmaf(sa, bv[3], vi * kv[3]));
            float yi = sum16(x.x * rv[0] + x.y * rv[1] + x.z * rv[2] + x.w * rv[3]);
            if constexpr (GATED) yi = (yi * 0.125f + uu * vi) * lds1<IO>(base + O_G, rg + 16 * q);
            *sp = x;
            if (cg == 0) y[u * kHead + rg + 16 * q] = from_f32<IO>(yi);
        }
        fence_proxy_async_smem();  // the updated state is read by the bulk store (async proxy)
        mbar_arrive(&done[j % NST]);
    }
}

template <typename IO, typename WT, bool PRO, bool GATED>
cudaError_t launch_typed(const DecodeArgs& p, int* status, cudaStream_t stream) {
    auto kern = wkv7_decode_kernel<IO, WT, PRO, GATED>;
    static std::atomic<unsigned long long> configured{0};
    cudaError_t e = configure_smem_once(kern, static_cast<int>(SMEM_BYTES), configured);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long units = static_cast<long>(p.B) * p.H;
    const long slots = static_cast<long>(BLOCKS_PER_SM) * sms;
    const long grid = units < slots ? units : slots;
    kern<<<static_cast<unsigned>(grid), NTHR, SMEM_BYTES, stream>>>(
        static_cast<const IO*>(p.r), static_cast<const WT*>(p.w_log), static_cast<const IO*>(p.k),
        static_cast<const IO*>(p.v), static_cast<const IO*>(p.a), static_cast<const IO*>(p.b), p.s_in,
        static_cast<IO*>(p.y), p.s_out, units, status, p.H, PRO ? p.H_kv : p.H, p.rk,
        static_cast<const IO*>(p.g));
    return cudaGetLastError();
}

template <typename IO, typename WT>
cudaError_t launch_io(const DecodeArgs& p, int* status, cudaStream_t stream) {
    if (!p.prologue) return launch_typed<IO, WT, false, false>(p, status, stream);
    return p.rk ? launch_typed<IO, WT, true, true>(p, status, stream)
                : launch_typed<IO, WT, true, false>(p, status, stream);
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& p, int io_dtype, int w_dtype, int* status, cudaStream_t stream) {
    if (io_dtype == WKV7_BF16) {
        return w_dtype == WKV7_BF16 ? launch_io<__nv_bfloat16, __nv_bfloat16>(p, status, stream)
                                    : launch_io<__nv_bfloat16, float>(p, status, stream);
    }
    return w_dtype == WKV7_BF16 ? launch_io<float, __nv_bfloat16>(p, status, stream)
                                : launch_io<float, float>(p, status, stream);
}

}  // namespace wkv7
