// wkv7_prefill_long.cu — two-phase prefill for batches with few (sequence, head)
// units and long sequences (wkv7_forward_long), bf16 inputs.
//
// The chunk algebra of wkv7_prefill_pipe.cu splits every chunk's outputs into a
// state-independent part and one product with the chunk's start state S0:
//   [Y; S_L^T - Gamma_L (.) S0^T] = OUTpre + [R'; Bh^T W] S0^T
// (Y over the state rows; see that file).  One sequence's chunks are serial only
// through S0, so:
//   phase 1: the prefill kernel in export mode runs every chunk's state-independent
//            work on a persistent grid (one block per SM, each taking every SM-th
//            (chunk, head) through one continuous pipeline) and writes
//            [R'; Bh^T W] (bf16, 16 KB), OUTpre (fp32, 32 KB) and Gamma_L (256 B)
//            per chunk and head to the workspace;
//   phase 2: wkv7_long_scan_kernel carries the state through the chunks: per chunk
//            one tcgen05 product D = [R'; Bh^T W] S0^T, then y = D + OUTpre (token
//            rows) and S^T <- Gamma_L (.) S^T + D + OUTpre (key rows) in fp32
//            registers.  Every value column of the state (column of S0^T) evolves
//            on its own, so a (sequence, head) is split over 64 / NV blocks of NV
//            value columns each: a block keeps its columns of S0^T in the first NV
//            columns of its operand tile (the rest stay zero), reads the whole
//            [R'; Bh^T W] tile but only its NV columns of OUTpre, and writes its NV
//            columns of y and sT.
// Phase 2 streams the workspace through a ring of bulk copies (4 or 6 stages)
// issued by a producer warp (full / empty mbarriers, bounded waits), which also
// prefetches the chunk one ring-depth ahead into L2.  The product is issued as
// tcgen05 (N = 64, the block's NV columns first in the operand tile, zeros after; an
// N = NV product over a K-major operand, one row per value column, needs NV 2-byte
// stores per thread and chunk and took 3 % longer per call with NV = 16):
// a warp-level mma.sync form of it, with the state in accumulator registers, was
// measured slower on B1 T16384 H40 (268 us with four warps, 329 us with eight,
// against 176 us: each warp has ~180 dependent instructions per chunk).
#include "prefill_common.cuh"
#include "sm100_ptx.cuh"
#include "wkv7_internal.cuh"

namespace wkv7 {
namespace {

constexpr int L = 64;
constexpr uint32_t AS_BYTES = 16384;     // [R'; Bh^T W], 128 rows x 64 bf16, 128-byte swizzled
constexpr uint32_t OUT_BYTES = 32768;    // OUTpre, 128 x 64 fp32 (column quads, quad-major)
constexpr uint32_t GAM_BYTES = 256;      // Gamma_L, 64 fp32
constexpr uint32_t SLOT_BYTES = AS_BYTES + OUT_BYTES + GAM_BYTES;
constexpr int NCOMP = 128;               // compute threads: TMEM lanes 0..127
constexpr int NTHR = NCOMP + 32;         // + one producer warp
constexpr uint64_t WAIT_NS = 1000000000ull;
constexpr uint32_t ID_KM64 = idesc_f32acc(1, 128, 64, 0, 1);  // bf16, B MN-major, N = 64

// per-block geometry for NV value columns (16 or 64), four chunks in flight: with 16
// columns two blocks share an SM
template <int NV>
struct ScanGeom {
    static_assert(NV == 16 || NV == 64, "value columns per block");
    static constexpr uint32_t OUT_PART = NV * 512u;  // this block's columns of OUTpre (NV / 4 quads)
    static constexpr uint32_t BYTES = AS_BYTES + OUT_PART + GAM_BYTES;  // one chunk's bulk copies
    static constexpr uint32_t STAGE = (BYTES + 1023u) / 1024u * 1024u;  // the AS tile is 1024-aligned
    static constexpr int NST = 4;                                       // ring stages
    static constexpr uint32_t OFF_ST = NST * STAGE;                     // S0^T, bf16 MN-major (64 x 64)
    static constexpr uint32_t OFF_BAR = OFF_ST + 8192;                  // full[NST], empty[NST], mma, tmem slot
    static constexpr uint32_t SMEM = OFF_BAR + (2 * NST + 2) * 8 + 1024;
    static_assert(SMEM <= 227u * 1024u, "shared memory");
};

// L2 prefetch of global bytes (a hint: nothing waits for it); 16-byte aligned, size a
// multiple of 16, all inside one allocation
__device__ __forceinline__ void prefetch_l2_bulk(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// the first NV fp32 columns of this thread's TMEM lane (NV = 16 or 64)
template <int NV>
__device__ __forceinline__ void tmem_load_cols(uint32_t taddr, float (&o)[NV]) {
    if constexpr (NV == 16) {
        float x[32];
        tmem_load32(taddr, x);  // columns 16 .. 31 are D of the zero columns of S0^T
#pragma unroll
        for (int i = 0; i < 16; ++i) o[i] = x[i];
    } else {
#pragma unroll
        for (int q = 0; q < NV / 32; ++q) tmem_load32(taddr + 32 * q, *reinterpret_cast<float(*)[32]>(o + 32 * q));
    }
}

// the first NV elements of row `row` of a bf16 MN-major 64 x 64 operand tile
template <int NV>
__device__ __forceinline__ void st_row_head(uint8_t* tile, int row, const float (&x)[NV]) {
#pragma unroll
    for (int c = 0; c < NV; c += 8) {
        *reinterpret_cast<uint4*>(tile + swz(row, 2 * c, 64)) =
            make_uint4(pack_bf16x2(x[c], x[c + 1]), pack_bf16x2(x[c + 2], x[c + 3]), pack_bf16x2(x[c + 4], x[c + 5]),
                       pack_bf16x2(x[c + 6], x[c + 7]));
    }
}

template <int NV>
__global__ void __launch_bounds__(NTHR, 1)
    wkv7_long_scan_kernel(const uint8_t* __restrict__ ex_as, const float* __restrict__ ex_out,
                          const float* __restrict__ ex_gam, const float* s0, __nv_bfloat16* __restrict__ y,
                          float* sT, int T, int H, int* status) {
    using G = ScanGeom<NV>;
    constexpr int NPART = 64 / NV, NST = G::NST;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + G::OFF_BAR);
    uint64_t* empty = full + NST;
    uint64_t* mma_bar = full + 2 * NST;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(full + 2 * NST + 1);
    __shared__ int abort_flag;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int part = blockIdx.x % NPART, unit = blockIdx.x / NPART, h = unit % H, n = unit / H;
    const int v0 = part * NV;  // this block's value columns v0 .. v0 + NV - 1
    const int nch = static_cast<int>((static_cast<long>(T) + L - 1) / L);
    const long cbase = static_cast<long>(n) * nch;  // the sequence's first chunk over the batch
    const long tstride = static_cast<long>(H) * kHead, hoff = static_cast<long>(h) * kHead;
    const long sbase = (static_cast<long>(n) * H + h) * kHead * kHead;

    if (tid == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(mma_bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 64);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == NCOMP / 32) {
        // ------------------------------------------------------------ producer
        if ((tid & 31) == 0) {
            int issued = 0;
            for (int c = 0; c < nch; ++c) {
                const int st = c % NST;
                if (c >= NST) {
                    if (!mbar_wait(&empty[st], static_cast<uint32_t>(c / NST - 1) & 1u, WAIT_NS)) {
                        report_status(status, WKV7_ERR_DEVICE_TIMEOUT);
                        break;
                    }
                }
                if (*reinterpret_cast<volatile int*>(&abort_flag)) break;
                const long slot = (cbase + c) * H + h;
                if (c + NST < nch) {  // the chunk one ring-depth ahead: from DRAM into L2
                    const long ps = slot + static_cast<long>(NST) * H;
                    prefetch_l2_bulk(ex_as + ps * AS_BYTES, AS_BYTES);
                    prefetch_l2_bulk(ex_out + ps * (OUT_BYTES / 4) + v0 * 128, G::OUT_PART);
                }
                uint8_t* stage = sm + st * G::STAGE;
                mbar_arrive_expect_tx(&full[st], G::BYTES);
                bulk_load(stage, ex_as + slot * AS_BYTES, AS_BYTES, &full[st]);
                bulk_load(stage + AS_BYTES, ex_out + slot * (OUT_BYTES / 4) + v0 * 128, G::OUT_PART, &full[st]);
                bulk_load(stage + AS_BYTES + G::OUT_PART, ex_gam + slot * 64, GAM_BYTES, &full[st]);
                ++issued;
            }
            // every copy still in flight lands before the block exits: the last phase of
            // each of the (at most NST) most recent stages
            for (int c = issued - NST < 0 ? 0 : issued - NST; c < issued; ++c)
                mbar_wait(&full[c % NST], static_cast<uint32_t>(c / NST) & 1u, WAIT_NS);
        }
    } else {
        // ------------------------------------------------------------ state pass
        const int ts = tid;
        const uint32_t bar_id = 1;
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        uint8_t* St = sm + G::OFF_ST;
        const uint64_t dSt = mnmajor_desc<false>(St, 64, 0);
        float S[NV];
        const int x = ts - 64;  // key channel owned by lanes 64..127
        if (ts >= 64) {
            // row x of S0^T: this block's NV columns first, zeros after them
            float row[64];
#pragma unroll
            for (int i = 0; i < 64; ++i) row[i] = 0.f;
#pragma unroll
            for (int i = 0; i < NV; ++i) row[i] = S[i] = s0 ? s0[sbase + (v0 + i) * kHead + x] : 0.f;
            st_op_row32<false>(St, 64, x, 0, row);
            st_op_row32<false>(St, 64, x, 32, row + 32);
        }
        fence_proxy_async_smem();
        group_sync(bar_id, NCOMP);
        bool ok = true, mma_pending = false;
        uint32_t mma_phase = 0;
        for (int c = 0; c < nch; ++c) {
            const int st = c % NST;
            const uint8_t* stage = sm + st * G::STAGE;
            const long row0 = static_cast<long>(n) * T + static_cast<long>(c) * L;
            const int nv = T - c * L < L ? T - c * L : L;
            // one thread waits for the stage, issues the product and waits for it; the
            // product's completion means every copy of the stage has landed (one full
            // barrier), so the other threads only wait for the product
            bool w_ok = true;
            if (ts == 0) {
                w_ok = mbar_wait(&full[st], static_cast<uint32_t>(c / NST) & 1u, WAIT_NS);
                if (w_ok) {
                    tc_fence_after();
                    const uint64_t dAS = kmajor_desc<false>(stage, 128, 0);
#pragma unroll
                    for (uint32_t s = 0; s < 4; ++s) mma_ss<false>(tmem, dAS + 2 * s, dSt + 128 * s, ID_KM64, s > 0);
                    mma_commit(mma_bar);
                    mma_pending = true;
                    w_ok = mbar_wait(mma_bar, mma_phase, WAIT_NS);
                }
            }
            ok = group_sync_and(bar_id, NCOMP, w_ok);
            if (!ok) break;
            mma_pending = false;
            mma_phase ^= 1u;
            tc_fence_after();
            // OUTpre and Gamma_L from the stage first (the TMEM read below is fenced against
            // reordering, so the shared loads are issued ahead of it explicitly)
            const float* pre = reinterpret_cast<const float*>(stage + AS_BYTES) + ts * 4;
            float4 p4[NV / 4];
#pragma unroll
            for (int i = 0; i < NV / 4; ++i) p4[i] = *reinterpret_cast<const float4*>(pre + i * 512);
            const float GL = ts >= 64 ? reinterpret_cast<const float*>(stage + AS_BYTES + G::OUT_PART)[x] : 1.f;
            float o[NV];
            tmem_load_cols<NV>(tmem + lane_base, o);
#pragma unroll
            for (int i = 0; i < NV / 4; ++i) {
                o[4 * i] += p4[i].x;
                o[4 * i + 1] += p4[i].y;
                o[4 * i + 2] += p4[i].z;
                o[4 * i + 3] += p4[i].w;
            }
            if (ts < 64) {
                if (ts < nv && y != nullptr) {
                    __nv_bfloat16* dst = y + (row0 + ts) * tstride + hoff + v0;
#pragma unroll
                    for (int i = 0; i < NV; i += 8)
                        *reinterpret_cast<uint4*>(dst + i) =
                            make_uint4(pack_bf16x2(o[i], o[i + 1]), pack_bf16x2(o[i + 2], o[i + 3]),
                                       pack_bf16x2(o[i + 4], o[i + 5]), pack_bf16x2(o[i + 6], o[i + 7]));
                }
            } else {
                // 1 / Gamma_t must stay far inside the fp32 / bf16 range (false for NaN too)
                if (!(GL >= kMinGammaL)) report_status(status, WKV7_ERR_DECAY_RANGE);
#pragma unroll
                for (int i = 0; i < NV; ++i) S[i] = fmaf(GL, S[i], o[i]);
                st_row_head<NV>(St, x, S);
            }
            fence_proxy_async_smem();  // S0^T for the next product
            tc_fence_before();         // D read before the next product overwrites it
            group_sync(bar_id, NCOMP);
            if (ts == 0) mbar_arrive(&empty[st]);  // the stage has been read (product complete)
        }
        if (!ok) {
            if (ts == 0) {
                report_status(status, WKV7_ERR_DEVICE_TIMEOUT);
                abort_flag = 1;
                if (mma_pending) mbar_wait(mma_bar, mma_phase, WAIT_NS);
            }
        } else if (sT && ts >= 64) {
#pragma unroll
            for (int i = 0; i < NV; ++i) sT[sbase + (v0 + i) * kHead + x] = S[i];
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 64);
    }
}

template <int NV>
cudaError_t launch_scan(const PrefillArgs& p, const PrefillArgs& q, cudaStream_t stream) {
    static std::atomic<unsigned long long> configured{0};
    auto kern = wkv7_long_scan_kernel<NV>;
    const cudaError_t e = configure_smem_once(kern, static_cast<int>(ScanGeom<NV>::SMEM), configured);
    if (e != cudaSuccess) return e;
    kern<<<static_cast<unsigned>(static_cast<long>(p.B) * p.H * (64 / NV)), NTHR, ScanGeom<NV>::SMEM, stream>>>(
        q.ex_as, q.ex_out, q.ex_gam, p.s0, static_cast<__nv_bfloat16*>(p.y), p.sT, p.T, p.H, p.status);
    return cudaGetLastError();
}

}  // namespace

size_t prefill_long_workspace_bytes(int B, int T, int H) {
    const size_t nch = (static_cast<size_t>(T) + L - 1) / L;
    return static_cast<size_t>(B) * nch * H * SLOT_BYTES;
}

cudaError_t launch_prefill_long(const PrefillArgs& p, int w_dtype, void* ws, cudaStream_t stream) {
    const size_t slots = static_cast<size_t>(p.B) * ((static_cast<size_t>(p.T) + L - 1) / L) * p.H;
    PrefillArgs q = p;
    q.ex_as = static_cast<uint8_t*>(ws);
    q.ex_out = reinterpret_cast<float*>(q.ex_as + slots * AS_BYTES);
    q.ex_gam = q.ex_out + slots * (OUT_BYTES / 4);
    cudaError_t e = launch_prefill_pipe_export(q, w_dtype, stream);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    // value columns per block: 16 while the four blocks of every unit stay resident at
    // once (two per SM), else one block of all 64 columns per unit.  (Two blocks of 32
    // columns, one per SM, never beat the 16-column split where both fit: 198 against
    // ~171 us on B1 T16384 H40.)
    const long units = static_cast<long>(p.B) * p.H;
    if (units * 4 <= 2L * sms) return launch_scan<16>(p, q, stream);
    return launch_scan<64>(p, q, stream);
}

}  // namespace wkv7
