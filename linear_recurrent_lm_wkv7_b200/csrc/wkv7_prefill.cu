// wkv7_prefill.cu — chunked WKV-7 prefill on the sm_100a tensor cores.
//
// The recurrence (generalized delta rule of "RWKV-7 Goose: Expressive Dynamic
// State Evolution", section "Generalized Delta rule"; argument roles from the
// WKV call of the hxa07D forward listing) is
//     S_t = S_{t-1} diag(w_t) + (S_{t-1} a_t) b_t^T + v_t k_t^T,   y_t = S_t r_t.
// The pages state that the WKV computation parallelises chunk-wise ("RWKV-7
// Goose architecture analysis", training section); the chunk algebra below is
// derived here from the recurrence.
//
// One chunk of L = 64 tokens, start state S0, Gamma_t = prod_{s<=t} w_s (per key
// channel, Gamma_0 = 1).  Scaled operands (rows = tokens):
//   Rt = r (.) Gamma_t       At = a (.) Gamma_{t-1}
//   Kt = k / Gamma_t         Bt = b / Gamma_t
//   Kh = k (.) Gamma_L / Gamma_t,  Bh = b (.) Gamma_L / Gamma_t
// With u_t = S_{t-1} a_t (rows of U), unrolling the recurrence gives
//   U = At S0^T + Mak V + Nab U,   Nab = strict_tril(At Bt^T), Mak = strict_tril(At Kt^T)
//   Y = Rt S0^T + Mrk V + Mrb U,   Mrk = tril(Rt Kt^T),        Mrb = tril(Rt Bt^T)
//   S_L = S0 diag(Gamma_L) + V^T Kh + U^T Bh.
// Solving the unit lower-triangular system, [W | Z] = (I - Nab)^{-1} [At | Mak],
// gives U = W S0^T + Z V, hence the chunk is an affine map of the state:
//   Y     = (Rt + Mrb W) S0^T + (Mrk + Mrb Z) V
//   S_L^T = Gamma_L (.) S0^T  + (Bh^T W) S0^T + (Kh^T + Bh^T Z) V
// Everything except the two products with S0^T is independent of the state.
//
// Tensor-core schedule per chunk (M = 128 rows by stacking two 64-row blocks):
//   G   = [Rt; At] [Bt; Kt]^T               -> Mrb | Mrk over Nab | Mak   (TMEM)
//   P   = [Mrb; Bh^T] [W | Z]               -> Mrb W | Mrb Z over Bh^T W | Bh^T Z
//   OUT = [Er; Eq] V + [R'; Bh^T W] S0^T    -> Y over S_L^T - Gamma_L (.) S0^T
// with R' = Rt + Mrb W, Er = Mrk + Mrb Z, Eq = Kh^T + Bh^T Z.  The triangular
// solve runs on the CUDA cores in fp32 (one column per thread).  The state is
// kept in fp32 registers of the threads that own TMEM lanes 64..127 (one key
// channel each); its decay Gamma_L is applied there in fp32, and a rounded copy
// of S^T is the B operand of the last product.
//
// Operand precision: bf16 tiles and kind::f16 MMAs for bf16 inputs, tf32 tiles
// and kind::tf32 MMAs for fp32 inputs; accumulation, the solve, the decay and
// the state are fp32.  All A operands and [W | Z] are K-major.  V and S^T are
// MN-major B operands (rows = tokens / keys, as they arrive) for bf16; for tf32
// they are stored transposed, K-major, because kind::tf32 with an MN-major
// SWIZZLE_128B operand does not produce the product (measured on B200).
#include <cuda.h>

#include <cstring>

#include "prefill_common.cuh"
#include "tma_host.cuh"
#include "sm100_ptx.cuh"
#include "wkv7_internal.cuh"

namespace wkv7 {
namespace {

constexpr int L = 64;          // chunk length (tokens)
constexpr int NT = 128;        // threads per block: one per TMEM lane
constexpr int NSTRIDE = 68;    // fp32 row stride of the solver matrices (bank-conflict padding)
constexpr uint32_t COL_G = 0;    // TMEM columns of G   (128)
constexpr uint32_t COL_P = 128;  // TMEM columns of P   (128)
constexpr uint32_t COL_O = 0;    // TMEM columns of OUT (64): reuses G columns 0..63, dead by then
constexpr uint32_t TMEM_COLS = 256;
constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;  // 1 s: far above any legitimate wait

struct Smem {
    uint8_t* RA;   // [Rt ; At]            128 x 64, K-major over key channels
    uint8_t* BK;   // [Bt ; Kt]            128 x 64, K-major over key channels   (then [W | Z])
    uint8_t* WZ;   // [W | Z]^T            128 columns x 64 tokens, K-major       (aliases BK)
    uint8_t* BH;   // [Mrb ; Bh^T]         128 x 64, K-major over tokens          (then [Er ; Eq])
    uint8_t* AQ;   // [Er ; Eq]            128 x 64, K-major over tokens          (aliases BH)
    uint8_t* KH;   // Kh^T                 64 keys x 64 tokens
    float* NAB;    // Nab fp32             64 x NSTRIDE                           (then AS)
    float* MAK;    // Mak fp32             64 x NSTRIDE
    uint8_t* AS;   // [R' ; Bh^T W]        128 x 64, K-major over key channels    (aliases NAB, MAK)
    uint8_t* V[2]; // V: bf16 64 tokens x 64 values (MN-major, two TMA slots); tf32 64 values x 64 tokens (K-major)
    uint8_t* S;    // S^T: bf16 64 keys x 64 values (MN-major); tf32 64 values x 64 keys (K-major)
    uint8_t* raw;  // bf16 only: TMA staging of r, k, a, b (64 x 64 each, row-major) and w_log
    float* gammaL; // Gamma_L per key channel
    float* red;    // per-half products of w (2 x 64), then (prologue) 1 / ||k_t|| per token (64)
    uint64_t* bar; // MMA completion barrier
    uint64_t* raw_bar; // TMA completion barrier (bf16 only)
    uint32_t* tmem_slot;
};


// Bytes of the raw staging area (bf16 inputs): r, k, a, b tiles + the w_log tile.
template <bool TF32, uint32_t WB>
__host__ __device__ constexpr uint32_t raw_bytes() {
    return TF32 ? 0u : 4u * 64u * 64u * 2u + 64u * 64u * WB;
}

template <bool TF32, uint32_t WB>
__host__ __device__ constexpr uint32_t smem_bytes_needed() {
    using O = OpType<TF32>;
    constexpr uint32_t solver = 2u * 64u * NSTRIDE * 4u;
    constexpr uint32_t r4 = ((solver > O::TILE128 ? solver : O::TILE128) + 1023u) & ~1023u;
    constexpr uint32_t nv = TF32 ? 1u : 2u;
    return 1024u /* alignment slack */ + 3u * O::TILE128 + O::TILE64 + r4 + (nv + 1u) * O::TILE64 +
           raw_bytes<TF32, WB>() + 64u * 4u + 192u * 4u + 64u;
}

template <bool TF32, uint32_t WB>
__device__ __forceinline__ Smem carve(uint8_t* raw) {
    using O = OpType<TF32>;
    constexpr uint32_t solver = 2u * 64u * NSTRIDE * 4u;
    constexpr uint32_t r4 = ((solver > O::TILE128 ? solver : O::TILE128) + 1023u) & ~1023u;
    uint8_t* p = raw + ((1024u - (smem_u32(raw) & 1023u)) & 1023u);  // stays in the shared address space
    Smem s;
    s.RA = p; p += O::TILE128;
    s.BK = p; s.WZ = p; p += O::TILE128;
    s.BH = p; s.AQ = p; p += O::TILE128;
    s.KH = p; p += O::TILE64;
    s.NAB = reinterpret_cast<float*>(p); s.MAK = s.NAB + 64 * NSTRIDE; s.AS = p; p += r4;
    s.V[0] = p; p += O::TILE64;
    if constexpr (!TF32) { s.V[1] = p; p += O::TILE64; } else { s.V[1] = s.V[0]; }
    s.S = p; p += O::TILE64;
    s.raw = p; p += raw_bytes<TF32, WB>();
    s.gammaL = reinterpret_cast<float*>(p); p += 64 * 4;
    s.red = reinterpret_cast<float*>(p); p += 192 * 4;
    s.bar = reinterpret_cast<uint64_t*>(p); p += 8;
    s.raw_bar = reinterpret_cast<uint64_t*>(p); p += 8;
    s.tmem_slot = reinterpret_cast<uint32_t*>(p);
    return s;
}

// Issues the TMA loads of chunk tokens [row0, row0 + 64) of head h: raw r, k,
// a, b, w_log tiles and the (swizzled) V tile.  One thread.
template <uint32_t WB>
__device__ __forceinline__ void issue_chunk_loads(const TmaMaps& m, const Smem& sm, uint8_t* vdst, int h, long row0) {
    constexpr uint32_t tile = 64u * 64u * 2u;
    mbar_arrive_expect_tx(sm.raw_bar, 5u * tile + 64u * 64u * WB);
    const int t0 = static_cast<int>(row0);
    tma_load_3d(sm.raw + 0 * tile, &m.r, sm.raw_bar, 0, h, t0);
    tma_load_3d(sm.raw + 1 * tile, &m.k, sm.raw_bar, 0, h, t0);
    tma_load_3d(sm.raw + 2 * tile, &m.a, sm.raw_bar, 0, h, t0);
    tma_load_3d(sm.raw + 3 * tile, &m.b, sm.raw_bar, 0, h, t0);
    tma_load_3d(sm.raw + 4 * tile, &m.wl, sm.raw_bar, 0, h, t0);
    tma_load_3d(vdst, &m.v, sm.raw_bar, 0, h, t0);
}

// Row jj of S^T (key channel jj, all 64 value channels) into the S operand tile.
template <bool TF32>
__device__ __forceinline__ void store_state_operand(uint8_t* tile, int jj, const float* S) {
    if constexpr (TF32) {
#pragma unroll
        for (int i = 0; i < 64; ++i) st_op<true>(tile, 64, i, jj, S[i]);  // K-major: row = value channel
    } else {
        st_op_row32<false>(tile, 64, jj, 0, S);  // MN-major: row = key channel
        st_op_row32<false>(tile, 64, jj, 32, S + 32);
    }
}

// Loads 16 bytes of one value row into the V tile (rows beyond nv are zeroed).
template <typename IO, bool TF32>
__device__ __forceinline__ void load_v_tile(const IO* __restrict__ v, long row0, long tstride, long hoff, int nv,
                                            uint8_t* tile, int tid) {
    if constexpr (TF32) {
        // fp32 values: 16 chunks of 4 per row, 64 rows
#pragma unroll
        for (int it = 0; it < 8; ++it) {
            const int q = tid + it * NT;
            const int row = q >> 4, ch = q & 15;
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (row < nv) {
                const float* src = reinterpret_cast<const float*>(v) + (row0 + row) * tstride + hoff + 4 * ch;
                x = __ldg(reinterpret_cast<const float4*>(src));
            }
            // K-major: row = value channel, column = token
            st_op<true>(tile, 64, 4 * ch + 0, row, x.x);
            st_op<true>(tile, 64, 4 * ch + 1, row, x.y);
            st_op<true>(tile, 64, 4 * ch + 2, row, x.z);
            st_op<true>(tile, 64, 4 * ch + 3, row, x.w);
        }
    } else {
        // bf16 values: 8 chunks of 8 per row, 64 rows
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int q = tid + it * NT;
            const int row = q >> 3, ch = q & 7;
            uint4 x = make_uint4(0, 0, 0, 0);
            if (row < nv) {
                const __nv_bfloat16* src =
                    reinterpret_cast<const __nv_bfloat16*>(v) + (row0 + row) * tstride + hoff + 8 * ch;
                x = __ldg(reinterpret_cast<const uint4*>(src));
            }
            *reinterpret_cast<uint4*>(tile + swz(row, ch * 16, 64)) = x;
        }
    }
}

// PRO (fp32 inputs only): the prologue of the WKV call is applied to the raw
// inputs in the element-wise stage (wkv7_forward_fused): k and v are rows of kv
// head h / (H / H_kv), `a` carries a_lr, and per token
//   kk = k / max(||k||, 1e-12),  a = -kk,  b = kk a_lr,  k <- k (1 - w + a_lr);
// `b` is not read.
template <typename IO, typename WT, bool TF32, bool PRO>
__global__ void __launch_bounds__(NT, 1)
    wkv7_prefill_kernel(const IO* __restrict__ r, const WT* __restrict__ wl, const IO* __restrict__ k,
                        const IO* __restrict__ v, const IO* __restrict__ a, const IO* __restrict__ b,
                        const float* s0, IO* __restrict__ y, float* sT, int T, int H,
                        const int32_t* __restrict__ seq_offsets, int* status, int H_kv,
                        const __grid_constant__ TmaMaps maps) {
    static_assert(TF32 || !PRO, "the prologue is fused into the fp32 path only");
    using O = OpType<TF32>;
    constexpr uint32_t WB = sizeof(WT);
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const Smem sm = carve<TF32, WB>(smem_raw);
    const int tid = threadIdx.x;
    const int warp = tid >> 5;

    // ---- which (sequence, head) unit, and its tokens
    const int unit = blockIdx.x;
    const int n = unit / H, h = unit % H;
    long tb = 0, len = 0;
    bool bad = false;
    if (seq_offsets) {
        const long o0 = seq_offsets[n], o1 = seq_offsets[n + 1];
        if (o0 < 0 || o1 < o0 || o1 > T) {
            bad = true;
        } else {
            tb = o0;
            len = o1 - o0;
        }
    } else {
        tb = static_cast<long>(n) * T;
        len = T;
    }
    if (bad) {
        if (tid == 0) report_status(status, WKV7_ERR_DEVICE_BOUNDS);
        return;  // nothing allocated yet
    }
    const long tstride = static_cast<long>(H) * kHead;  // elements between consecutive tokens
    const long hoff = static_cast<long>(h) * kHead;
    const long tstride_kv = PRO ? static_cast<long>(H_kv) * kHead : tstride;  // k and v rows
    const long hoff_kv = PRO ? static_cast<long>(h / (H / H_kv)) * kHead : hoff;
    const long sbase = (static_cast<long>(n) * H + h) * kHead * kHead;

    // ---- set-up: barrier, TMEM
    const int nchunks = static_cast<int>((len + L - 1) / L);
    if (tid == 0) {
        mbar_init(sm.bar, 1);
        mbar_init(sm.raw_bar, 1);
        fence_mbar_init();
        if constexpr (!TF32) {
            if (nchunks > 0) issue_chunk_loads<WB>(maps, sm, sm.V[0], h, tb);
        }
    }
    if (warp == 0) {
        tmem_alloc(sm.tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *sm.tmem_slot;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;

    // ---- state: threads 64..127 own key channel j = tid - 64 (a row of S^T)
    float S[64];
    const int jj = tid - 64;
    if (tid >= 64) {
#pragma unroll
        for (int i = 0; i < 64; ++i) S[i] = s0 ? s0[sbase + i * kHead + jj] : 0.f;
        store_state_operand<TF32>(sm.S, jj, S);
    }

    bool ok = true;
    uint32_t phase = 0;          // parity of the next MMA completion
    bool mma_pending = false;    // an MMA commit not yet waited for
    int tma_issued = (!TF32 && nchunks > 0) ? 1 : 0;  // chunks whose TMA loads were issued
    int tma_consumed = 0;                              // chunks whose TMA loads were waited for
    for (int c = 0; c < nchunks && ok; ++c) {
        const long row0 = tb + static_cast<long>(c) * L;  // first token of the chunk
        const int nv = static_cast<int>(len - static_cast<long>(c) * L < L ? len - static_cast<long>(c) * L : L);

        // ---- p1: decay products and scaled operand tiles.  Thread (j, half).
        if constexpr (!TF32) {
            ok = __syncthreads_and(mbar_wait(sm.raw_bar, static_cast<uint32_t>(c) & 1u, WAIT_LIMIT_NS));
            if (!ok) break;
            tma_consumed = c + 1;
        }
        {
            const int j = tid & 63, hf = tid >> 6;
            const __nv_bfloat16* raw16 = reinterpret_cast<const __nv_bfloat16*>(sm.raw);
            const WT* rawl = reinterpret_cast<const WT*>(sm.raw + 4 * 64 * 64 * 2);
            float cp[32];
            float prod = 1.f;
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                const int t = hf * 32 + q;
                float w = 1.f;
                if (t < nv) {
                    const float l = TF32 ? to_f32(wl[(row0 + t) * tstride + hoff + j]) : to_f32(rawl[t * 64 + j]);
                    w = expf(-expf(l));
                }
                prod *= w;
                cp[q] = prod;
            }
            sm.red[hf * 64 + j] = prod;
            if constexpr (PRO) {
                // 1 / max(||k_t||, 1e-12) of token t = tid / 2: each thread of the pair sums 32 channels
                const int t = tid >> 1, c0 = (tid & 1) * 32;
                float ss = 0.f;
                if (t < nv) {
                    const IO* kr = k + (row0 + t) * tstride_kv + hoff_kv + c0;
#pragma unroll 8
                    for (int i = 0; i < 32; ++i) {
                        const float x = to_f32(kr[i]);
                        ss = fmaf(x, x, ss);
                    }
                }
                ss += __shfl_xor_sync(0xffffffffu, ss, 1);
                if ((tid & 1) == 0) sm.red[128 + t] = 1.f / fmaxf(sqrtf(ss), 1e-12f);
            }
            __syncthreads();
            const float pre = hf ? sm.red[j] : 1.f;
            const float GL = sm.red[j] * sm.red[64 + j];
            if (hf == 0) sm.gammaL[j] = GL;
            float gprev = pre;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                // batches of 8 tokens: all loads of a batch are issued before its stores
                float rr[8], kk[8], aa[8], bb[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int t = hf * 32 + g * 8 + e;
                    rr[e] = kk[e] = aa[e] = bb[e] = 0.f;
                    if (t < nv) {
                        if constexpr (TF32) {
                            const long off = (row0 + t) * tstride + hoff + j;
                            rr[e] = to_f32(r[off]);
                            aa[e] = to_f32(a[off]);
                            if constexpr (PRO) {
                                kk[e] = to_f32(k[(row0 + t) * tstride_kv + hoff_kv + j]);
                            } else {
                                kk[e] = to_f32(k[off]);
                                bb[e] = to_f32(b[off]);
                            }
                        } else {
                            rr[e] = to_f32(raw16[0 * 4096 + t * 64 + j]);
                            kk[e] = to_f32(raw16[1 * 4096 + t * 64 + j]);
                            aa[e] = to_f32(raw16[2 * 4096 + t * 64 + j]);
                            bb[e] = to_f32(raw16[3 * 4096 + t * 64 + j]);
                        }
                    }
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int t = hf * 32 + g * 8 + e;
                    const float G = pre * cp[g * 8 + e];
                    const float inv = 1.f / G;
                    const float invL = inv * GL;
                    if constexpr (PRO) {
                        const float w = G / gprev, kn = kk[e] * sm.red[128 + t];  // w_t and kk
                        bb[e] = kn * aa[e];
                        kk[e] *= 1.f - w + aa[e];
                        aa[e] = -kn;
                    }
                    st_op<TF32>(sm.RA, 128, t, j, rr[e] * G);
                    st_op<TF32>(sm.RA, 128, 64 + t, j, aa[e] * gprev);
                    st_op<TF32>(sm.BK, 128, t, j, bb[e] * inv);
                    st_op<TF32>(sm.BK, 128, 64 + t, j, kk[e] * inv);
                    st_op<TF32>(sm.BH, 128, 64 + j, t, bb[e] * invL);
                    st_op<TF32>(sm.KH, 64, j, t, kk[e] * invL);
                    gprev = G;
                }
            }
            if constexpr (TF32) load_v_tile<IO, TF32>(v, row0, tstride_kv, hoff_kv, nv, sm.V[0], tid);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- G = [Rt; At] [Bt; Kt]^T; then prefetch the next chunk's inputs
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idesc = idesc_f32acc(O::FMT, 128, 128, 0, 0);
#pragma unroll
            for (uint32_t s = 0; s < O::KSTEPS; ++s)
                mma_ss<TF32>(tmem + COL_G, kmajor_desc<TF32>(sm.RA, 128, s), kmajor_desc<TF32>(sm.BK, 128, s), idesc,
                             s > 0);
            mma_commit(sm.bar);
            if constexpr (!TF32) {
                // the raw tiles were consumed by p1 (fenced above); the other V slot
                // was last read by the previous chunk's OUT product, which has completed
                if (c + 1 < nchunks) issue_chunk_loads<WB>(maps, sm, sm.V[(c + 1) & 1], h, row0 + L);
            }
        }
        if (!TF32 && c + 1 < nchunks) tma_issued = c + 2;
        mma_pending = true;
        ok = __syncthreads_and(mbar_wait(sm.bar, phase, WAIT_LIMIT_NS));
        if (!ok) break;
        mma_pending = false;
        phase ^= 1u;
        tc_fence_after();

        // ---- masks: Mrb (incl. diagonal) -> BH rows 0..63; Nab, Mak (strict) -> fp32 solver inputs
        {
            float g[32];
            if (tid < 64) {
                const int t = tid;
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    tmem_load32(tmem + lane_base + COL_G + 32 * q, g);
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (32 * q + i > t) g[i] = 0.f;
                    st_op_row32<TF32>(sm.BH, 128, t, 32 * q, g);
                }
            } else {
                const int t = tid - 64;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    tmem_load32(tmem + lane_base + COL_G + 32 * q, g);
                    float* dst = (q < 2 ? sm.NAB : sm.MAK) + t * NSTRIDE + 32 * (q & 1);
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        float4 x;
                        x.x = (32 * (q & 1) + i + 0 < t) ? g[i + 0] : 0.f;
                        x.y = (32 * (q & 1) + i + 1 < t) ? g[i + 1] : 0.f;
                        x.z = (32 * (q & 1) + i + 2 < t) ? g[i + 2] : 0.f;
                        x.w = (32 * (q & 1) + i + 3 < t) ? g[i + 3] : 0.f;
                        *reinterpret_cast<float4*>(dst + i) = x;
                    }
                }
            }
        }
        tc_fence_before();
        __syncthreads();

        // ---- [W | Z] = (I - Nab)^{-1} [At | Mak]: forward substitution, column `tid`
        {
            const int col = tid;
            float x[64];
#pragma unroll
            for (int t = 0; t < 64; ++t) x[t] = 0.f;
#pragma unroll
            for (int t = 0; t < 64; ++t) {
                float acc = col < 64 ? ld_op<TF32>(sm.RA, 128, 64 + t, col) : sm.MAK[t * NSTRIDE + (col - 64)];
                const float* nrow = sm.NAB + t * NSTRIDE;
#pragma unroll
                for (int i = 0; i < t; i += 4) {
                    const float4 nv4 = *reinterpret_cast<const float4*>(nrow + i);
                    acc = fmaf(nv4.x, x[i], acc);
                    acc = fmaf(nv4.y, x[i + 1], acc);
                    acc = fmaf(nv4.z, x[i + 2], acc);
                    acc = fmaf(nv4.w, x[i + 3], acc);
                }
                x[t] = acc;
            }
            st_op_row32<TF32>(sm.WZ, 128, col, 0, x);
            st_op_row32<TF32>(sm.WZ, 128, col, 32, x + 32);
        }
        fence_proxy_async_smem();
        __syncthreads();

        // ---- P = [Mrb; Bh^T] [W | Z]
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idesc = idesc_f32acc(O::FMT, 128, 128, 0, 0);
#pragma unroll
            for (uint32_t s = 0; s < O::KSTEPS; ++s)
                mma_ss<TF32>(tmem + COL_P, kmajor_desc<TF32>(sm.BH, 128, s), kmajor_desc<TF32>(sm.WZ, 128, s),
                             idesc, s > 0);
            mma_commit(sm.bar);
        }
        mma_pending = true;
        ok = __syncthreads_and(mbar_wait(sm.bar, phase, WAIT_LIMIT_NS));
        if (!ok) break;
        mma_pending = false;
        phase ^= 1u;
        tc_fence_after();

        // ---- R' = Rt + Mrb W, Er = Mrk + Mrb Z (lanes 0..63); Bh^T W, Eq = Kh^T + Bh^T Z (lanes 64..127)
        {
            float p[32], e[32];
            if (tid < 64) {
                const int t = tid;
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    tmem_load32(tmem + lane_base + COL_P + 32 * q, p);
                    ld_op_row32<TF32>(sm.RA, 128, t, 32 * q, e);
#pragma unroll
                    for (int i = 0; i < 32; ++i) p[i] += e[i];
                    st_op_row32<TF32>(sm.AS, 128, t, 32 * q, p);
                }
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    tmem_load32(tmem + lane_base + COL_P + 64 + 32 * q, p);
                    tmem_load32(tmem + lane_base + COL_G + 64 + 32 * q, e);
#pragma unroll
                    for (int i = 0; i < 32; ++i) p[i] += (32 * q + i <= t) ? e[i] : 0.f;
                    st_op_row32<TF32>(sm.AQ, 128, t, 32 * q, p);
                }
            } else {
                const int j = tid - 64;
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    tmem_load32(tmem + lane_base + COL_P + 32 * q, p);
                    st_op_row32<TF32>(sm.AS, 128, 64 + j, 32 * q, p);
                }
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    tmem_load32(tmem + lane_base + COL_P + 64 + 32 * q, p);
                    ld_op_row32<TF32>(sm.KH, 64, j, 32 * q, e);
#pragma unroll
                    for (int i = 0; i < 32; ++i) p[i] += e[i];
                    st_op_row32<TF32>(sm.AQ, 128, 64 + j, 32 * q, p);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- OUT = [Er; Eq] V + [R'; Bh^T W] S0^T
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idesc = idesc_f32acc(O::FMT, 128, 64, 0, TF32 ? 0 : 1);
#pragma unroll
            for (uint32_t s = 0; s < O::KSTEPS; ++s) {
                const uint64_t bd = TF32 ? kmajor_desc<TF32>(sm.V[0], 64, s) : mnmajor_desc<TF32>(sm.V[c & 1], 64, s);
                mma_ss<TF32>(tmem + COL_O, kmajor_desc<TF32>(sm.AQ, 128, s), bd, idesc, s > 0);
            }
#pragma unroll
            for (uint32_t s = 0; s < O::KSTEPS; ++s) {
                const uint64_t bd = TF32 ? kmajor_desc<TF32>(sm.S, 64, s) : mnmajor_desc<TF32>(sm.S, 64, s);
                mma_ss<TF32>(tmem + COL_O, kmajor_desc<TF32>(sm.AS, 128, s), bd, idesc, 1);
            }
            mma_commit(sm.bar);
        }
        mma_pending = true;
        ok = __syncthreads_and(mbar_wait(sm.bar, phase, WAIT_LIMIT_NS));
        if (!ok) break;
        mma_pending = false;
        phase ^= 1u;
        tc_fence_after();

        // ---- y rows (lanes 0..63) and the state update (lanes 64..127)
        {
            float o[32];
            if (tid < 64) {
                const int t = tid;
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    tmem_load32(tmem + lane_base + COL_O + 32 * q, o);
                    if (t < nv) {
                        IO* dst = y + (row0 + t) * tstride + hoff + 32 * q;
                        if constexpr (TF32) {
#pragma unroll
                            for (int i = 0; i < 32; i += 4)
                                *reinterpret_cast<float4*>(dst + i) = make_float4(o[i], o[i + 1], o[i + 2], o[i + 3]);
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; i += 8) {
                                uint4 pk;
                                uint32_t* w = reinterpret_cast<uint32_t*>(&pk);
#pragma unroll
                                for (int e2 = 0; e2 < 4; ++e2) {
                                    __nv_bfloat162 bb2 = __floats2bfloat162_rn(o[i + 2 * e2], o[i + 2 * e2 + 1]);
                                    w[e2] = *reinterpret_cast<uint32_t*>(&bb2);
                                }
                                *reinterpret_cast<uint4*>(dst + i) = pk;
                            }
                        }
                    }
                }
            } else {
                const float GL = sm.gammaL[jj];
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    tmem_load32(tmem + lane_base + COL_O + 32 * q, o);
#pragma unroll
                    for (int i = 0; i < 32; ++i) S[32 * q + i] = fmaf(GL, S[32 * q + i], o[i]);
                }
                store_state_operand<TF32>(sm.S, jj, S);
            }
        }
        tc_fence_before();
        __syncthreads();
    }

    if (!ok) {
        if (tid == 0) report_status(status, WKV7_ERR_DEVICE_TIMEOUT);
        // let MMAs and TMA loads still in flight finish (bounded) before the
        // block releases TMEM and its shared memory
        if (mma_pending) mbar_wait(sm.bar, phase, WAIT_LIMIT_NS);
        for (int ci = tma_consumed; ci < tma_issued; ++ci)
            mbar_wait(sm.raw_bar, static_cast<uint32_t>(ci) & 1u, WAIT_LIMIT_NS);
    } else if (sT && tid >= 64) {
#pragma unroll
        for (int i = 0; i < 64; ++i) sT[sbase + i * kHead + jj] = S[i];
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

template <typename IO, typename WT, bool TF32, bool PRO>
cudaError_t launch_typed(const PrefillArgs& p, cudaStream_t stream) {
    constexpr uint32_t smem = smem_bytes_needed<TF32, sizeof(WT)>();
    TmaMaps maps;  // unused by the fp32 path
    memset(&maps, 0, sizeof(maps));
    if constexpr (!TF32) {
        const uint64_t ntok = p.seq_offsets ? static_cast<uint64_t>(p.T) : static_cast<uint64_t>(p.B) * p.T;
        if (!make_prefill_maps(&maps, p.r, p.w_log, p.k, p.v, p.a, p.b, p.H, p.H, ntok, sizeof(WT)))
            return cudaErrorInvalidValue;
    }
    auto kern = wkv7_prefill_kernel<IO, WT, TF32, PRO>;
    static unsigned long long configured = 0;  // one bit per device ordinal
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(configured & bit)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        configured |= bit;
    }
    const long units = static_cast<long>(p.B) * p.H;
    kern<<<static_cast<unsigned>(units), NT, smem, stream>>>(
        static_cast<const IO*>(p.r), static_cast<const WT*>(p.w_log), static_cast<const IO*>(p.k),
        static_cast<const IO*>(p.v), static_cast<const IO*>(p.a), static_cast<const IO*>(p.b), p.s0,
        static_cast<IO*>(p.y), p.sT, p.T, p.H, p.seq_offsets, p.status, PRO ? p.H_kv : p.H, maps);
    return cudaGetLastError();
}

__global__ void expire_wait_kernel(int spins, int* status) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        // nothing ever arrives on `bar`: the bounded wait must give up
        if (!mbar_wait_spins(&bar, 0, static_cast<uint32_t>(spins))) report_status(status, WKV7_ERR_DEVICE_TIMEOUT);
    }
}

}  // namespace

cudaError_t launch_prefill(const PrefillArgs& p, int io_dtype, int w_dtype, cudaStream_t stream) {
    if (io_dtype == WKV7_BF16) return launch_prefill_pipe(p, w_dtype, stream);
    if (p.prologue)
        return w_dtype == WKV7_BF16 ? launch_typed<float, __nv_bfloat16, true, true>(p, stream)
                                    : launch_typed<float, float, true, true>(p, stream);
    return w_dtype == WKV7_BF16 ? launch_typed<float, __nv_bfloat16, true, false>(p, stream)
                                : launch_typed<float, float, true, false>(p, stream);
}

cudaError_t launch_expire_wait(int spins, int* status, cudaStream_t stream) {
    expire_wait_kernel<<<1, 32, 0, stream>>>(spins, status);
    return cudaGetLastError();
}

}  // namespace wkv7
