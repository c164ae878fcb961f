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
// This kernel serves fp32 inputs (bf16 inputs go to wkv7_prefill_pipe.cu):
// tf32 tiles and kind::tf32 MMAs; accumulation, the solve, the decay and the
// state are fp32.  All A operands and [W | Z] are K-major; V and S^T are stored
// transposed, K-major, because kind::tf32 with an MN-major SWIZZLE_128B operand
// does not produce the product (measured on B200).  Inputs are read with plain
// loads.  The operand-type template parameter (TF32) of the shared tile helpers
// is fixed to true here.
#include "prefill_common.cuh"
#include "sm100_ptx.cuh"
#include "wkv7_internal.cuh"

namespace wkv7 {
namespace {

constexpr int L = 64;          // chunk length (tokens)
constexpr int NT = 256;        // threads per block: the first 128 own one TMEM lane each
constexpr int NL = 128;        // TMEM lanes (and columns of the triangular solve)
constexpr int XSTRIDE = 132;   // fp32 row stride of the solver's columns (bank spread of 4 per row)
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
    uint8_t* V;    // V: 64 values x 64 tokens (K-major)
    uint8_t* S;    // S^T: 64 values x 64 keys (K-major)
    float* XS;     // solver columns: XS[t][col], 64 tokens x 128 columns fp32 (row stride XSTRIDE)
    float* gammaL; // Gamma_L per key channel
    float* red;    // per-quarter products of w (4 x 64), then (prologue) 1 / ||k_t|| per token (64)
    uint64_t* bar; // MMA completion barrier
    uint32_t* tmem_slot;
};


template <bool TF32>
__host__ __device__ constexpr uint32_t smem_bytes_needed() {
    using O = OpType<TF32>;
    constexpr uint32_t solver = 2u * 64u * NSTRIDE * 4u;
    constexpr uint32_t r4 = ((solver > O::TILE128 ? solver : O::TILE128) + 1023u) & ~1023u;
    return 1024u /* alignment slack */ + 3u * O::TILE128 + O::TILE64 + r4 + 2u * O::TILE64 + 64u * XSTRIDE * 4u +
           64u * 4u + 320u * 4u + 64u;
}

template <bool TF32>
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
    s.V = p; p += O::TILE64;
    s.S = p; p += O::TILE64;
    s.XS = reinterpret_cast<float*>(p); p += 64 * XSTRIDE * 4;
    s.gammaL = reinterpret_cast<float*>(p); p += 64 * 4;
    s.red = reinterpret_cast<float*>(p); p += 320 * 4;
    s.bar = reinterpret_cast<uint64_t*>(p); p += 8;
    s.tmem_slot = reinterpret_cast<uint32_t*>(p);
    return s;
}

// S^T as the tf32 K-major B operand of the state product: row = value channel.
__device__ __forceinline__ void store_state_operand(uint8_t* tile, int jj, const float* S) {
#pragma unroll
    for (int i = 0; i < 64; ++i) st_op<true>(tile, 64, i, jj, S[i]);
}

// Loads the chunk's fp32 value rows into the K-major V tile (row = value
// channel, column = token); tokens beyond nv are zero.
__device__ __forceinline__ void load_v_tile(const float* __restrict__ v, long row0, long tstride, long hoff, int nv,
                                            uint8_t* tile, int tid) {
#pragma unroll
    for (int it = 0; it < 1024 / NT; ++it) {
        const int q = tid + it * NT;
        const int row = q >> 4, ch = q & 15;
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (row < nv) x = __ldg(reinterpret_cast<const float4*>(v + (row0 + row) * tstride + hoff + 4 * ch));
        st_op<true>(tile, 64, 4 * ch + 0, row, x.x);
        st_op<true>(tile, 64, 4 * ch + 1, row, x.y);
        st_op<true>(tile, 64, 4 * ch + 2, row, x.z);
        st_op<true>(tile, 64, 4 * ch + 3, row, x.w);
    }
}

constexpr float kLog2e = 1.4426950408889634f;

// L2 prefetch of the rows of one chunk (up to 64 tokens from row0, nrows of them):
// thread tid takes token tid / 2 and one 128-byte half of each 256-byte fp32 row.
template <typename IO, typename WT>
__device__ __forceinline__ void prefetch_chunk_rows(const IO* r, const WT* wl, const IO* k, const IO* v, const IO* a,
                                                    const IO* b, long row0, long nrows, long tstride, long hoff,
                                                    long tstride_kv, long hoff_kv, int tid, bool pro) {
    const int t = tid >> 1, half = tid & 1;
    if (tid >= 2 * L || t >= nrows) return;
    const long off = (row0 + t) * tstride + hoff + 32 * half;
    const long offkv = (row0 + t) * tstride_kv + hoff_kv + 32 * half;
    prefetch_line_l2(r + off);
    prefetch_line_l2(a + off);
    prefetch_line_l2(k + offkv);
    prefetch_line_l2(v + offkv);
    if (!pro) prefetch_line_l2(b + off);
    prefetch_line_l2(wl + (row0 + t) * tstride + hoff + (sizeof(WT) == 4 ? 32 * half : 0));
}

template <typename IO, typename WT, bool TF32, bool PRO>
__global__ void __launch_bounds__(NT, 1)
    wkv7_prefill_kernel(const IO* __restrict__ r, const WT* __restrict__ wl, const IO* __restrict__ k,
                        const IO* __restrict__ v, const IO* __restrict__ a, const IO* __restrict__ b,
                        const float* s0, IO* __restrict__ y, float* sT, int T, int H,
                        const int32_t* __restrict__ seq_offsets, int* status, int H_kv, int map_flags) {
    static_assert(TF32, "this kernel serves fp32 inputs (tf32 operands) only");
    using O = OpType<TF32>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const Smem sm = carve<TF32>(smem_raw);
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
        fence_mbar_init();
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
    if (tid >= 64 && tid < NL) {
#pragma unroll
        for (int i = 0; i < 64; ++i)
            S[i] = (map_flags & 2) ? (i == jj ? 1.f : 0.f) : (s0 ? s0[sbase + i * kHead + jj] : 0.f);
        store_state_operand(sm.S, jj, S);
    }

    if (nchunks > 0) prefetch_chunk_rows(r, wl, k, v, a, b, tb, len, tstride, hoff, tstride_kv, hoff_kv, tid, PRO);
    bool ok = true;
    uint32_t phase = 0;          // parity of the next MMA completion
    bool mma_pending = false;    // an MMA commit not yet waited for
    for (int c = 0; c < nchunks && ok; ++c) {
        const long row0 = tb + static_cast<long>(c) * L;  // first token of the chunk
        const int nv = static_cast<int>(len - static_cast<long>(c) * L < L ? len - static_cast<long>(c) * L : L);

        // the next chunk's rows into L2 while this one is worked on (its loads then hit L2)
        if (c + 1 < nchunks) prefetch_chunk_rows(r, wl, k, v, a, b, row0 + L, len - static_cast<long>(c + 1) * L,
                                                  tstride, hoff, tstride_kv, hoff_kv, tid, PRO);
        // ---- p1: decay products and scaled operand tiles.  Thread (j, half).
        {
            const int j = tid & 63, hf = tid >> 6;  // key channel j, tokens 16 hf .. 16 hf + 15
            float cp[16];
            float prod = 1.f;
            // every decay logit of the thread's 16 tokens is loaded before the first product
            float lv[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const int t = hf * 16 + q;
                lv[q] = t < nv ? to_f32(wl[(row0 + t) * tstride + hoff + j]) : -INFINITY;
            }
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                // w = exp(-exp(l)) by the hardware 2^x (w_log = -inf gives w = 1 exactly)
                prod *= ex2_ftz(-kLog2e * ex2_ftz(kLog2e * lv[q]));
                cp[q] = prod;
            }
            sm.red[hf * 64 + j] = prod;
            if constexpr (PRO) {
                // 1 / max(||k_t||, 1e-12) of token t = tid / 4: each thread of the quad sums 16 channels
                const int t = tid >> 2, c0 = (tid & 3) * 16;
                float ss = 0.f;
                if (t < nv) {
                    const IO* kr = k + (row0 + t) * tstride_kv + hoff_kv + c0;
#pragma unroll 8
                    for (int i = 0; i < 16; ++i) {
                        const float x = to_f32(kr[i]);
                        ss = fmaf(x, x, ss);
                    }
                }
                ss += __shfl_xor_sync(0xffffffffu, ss, 1);
                ss += __shfl_xor_sync(0xffffffffu, ss, 2);
                if ((tid & 3) == 0) sm.red[256 + t] = 1.f / fmaxf(sqrtf(ss), 1e-12f);
            }
            __syncthreads();
            float pre = 1.f, GL = 1.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float x = sm.red[q * 64 + j];
                if (q < hf) pre *= x;
                GL *= x;
            }
            if (hf == 0) sm.gammaL[j] = GL;
            float gprev = pre;
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                // batches of 8 tokens: all loads of a batch are issued before its stores
                float rr[8], kk[8], aa[8], bb[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int t = hf * 16 + g * 8 + e;
                    rr[e] = kk[e] = aa[e] = bb[e] = 0.f;
                    if (t < nv) {
                        const long off = (row0 + t) * tstride + hoff + j;
                        rr[e] = to_f32(r[off]);
                        aa[e] = to_f32(a[off]);
                        if constexpr (PRO) {
                            kk[e] = to_f32(k[(row0 + t) * tstride_kv + hoff_kv + j]);
                        } else {
                            kk[e] = to_f32(k[off]);
                            bb[e] = to_f32(b[off]);
                        }
                    }
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int t = hf * 16 + g * 8 + e;
                    const float G = pre * cp[g * 8 + e];
                    const float inv = 1.f / G;
                    const float invL = inv * GL;
                    if constexpr (PRO) {
                        const float w = G / gprev, kn = kk[e] * sm.red[256 + t];  // w_t and kk
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
            load_v_tile(v, row0, tstride_kv, hoff_kv, (map_flags & 1) ? 0 : nv, sm.V, tid);  // v = 0: no rows
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- G = [Rt; At] [Bt; Kt]^T
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idesc = idesc_f32acc(O::FMT, 128, 128, 0, 0);
#pragma unroll
            for (uint32_t s = 0; s < O::KSTEPS; ++s)
                mma_ss<TF32>(tmem + COL_G, kmajor_desc<TF32>(sm.RA, 128, s), kmajor_desc<TF32>(sm.BK, 128, s), idesc,
                             s > 0);
            mma_commit(sm.bar);
        }
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
            } else if (tid < NL) {
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

        // ---- [W | Z] = (I - Nab)^{-1} [At | Mak]: forward substitution of 128 columns in blocks of
        // sixteen rows.  Warp w takes columns 16 w .. 16 w + 15; lanes l and l + 16 share a column and
        // split the products with the solved rows above a block (alternate groups of four rows,
        // which the row stride of XS puts in different banks), add them with shuffles, and both
        // take the 16 x 16 triangle; the column lives in XS
        {
            const int lane = tid & 31, part = lane >> 4;
            const int col = 16 * warp + (lane & 15);
            float* xs = sm.XS;
#pragma unroll 1
            for (int t0 = 0; t0 < 64; t0 += 16) {
                float acc[16];
#pragma unroll
                for (int q = 0; q < 16; ++q)
                    acc[q] = part ? 0.f
                                  : (col < 64 ? ld_op<TF32>(sm.RA, 128, 64 + t0 + q, col)
                                              : sm.MAK[(t0 + q) * NSTRIDE + (col - 64)]);
                const float* n0 = sm.NAB + t0 * NSTRIDE;  // rows t0 .. t0 + 15
#pragma unroll 2
                for (int i = 4 * part; i < t0; i += 8) {
                    const float x0 = xs[i * XSTRIDE + col], x1 = xs[(i + 1) * XSTRIDE + col];
                    const float x2 = xs[(i + 2) * XSTRIDE + col], x3 = xs[(i + 3) * XSTRIDE + col];
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const float4 n4 = *reinterpret_cast<const float4*>(n0 + q * NSTRIDE + i);
                        acc[q] = fmaf(n4.x, x0, acc[q]);
                        acc[q] = fmaf(n4.y, x1, acc[q]);
                        acc[q] = fmaf(n4.z, x2, acc[q]);
                        acc[q] = fmaf(n4.w, x3, acc[q]);
                    }
                }
#pragma unroll
                for (int q = 0; q < 16; ++q) acc[q] += __shfl_xor_sync(0xffffffffu, acc[q], 16);
                // the 16 x 16 unit lower triangle of the block
                float yv[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    float yq = acc[q];
#pragma unroll
                    for (int r = 0; r < q; ++r) yq = fmaf(n0[q * NSTRIDE + t0 + r], yv[r], yq);
                    yv[q] = yq;
                }
                if (part == 0) {
#pragma unroll
                    for (int q = 0; q < 16; ++q) xs[(t0 + q) * XSTRIDE + col] = yv[q];
                }
                __syncwarp();  // the block's rows are in XS for both lanes of the column
            }
            // the column -> the K-major [W | Z]^T tile: one half of it per lane of the pair
            float x[32];
#pragma unroll
            for (int q = 0; q < 32; ++q) x[q] = xs[(32 * part + q) * XSTRIDE + col];
            st_op_row32<TF32>(sm.WZ, 128, col, 32 * part, x);
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
            } else if (tid < NL) {
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
            constexpr uint32_t idesc = idesc_f32acc(O::FMT, 128, 64, 0, 0);
#pragma unroll
            for (uint32_t s = 0; s < O::KSTEPS; ++s)
                mma_ss<TF32>(tmem + COL_O, kmajor_desc<TF32>(sm.AQ, 128, s), kmajor_desc<TF32>(sm.V, 64, s), idesc,
                             s > 0);
#pragma unroll
            for (uint32_t s = 0; s < O::KSTEPS; ++s)
                mma_ss<TF32>(tmem + COL_O, kmajor_desc<TF32>(sm.AS, 128, s), kmajor_desc<TF32>(sm.S, 64, s), idesc, 1);
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
                    if (t < nv && y != nullptr) {
                        IO* dst = y + (row0 + t) * tstride + hoff + 32 * q;
#pragma unroll
                        for (int i = 0; i < 32; i += 4)
                            *reinterpret_cast<float4*>(dst + i) = make_float4(o[i], o[i + 1], o[i + 2], o[i + 3]);
                    }
                }
            } else if (tid < NL) {
                const float GL = sm.gammaL[jj];
                // 1 / Gamma_t must stay far inside the fp32 range (false for NaN too)
                if (!(GL >= kMinGammaL)) report_status(status, WKV7_ERR_DECAY_RANGE);
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    tmem_load32(tmem + lane_base + COL_O + 32 * q, o);
#pragma unroll
                    for (int i = 0; i < 32; ++i) S[32 * q + i] = fmaf(GL, S[32 * q + i], o[i]);
                }
                store_state_operand(sm.S, jj, S);
            }
        }
        tc_fence_before();
        __syncthreads();
    }

    if (!ok) {
        if (tid == 0) report_status(status, WKV7_ERR_DEVICE_TIMEOUT);
        // let an MMA still in flight finish (bounded) before the block releases
        // TMEM and its shared memory
        if (mma_pending) mbar_wait(sm.bar, phase, WAIT_LIMIT_NS);
    } else if (sT && tid >= 64 && tid < NL) {
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
    constexpr uint32_t smem = smem_bytes_needed<TF32>();
    auto kern = wkv7_prefill_kernel<IO, WT, TF32, PRO>;
    static std::atomic<unsigned long long> configured{0};
    const cudaError_t e = configure_smem_once(kern, static_cast<int>(smem), configured);
    if (e != cudaSuccess) return e;
    const long units = static_cast<long>(p.B) * p.H;
    kern<<<static_cast<unsigned>(units), NT, smem, stream>>>(
        static_cast<const IO*>(p.r), static_cast<const WT*>(p.w_log), static_cast<const IO*>(p.k),
        static_cast<const IO*>(p.v), static_cast<const IO*>(p.a), static_cast<const IO*>(p.b), p.s0,
        static_cast<IO*>(p.y), p.sT, p.T, p.H, p.seq_offsets, p.status, PRO ? p.H_kv : p.H,
        (p.zero_v ? 1 : 0) | (p.s0_identity ? 2 : 0));
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
