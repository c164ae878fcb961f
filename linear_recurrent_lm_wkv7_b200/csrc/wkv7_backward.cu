// wkv7_backward.cu — gradient of the WKV-7 recurrence in recurrent form, for fp32
// inputs (fp32 arithmetic throughout, which their tighter bound needs; bf16 inputs
// take the chunked form of wkv7_backward_chunk.cu).  Also the entry point's
// workspace size and dispatch.
//
// For L = sum_t <dy_t, y_t> + <dsT, S_T> the chain rule through one step
// S_t = S_{t-1} diag(w_t) + (S_{t-1} a_t) b_t^T + v_t k_t^T, y_t = S_t r_t gives,
// sweeping t downwards with G = dL/dS_t (G = dsT at t = T):
//   G += dy_t r_t^T;   dr_t = S_t^T dy_t;   dv_t = G k_t;   dk_t = G^T v_t
//   q = G b_t;   p = S_{t-1} a_t;   da_t = S_{t-1}^T q;   db_t = G^T p
//   dw_t[j] = sum_i G[i][j] S_{t-1}[i][j];   d w_log_t = dw_t (-exp(w_log_t) w_t)
//   G <- G diag(w_t) + q a_t^T                         (and ds0 = G at the end)
// (the derivative of the generalized delta rule of "RWKV-7 Goose: Expressive
// Dynamic State Evolution", section "Generalized Delta rule", with the argument
// roles of the hxa07D WKV call; the pages themselves print no backward).
//
// One 256-thread block per (sequence, head) unit.  Thread (rg, cg) = (tid / 16,
// tid % 16) owns value rows rg, rg + 16, rg + 32, rg + 48 and key columns
// 4 cg .. 4 cg + 3 of both S and G, so row sums are 16-lane shuffles and column
// sums go through shared memory (one block barrier per token, double-buffered).
//   1. forward over the sequence, writing the state at every chunk start to the
//      workspace (checkpoints);
//   2. chunks in reverse: stage the chunk's inputs in shared memory (fp32),
//      recompute its 64 states from the checkpoint into a per-unit scratch of
//      the workspace (1 MB), then sweep its tokens downwards.
#include <cstdint>

#include "wkv7_internal.cuh"

namespace wkv7 {
namespace {

constexpr int L = 64;
constexpr int NTHR = 256;
constexpr int NWARP = NTHR / 32;
constexpr int SQ = kHead * kHead;  // floats per state

// staged chunk inputs, [L][64] fp32 each
enum { IN_R = 0, IN_W, IN_DLW, IN_K, IN_V, IN_A, IN_B, IN_DY, N_IN };
constexpr int NRED = 5;  // column sums per token: dr, dk, da, db, dw
constexpr size_t SMEM_BYTES = sizeof(float) * (N_IN * L * kHead + 2 * NWARP * NRED * kHead);

__device__ __forceinline__ float sum16(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 8);
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    return x;
}

// Stages tokens [row0, row0 + nv) of one head into sm (fp32); rows beyond nv are
// identity steps (w = 1, everything else 0).  `all` = false stages only what the
// forward step needs.
template <typename IO, typename WT>
__device__ void stage_chunk(float* sm, const IO* r, const WT* wl, const IO* k, const IO* v, const IO* a, const IO* b,
                            const IO* dy, long row0, long tstride, long hoff, int nv, bool all) {
    for (int e = threadIdx.x; e < L * kHead; e += NTHR) {
        const int t = e >> 6, j = e & 63;
        float rr = 0.f, w = 1.f, dlw = 0.f, kk = 0.f, vv = 0.f, aa = 0.f, bb = 0.f, dd = 0.f;
        if (t < nv) {
            const long off = (row0 + t) * tstride + hoff + j;
            const float l = to_f32(wl[off]);
            const float el = expf(l);
            w = expf(-el);
            dlw = -el * w;
            kk = to_f32(k[off]);
            vv = to_f32(v[off]);
            aa = to_f32(a[off]);
            bb = to_f32(b[off]);
            if (all) {
                rr = to_f32(r[off]);
                dd = to_f32(dy[off]);
            }
        }
        sm[IN_R * L * kHead + e] = rr;
        sm[IN_W * L * kHead + e] = w;
        sm[IN_DLW * L * kHead + e] = dlw;
        sm[IN_K * L * kHead + e] = kk;
        sm[IN_V * L * kHead + e] = vv;
        sm[IN_A * L * kHead + e] = aa;
        sm[IN_B * L * kHead + e] = bb;
        sm[IN_DY * L * kHead + e] = dd;
    }
}

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }

// One forward step on this thread's 16 elements: S <- S diag(w) + (S a) b^T + v k^T.
__device__ __forceinline__ void fwd_step(float (&S)[4][4], const float* sm, int tt, int rg, int cg) {
    const float* base = sm + tt * kHead;
    const float4 w = ld4(base + IN_W * L * kHead + 4 * cg), kk = ld4(base + IN_K * L * kHead + 4 * cg);
    const float4 a = ld4(base + IN_A * L * kHead + 4 * cg), b = ld4(base + IN_B * L * kHead + 4 * cg);
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const float vi = base[IN_V * L * kHead + rg + 16 * m];
        const float sa = sum16(S[m][0] * a.x + S[m][1] * a.y + S[m][2] * a.z + S[m][3] * a.w);
        S[m][0] = fmaf(S[m][0], w.x, fmaf(sa, b.x, vi * kk.x));
        S[m][1] = fmaf(S[m][1], w.y, fmaf(sa, b.y, vi * kk.y));
        S[m][2] = fmaf(S[m][2], w.z, fmaf(sa, b.z, vi * kk.z));
        S[m][3] = fmaf(S[m][3], w.w, fmaf(sa, b.w, vi * kk.w));
    }
}

__device__ __forceinline__ void st_state(float* dst, const float (&S)[4][4], int rg, int cg) {
#pragma unroll
    for (int m = 0; m < 4; ++m)
        *reinterpret_cast<float4*>(dst + (rg + 16 * m) * kHead + 4 * cg) = make_float4(S[m][0], S[m][1], S[m][2], S[m][3]);
}
__device__ __forceinline__ void ld_state(const float* src, float (&S)[4][4], int rg, int cg) {
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const float4 x = ld4(src + (rg + 16 * m) * kHead + 4 * cg);
        S[m][0] = x.x; S[m][1] = x.y; S[m][2] = x.z; S[m][3] = x.w;
    }
}

template <typename IO, typename WT>
__global__ void __launch_bounds__(NTHR, 1)
    wkv7_backward_kernel(const IO* __restrict__ r, const WT* __restrict__ wl, const IO* __restrict__ k,
                         const IO* __restrict__ v, const IO* __restrict__ a, const IO* __restrict__ b,
                         const float* __restrict__ s0, const IO* __restrict__ dy, const float* __restrict__ dsT,
                         IO* __restrict__ dr, WT* __restrict__ dwl, IO* __restrict__ dk, IO* __restrict__ dv,
                         IO* __restrict__ da, IO* __restrict__ db, float* __restrict__ ds0, float* __restrict__ ws,
                         int B, int T, int H, const int32_t* __restrict__ seq_offsets, long ckpt_chunks,
                         int* status) {
    extern __shared__ __align__(16) float smf[];
    float* red = smf + N_IN * L * kHead;  // [2][NWARP][NRED][64]
    const int tid = threadIdx.x, warp = tid >> 5;
    const int rg = tid >> 4, cg = tid & 15;
    const int unit = blockIdx.x;
    const int n = unit / H, h = unit % H;

    // ---- the unit's tokens and the index of its first chunk checkpoint
    long tb = 0, len = 0, cbase = 0;
    if (seq_offsets) {
        const long o0 = seq_offsets[n], o1 = seq_offsets[n + 1];
        if (o0 < 0 || o1 < o0 || o1 > T) {
            if (tid == 0) report_status(status, WKV7_ERR_DEVICE_BOUNDS);
            return;
        }
        tb = o0;
        len = o1 - o0;
        for (int m = 0; m < n; ++m) {
            const long lm = static_cast<long>(seq_offsets[m + 1]) - seq_offsets[m];
            cbase += lm > 0 ? (lm + L - 1) / L : 0;
        }
        if (cbase + (len + L - 1) / L > ckpt_chunks) {  // offsets inconsistent with the workspace size
            if (tid == 0) report_status(status, WKV7_ERR_DEVICE_BOUNDS);
            return;
        }
    } else {
        tb = static_cast<long>(n) * T;
        len = T;
        cbase = static_cast<long>(n) * ((T + L - 1) / L);
    }
    const int nchunks = static_cast<int>((len + L - 1) / L);
    const long tstride = static_cast<long>(H) * kHead, hoff = static_cast<long>(h) * kHead;
    const long sbase = (static_cast<long>(n) * H + h) * SQ;
    float* ckpt = ws;                                          // [ckpt_chunks][H][SQ]
    float* cs = ws + ckpt_chunks * H * SQ + static_cast<long>(unit) * L * SQ;  // [L][SQ] of this unit

    // ---- 1. forward: checkpoints at chunk starts
    float S[4][4];
    if (s0) {
        ld_state(s0 + sbase, S, rg, cg);
    } else {
#pragma unroll
        for (int m = 0; m < 4; ++m) S[m][0] = S[m][1] = S[m][2] = S[m][3] = 0.f;
    }
    for (int c = 0; c < nchunks; ++c) {
        const long row0 = tb + static_cast<long>(c) * L;
        const int nv = static_cast<int>(len - static_cast<long>(c) * L < L ? len - static_cast<long>(c) * L : L);
        st_state(ckpt + ((cbase + c) * H + h) * SQ, S, rg, cg);
        __syncthreads();  // the previous chunk's staged inputs are no longer read
        stage_chunk<IO, WT>(smf, r, wl, k, v, a, b, dy, row0, tstride, hoff, nv, false);
        __syncthreads();
        for (int tt = 0; tt < nv; ++tt) fwd_step(S, smf, tt, rg, cg);
    }

    // ---- 2. backward, chunks in reverse
    float G[4][4];
    if (dsT) {
        ld_state(dsT + sbase, G, rg, cg);
    } else {
#pragma unroll
        for (int m = 0; m < 4; ++m) G[m][0] = G[m][1] = G[m][2] = G[m][3] = 0.f;
    }
    int tok = 0;  // tokens swept so far (reduction buffer parity)
    for (int c = nchunks - 1; c >= 0; --c) {
        const long row0 = tb + static_cast<long>(c) * L;
        const int nv = static_cast<int>(len - static_cast<long>(c) * L < L ? len - static_cast<long>(c) * L : L);
        __syncthreads();  // every read of the previous chunk's staged inputs is done
        stage_chunk<IO, WT>(smf, r, wl, k, v, a, b, dy, row0, tstride, hoff, nv, true);
        __syncthreads();
        // recompute the chunk's states: cs[tt] = state before token tt (each thread its own elements)
        ld_state(ckpt + ((cbase + c) * H + h) * SQ, S, rg, cg);
        for (int tt = 0; tt < nv; ++tt) {
            st_state(cs + static_cast<long>(tt) * SQ, S, rg, cg);
            fwd_step(S, smf, tt, rg, cg);
        }
        // S is now the state after the chunk's last token; the state before each token is
        // loaded one token ahead (its own elements: no barrier needed)
        float Sn[4][4];
        if (nv > 0) ld_state(cs + static_cast<long>(nv - 1) * SQ, Sn, rg, cg);
        for (int tt = nv - 1; tt >= 0; --tt, ++tok) {
            const float* base = smf + tt * kHead;
            float Sp[4][4];
#pragma unroll
            for (int m = 0; m < 4; ++m)
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) Sp[m][c4] = Sn[m][c4];
            if (tt > 0) ld_state(cs + static_cast<long>(tt - 1) * SQ, Sn, rg, cg);
            const float4 rj = ld4(base + IN_R * L * kHead + 4 * cg), kj = ld4(base + IN_K * L * kHead + 4 * cg);
            const float4 aj = ld4(base + IN_A * L * kHead + 4 * cg), bj = ld4(base + IN_B * L * kHead + 4 * cg);
            const float4 wj = ld4(base + IN_W * L * kHead + 4 * cg);
            const float rv[4] = {rj.x, rj.y, rj.z, rj.w}, kv[4] = {kj.x, kj.y, kj.z, kj.w};
            const float av[4] = {aj.x, aj.y, aj.z, aj.w}, bv[4] = {bj.x, bj.y, bj.z, bj.w};
            const float wv[4] = {wj.x, wj.y, wj.z, wj.w};
            float part[NRED][4];
#pragma unroll
            for (int q = 0; q < NRED; ++q) part[q][0] = part[q][1] = part[q][2] = part[q][3] = 0.f;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int i = rg + 16 * m;
                const float dyi = base[IN_DY * L * kHead + i], vi = base[IN_V * L * kHead + i];
                float gk = 0.f, gb = 0.f, sa = 0.f;
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    G[m][c4] = fmaf(dyi, rv[c4], G[m][c4]);     // G += dy r^T
                    part[0][c4] = fmaf(S[m][c4], dyi, part[0][c4]);   // dr = S_t^T dy
                    part[1][c4] = fmaf(G[m][c4], vi, part[1][c4]);    // dk = G^T v
                    gk = fmaf(G[m][c4], kv[c4], gk);
                    gb = fmaf(G[m][c4], bv[c4], gb);
                    sa = fmaf(Sp[m][c4], av[c4], sa);
                }
                gk = sum16(gk);  // dv_i
                gb = sum16(gb);  // q_i
                sa = sum16(sa);  // p_i
                if (cg == 0) {
                    const long off = (row0 + tt) * tstride + hoff + i;
                    dv[off] = from_f32<IO>(gk);
                }
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    part[2][c4] = fmaf(Sp[m][c4], gb, part[2][c4]);   // da = S_{t-1}^T q
                    part[3][c4] = fmaf(G[m][c4], sa, part[3][c4]);    // db = G^T p
                    part[4][c4] = fmaf(G[m][c4], Sp[m][c4], part[4][c4]);  // dw
                    G[m][c4] = fmaf(G[m][c4], wv[c4], gb * av[c4]);   // G <- G diag(w) + q a^T
                    S[m][c4] = Sp[m][c4];
                }
            }
            // column sums: the two row groups of a warp, then the warps through shared memory
            float* rb = red + (tok & 1) * NWARP * NRED * kHead;
#pragma unroll
            for (int q = 0; q < NRED; ++q)
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) part[q][c4] += __shfl_xor_sync(0xffffffffu, part[q][c4], 16);
            if ((tid & 16) == 0) {
#pragma unroll
                for (int q = 0; q < NRED; ++q)
                    *reinterpret_cast<float4*>(rb + (warp * NRED + q) * kHead + 4 * cg) =
                        make_float4(part[q][0], part[q][1], part[q][2], part[q][3]);
            }
            __syncthreads();
            for (int o = tid; o < NRED * kHead; o += NTHR) {
                const int q = o >> 6, j = o & 63;
                float s = 0.f;
#pragma unroll
                for (int w8 = 0; w8 < NWARP; ++w8) s += rb[(w8 * NRED + q) * kHead + j];
                const long off = (row0 + tt) * tstride + hoff + j;
                if (q == 0) dr[off] = from_f32<IO>(s);
                else if (q == 1) dk[off] = from_f32<IO>(s);
                else if (q == 2) da[off] = from_f32<IO>(s);
                else if (q == 3) db[off] = from_f32<IO>(s);
                else dwl[off] = from_f32<WT>(s * base[IN_DLW * L * kHead + j]);
            }
        }
    }
    st_state(ds0 + sbase, G, rg, cg);
}

template <typename IO, typename WT>
cudaError_t launch_bwd_typed(const BackwardArgs& p, cudaStream_t stream) {
    auto kern = wkv7_backward_kernel<IO, WT>;
    static std::atomic<unsigned long long> configured{0};
    const cudaError_t e = configure_smem_once(kern, static_cast<int>(SMEM_BYTES), configured);
    if (e != cudaSuccess) return e;
    const long units = static_cast<long>(p.B) * p.H;
    kern<<<static_cast<unsigned>(units), NTHR, SMEM_BYTES, stream>>>(
        static_cast<const IO*>(p.r), static_cast<const WT*>(p.w_log), static_cast<const IO*>(p.k),
        static_cast<const IO*>(p.v), static_cast<const IO*>(p.a), static_cast<const IO*>(p.b), p.s0,
        static_cast<const IO*>(p.dy), p.dsT, static_cast<IO*>(p.dr), static_cast<WT*>(p.dw_log),
        static_cast<IO*>(p.dk), static_cast<IO*>(p.dv), static_cast<IO*>(p.da), static_cast<IO*>(p.db), p.ds0,
        p.ws, p.B, p.T, p.H, p.seq_offsets, p.ckpt_chunks, p.status);
    return cudaGetLastError();
}

}  // namespace

long backward_ckpt_chunks(int B, int T, int packed) {
    const long per = (static_cast<long>(T) + L - 1) / L;
    return packed ? per + B : static_cast<long>(B) * per;
}

// The larger of the two forms' needs, so that one size serves both input types.
size_t backward_workspace_floats(int B, int T, int H, int packed) {
    const size_t recurrent = static_cast<size_t>(backward_ckpt_chunks(B, T, packed)) * H * SQ +
                             static_cast<size_t>(B) * H * L * SQ;
    const size_t chunked = backward_chunked_workspace_floats(B, T, H, packed);
    return recurrent > chunked ? recurrent : chunked;
}

// bf16 inputs take the chunked form (wkv7_backward_chunk.cu); fp32 inputs keep
// this recurrent kernel, whose fp32 arithmetic holds their tighter bound.
cudaError_t launch_backward(const BackwardArgs& p, int io_dtype, int w_dtype, cudaStream_t stream) {
    if (io_dtype == WKV7_BF16) return launch_backward_chunked(p, w_dtype, stream);
    return w_dtype == WKV7_BF16 ? launch_bwd_typed<float, __nv_bfloat16>(p, stream)
                                : launch_bwd_typed<float, float>(p, stream);
}

}  // namespace wkv7
