// wkv7_backward.cu — gradient of the WKV-7 recurrence in chunked (WY) form, for
// bf16 and fp32 inputs; also the entry point's workspace size and dispatch.
//
// Per 64-token chunk, tokens as rows (row t of X is token t of the chunk), with
// Gamma_t = prod_{s<=t} w_s (per key column), Gamma_{-1} = 1, Gamma_L its last row:
//   At = a (.) Gamma_{t-1},  Rt = r (.) Gamma_t,  Bt = b / Gamma_t,  Kt = k / Gamma_t
//   Nab = tril(At Bt^T, -1), Nak = tril(At Kt^T, -1), Mrb = tril(Rt Bt^T), Mrk = tril(Rt Kt^T)
//   T = (I - Nab)^{-1},  U = T (At S0^T + Nak V)     (row t of U: S_{t-1} a_t)
//   Y = Rt S0^T + Mrb U + Mrk V,   S_L = S0 diag(Gamma_L) + U^T Bt diag(Gamma_L) + V^T Kt diag(Gamma_L)
// (the chunk-parallel form of the generalized delta rule of "RWKV-7 Goose:
// Expressive Dynamic State Evolution", section "Generalized Delta rule"; the
// pages call the model trainable in parallel but print no backward).
//
// Reverse-mode through these products, with dSLg = dS_L diag(Gamma_L):
//   dX = T^T (Mrb^T dY + Bt dSLg^T)                      dV = Mrk^T dY + Kt dSLg^T + Nak^T dX
//   dNab = tril(dX U^T, -1), dNak = tril(dX V^T, -1), dMrb = tril(dY U^T), dMrk = tril(dY V^T)
//   dAt = dX S0 + dNab Bt + dNak Kt                       dRt = dY S0 + dMrb Bt + dMrk Kt
//   dBt' = U dSLg + dNab^T At + dMrb^T Rt                 dKt' = V dSLg + dNak^T At + dMrk^T Rt
//   da = dAt (.) Gamma_{t-1},  dr = dRt (.) Gamma_t,  db = dBt' / Gamma_t,  dk = dKt' / Gamma_t
//   d log w_s = sum_{t>=s} (dr_t r_t - db_t b_t - dk_t k_t) + sum_{t>s} da_t a_t
//               + colsum(dS_L (.) S_L)                 d w_log = d log w (.) (-exp(w_log))
// and the chunk's maps between its end and start: S_L = S0 M^T + Qf and
// dS0 = Q + dS_L M with
//   M = diag(Gamma_L) (I + Bt^T T At),  Q = dY^T (Rt + Mrb T At),
//   Qf = V^T (Kt + Nak^T T^T Bt) diag(Gamma_L).
//
// Three launches:
//   1. bwd_map_kernel, a persistent grid over the (chunk, head) items: M, Q, Qf of each chunk;
//   2. bwd_scan_kernel, one block per (sequence, head) and direction: the forward
//      scan S <- S M^T + Qf writes the state at every chunk boundary, the backward
//      scan dS <- Q + dS M writes dS_L of every chunk and ds0 (the carried state
//      enters each product as tf32 high and low parts, which keeps fp32 accuracy);
//   3. bwd_grad_kernel, one block per (chunk, head): every gradient of the chunk.
// Products are warp-level tf32 tensor-core products (m16n8k8, fp32 accumulate)
// on fp32 tiles in shared memory: 64 x 64 products chained through elementwise
// steps and masks, each small enough that a register accumulator beats a round
// trip through tensor memory.  bf16 inputs: the tiles are rounded to tf32 and
// every product is one tensor-core product.  fp32 inputs: the tiles keep full
// fp32 values and every product is formed from their tf32 high and low parts
// (hi hi + hi lo + lo hi, three tensor-core products), which keeps fp32 accuracy.
// Both share the decay range of the prefill: a chunk whose Gamma_L falls below
// kMinGammaL reports WKV7_ERR_DECAY_RANGE.
#include <cstdint>

#include "prefill_common.cuh"
#include "wkv7_internal.cuh"

namespace wkv7 {
namespace {

constexpr int L = 64;
constexpr int D = kHead;
constexpr int SQ = D * D;
constexpr int NTHR = 512;  // 16 warps; warp w owns the 16 x 16 block (16 (w / 4), 16 (w % 4)) of a 64 x 64 result
constexpr int TILE = 64 * 64;

// 64 x 64 fp32 tile, row-major, with the 8-column groups of row r XOR-permuted by
// h(r) = (r mod 4) ^ bit 2 of r, which depends on r mod 8 only.  The permutation
// leaves the offset within a group alone, so a step of 8 columns is one XOR away
// and a step of 8 rows is additive; every fragment pattern below hits 32
// distinct banks per 16 lanes.
__device__ __forceinline__ int hsw(int row) { return (row & 3) ^ ((row >> 2) & 1); }
__device__ __forceinline__ int sx(int row, int col) { return (row << 6) + (col ^ (hsw(row) << 3)); }

__device__ __forceinline__ void mma_tf32(float* d, const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Fragment offsets of one operand, per lane, for the k-steps of one product.
// An m16n8k8 product sums over its 8 k in any order both operands agree on:
// lane t4 supplies k = t4 from position 2 t4 of the 8-step and k = t4 + 4 from
// 2 t4 + 1, so a row-contiguous operand reads both with one 64-bit load.
//   along rows (the 16 or 8 rows r0 + l of the operand run along its M or N; the
//   k-steps run along its columns from c0): offsets of (r0 + l, c0 + 8 s + 2 t4)
//   across rows (the k-steps run down its rows from k0; the M or N positions
//   are columns c0 + l): offsets of (k0 + 8 s + 2 t4 + e, c0 + l)
// r0, c0, k0 are multiples of 8 (all callers use multiples of 16 or 8).
struct AlongRows {
    int base, q0, h;  // row offset, first 8-column group, row's permutation
    __device__ __forceinline__ AlongRows(int row, int c0, int t4) : base((row << 6) + 2 * t4), q0(c0 >> 3), h(hsw(row)) {}
    __device__ __forceinline__ int at(int s) const { return base + (((q0 + s) ^ h) << 3); }
};
struct AcrossRows {
    int base0, base1;  // offsets of (k0 + 2 t4 + e, col)
    __device__ __forceinline__ AcrossRows(int k0, int col, int t4) {
        const int r0 = k0 + 2 * t4;
        base0 = (r0 << 6) + (col ^ (hsw(r0) << 3));
        base1 = ((r0 + 1) << 6) + (col ^ (hsw(r0 + 1) << 3));
    }
};

// tf32 high and low parts of fp32 values: x = hi + lo to about 2^-22 relative
__device__ __forceinline__ void split_tf32(uint32_t x, uint32_t& hi, uint32_t& lo) {
    const float h = round_tf32(__uint_as_float(x));
    hi = __float_as_uint(h);
    lo = __float_as_uint(round_tf32(__uint_as_float(x) - h));
}
// The two products of one k-step (n-tiles p and q).  SP: the tiles hold full fp32
// values, and each product is formed from tf32 parts as hi*hi + hi*lo + lo*hi,
// which keeps fp32 accuracy (the fp32-input path).
template <bool SP>
__device__ __forceinline__ void mma_pair(float (&acc)[8], const uint32_t (&a)[4], const uint32_t (&p)[2],
                                         const uint32_t (&q)[2]) {
    if constexpr (!SP) {
        mma_tf32(acc, a, p);
        mma_tf32(acc + 4, a, q);
    } else {
        uint32_t ah[4], al[4], ph[2], pl[2], qh[2], ql[2];
#pragma unroll
        for (int i = 0; i < 4; ++i) split_tf32(a[i], ah[i], al[i]);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            split_tf32(p[i], ph[i], pl[i]);
            split_tf32(q[i], qh[i], ql[i]);
        }
        mma_tf32(acc, al, ph);
        mma_tf32(acc + 4, al, qh);
        mma_tf32(acc, ah, pl);
        mma_tf32(acc + 4, ah, ql);
        mma_tf32(acc, ah, ph);
        mma_tf32(acc + 4, ah, qh);
    }
}

// acc (16 x 16) += sum_{kk < 8 nk} op(A)(ar + m, ac + kk) op(B)(bk + kk, bn + n)   (one warp)
// with op(X) = X, or X^T when the flag is set.  acc[4 h + 2 q + e] is row
// gq + 8 q, column 8 h + 2 t4 + e of the block (lane = 4 gq + t4).
template <bool TA, bool TB, bool SP = false>
__device__ __forceinline__ void gemm16(float (&acc)[8], const float* A, int ar, int ac, const float* B, int bk, int bn,
                                       int nk, int gq, int t4) {
    if (!TA && !TB) {
        const AlongRows a0(ar + gq, ac, t4), a1(ar + gq + 8, ac, t4);
        const AcrossRows b0(bk, bn + gq, t4), b1(bk, bn + 8 + gq, t4);
#pragma unroll(SP ? 1 : 4)
        for (int s = 0; s < nk; ++s) {
            const float2 x0 = *reinterpret_cast<const float2*>(A + a0.at(s));
            const float2 x1 = *reinterpret_cast<const float2*>(A + a1.at(s));
            const uint32_t a[4] = {__float_as_uint(x0.x), __float_as_uint(x1.x), __float_as_uint(x0.y),
                                   __float_as_uint(x1.y)};
            const uint32_t p[2] = {__float_as_uint(B[b0.base0 + 512 * s]), __float_as_uint(B[b0.base1 + 512 * s])};
            const uint32_t q[2] = {__float_as_uint(B[b1.base0 + 512 * s]), __float_as_uint(B[b1.base1 + 512 * s])};
            mma_pair<SP>(acc, a, p, q);
        }
    } else if (!TA && TB) {
        const AlongRows a0(ar + gq, ac, t4), a1(ar + gq + 8, ac, t4);
        const AlongRows b0(bn + gq, bk, t4), b1(bn + 8 + gq, bk, t4);
#pragma unroll(SP ? 1 : 4)
        for (int s = 0; s < nk; ++s) {
            const float2 x0 = *reinterpret_cast<const float2*>(A + a0.at(s));
            const float2 x1 = *reinterpret_cast<const float2*>(A + a1.at(s));
            const float2 y0 = *reinterpret_cast<const float2*>(B + b0.at(s));
            const float2 y1 = *reinterpret_cast<const float2*>(B + b1.at(s));
            const uint32_t a[4] = {__float_as_uint(x0.x), __float_as_uint(x1.x), __float_as_uint(x0.y),
                                   __float_as_uint(x1.y)};
            const uint32_t p[2] = {__float_as_uint(y0.x), __float_as_uint(y0.y)};
            const uint32_t q[2] = {__float_as_uint(y1.x), __float_as_uint(y1.y)};
            mma_pair<SP>(acc, a, p, q);
        }
    } else if (TA && !TB) {
        const AcrossRows a0(ac, ar + gq, t4), a1(ac, ar + gq + 8, t4);
        const AcrossRows b0(bk, bn + gq, t4), b1(bk, bn + 8 + gq, t4);
#pragma unroll(SP ? 1 : 4)
        for (int s = 0; s < nk; ++s) {
            const int o = 512 * s;
            const uint32_t a[4] = {__float_as_uint(A[a0.base0 + o]), __float_as_uint(A[a1.base0 + o]),
                                   __float_as_uint(A[a0.base1 + o]), __float_as_uint(A[a1.base1 + o])};
            const uint32_t p[2] = {__float_as_uint(B[b0.base0 + o]), __float_as_uint(B[b0.base1 + o])};
            const uint32_t q[2] = {__float_as_uint(B[b1.base0 + o]), __float_as_uint(B[b1.base1 + o])};
            mma_pair<SP>(acc, a, p, q);
        }
    } else {
        const AcrossRows a0(ac, ar + gq, t4), a1(ac, ar + gq + 8, t4);
        const AlongRows b0(bn + gq, bk, t4), b1(bn + 8 + gq, bk, t4);
#pragma unroll(SP ? 1 : 4)
        for (int s = 0; s < nk; ++s) {
            const int o = 512 * s;
            const float2 y0 = *reinterpret_cast<const float2*>(B + b0.at(s));
            const float2 y1 = *reinterpret_cast<const float2*>(B + b1.at(s));
            const uint32_t a[4] = {__float_as_uint(A[a0.base0 + o]), __float_as_uint(A[a1.base0 + o]),
                                   __float_as_uint(A[a0.base1 + o]), __float_as_uint(A[a1.base1 + o])};
            const uint32_t p[2] = {__float_as_uint(y0.x), __float_as_uint(y0.y)};
            const uint32_t q[2] = {__float_as_uint(y1.x), __float_as_uint(y1.y)};
            mma_pair<SP>(acc, a, p, q);
        }
    }
}

// The fragments of one k-step of gemm16's operands, as separate loaders, so that
// gemm16_2 can run two independent products through the same k-steps.
template <bool T>
struct OpA;  // A: 16 rows (M) x 8 k
template <>
struct OpA<false> {
    AlongRows r0, r1;
    __device__ __forceinline__ OpA(int ar, int ac, int gq, int t4) : r0(ar + gq, ac, t4), r1(ar + gq + 8, ac, t4) {}
    __device__ __forceinline__ void load(const float* A, int s, uint32_t (&a)[4]) const {
        const float2 x0 = *reinterpret_cast<const float2*>(A + r0.at(s));
        const float2 x1 = *reinterpret_cast<const float2*>(A + r1.at(s));
        a[0] = __float_as_uint(x0.x);
        a[1] = __float_as_uint(x1.x);
        a[2] = __float_as_uint(x0.y);
        a[3] = __float_as_uint(x1.y);
    }
};
template <>
struct OpA<true> {
    AcrossRows c0, c1;
    __device__ __forceinline__ OpA(int ar, int ac, int gq, int t4) : c0(ac, ar + gq, t4), c1(ac, ar + gq + 8, t4) {}
    __device__ __forceinline__ void load(const float* A, int s, uint32_t (&a)[4]) const {
        const int o = 512 * s;
        a[0] = __float_as_uint(A[c0.base0 + o]);
        a[1] = __float_as_uint(A[c1.base0 + o]);
        a[2] = __float_as_uint(A[c0.base1 + o]);
        a[3] = __float_as_uint(A[c1.base1 + o]);
    }
};
template <bool T>
struct OpB;  // B: 8 k x 16 columns (N), as two n-tiles
template <>
struct OpB<false> {
    AcrossRows b0, b1;
    __device__ __forceinline__ OpB(int bk, int bn, int gq, int t4) : b0(bk, bn + gq, t4), b1(bk, bn + 8 + gq, t4) {}
    __device__ __forceinline__ void load(const float* B, int s, uint32_t (&p)[2], uint32_t (&q)[2]) const {
        const int o = 512 * s;
        p[0] = __float_as_uint(B[b0.base0 + o]);
        p[1] = __float_as_uint(B[b0.base1 + o]);
        q[0] = __float_as_uint(B[b1.base0 + o]);
        q[1] = __float_as_uint(B[b1.base1 + o]);
    }
};
template <>
struct OpB<true> {
    AlongRows b0, b1;
    __device__ __forceinline__ OpB(int bk, int bn, int gq, int t4) : b0(bn + gq, bk, t4), b1(bn + 8 + gq, bk, t4) {}
    __device__ __forceinline__ void load(const float* B, int s, uint32_t (&p)[2], uint32_t (&q)[2]) const {
        const float2 y0 = *reinterpret_cast<const float2*>(B + b0.at(s));
        const float2 y1 = *reinterpret_cast<const float2*>(B + b1.at(s));
        p[0] = __float_as_uint(y0.x);
        p[1] = __float_as_uint(y0.y);
        q[0] = __float_as_uint(y1.x);
        q[1] = __float_as_uint(y1.y);
    }
};

// Two independent products of gemm16's form (each with its own operand orientations
// and k-step count), advanced together: each k-step issues both products' fragment
// loads and then their four products, so the two accumulator chains overlap.
template <bool TA1, bool TB1, bool TA2, bool TB2, bool SP>
__device__ __forceinline__ void gemm16_2(float (&acc1)[8], const float* A1, int ar1, int ac1, const float* B1, int bk1,
                                         int bn1, int nk1, float (&acc2)[8], const float* A2, int ar2, int ac2,
                                         const float* B2, int bk2, int bn2, int nk2, int gq, int t4) {
    const OpA<TA1> x1(ar1, ac1, gq, t4);
    const OpA<TA2> x2(ar2, ac2, gq, t4);
    const OpB<TB1> y1(bk1, bn1, gq, t4);
    const OpB<TB2> y2(bk2, bn2, gq, t4);
    const int nk = nk1 > nk2 ? nk1 : nk2;
#pragma unroll(SP ? 1 : 2)
    for (int s = 0; s < nk; ++s) {
        uint32_t a1[4], a2[4], p1[2], q1[2], p2[2], q2[2];
        if (s < nk1) {
            x1.load(A1, s, a1);
            y1.load(B1, s, p1, q1);
        }
        if (s < nk2) {
            x2.load(A2, s, a2);
            y2.load(B2, s, p2, q2);
        }
        if (s < nk1) mma_pair<SP>(acc1, a1, p1, q1);
        if (s < nk2) mma_pair<SP>(acc2, a2, p2, q2);
    }
}

constexpr float kLog2e = 1.4426950408889634f;
// w = exp(-exp(l)) and exp(l) by the hardware 2^x (subnormals flushed: a w that
// small fails the decay-range check anyway)
__device__ __forceinline__ float decay(float l) { return ex2_ftz(-kLog2e * ex2_ftz(kLog2e * l)); }
__device__ __forceinline__ float exp_l(float l) { return ex2_ftz(kLog2e * l); }

__device__ __forceinline__ void zero8(float (&acc)[8]) {
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
}

// row / column of acc[e] within the warp's 16 x 16 block
__device__ __forceinline__ int frag_row(int e, int gq) { return gq + 8 * ((e >> 1) & 1); }
__device__ __forceinline__ int frag_col(int e, int t4) { return 8 * (e >> 2) + 2 * t4 + (e & 1); }

// Stores acc as the block (r0, c0) of C (tf32-rounded).  MASK 1 keeps col < row,
// MASK 2 keeps col <= row (row, col in C's coordinates).
template <int MASK, bool RND = true>
__device__ __forceinline__ void st16(float* C, const float (&acc)[8], int r0, int c0, int gq, int t4) {
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
        const int row = r0 + frag_row(e, gq), col = c0 + frag_col(e, t4);
        float x0 = acc[e], x1 = acc[e + 1];
        if (MASK == 1) {
            x0 = col < row ? x0 : 0.f;
            x1 = col + 1 < row ? x1 : 0.f;
        } else if (MASK == 2) {
            x0 = col <= row ? x0 : 0.f;
            x1 = col + 1 <= row ? x1 : 0.f;
        }
        *reinterpret_cast<float2*>(C + sx(row, col)) =
            RND ? make_float2(round_tf32(x0), round_tf32(x1)) : make_float2(x0, x1);
    }
}

__device__ __forceinline__ float2 bf2_to_f2(uint32_t u) { return make_float2(bf16lo_to_f32(u), bf16hi_to_f32(u)); }
__device__ __forceinline__ void unpack8(uint4 u, float (&x)[8]) {
    float2 p = bf2_to_f2(u.x);
    x[0] = p.x; x[1] = p.y;
    p = bf2_to_f2(u.y);
    x[2] = p.x; x[3] = p.y;
    p = bf2_to_f2(u.z);
    x[4] = p.x; x[5] = p.y;
    p = bf2_to_f2(u.w);
    x[6] = p.x; x[7] = p.y;
}
// eight consecutive values as fp32 (decay logits, and the inputs of either type)
__device__ __forceinline__ void ld_wlog8(const float* p, float (&x)[8]) {
    const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
__device__ __forceinline__ void ld_wlog8(const __nv_bfloat16* p, float (&x)[8]) {
    unpack8(*reinterpret_cast<const uint4*>(p), x);
}
__device__ __forceinline__ void st8(float* tile, int row, int c0, const float (&x)[8], bool rnd) {
    float y[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] = rnd ? round_tf32(x[e]) : x[e];
    *reinterpret_cast<float4*>(tile + sx(row, c0)) = make_float4(y[0], y[1], y[2], y[3]);
    *reinterpret_cast<float4*>(tile + sx(row, c0 + 4)) = make_float4(y[4], y[5], y[6], y[7]);
}
__device__ __forceinline__ void ld8(const float* tile, int row, int c0, float (&x)[8]) {
    const float4 a = *reinterpret_cast<const float4*>(tile + sx(row, c0));
    const float4 b = *reinterpret_cast<const float4*>(tile + sx(row, c0 + 4));
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

// Where one chunk sits: its first token row, its length, and the workspace
// region of its (sequence, head) unit.  A unit of nch chunks owns 3 (nch + 1)
// states of D x D floats: M[0..nch], Q[0..nch] (dS_L after the backward scan),
// and Qf[0..nch] (the state at every chunk boundary S[0..nch] after the forward
// scan, which writes S[c] once it has read Qf[c]); the units of sequence n start
// at state 3 H (cbase_n + n), head h at 3 h (nch_n + 1) within.
struct ChunkLoc {
    long row0;    // token row of the chunk's first token
    long region;  // float offset of the unit's region in the workspace
    int c;        // chunk index within the sequence
    int nch;      // chunks of the sequence
    int nv;       // tokens of the chunk (1 .. 64)
};

__device__ __forceinline__ long unit_region(long cbase, int n, int h, int H, int nch) {
    return (3L * H * (cbase + n) + 3L * h * (nch + 1)) * SQ;
}

// Chunk g (counted over all sequences) of head h.  Returns false past the last
// chunk, or after reporting WKV7_ERR_DEVICE_BOUNDS for offsets that are not
// monotone, leave [0, T], or need more chunks than the workspace holds.
__device__ bool locate_chunk(long g, int h, int B, int T, int H, const int32_t* offs, long ckpt_chunks, int* status,
                             ChunkLoc& o) {
    if (!offs) {
        const long cps = (static_cast<long>(T) + L - 1) / L;
        if (cps == 0 || g >= static_cast<long>(B) * cps) return false;
        const int n = static_cast<int>(g / cps);
        o.c = static_cast<int>(g % cps);
        o.nch = static_cast<int>(cps);
        o.row0 = static_cast<long>(n) * T + static_cast<long>(o.c) * L;
        const long rest = static_cast<long>(T) - static_cast<long>(o.c) * L;
        o.nv = static_cast<int>(rest < L ? rest : L);
        o.region = unit_region(static_cast<long>(n) * cps, n, h, H, o.nch);
        return true;
    }
    long cbase = 0;
    for (int n = 0; n < B; ++n) {
        const long o0 = offs[n], o1 = offs[n + 1];
        if (o0 < 0 || o1 < o0 || o1 > T) {
            report_status(status, WKV7_ERR_DEVICE_BOUNDS);
            return false;
        }
        const long nc = (o1 - o0 + L - 1) / L;
        if (g < cbase + nc) {
            if (cbase + nc > ckpt_chunks) {
                report_status(status, WKV7_ERR_DEVICE_BOUNDS);
                return false;
            }
            o.c = static_cast<int>(g - cbase);
            o.nch = static_cast<int>(nc);
            o.row0 = o0 + static_cast<long>(o.c) * L;
            const long rest = o1 - o.row0;
            o.nv = static_cast<int>(rest < L ? rest : L);
            o.region = unit_region(cbase, n, h, H, o.nch);
            return true;
        }
        cbase += nc;
    }
    return false;
}

// Thread 0 locates the block's chunk; the others read it from shared memory.
__device__ bool locate_block_chunk(int B, int T, int H, const int32_t* offs, long ckpt_chunks, int* status,
                                   ChunkLoc& o, ChunkLoc* sh, int* sh_ok) {
    if (threadIdx.x == 0) {
        ChunkLoc x{};
        const bool ok = locate_chunk(blockIdx.x, blockIdx.y, B, T, H, offs, ckpt_chunks, status, x);
        *sh = x;
        *sh_ok = ok ? 1 : 0;
    }
    __syncthreads();
    o = *sh;
    return *sh_ok != 0;
}

// L2 prefetch of the inputs of the block `ahead` places later in launch order
// (dense batches; with one block per SM that is about the next block this SM
// runs, so its staging finds its rows in L2).  One thread per 128-byte row piece.
template <typename IO, typename WT>
__device__ __forceinline__ void prefetch_ahead(const IO* r, const WT* wl, const IO* k, const IO* v, const IO* a,
                                               const IO* b, const IO* dy, int B, int T, int H, const int32_t* offs,
                                               unsigned ahead) {
    if (offs || threadIdx.x >= 64) return;
    const unsigned id = blockIdx.y * gridDim.x + blockIdx.x + ahead;
    if (id >= gridDim.x * gridDim.y) return;
    const long cps = (static_cast<long>(T) + L - 1) / L;
    const int h = static_cast<int>(id / gridDim.x);
    const long g = id % gridDim.x;
    const long n = g / cps, c = g % cps;
    const int t = threadIdx.x;
    if (n >= B || c * L + t >= T) return;
    const long off = (n * T + c * L + t) * static_cast<long>(H) * D + static_cast<long>(h) * D;
    const void* rows[7] = {r + off, k + off, v + off, a + off, b + off, dy + off, wl + off};
#pragma unroll
    for (int q = 0; q < 7; ++q) asm volatile("prefetch.global.L2 [%0];" ::"l"(rows[q]));
    if constexpr (sizeof(IO) == 4) {
        const void* rows2[6] = {r + off + 32, k + off + 32, v + off + 32, a + off + 32, b + off + 32, dy + off + 32};
#pragma unroll
        for (int q = 0; q < 6; ++q) asm volatile("prefetch.global.L2 [%0];" ::"l"(rows2[q]));
    }
    if constexpr (sizeof(WT) == 4) asm volatile("prefetch.global.L2 [%0];" ::"l"(wl + off + 32));
}

// Stages the chunk's inputs of one head as fp32 tiles: GAM = Gamma (running
// products of w = exp(-exp(w_log)) down the tokens), AT, RT, BT, KT (the scaled
// operands, tf32-rounded), VV and DY (bf16 values, exact in tf32); GL = Gamma_L.
// Rows t >= nv are identity steps (w = 1, every other input 0).  The inputs are
// read from rows 0 .. nv - 1 of r .. dy (each pointing at the chunk's first token
// row of this head) with a row stride of rs elements: the tensors in global
// memory, or copies of the rows in shared memory.  seg: 8 x 64 floats of
// scratch.  Ends with a block barrier.
template <typename IO, typename WT>
__device__ void stage_chunk(float* GAM, float* AT, float* RT, float* BT, float* KT, float* VV, float* DY, float* GL,
                            float* seg, const IO* r, const WT* wl, const IO* k, const IO* v, const IO* a, const IO* b,
                            const IO* dy, long rs, int nv) {
    constexpr bool RND = sizeof(IO) == 2;  // bf16 inputs: tf32 operand tiles; fp32 inputs: full fp32 tiles
    const int tid = threadIdx.x;
    const int t = tid >> 3, c0 = 8 * (tid & 7);
    float rr[8], kk[8], aa[8], bb[8], x[8];
    if (t < nv) {
        const long off = t * rs + c0;
        ld_wlog8(r + off, rr);
        ld_wlog8(k + off, kk);
        ld_wlog8(a + off, aa);
        ld_wlog8(b + off, bb);
        ld_wlog8(v + off, x);
        st8(VV, t, c0, x, false);
        ld_wlog8(dy + off, x);
        st8(DY, t, c0, x, false);
        ld_wlog8(wl + off, x);
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = decay(x[e]);
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            rr[e] = kk[e] = aa[e] = bb[e] = 0.f;
            x[e] = 0.f;
        }
        st8(VV, t, c0, x, false);
        st8(DY, t, c0, x, false);
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = 1.f;
    }
    st8(GAM, t, c0, x, false);
    __syncthreads();
    {
        // running products: thread (column j, segment s of 8 tokens)
        const int j = tid & 63, s = tid >> 6;
        float p[8], run = 1.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            run *= GAM[sx(8 * s + i, j)];
            p[i] = run;
        }
        seg[s * 64 + j] = run;
        __syncthreads();
        float pre = 1.f;
        for (int q = 0; q < s; ++q) pre *= seg[q * 64 + j];
#pragma unroll
        for (int i = 0; i < 8; ++i) GAM[sx(8 * s + i, j)] = pre * p[i];
        if (s == 7) GL[j] = pre * p[7];
    }
    __syncthreads();
    {
        float g[8], gp[8];
        ld8(GAM, t, c0, g);
        if (t > 0) {
            ld8(GAM, t - 1, c0, gp);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) gp[e] = 1.f;
        }
        float o1[8], o2[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            o1[e] = aa[e] * gp[e];
            o2[e] = rr[e] * g[e];
        }
        st8(AT, t, c0, o1, RND);
        st8(RT, t, c0, o2, RND);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float inv = __frcp_rn(g[e]);
            o1[e] = bb[e] * inv;
            o2[e] = kk[e] * inv;
        }
        st8(BT, t, c0, o1, RND);
        st8(KT, t, c0, o2, RND);
    }
    __syncthreads();
}

// Tm = (I - N)^{-1} for strictly lower-triangular N (both 64 x 64 tiles):
//  (1) the 16 x 16 diagonal blocks D_b = (I - N_bb)^{-1}: thread 16 b + c computes
//      column c by forward substitution;
//  (2) T_{b+1,b} = D_{b+1} (N_{b+1,b} D_b) for b = 0, 2;
//  (3) T_hl = T_hi (N_hl T_lo) for the 32 x 32 halves.
// Intermediate products live in the upper-right 32 x 32 quadrant of Tm (zero in
// T), which is cleared at the end.  Every thread of the block calls this; it
// starts and ends with the caller's data in place (barriers inside).
template <bool SP>
__device__ void invert_unit_lower(const float* N, float* Tm) {
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31, gq = lane >> 2, t4 = lane & 3;
    if (tid < 64) {
        const int r0 = 16 * (tid >> 4), c = tid & 15;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float p = (i == c) ? 1.f : 0.f;
#pragma unroll
            for (int j = 0; j < i; ++j) p = fmaf(N[sx(r0 + i, r0 + j)], x[j], p);
            x[i] = p;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) Tm[sx(r0 + i, r0 + c)] = SP ? x[i] : round_tf32(x[i]);
    } else {
        // blocks (0, 1) and (2, 3) are zero in T and not used as scratch
        for (int e = tid - 64; e < 512; e += NTHR - 64) {
            const int row = e >> 4, col = e & 15;  // 32 rows x 16 columns
            if (row < 16) Tm[sx(row, 16 + col)] = 0.f;   // rows 0 .. 15, columns 16 .. 31
            else Tm[sx(16 + row, 48 + col)] = 0.f;       // rows 32 .. 47, columns 48 .. 63
        }
    }
    __syncthreads();
    if (w < 2) {
        // Y_b = N_{b+1,b} D_b -> quadrant block (w, 2 + w)
        float acc[8];
        zero8(acc);
        const int b0 = 32 * w;
        gemm16<false, false, SP>(acc, N, b0 + 16, b0, Tm, b0, b0, 2, gq, t4);
        st16<0, !SP>(Tm, acc, 16 * w, 32 + 16 * w, gq, t4);
    }
    __syncthreads();
    if (w < 2) {
        // T_{b+1,b} = D_{b+1} Y_b
        float acc[8];
        zero8(acc);
        const int b0 = 32 * w;
        gemm16<false, false, SP>(acc, Tm, b0 + 16, b0 + 16, Tm, 16 * w, 32 + 16 * w, 2, gq, t4);
        st16<0, !SP>(Tm, acc, b0 + 16, b0, gq, t4);
    }
    __syncthreads();
    if (w < 4) {
        // X = N_hl T_lo -> quadrant (T_lo is zero above its diagonal: k from 16 ni)
        const int mi = w >> 1, ni = w & 1;
        float acc[8];
        zero8(acc);
        gemm16<false, false, SP>(acc, N, 32 + 16 * mi, 16 * ni, Tm, 16 * ni, 16 * ni, 4 - 2 * ni, gq, t4);
        st16<0, !SP>(Tm, acc, 16 * mi, 32 + 16 * ni, gq, t4);
    }
    __syncthreads();
    if (w < 4) {
        // T_hl = T_hi X (T_hi is zero right of its diagonal: k up to 16 mi + 16)
        const int mi = w >> 1, ni = w & 1;
        float acc[8];
        zero8(acc);
        gemm16<false, false, SP>(acc, Tm, 32 + 16 * mi, 32, Tm, 0, 32 + 16 * ni, 2 + 2 * mi, gq, t4);
        st16<0, !SP>(Tm, acc, 32 + 16 * mi, 16 * ni, gq, t4);
    }
    __syncthreads();
    for (int e = tid; e < 1024; e += NTHR) Tm[sx(e >> 5, 32 + (e & 31))] = 0.f;
    __syncthreads();
}

// shared memory of the map and gradient kernels: 13 tiles, Gamma_L, 8 x 64 scratch,
// 64 column sums, the chunk's location
constexpr int N_TILES = 13;
constexpr size_t SMEM_BYTES =
    sizeof(float) * (N_TILES * TILE + 64 + 8 * 64 + 64) + 2 * sizeof(ChunkLoc) + 16;

struct Smem {
    float* tile[N_TILES];
    float* GL;
    float* seg;
    float* csum;
    ChunkLoc* loc;
    int* ok;
};
__device__ __forceinline__ Smem carve(float* smf) {
    Smem s;
#pragma unroll
    for (int i = 0; i < N_TILES; ++i) s.tile[i] = smf + i * TILE;
    s.GL = smf + N_TILES * TILE;
    s.seg = s.GL + 64;
    s.csum = s.seg + 8 * 64;
    s.loc = reinterpret_cast<ChunkLoc*>(s.csum + 64);  // two slots (the map kernel's current and next chunk)
    s.ok = reinterpret_cast<int*>(s.loc + 2);
    return s;
}

// acc -> block (r0, c0) of a row-major 64 x 64 fp32 matrix in global memory
__device__ __forceinline__ void st16_global(float* G, const float (&acc)[8], int r0, int c0, int gq, int t4) {
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
        const int row = r0 + frag_row(e, gq), col = c0 + frag_col(e, t4);
        *reinterpret_cast<float2*>(G + row * 64 + col) = make_float2(acc[e], acc[e + 1]);
    }
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Nab = tril(At Bt^T, -1), Nak = tril(At Kt^T, -1), Mrb = tril(Rt Bt^T) (each warp its
// block of all three; blocks above the diagonal are zero)
template <bool SP>
__device__ __forceinline__ void masks_abk(const float* AT, const float* RT, const float* BT, const float* KT,
                                          float* NAB, float* NAK, float* MRB, int m0, int n0, int gq, int t4) {
    float acc[8];
    zero8(acc);
    if (n0 > m0) {
        st16<0, !SP>(NAB, acc, m0, n0, gq, t4);
        st16<0, !SP>(NAK, acc, m0, n0, gq, t4);
        st16<0, !SP>(MRB, acc, m0, n0, gq, t4);
        return;
    }
    gemm16<false, true, SP>(acc, AT, m0, 0, BT, 0, n0, 8, gq, t4);
    st16<1, !SP>(NAB, acc, m0, n0, gq, t4);
    zero8(acc);
    gemm16<false, true, SP>(acc, AT, m0, 0, KT, 0, n0, 8, gq, t4);
    st16<1, !SP>(NAK, acc, m0, n0, gq, t4);
    zero8(acc);
    gemm16<false, true, SP>(acc, RT, m0, 0, BT, 0, n0, 8, gq, t4);
    st16<2, !SP>(MRB, acc, m0, n0, gq, t4);
}

enum { T_GAM = 0, T_AT, T_RT, T_BT, T_KT, T_VV, T_DY, T_X0, T_X1, T_X2, T_X3, T_X4, T_X5 };

// Raw input rows of one chunk and head into shared memory (per-thread 16-byte
// cp.async): rows 0 .. nv - 1 of r, k, a, b, v, dy (bf16, 128 bytes each) into
// two 16 KB tiles' worth of row-major buffers R2 = [r | k], A2 = [a | b],
// V2 = [v | dy], and the w_log rows (64 or 128 bytes) into W1.  One commit group.
template <typename WT>
__device__ __forceinline__ void issue_raw(float* R2, float* A2, float* V2, float* W1, const __nv_bfloat16* r,
                                          const WT* wl, const __nv_bfloat16* k, const __nv_bfloat16* v,
                                          const __nv_bfloat16* a, const __nv_bfloat16* b, const __nv_bfloat16* dy,
                                          long o, long tstride, int nv) {
    const int tid = threadIdx.x, t = tid >> 3, pc = tid & 7;  // 64 rows x 8 pieces of 16 bytes
    if (t < nv) {
        const long go = o + t * tstride + 8 * pc;
        __nv_bfloat16* rr = reinterpret_cast<__nv_bfloat16*>(R2);
        __nv_bfloat16* aa = reinterpret_cast<__nv_bfloat16*>(A2);
        __nv_bfloat16* vv = reinterpret_cast<__nv_bfloat16*>(V2);
        const int so = t * 64 + 8 * pc;
        cp_async16(rr + so, r + go);
        cp_async16(rr + 4096 + so, k + go);
        cp_async16(aa + so, a + go);
        cp_async16(aa + 4096 + so, b + go);
        cp_async16(vv + so, v + go);
        cp_async16(vv + 4096 + so, dy + go);
        WT* ww = reinterpret_cast<WT*>(W1);
        constexpr int PER_ROW = 64 * sizeof(WT) / 16;  // 16-byte pieces per w_log row
#pragma unroll
        for (int q = pc; q < PER_ROW; q += 8) cp_async16(ww + t * 64 + q * (16 / sizeof(WT)), wl + o + t * tstride + q * (16 / sizeof(WT)));
    }
    cp_async_commit();
}

// ---- 1. the chunk's maps M, Q, Qf.  A persistent grid walks over the
// (chunk, head) items; while an item's last products run, the raw rows of the
// block's next item are copied into four tiles that are dead by then (NAK,
// MRB, TA, TB), so the next staging reads shared memory instead of waiting for
// global loads.
template <typename IO, typename WT>
__global__ void __launch_bounds__(NTHR, 1)
    bwd_map_kernel(const IO* __restrict__ r, const WT* __restrict__ wl, const IO* __restrict__ k,
                   const IO* __restrict__ v, const IO* __restrict__ a, const IO* __restrict__ b,
                   const IO* __restrict__ dy, float* __restrict__ ws, int B, int T, int H,
                   const int32_t* __restrict__ offs, long ckpt_chunks, int* status) {
    // bf16 inputs: tf32 products, raw rows of the next item copied ahead into dead tiles;
    // fp32 inputs: split products on full fp32 tiles, rows staged from global memory
    constexpr bool SP = sizeof(IO) == 4;
    extern __shared__ __align__(16) float smf[];
    const Smem sm = carve(smf);
    float *GAM = sm.tile[T_GAM], *AT = sm.tile[T_AT], *RT = sm.tile[T_RT], *BT = sm.tile[T_BT], *KT = sm.tile[T_KT];
    float *VV = sm.tile[T_VV], *DY = sm.tile[T_DY];
    float *NAB = sm.tile[T_X0], *NAK = sm.tile[T_X1], *MRB = sm.tile[T_X2], *TT = sm.tile[T_X3];
    float *TA = sm.tile[T_X4], *TB = sm.tile[T_X5];
    const int tid = threadIdx.x, w = tid >> 5, gq = (tid & 31) >> 2, t4 = tid & 3;
    const int m0 = 16 * (w >> 2), n0 = 16 * (w & 3);
    const long tstride = static_cast<long>(H) * D;
    const long n_items = ckpt_chunks * H;  // item = h * ckpt_chunks + chunk
    const __nv_bfloat16* raw = reinterpret_cast<const __nv_bfloat16*>(NAK);  // [r | k], then [a | b] in MRB ...
    const __nv_bfloat16* rawa = reinterpret_cast<const __nv_bfloat16*>(MRB);
    const __nv_bfloat16* rawv = reinterpret_cast<const __nv_bfloat16*>(TA);
    const WT* raww = reinterpret_cast<const WT*>(TB);
    auto locate_item = [&](long item, int slot) {  // thread 0
        ChunkLoc x{};
        const bool ok = item < n_items &&
                        locate_chunk(item % ckpt_chunks, static_cast<int>(item / ckpt_chunks), B, T, H, offs,
                                     ckpt_chunks, status, x);
        sm.loc[slot] = x;
        sm.ok[slot] = ok ? 1 : 0;
    };
    auto head_of = [&](long item) { return static_cast<long>(item / ckpt_chunks) * D; };

    long item = blockIdx.x;
    int cur = 0;
    if (tid == 0) locate_item(item, 0);
    __syncthreads();
    if constexpr (!SP) {
        if (sm.ok[0])
            issue_raw<WT>(NAK, MRB, TA, TB, r, wl, k, v, a, b, dy, sm.loc[0].row0 * tstride + head_of(item), tstride,
                          sm.loc[0].nv);
        else
            cp_async_commit();
    }
    for (; item < n_items; item += gridDim.x, cur ^= 1) {
        const long next = item + gridDim.x;
        if (tid == 0) locate_item(next, cur ^ 1);  // read by every thread after the barriers below
        cp_async_wait<0>();
        __syncthreads();  // this item's raw rows have landed; the previous item's products are done
        const ChunkLoc lc = sm.loc[cur];
        const bool ok = sm.ok[cur] != 0;
        auto prefetch_next = [&]() {
            if constexpr (!SP) {
                if (sm.ok[cur ^ 1])
                    issue_raw<WT>(NAK, MRB, TA, TB, r, wl, k, v, a, b, dy,
                                  sm.loc[cur ^ 1].row0 * tstride + head_of(next), tstride, sm.loc[cur ^ 1].nv);
                else
                    cp_async_commit();
            }
        };
        if (!ok) {
            prefetch_next();
            continue;
        }
        if constexpr (SP) {
            const long o = lc.row0 * tstride + head_of(item);
            stage_chunk<IO, WT>(GAM, AT, RT, BT, KT, VV, DY, sm.GL, sm.seg, r + o, wl + o, k + o, v + o, a + o, b + o,
                                dy + o, tstride, lc.nv);
        } else {
            stage_chunk<__nv_bfloat16, WT>(GAM, AT, RT, BT, KT, VV, DY, sm.GL, sm.seg, raw, raww, raw + 4096, rawv,
                                           rawa, rawa + 4096, rawv + 4096, 64, lc.nv);
        }
        if (tid < 64 && !(sm.GL[tid] >= kMinGammaL)) report_status(status, WKV7_ERR_DECAY_RANGE);
        masks_abk<SP>(AT, RT, BT, KT, NAB, NAK, MRB, m0, n0, gq, t4);
        __syncthreads();
        invert_unit_lower<SP>(NAB, TT);
        {
            float acc[8];
            zero8(acc);  // TA = T At (T is zero right of its diagonal)
            gemm16<false, false, SP>(acc, TT, m0, 0, AT, 0, n0, (m0 + 16) / 8, gq, t4);
            st16<0, !SP>(TA, acc, m0, n0, gq, t4);
            zero8(acc);  // TB = T^T Bt (T^T is zero left of its diagonal)
            gemm16<true, false, SP>(acc, TT, m0, m0, BT, m0, n0, (64 - m0) / 8, gq, t4);
            st16<0, !SP>(TB, acc, m0, n0, gq, t4);
        }
        __syncthreads();
        float* Mg = ws + lc.region + static_cast<long>(lc.c) * SQ;
        float* Qg = ws + lc.region + static_cast<long>(lc.nch + 1 + lc.c) * SQ;
        float* Qfg = ws + lc.region + static_cast<long>(2 * (lc.nch + 1) + lc.c) * SQ;
        {
            float acc[8], accw[8];
            // M = diag(Gamma_L) (I + Bt^T TA), and W = Rt + Mrb TA -> NAB (one after the other: run
            // together, as in the gradient kernel, they were slower here)
            zero8(acc);
            zero8(accw);
            gemm16<true, false, SP>(acc, BT, m0, 0, TA, 0, n0, 8, gq, t4);
            gemm16<false, false, SP>(accw, MRB, m0, 0, TA, 0, n0, (m0 + 16) / 8, gq, t4);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int row = m0 + frag_row(e, gq), col = n0 + frag_col(e, t4);
                const float mv = sm.GL[row] * (acc[e] + (row == col ? 1.f : 0.f));
                acc[e] = SP ? mv : round_tf32(mv);  // an operand of the scan (tf32 unless split)
            }
            st16_global(Mg, acc, m0, n0, gq, t4);
#pragma unroll
            for (int e = 0; e < 8; ++e) accw[e] += RT[sx(m0 + frag_row(e, gq), n0 + frag_col(e, t4))];
            st16<0, !SP>(NAB, accw, m0, n0, gq, t4);
            zero8(acc);  // Z = Kt + Nak^T TB -> TT
            gemm16<true, false, SP>(acc, NAK, m0, m0, TB, m0, n0, (64 - m0) / 8, gq, t4);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] += KT[sx(m0 + frag_row(e, gq), n0 + frag_col(e, t4))];
            st16<0, !SP>(TT, acc, m0, n0, gq, t4);
        }
        __syncthreads();
        prefetch_next();  // NAK, MRB, TA and TB are dead: the next item's raw rows go there
        {
            float acc[8], accf[8];
            // Q = dY^T W, and Qf = V^T Z diag(Gamma_L)
            zero8(acc);
            zero8(accf);
            gemm16<true, false, SP>(acc, DY, m0, 0, NAB, 0, n0, 8, gq, t4);
            gemm16<true, false, SP>(accf, VV, m0, 0, TT, 0, n0, 8, gq, t4);
            st16_global(Qg, acc, m0, n0, gq, t4);
#pragma unroll
            for (int e = 0; e < 8; ++e) accf[e] *= sm.GL[n0 + frag_col(e, t4)];
            st16_global(Qfg, accf, m0, n0, gq, t4);
        }
    }
    cp_async_wait<0>();  // nothing may still be landing when the block exits
}

// ---- 2. the scans over a unit's chunks: direction 0 runs S <- S M^T + Qf
// forward from s0 and writes S[c] before every chunk c and S[nch] at the end;
// direction 1 runs dS <- Q + dS M backward from dsT, writes dS_L[c] over the Q
// slot c after reading it, and ds0 at the end.  Warp w keeps rows 16 w ..
// 16 w + 15 of the state in registers, laid out as the accumulator of m16n8k8
// products; with the k order of gemm16 those registers are also the A
// fragments of the next product, so the state never leaves the registers.  M
// (tf32 from the map kernel) and the addend stream through a three-stage
// cp.async ring; the state enters the product as tf32 high and low parts
// (S = S_hi + S_lo, two products), which keeps the scan at fp32 accuracy over
// many chunks.
constexpr int SCAN_THR = 128;


// row-major 64 x 64 fp32 matrix (global) -> tile in the sx layout, by a block of NT threads
template <int NT>
__device__ __forceinline__ void tile_async(float* tile, const float* g) {
#pragma unroll
    for (int i = 0; i < 1024 / NT; ++i) {
        const int q = threadIdx.x + NT * i, row = q >> 4, col = (q & 15) << 2;
        cp_async16(tile + sx(row, col), g + row * 64 + col);
    }
}

constexpr int SCAN_STAGES = 3;
constexpr size_t SCAN_SMEM = sizeof(float) * 2 * SCAN_STAGES * TILE;

template <bool SP>
__global__ void __launch_bounds__(SCAN_THR)
    bwd_scan_kernel(const float* __restrict__ s0, const float* __restrict__ dsT, float* __restrict__ ds0,
                    float* __restrict__ ws, int B, int T, int H, const int32_t* __restrict__ offs, long ckpt_chunks,
                    int* status) {
    extern __shared__ __align__(128) float scan_smem[];  // M[stage] then addend[stage], sx layout
    __shared__ long sh_cbase;
    __shared__ int sh_nch, sh_ok;
    const int tid = threadIdx.x, unit = blockIdx.x, dir = blockIdx.y;
    const int n = unit / H, h = unit % H;
    if (tid == 0) {
        long cbase = 0;
        int nch = 0, ok = 1;
        if (!offs) {
            const long cps = (static_cast<long>(T) + L - 1) / L;
            cbase = static_cast<long>(n) * cps;
            nch = static_cast<int>(cps);
        } else {
            for (int m = 0; m <= n && ok; ++m) {
                const long o0 = offs[m], o1 = offs[m + 1];
                if (o0 < 0 || o1 < o0 || o1 > T) {
                    ok = 0;
                } else if (m < n) {
                    cbase += (o1 - o0 + L - 1) / L;
                } else {
                    nch = static_cast<int>((o1 - o0 + L - 1) / L);
                }
            }
            if (ok && cbase + nch > ckpt_chunks) ok = 0;
            if (!ok) report_status(status, WKV7_ERR_DEVICE_BOUNDS);
        }
        sh_cbase = cbase;
        sh_nch = nch;
        sh_ok = ok;
    }
    __syncthreads();
    if (!sh_ok) return;
    const int nch = sh_nch;
    float* Mb = ws + unit_region(sh_cbase, n, h, H, nch);
    float* Qb = Mb + static_cast<long>(nch + 1) * SQ;
    float* Qfb = Qb + static_cast<long>(nch + 1) * SQ;
    float* Sb = Qfb;  // S[c] goes over Qf[c], which the forward scan has read by then
    const float* addb = dir == 0 ? Qfb : Qb;
    const int w = tid >> 5, gq = (tid & 31) >> 2, t4 = tid & 3, r0 = 16 * w;
    const long sbase = static_cast<long>(unit) * SQ;
    // element e of n-tile j: row r0 + gq + 8 (e >> 1), column 8 j + 2 t4 + (e & 1)
    auto frow = [&](int e) { return r0 + gq + 8 * (e >> 1); };
    auto fcol = [&](int j) { return 8 * j + 2 * t4; };

    float st[8][4];
    {
        const float* init = dir == 0 ? s0 : dsT;
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
                const float2 x = init ? *reinterpret_cast<const float2*>(init + sbase + frow(e) * 64 + fcol(j))
                                      : make_float2(0.f, 0.f);
                st[j][e] = x.x;
                st[j][e + 1] = x.y;
            }
    }
    auto chunk_of = [&](int s) { return dir == 0 ? s : nch - 1 - s; };
    auto fetch = [&](int s) {  // M and addend of step s -> stage s % 3 (one commit group per step)
        if (s < nch) {
            const long c = chunk_of(s);
            float* stage = scan_smem + 2 * (s % SCAN_STAGES) * TILE;
            tile_async<SCAN_THR>(stage, Mb + c * SQ);
            tile_async<SCAN_THR>(stage + TILE, addb + c * SQ);
        }
        cp_async_commit();
    };
    fetch(0);
    fetch(1);
    for (int s = 0; s < nch; ++s) {
        const int c = chunk_of(s);
        fetch(s + 2);
        cp_async_wait<2>();
        __syncthreads();  // step s's tiles have landed for every thread
        const float* M = scan_smem + 2 * (s % SCAN_STAGES) * TILE;
        const float* A = M + TILE;
        // the state before chunk c: forward S[c]; backward dS_L[c] over the Q slot, whose copy has completed
        float* out = (dir == 0 ? Sb : Qb) + static_cast<long>(c) * SQ;
        float acc[8][4];
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
                *reinterpret_cast<float2*>(out + frow(e) * 64 + fcol(j)) = make_float2(st[j][e], st[j][e + 1]);
                const float2 x = *reinterpret_cast<const float2*>(A + sx(frow(e), fcol(j)));
                acc[j][e] = x.x;
                acc[j][e + 1] = x.y;
            }
#pragma unroll
        for (int kb = 0; kb < 8; ++kb) {
            uint32_t ahi[4], alo[4];
            const float av[4] = {st[kb][0], st[kb][2], st[kb][1], st[kb][3]};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float hi = round_tf32(av[i]);
                ahi[i] = __float_as_uint(hi);
                alo[i] = __float_as_uint(round_tf32(av[i] - hi));
            }
            uint32_t bf[8][2], bl[8][2];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float y0, y1;
                if (dir == 0) {  // B(k, n) = M[n][k]
                    const float2 y = *reinterpret_cast<const float2*>(M + sx(8 * j + gq, 8 * kb + 2 * t4));
                    y0 = y.x;
                    y1 = y.y;
                } else {         // B(k, n) = M[k][n]
                    y0 = M[sx(8 * kb + 2 * t4, 8 * j + gq)];
                    y1 = M[sx(8 * kb + 2 * t4 + 1, 8 * j + gq)];
                }
                if constexpr (SP) {  // an fp32 map: its high and low tf32 parts
                    split_tf32(__float_as_uint(y0), bf[j][0], bl[j][0]);
                    split_tf32(__float_as_uint(y1), bf[j][1], bl[j][1]);
                } else {             // the map is tf32 already
                    bf[j][0] = __float_as_uint(y0);
                    bf[j][1] = __float_as_uint(y1);
                }
            }
            // the high parts into all eight accumulators, then the low parts: eight
            // independent products between two that share an accumulator
#pragma unroll
            for (int j = 0; j < 8; ++j) mma_tf32(acc[j], ahi, bf[j]);
#pragma unroll
            for (int j = 0; j < 8; ++j) mma_tf32(acc[j], alo, bf[j]);
            if constexpr (SP) {
#pragma unroll
                for (int j = 0; j < 8; ++j) mma_tf32(acc[j], ahi, bl[j]);
            }
        }
        __syncthreads();  // every warp is done with this stage before step s + 3 refills it
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) st[j][e] = acc[j][e];
    }
    cp_async_wait<0>();
    float* fin = dir == 0 ? Sb + static_cast<long>(nch) * SQ : ds0 + sbase;
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; e += 2)
            *reinterpret_cast<float2*>(fin + frow(e) * 64 + fcol(j)) = make_float2(st[j][e], st[j][e + 1]);
}

// two consecutive outputs of a [tokens][H][D] tensor, in its storage type
__device__ __forceinline__ void st_pair(__nv_bfloat16* p, float x0, float x1) {
    *reinterpret_cast<uint32_t*>(p) = pack_bf16x2(x0, x1);
}
__device__ __forceinline__ void st_pair(float* p, float x0, float x1) {
    *reinterpret_cast<float2*>(p) = make_float2(x0, x1);
}

// ---- 3. every gradient of one chunk, from S0 = S[c], S_L = S[c + 1] and dS_L
template <typename IO, typename WT>
__global__ void __launch_bounds__(NTHR, 1)
    bwd_grad_kernel(const IO* __restrict__ r, const WT* __restrict__ wl, const IO* __restrict__ k,
                    const IO* __restrict__ v, const IO* __restrict__ a, const IO* __restrict__ b,
                    const IO* __restrict__ dy, IO* __restrict__ dr, WT* __restrict__ dwl, IO* __restrict__ dk,
                    IO* __restrict__ dv, IO* __restrict__ da, IO* __restrict__ db, const float* __restrict__ ws, int B,
                    int T, int H, const int32_t* __restrict__ offs, long ckpt_chunks, int* status) {
    constexpr bool SP = sizeof(IO) == 4;  // fp32 inputs: split products on full fp32 tiles, fp32 outputs
    extern __shared__ __align__(16) float smf[];
    const Smem sm = carve(smf);
    ChunkLoc lc;
    if (!locate_block_chunk(B, T, H, offs, ckpt_chunks, status, lc, sm.loc, sm.ok)) return;
    float *GAM = sm.tile[T_GAM], *AT = sm.tile[T_AT], *RT = sm.tile[T_RT], *BT = sm.tile[T_BT], *KT = sm.tile[T_KT];
    float *VV = sm.tile[T_VV], *DY = sm.tile[T_DY];
    float *W0 = sm.tile[T_X0], *W1 = sm.tile[T_X1], *W2 = sm.tile[T_X2], *W3 = sm.tile[T_X3];
    float *S0 = sm.tile[T_X4], *DS = sm.tile[T_X5];
    const int tid = threadIdx.x, w = tid >> 5, gq = (tid & 31) >> 2, t4 = tid & 3;
    const int m0 = 16 * (w >> 2), n0 = 16 * (w & 3);
    const long tstride = static_cast<long>(H) * D, hoff = static_cast<long>(blockIdx.y) * D;
    const int nv = lc.nv;
    {
        // S0 -> S0, dS_L -> DS, S_L -> W3 (free until the inverse), in flight during the staging
        const float* S0g = ws + lc.region + static_cast<long>(2 * (lc.nch + 1) + lc.c) * SQ;
        const float* dSg = ws + lc.region + static_cast<long>(lc.nch + 1 + lc.c) * SQ;
        tile_async<NTHR>(S0, S0g);
        tile_async<NTHR>(DS, dSg);
        tile_async<NTHR>(W3, S0g + SQ);
        cp_async_commit();
    }
    prefetch_ahead<IO, WT>(r, wl, k, v, a, b, dy, B, T, H, offs, 148);
    {
        const long o = lc.row0 * tstride + hoff;
        stage_chunk<IO, WT>(GAM, AT, RT, BT, KT, VV, DY, sm.GL, sm.seg, r + o, wl + o, k + o, v + o, a + o, b + o, dy + o,
                        tstride, nv);
    }
    cp_async_wait<0>();
    __syncthreads();
    {
        // S0 tf32-rounded and dSLg = dS_L diag(Gamma_L) in place; column sums of dS_L (.) S_L
        const int j = tid & 63, s = tid >> 6;
        const float gl = sm.GL[j];
        float cs = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int ix = sx(8 * s + i, j);
            const float d = DS[ix];
            cs = fmaf(d, W3[ix], cs);
            S0[ix] = SP ? S0[ix] : round_tf32(S0[ix]);
            DS[ix] = SP ? d * gl : round_tf32(d * gl);
        }
        sm.seg[s * 64 + j] = cs;
    }
    masks_abk<SP>(AT, RT, BT, KT, W0, W1, W2, m0, n0, gq, t4);  // W0 = Nab, W1 = Nak, W2 = Mrb
    __syncthreads();
    if (tid < 64) {
        float cs = 0.f;
#pragma unroll
        for (int s = 0; s < 8; ++s) cs += sm.seg[s * 64 + tid];
        sm.csum[tid] = cs;
    }
    invert_unit_lower<SP>(W0, W3);  // W3 = T
    float acc[8];
    // X = At S0^T + Nak V -> W0
    {
        float acc2[8];
        zero8(acc);
        zero8(acc2);
        gemm16_2<false, true, false, false, SP>(acc, AT, m0, 0, S0, 0, n0, 8, acc2, W1, m0, 0, VV, 0, n0,
                                                (m0 + 16) / 8, gq, t4);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += acc2[e];
    }
    st16<0, !SP>(W0, acc, m0, n0, gq, t4);
    __syncthreads();
    // U = T X -> W0
    zero8(acc);
    gemm16<false, false, SP>(acc, W3, m0, 0, W0, 0, n0, (m0 + 16) / 8, gq, t4);
    __syncthreads();
    st16<0, !SP>(W0, acc, m0, n0, gq, t4);
    // dU = Mrb^T dY + Bt dSLg^T -> W2
    {
        float acc2[8];
        zero8(acc);
        zero8(acc2);
        gemm16_2<true, false, false, true, SP>(acc, W2, m0, m0, DY, m0, n0, (64 - m0) / 8, acc2, BT, m0, 0, DS, 0, n0,
                                               8, gq, t4);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += acc2[e];
    }
    __syncthreads();
    st16<0, !SP>(W2, acc, m0, n0, gq, t4);
    __syncthreads();
    // dX = T^T dU -> W3
    zero8(acc);
    gemm16<true, false, SP>(acc, W3, m0, m0, W2, m0, n0, (64 - m0) / 8, gq, t4);
    __syncthreads();
    st16<0, !SP>(W3, acc, m0, n0, gq, t4);
    // Mrk = tril(Rt Kt^T) -> W2
    zero8(acc);
    if (n0 <= m0) gemm16<false, true, SP>(acc, RT, m0, 0, KT, 0, n0, 8, gq, t4);
    st16<2, !SP>(W2, acc, m0, n0, gq, t4);
    __syncthreads();
    // dV = Mrk^T dY + Kt dSLg^T + Nak^T dX
    {
        float acc2[8];
        zero8(acc);
        zero8(acc2);
        gemm16_2<false, true, true, false, SP>(acc, KT, m0, 0, DS, 0, n0, 8, acc2, W1, m0, m0, W3, m0, n0,
                                               (64 - m0) / 8, gq, t4);
        gemm16<true, false, SP>(acc2, W2, m0, m0, DY, m0, n0, (64 - m0) / 8, gq, t4);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += acc2[e];
    }
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
        const int row = m0 + frag_row(e, gq), col = n0 + frag_col(e, t4);
        if (row < nv) st_pair(dv + (lc.row0 + row) * tstride + hoff + col, acc[e], acc[e + 1]);
    }
    // the four accumulated gradients: dAt, dRt, dBt', dKt'
    float gA[8], gR[8], gB[8], gK[8];
    zero8(gA);
    zero8(gR);
    zero8(gB);
    zero8(gK);
    gemm16_2<false, false, false, false, SP>(gA, W3, m0, 0, S0, 0, n0, 8, gR, DY, m0, 0, S0, 0, n0, 8, gq,
                                             t4);  // dX S0, dY S0
    gemm16_2<false, false, false, false, SP>(gB, W0, m0, 0, DS, 0, n0, 8, gK, VV, m0, 0, DS, 0, n0, 8, gq,
                                             t4);  // U dSLg, V dSLg
    __syncthreads();
    // dNab = tril(dX U^T, -1) -> W1, dNak = tril(dX V^T, -1) -> W2
    {
        float acc2[8];
        zero8(acc);
        zero8(acc2);
        if (n0 <= m0)
            gemm16_2<false, true, false, true, SP>(acc, W3, m0, 0, W0, 0, n0, 8, acc2, W3, m0, 0, VV, 0, n0, 8, gq, t4);
        st16<1, !SP>(W1, acc, m0, n0, gq, t4);
        st16<1, !SP>(W2, acc2, m0, n0, gq, t4);
    }
    __syncthreads();
    {
        float tmp[8];  // dNak Kt, added to gA after the pair
        zero8(tmp);
        gemm16_2<false, false, false, false, SP>(gA, W1, m0, 0, BT, 0, n0, (m0 + 16) / 8, tmp, W2, m0, 0, KT, 0, n0,
                                                 (m0 + 16) / 8, gq, t4);
#pragma unroll
        for (int e = 0; e < 8; ++e) gA[e] += tmp[e];
    }
    // dNab^T At, dNak^T At
    gemm16_2<true, false, true, false, SP>(gB, W1, m0, m0, AT, m0, n0, (64 - m0) / 8, gK, W2, m0, m0, AT, m0, n0,
                                           (64 - m0) / 8, gq, t4);
    __syncthreads();
    // dMrb = tril(dY U^T) -> W1, dMrk = tril(dY V^T) -> W2
    {
        float acc2[8];
        zero8(acc);
        zero8(acc2);
        if (n0 <= m0)
            gemm16_2<false, true, false, true, SP>(acc, DY, m0, 0, W0, 0, n0, 8, acc2, DY, m0, 0, VV, 0, n0, 8, gq, t4);
        st16<2, !SP>(W1, acc, m0, n0, gq, t4);
        st16<2, !SP>(W2, acc2, m0, n0, gq, t4);
    }
    __syncthreads();
    {
        float tmp[8];  // dMrk Kt, added to gR after the pair
        zero8(tmp);
        gemm16_2<false, false, false, false, SP>(gR, W1, m0, 0, BT, 0, n0, (m0 + 16) / 8, tmp, W2, m0, 0, KT, 0, n0,
                                                 (m0 + 16) / 8, gq, t4);
#pragma unroll
        for (int e = 0; e < 8; ++e) gR[e] += tmp[e];
    }
    // dMrb^T Rt, dMrk^T Rt
    gemm16_2<true, false, true, false, SP>(gB, W1, m0, m0, RT, m0, n0, (64 - m0) / 8, gK, W2, m0, m0, RT, m0, n0,
                                           (64 - m0) / 8, gq, t4);
    __syncthreads();
    // d log w needs exp(w_log) of this thread's column j and tokens 8 s .. 8 s + 7 at the end:
    // load them now, behind the element-wise work
    const int jc = tid & 63, sc = tid >> 6;
    float el[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int t = 8 * sc + i;
        el[i] = t < nv ? to_f32(wl[(lc.row0 + t) * tstride + hoff + jc]) : 0.f;
    }
    // da, dr, db, dk -> bf16 rows in OB (the dead S0 and DS tiles: 4 x 64 rows of 128 bytes, 32-bit
    // words XOR-permuted by 4 (row mod 8)); the terms of d log w: W1 = da (.) a,
    // W2 = dr (.) r - db (.) b - dk (.) k
    uint32_t* OB = reinterpret_cast<uint32_t*>(S0);
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
        const int row = m0 + frag_row(e, gq), col = n0 + frag_col(e, t4);
        float o[4][2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int cc = col + u, ix = sx(row, cc);
            const float g = GAM[ix], gp = row > 0 ? GAM[sx(row - 1, cc)] : 1.f, ig = __frcp_rn(g);
            const float xa = gA[e + u], xr = gR[e + u], xb = gB[e + u], xk = gK[e + u];
            o[0][u] = xa * gp;
            o[1][u] = xr * g;
            o[2][u] = xb * ig;
            o[3][u] = xk * ig;
            W1[ix] = xa * AT[ix];
            W2[ix] = xr * RT[ix] - xb * BT[ix] - xk * KT[ix];
        }
        if constexpr (SP) {
            if (row < nv) {
                const long off = (lc.row0 + row) * tstride + hoff + col;
                st_pair(da + off, o[0][0], o[0][1]);
                st_pair(dr + off, o[1][0], o[1][1]);
                st_pair(db + off, o[2][0], o[2][1]);
                st_pair(dk + off, o[3][0], o[3][1]);
            }
        } else {
            const int word = (row << 5) + ((col >> 1) ^ ((row & 7) << 2));
#pragma unroll
            for (int q = 0; q < 4; ++q) OB[q * 2048 + word] = pack_bf16x2(o[q][0], o[q][1]);
        }
    }
    __syncthreads();
    if constexpr (!SP) {
        // coalesced copy-out: 4 tensors x 64 rows x 8 pieces of 16 bytes
        IO* const dst[4] = {da, dr, db, dk};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int q = tid + NTHR * i, tsr = q >> 9, row = (q >> 3) & 63, pc = q & 7;
            if (row < nv) {
                const uint4 x = *reinterpret_cast<const uint4*>(OB + tsr * 2048 + (row << 5) + ((4 * pc) ^ ((row & 7) << 2)));
                *reinterpret_cast<uint4*>(dst[tsr] + (lc.row0 + row) * tstride + hoff + 8 * pc) = x;
            }
        }
    }
    {
        // d log w_s = sum_{t >= s} g_t with g_t = W2[t] + W1[t + 1] (t < 63) and
        // g_63 = W2[63] + colsum(dS_L (.) S_L): thread (column j, tokens 8 s .. 8 s + 7)
        const int j = jc, s = sc;
        float x[8], run = 0.f;
#pragma unroll
        for (int i = 7; i >= 0; --i) {
            const int t = 8 * s + i;
            run += W2[sx(t, j)] + (t < 63 ? W1[sx(t + 1, j)] : sm.csum[j]);
            x[i] = run;
        }
        sm.seg[s * 64 + j] = run;
        __syncthreads();
        float later = 0.f;
        for (int q = s + 1; q < 8; ++q) later += sm.seg[q * 64 + j];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int t = 8 * s + i;
            if (t < nv) {
                const long off = (lc.row0 + t) * tstride + hoff + j;
                dwl[off] = from_f32<WT>(-(x[i] + later) * exp_l(el[i]));
            }
        }
    }
}

template <typename IO, typename WT>
cudaError_t launch_chunked_typed(const BackwardArgs& p, cudaStream_t stream) {
    constexpr bool SP = sizeof(IO) == 4;
    static std::atomic<unsigned long long> cfg_map{0}, cfg_grad{0}, cfg_scan{0};
    auto map = bwd_map_kernel<IO, WT>;
    auto grad = bwd_grad_kernel<IO, WT>;
    auto scan = bwd_scan_kernel<SP>;
    cudaError_t e = configure_smem_once(map, static_cast<int>(SMEM_BYTES), cfg_map);
    if (e != cudaSuccess) return e;
    e = configure_smem_once(grad, static_cast<int>(SMEM_BYTES), cfg_grad);
    if (e != cudaSuccess) return e;
    e = configure_smem_once(scan, static_cast<int>(SCAN_SMEM), cfg_scan);
    if (e != cudaSuccess) return e;
    const IO *r = static_cast<const IO*>(p.r), *k = static_cast<const IO*>(p.k), *v = static_cast<const IO*>(p.v);
    const IO *a = static_cast<const IO*>(p.a), *b = static_cast<const IO*>(p.b), *dy = static_cast<const IO*>(p.dy);
    const WT* wl = static_cast<const WT*>(p.w_log);
    const dim3 cgrid(static_cast<unsigned>(p.ckpt_chunks), static_cast<unsigned>(p.H));
    if (p.ckpt_chunks > 0) {
        int dev = 0, sms = 0;
        e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        const long items = p.ckpt_chunks * p.H;
        const unsigned mgrid = static_cast<unsigned>(items < sms ? items : sms);
        map<<<mgrid, NTHR, SMEM_BYTES, stream>>>(r, wl, k, v, a, b, dy, p.ws, p.B, p.T, p.H, p.seq_offsets,
                                                 p.ckpt_chunks, p.status);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    scan<<<dim3(static_cast<unsigned>(p.B) * p.H, 2), SCAN_THR, SCAN_SMEM, stream>>>(
        p.s0, p.dsT, p.ds0, p.ws, p.B, p.T, p.H, p.seq_offsets, p.ckpt_chunks, p.status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (p.ckpt_chunks > 0) {
        grad<<<cgrid, NTHR, SMEM_BYTES, stream>>>(r, wl, k, v, a, b, dy, static_cast<IO*>(p.dr),
                                                  static_cast<WT*>(p.dw_log), static_cast<IO*>(p.dk),
                                                  static_cast<IO*>(p.dv), static_cast<IO*>(p.da), static_cast<IO*>(p.db),
                                                  p.ws, p.B, p.T, p.H, p.seq_offsets, p.ckpt_chunks, p.status);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace

long backward_ckpt_chunks(int B, int T, int packed) {
    const long per = (static_cast<long>(T) + L - 1) / L;
    return packed ? per + B : static_cast<long>(B) * per;
}

// three 64 x 64 fp32 states per chunk and one more per sequence (see unit_region)
size_t backward_workspace_floats(int B, int T, int H, int packed) {
    return static_cast<size_t>(3) * H * (backward_ckpt_chunks(B, T, packed) + B) * SQ;
}

cudaError_t launch_backward(const BackwardArgs& p, int io_dtype, int w_dtype, cudaStream_t stream) {
    using bf = __nv_bfloat16;
    if (io_dtype == WKV7_F32)
        return w_dtype == WKV7_BF16 ? launch_chunked_typed<float, bf>(p, stream) : launch_chunked_typed<float, float>(p, stream);
    return w_dtype == WKV7_BF16 ? launch_chunked_typed<bf, bf>(p, stream) : launch_chunked_typed<bf, float>(p, stream);
}

}  // namespace wkv7
