// wkv7_prefill_pipe.cu — warp-specialised chunked WKV-7 prefill for bf16 inputs.
//
// Same chunk algebra as wkv7_prefill.cu (derived from the generalized delta
// rule of "RWKV-7 Goose: Expressive Dynamic State Evolution", section
// "Generalized Delta rule", with the argument roles of the hxa07D WKV call):
// per 64-token chunk with start state S0 and Gamma_t = prod_{s<=t} w_s,
//   Y     = (Rt + Mrb W) S0^T + (Mrk + Mrb Z) V
//   S_L^T = Gamma_L (.) S0^T  + (Bh^T W) S0^T + (Kh^T + Bh^T Z) V
// with [W | Z] = T [At | Mak] and T = (I - Nab)^{-1}.  T is formed explicitly
// in fp32 (16 x 16 diagonal blocks by substitution on the CUDA cores, the
// blocks below them by warp-level tf32 tensor-core products) and folded into
// tcgen05 products:
//   G   = [Rt; At] [Bt; Kt]^T                        (Mrb | Mrk over Nab | Mak)
//   Q   = [Mrb; Bh^T] T
//   P   = Q [At | Mak]                               (Mrb W | Mrb Z over Bh^T W | Bh^T Z)
//   OUT = [Mrb Z; Bh^T Z] V + [Mrk; Kh^T] V + [Rt + Mrb W; Bh^T W] S0^T
//                                                    (Y over S_L^T - Gamma_L (.) S0^T)
// Only the last product depends on the state.
//
// Block of 384 threads, one (sequence, head) unit:
//   warps 0-3  prep group 0: chunks 0, 2, 4, ...   (everything up to OUT without S0)
//   warps 4-7  prep group 1: chunks 1, 3, 5, ...
//   warps 8-11 serial group: for every chunk in order, the S0-dependent product,
//              the y rows and the fp32 state update (state held in registers
//              of the threads owning TMEM lanes 64..127, one key channel each).
// The two prep groups overlap each other's latencies and run ahead of the
// serial group; each owns its shared-memory tiles and TMEM columns, except the
// [R'; Bh^T W] tile that the serial group reads, which is shared.
// Synchronisation: a prep group hands a chunk to the serial group through
// `ready[g]` (MMA commit + release arrive).  The serial group releases the
// shared tile through `asfree[g]` as soon as its product has read it, and the
// group's OUT columns through `freeg[g]` once it has read them; both have one
// barrier per prep group, whose phases are that group's chunks.  A waiter has
// always waited for the phase before the one it waits for (during the group's
// previous chunk), so no parity wait can be two phases behind (it would then
// return on the wrong phase).
// Inputs arrive by TMA into tiles of the group that are dead at that point of
// the previous chunk: w_log of chunk c + 2 into BK once T is built, r and k into
// NQ once P has consumed Q, a and b into RAM once the conversion has read Rt; V
// goes straight into the group's MN-major V tile once the previous OUT product
// has read it.  Waits are polled by one thread while the others sleep on the
// group's named barrier; every wait is bounded.
#include <cstring>

#include "prefill_common.cuh"
#include "sm100_ptx.cuh"
#include "tma_host.cuh"
#include "wkv7_internal.cuh"

namespace wkv7 {
namespace {

constexpr int L = 64;
constexpr int NTHR = 384;
constexpr uint32_t GROUP = 128;
constexpr uint64_t WAIT_NS = 1000000000ull;  // 1 s

// per prep-group shared-memory tiles (bytes)
constexpr uint32_t OFF_RAM = 0;        // Rt (rows 0-63) | At (rows 64-127) | Mak (64 tokens x 64), 24 KB
constexpr uint32_t OFF_BK = 24576;     // raw w_log (16 KB), then T fp32 (64 x 64, tf_idx layout)
constexpr uint32_t OFF_BH = 40960;     // [Mrb; Bh^T] 16 KB, then [Mrb Z; Bh^T Z]
constexpr uint32_t OFF_MK = 57344;     // [Mrk; Kh^T] 16 KB, K-major over tokens
constexpr uint32_t OFF_NQ = 73728;     // raw r, k -> [Bt; Kt] 16 KB, then Nab fp32, then T bf16 (first 8 KB), then Q bf16
constexpr uint32_t OFF_V = 90112;      // V 8 KB (MN-major)
constexpr uint32_t GROUP_TILES = 98304;
constexpr uint32_t OFF_AS = 2 * GROUP_TILES;          // [R'; Bh^T W] 16 KB, shared by both groups
constexpr uint32_t OFF_S = OFF_AS + 16384;            // S^T bf16, 8 KB (serial group)
constexpr uint32_t OFF_GAMMA = OFF_S + 8192;          // Gamma_L [2 groups][2 slots][64] fp32
constexpr uint32_t OFF_RED = OFF_GAMMA + 2 * 2 * 64 * 4;  // block products [2 groups][4][64] fp32
constexpr uint32_t OFF_U = OFF_RED + 2 * 4 * 64 * 4;    // gated read-out: u [2 groups][2 slots][64] fp32
constexpr uint32_t OFF_BAR = OFF_U + 2 * 2 * 64 * 4;
constexpr uint32_t SMEM_USED = OFF_BAR + 22 * 8 + 16;
// raw TMA staging inside a group's tiles (dead at the time of the load)
constexpr uint32_t RAW_R = OFF_NQ, RAW_K = OFF_NQ + 8192, RAW_A = OFF_RAM, RAW_B = OFF_RAM + 8192, RAW_L = OFF_BK;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;      // alignment slack

// TMEM columns
constexpr uint32_t TM_GP = 0;    // + 256 g: G, then P (128 columns)
constexpr uint32_t TM_Q = 128;   // + 256 g: Q (64 columns)
constexpr uint32_t TM_OUT = 192; // + 256 g: OUT (64 columns)
constexpr uint32_t TMEM_COLS = 512;

constexpr uint32_t ID_G16 = idesc_f32acc(1, 128, 128, 0, 0);  // K-major A and B, N = 128
constexpr uint32_t ID_KM128 = idesc_f32acc(1, 128, 128, 0, 1); // B MN-major, N = 128
constexpr uint32_t ID_KM64 = idesc_f32acc(1, 128, 64, 0, 1);   // B MN-major, N = 64

// fp32 64 x 64 matrix with its 4-column groups XOR-permuted by row (bank spread)
__device__ __forceinline__ uint32_t tf_idx(uint32_t row, uint32_t col) {
    return row * 64u + (col ^ ((row & 7u) << 2));
}

// Warp-level tf32 tensor-core product on fp32 matrices held in the tf_idx layout.
// m16n8k8 fragments: lane = 4 gq + t4; A (16 x 8) holds rows gq, gq + 8 and
// columns t4, t4 + 4; B (8 x 8) rows t4, t4 + 4 and column gq; C (16 x 8) rows
// gq, gq + 8 and columns 2 t4, 2 t4 + 1.  Stored values are already tf32.
__device__ __forceinline__ void frag_a_tf32(const float* M, int r0, int c0, int gq, int t4, uint32_t (&a)[4]) {
    a[0] = __float_as_uint(M[tf_idx(r0 + gq, c0 + t4)]);
    a[1] = __float_as_uint(M[tf_idx(r0 + gq + 8, c0 + t4)]);
    a[2] = __float_as_uint(M[tf_idx(r0 + gq, c0 + t4 + 4)]);
    a[3] = __float_as_uint(M[tf_idx(r0 + gq + 8, c0 + t4 + 4)]);
}
__device__ __forceinline__ void frag_b_tf32(const float* M, int k0, int n0, int gq, int t4, uint32_t (&b)[2]) {
    b[0] = __float_as_uint(M[tf_idx(k0 + t4, n0 + gq)]);
    b[1] = __float_as_uint(M[tf_idx(k0 + t4 + 4, n0 + gq)]);
}
__device__ __forceinline__ void frag_c_store_tf32(float* M, int r0, int n0, int gq, int t4, const float (&d)[4]) {
    *reinterpret_cast<float2*>(M + tf_idx(r0 + gq, n0 + 2 * t4)) = make_float2(round_tf32(d[0]), round_tf32(d[1]));
    *reinterpret_cast<float2*>(M + tf_idx(r0 + gq + 8, n0 + 2 * t4)) = make_float2(round_tf32(d[2]), round_tf32(d[3]));
}
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// C[cr + 0..15][cc + 0..15] = sum over k-steps ks in [ks0, ks1) (0 <= ks0 < ks1 <= 4) of
//   A[ar + 0..15][ac + 8 ks + 0..7] * B[bk + 8 ks + 0..7][bn + 0..15]   (one warp)
// written to C (tf32, tf_idx layout) and/or to Cb (bf16, 128-byte swizzled rows); either may be null.
// All fragments are loaded before the first product, so the loads of the k-steps overlap.
__device__ __forceinline__ void tf32_tile16(const float* A, int ar, int ac, const float* B, int bk, int bn, int ks0,
                                            int ks1, float* C, uint8_t* Cb, int cr, int cc, int gq, int t4) {
    float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
    uint32_t af[4][4], b0[4][2], b1[4][2];
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
        if (ks >= ks0 && ks < ks1) {
            frag_a_tf32(A, ar, ac + 8 * ks, gq, t4, af[ks]);
            frag_b_tf32(B, bk + 8 * ks, bn, gq, t4, b0[ks]);
            frag_b_tf32(B, bk + 8 * ks, bn + 8, gq, t4, b1[ks]);
        }
    }
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
        if (ks >= ks0 && ks < ks1) {
            mma_tf32_16x8x8(d0, af[ks], b0[ks]);
            mma_tf32_16x8x8(d1, af[ks], b1[ks]);
        }
    }
    if (C) {
        frag_c_store_tf32(C, cr, cc, gq, t4, d0);
        frag_c_store_tf32(C, cr, cc + 8, gq, t4, d1);
    }
    if (Cb) {
        *reinterpret_cast<uint32_t*>(Cb + swz(cr + gq, 2 * (cc + 2 * t4), 64)) = pack_bf16x2(d0[0], d0[1]);
        *reinterpret_cast<uint32_t*>(Cb + swz(cr + gq + 8, 2 * (cc + 2 * t4), 64)) = pack_bf16x2(d0[2], d0[3]);
        *reinterpret_cast<uint32_t*>(Cb + swz(cr + gq, 2 * (cc + 8 + 2 * t4), 64)) = pack_bf16x2(d1[0], d1[1]);
        *reinterpret_cast<uint32_t*>(Cb + swz(cr + gq + 8, 2 * (cc + 8 + 2 * t4), 64)) = pack_bf16x2(d1[2], d1[3]);
    }
}

__device__ __forceinline__ float2 unpack_bf16x2(uint32_t u) { return make_float2(bf16lo_to_f32(u), bf16hi_to_f32(u)); }

// w_log of key channels j, j + 1 (element index i of the raw tile) as floats
__device__ __forceinline__ float2 ld_wlog2(const float* p, int i) { return *reinterpret_cast<const float2*>(p + i); }
__device__ __forceinline__ float2 ld_wlog2(const __nv_bfloat16* p, int i) {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(p + i);
    return make_float2(bf16lo_to_f32(u), bf16hi_to_f32(u));
}
// w = exp(-exp(w_log)) = 2^(-log2(e) 2^(log2(e) w_log)) for two key channels
__device__ __forceinline__ float2 decay2(float2 lv) {
    constexpr float kLog2e = 1.4426950408889634f;
    return make_float2(ex2_ftz(-kLog2e * ex2_ftz(kLog2e * lv.x)), ex2_ftz(-kLog2e * ex2_ftz(kLog2e * lv.y)));
}
__device__ __forceinline__ uint32_t pack2(float2 v) { return pack_bf16x2(v.x, v.y); }

template <typename WT>
__device__ __forceinline__ WT neg_inf_of();
template <>
__device__ __forceinline__ float neg_inf_of<float>() { return -INFINITY; }
template <>
__device__ __forceinline__ __nv_bfloat16 neg_inf_of<__nv_bfloat16>() { return __ushort_as_bfloat16(0xFF80u); }

struct Bars {
    uint64_t* mma;    // [2] prep-group MMA completions (G, Q, P)
    uint64_t* ready;  // [2] OUT-pre complete and chunk tiles published (count 2)
    uint64_t* freeg;  // [2] serial group done with a chunk of prep group g (shared tile, OUT columns)
    uint64_t* ser;    // serial MMA completion
    uint64_t* asfree; // [2] the serial product of a chunk of prep group g has read the shared tile
    uint64_t* rl;     // [2] TMA of a group's raw w_log tile
    uint64_t* rrk;    // [2] TMA of a group's raw r, k tiles
    uint64_t* rab;    // [2] TMA of a group's raw a, b tiles
    uint64_t* vld;    // [2] TMA of a group's V tile
    uint64_t* p1done; // [2] SERIAL_P1: the serial group has done pass 1 of a chunk of prep group g (from 2 on)
    uint64_t* rls;    // [2] SERIAL_P1: TMA of a group's raw w_log tile for its chunks from 2 on
    uint32_t* tmem_slot;
};

// Sum over a warp of 8 per-token partial sums (lane jp holds its share of
// tokens 0..7): a reduce-scatter over lane bits 4, 3, 2 leaves token
// (jp >> 2) & 7 in lanes 4m .. 4m + 3, and two more steps complete the sum, so
// lane 4m returns the total of token m.  9 shuffles for 8 tokens.
__device__ __forceinline__ float sum8_scatter(const float (&pd)[8], int jp) {
    const bool b4 = (jp & 16) != 0, b3 = (jp & 8) != 0, b2 = (jp & 4) != 0;
    float q4[4], q2[2];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        q4[i] = (b4 ? pd[4 + i] : pd[i]) + __shfl_xor_sync(0xffffffffu, b4 ? pd[i] : pd[4 + i], 16);
#pragma unroll
    for (int i = 0; i < 2; ++i)
        q2[i] = (b3 ? q4[2 + i] : q4[i]) + __shfl_xor_sync(0xffffffffu, b3 ? q4[i] : q4[2 + i], 8);
    float q1 = (b2 ? q2[1] : q2[0]) + __shfl_xor_sync(0xffffffffu, b2 ? q2[0] : q2[1], 4);
    q1 += __shfl_xor_sync(0xffffffffu, q1, 2);
    q1 += __shfl_xor_sync(0xffffffffu, q1, 1);
    return q1;
}

// Pass 1 of a chunk: the product of w over each thread's 16 tokens, per key channel
// (thread (jp, tq) of a 128-thread group: key channels 2 jp, 2 jp + 1, tokens
// 16 tq .. 16 tq + 15), into red[tq][j]; with fp32 w_log the running products
// overwrite the thread's own w_log elements.
template <typename WT>
__device__ __forceinline__ void decay_pass(WT* rawl, float* red, int tq, int j0) {
    float2 pw = make_float2(1.f, 1.f);
#pragma unroll 4
    for (int e = 0; e < 16; ++e) {
        const int i = (16 * tq + e) * 64 + j0;
        pw = __fmul2_rn(pw, decay2(ld_wlog2(rawl, i)));
        if constexpr (sizeof(WT) == 4) *reinterpret_cast<float2*>(rawl + i) = pw;
    }
    red[tq * 64 + j0] = pw.x;
    red[tq * 64 + j0 + 1] = pw.y;
}

// GATED: the output rows are z = (y / sqrt(D) + u v) (.) g with u = sum_d r k rk
// (the read-out of wkv7_forward_gated) instead of y.
// PRO: the prologue of the WKV call is applied to the raw inputs in the
// element-wise stage (wkv7_forward_fused): k and v are rows of kv head
// h / (H / H_kv), the `a` tile carries a_lr, and per token
//   kk = k / max(||k||, 1e-12),  a = -kk,  b = kk a_lr,  k <- k (1 - w + a_lr);
// `b` is not read.
// map_flags (wkv7_state_map; 0 otherwise): kMapZeroV treats v as zero (no V tile is
// loaded), kMapIdentity starts from the identity state (s0 ignored).  y == nullptr
// writes no y rows.
constexpr int kMapZeroV = 1, kMapIdentity = 2;
// EXPORT (first phase of wkv7_forward_long, dense batches): no chunk depends on
// another, so the grid is persistent: block i takes chunks i, i + gridDim.x, ...
// of the list of every (sequence n, chunk j, head h) in the order
// slot = (n * chunks per sequence + j) * H + h, through one continuous pipeline,
// and the serial group, instead of the state pass, writes each chunk's
// state-independent results to its workspace slot: the [R'; Bh^T W] tile as it
// is in shared memory (ex_as, 16 KB), the OUT product so far (ex_out, 128 rows x
// 64 fp32 in 16 column quads, quad-major: element (row, col) at
// ((col / 4) * 128 + row) * 4 + col % 4) and Gamma_L (ex_gam, 64 fp32).

template <typename WT, bool GATED, bool PRO, bool EXPORT = false>
__global__ void __launch_bounds__(NTHR, 1)
    wkv7_prefill_pipe_kernel(const __nv_bfloat16* __restrict__ r, const WT* __restrict__ wl,
                             const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                             const __nv_bfloat16* __restrict__ a, const __nv_bfloat16* __restrict__ b,
                             const float* s0, __nv_bfloat16* __restrict__ y, float* sT, int T, int H,
                             const int32_t* __restrict__ seq_offsets, int* status,
                             const float* __restrict__ rk, const __nv_bfloat16* __restrict__ gte, int H_kv,
                             int map_flags, int B, uint8_t* __restrict__ ex_as,
                             float* __restrict__ ex_out, float* __restrict__ ex_gam,
                             const __grid_constant__ TmaMaps maps) {
    // With the fused prologue (the longest pass 2) the serial group also runs pass 1 of each prep
    // group's chunks from the second on, off the prep chains (fused + gated 107 -> 100 us on
    // B4 T1024 H32 with 8 kv heads); for the other variants the extra work on the serial warps
    // cost more than it saved (plain +0.7 %, gated +3 %, packed +1.5 %), so they keep it.
    constexpr bool SERIAL_P1 = PRO;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base, derived from the shared array so that every tile pointer
    // stays in the shared address space (32-bit addressing)
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    Bars bars;
    {
        uint64_t* p = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
        bars.mma = p;
        bars.ready = p + 2;
        bars.ser = p + 4;
        bars.asfree = p + 16;
        bars.rl = p + 6;
        bars.rrk = p + 8;
        bars.rab = p + 10;
        bars.vld = p + 12;
        bars.freeg = p + 14;
        bars.p1done = p + 18;
        bars.rls = p + 20;
        bars.tmem_slot = reinterpret_cast<uint32_t*>(p + 22);
    }

    // ---- the unit and its tokens
    const int unit = blockIdx.x;
    const int h = unit % H;
    int n = unit / H;
    // A packed batch of at most NTHR sequences is taken longest first: blocks are
    // started roughly in index order, so the long sequences (the longest chains)
    // start early and the short ones fill in behind them.  Block n' runs the
    // sequence of length rank n' (ties by index); the ranks are a permutation even
    // for offsets that the bounds check below rejects.
    if (seq_offsets && static_cast<int>(gridDim.x) / H <= NTHR) {
        const int nseq = static_cast<int>(gridDim.x) / H;
        long* lens = reinterpret_cast<long*>(sm + OFF_AS);  // scratch, before the tile is used
        int* pick = reinterpret_cast<int*>(sm + OFF_AS + 8 * NTHR);
        if (tid < nseq) lens[tid] = static_cast<long>(seq_offsets[tid + 1]) - seq_offsets[tid];
        __syncthreads();
        if (tid < nseq) {
            const long li = lens[tid];
            int rank = 0;
            for (int j = 0; j < nseq; ++j) rank += (lens[j] > li || (lens[j] == li && j < tid)) ? 1 : 0;
            if (rank == n) *pick = tid;
        }
        __syncthreads();
        n = *pick;
        __syncthreads();  // every thread has its sequence before the scratch is reused
    }
    long tb = 0, len = 0;
    if (seq_offsets) {
        const long o0 = seq_offsets[n], o1 = seq_offsets[n + 1];
        if (o0 < 0 || o1 < o0 || o1 > T) {
            if (tid == 0) report_status(status, WKV7_ERR_DEVICE_BOUNDS);
            return;
        }
        tb = o0;
        len = o1 - o0;
    } else {
        tb = static_cast<long>(n) * T;
        len = T;
    }
    const long tstride = static_cast<long>(H) * kHead;
    const long hoff = static_cast<long>(h) * kHead;
    const long sbase = (static_cast<long>(n) * H + h) * kHead * kHead;
    int nchunks = static_cast<int>((len + L - 1) / L);
    // EXPORT: this block's c-th chunk is slot blockIdx.x + c * gridDim.x
    const long nch_seq = (static_cast<long>(T) + L - 1) / L;
    if constexpr (EXPORT) {
        const long total = static_cast<long>(B) * nch_seq * H;
        nchunks = static_cast<int>((total - blockIdx.x + gridDim.x - 1) / gridDim.x);
    }
    auto slot_of = [&](int c) { return static_cast<long>(blockIdx.x) + static_cast<long>(c) * gridDim.x; };
    // EXPORT: slot = (n * nch_seq + j) * H + h, in 32-bit arithmetic (the host keeps every slot
    // below 2^31)
    const uint32_t H32 = static_cast<uint32_t>(H), nch32 = static_cast<uint32_t>(nch_seq);
    auto slot_q = [&](int c) -> uint32_t { return static_cast<uint32_t>(slot_of(c)) / H32; };
    // kv head of k and v (the fused prologue shares them over H / H_kv heads); fixed per
    // block except in EXPORT mode, which has no prologue
    const int hk_unit = PRO ? h / (H / H_kv) : h;
    // valid rows of this block's c-th chunk
    auto chunk_nv = [&](int c) -> int {
        long rem;
        if constexpr (EXPORT) rem = T - static_cast<long>(slot_q(c) % nch32) * L;
        else rem = len - static_cast<long>(c) * L;
        return static_cast<int>(rem < L ? rem : L);
    };
    // EXPORT: (sequence n, chunk j, head h) of a prep group's chunk.  A group's consecutive
    // slots are 2 x gridDim.x apart; that step is split into heads, chunks and sequences once,
    // so each next position follows by additions with carries (no division per chunk)
    struct Pos {
        uint32_t n, j, h;
    };
    auto pos_of = [&](int c) -> Pos {
        if constexpr (EXPORT) {
            const uint32_t sl = static_cast<uint32_t>(slot_of(c)), q = sl / H32;
            return Pos{q / nch32, q % nch32, sl - q * H32};
        } else {
            return Pos{0u, 0u, 0u};
        }
    };
    const uint32_t step_q = EXPORT ? 2u * gridDim.x / H32 : 0u;
    const uint32_t step_h = EXPORT ? 2u * gridDim.x - step_q * H32 : 0u;
    const uint32_t step_j = EXPORT ? step_q % nch32 : 0u, step_n = EXPORT ? step_q / nch32 : 0u;
    auto advance2 = [&](Pos p) -> Pos {
        if constexpr (EXPORT) {
            p.h += step_h;
            uint32_t cy = p.h >= H32 ? 1u : 0u;
            p.h -= cy * H32;
            p.j += step_j + cy;  // < 2 nch32
            cy = p.j >= nch32 ? 1u : 0u;
            p.j -= cy * nch32;
            p.n += step_n + cy;
        }
        return p;
    };
    auto pos_t0 = [&](int c, const Pos& p) -> long {
        if constexpr (EXPORT) return static_cast<long>(p.n) * T + static_cast<long>(p.j) * L;
        else return tb + static_cast<long>(c) * L;
    };
    auto pos_h = [&](const Pos& p) -> int {
        if constexpr (EXPORT) return static_cast<int>(p.h);
        else return h;
    };
    auto pos_hk = [&](const Pos& p) -> int {
        if constexpr (EXPORT) return static_cast<int>(p.h);
        else return hk_unit;
    };
    auto pos_nv = [&](int c, const Pos& p) -> int {
        long rem;
        if constexpr (EXPORT) rem = T - static_cast<long>(p.j) * L;
        else rem = len - static_cast<long>(c) * L;
        return static_cast<int>(rem < L ? rem : L);
    };

    if (tid == 0) {
        for (int g = 0; g < 2; ++g) {
            mbar_init(&bars.mma[g], 1);
            mbar_init(&bars.ready[g], 2);
            mbar_init(&bars.rl[g], 1);
            mbar_init(&bars.rrk[g], 1);
            mbar_init(&bars.rab[g], 1);
            mbar_init(&bars.vld[g], 1);
            mbar_init(&bars.freeg[g], 1);
            mbar_init(&bars.p1done[g], 1);
            mbar_init(&bars.rls[g], 1);
        }
        mbar_init(bars.ser, 1);
        mbar_init(&bars.asfree[0], 1);
        mbar_init(&bars.asfree[1], 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(bars.tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *bars.tmem_slot;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    bool ok = true;
    // SERIAL_P1: pass 1 of chunk cn (>= 2) by the serial group (thread ts, named barrier 3)
    // for prep group cn & 1, run while that group finishes chunk cn - 2 (whose inverse has
    // released the tile the w_log of chunk cn lands in, on rls: the serial group is its only
    // waiter, one phase per chunk in order); the group waits on p1done instead of running
    // the pass on its own chain.
    auto serial_pass1 = [&](int cn, int ts) -> bool {
        const int gn = cn & 1;
        WT* rl_n = reinterpret_cast<WT*>(sm + gn * GROUP_TILES + RAW_L);
        float* red_n = reinterpret_cast<float*>(sm + OFF_RED) + gn * 256;
        if (!group_sync_and(3, GROUP,
                            ts == 0 ? mbar_wait(&bars.rls[gn], static_cast<uint32_t>((cn >> 1) - 1) & 1u, WAIT_NS)
                                    : true))
            return false;
        const int nvn = chunk_nv(cn);
        if (nvn < L) {  // tokens past the end of the sequence are identity steps (w = 1)
            for (int i = nvn * 64 + ts; i < L * 64; i += static_cast<int>(GROUP)) rl_n[i] = neg_inf_of<WT>();
            group_sync(3, GROUP);
        }
        decay_pass<WT>(rl_n, red_n, ts >> 5, 2 * (ts & 31));
        group_sync(3, GROUP);
        if (ts == 0) mbar_arrive(&bars.p1done[gn]);
        return true;
    };

    if (warp < 8) {
        // =========================================================== prep groups
        const int g = warp >> 2;
        const int tg = tid & 127;
        const uint32_t bar_id = 1 + g;
        uint8_t* gt = sm + g * GROUP_TILES;
        uint8_t* RAM = gt + OFF_RAM;
        uint8_t* BH = gt + OFF_BH;
        uint8_t* MK = gt + OFF_MK;
        float* Tf = reinterpret_cast<float*>(gt + OFF_BK);
        float* Nr = reinterpret_cast<float*>(gt + OFF_NQ);
        uint8_t* Tb = gt + OFF_NQ;  // bf16 T, over the rows of Nab no longer read
        uint8_t* Qt = gt + OFF_NQ;
        uint8_t* AS = sm + OFF_AS;
        uint8_t* Vt = gt + OFF_V;
        float* gam = reinterpret_cast<float*>(sm + OFF_GAMMA) + g * 128;
        float* red = reinterpret_cast<float*>(sm + OFF_RED) + g * 256;
        const uint32_t tm_gp = tmem + 256u * g + TM_GP;
        const uint32_t tm_q = tmem + 256u * g + TM_Q;
        const uint32_t tm_out = tmem + 256u * g + TM_OUT;
        uint32_t mma_phase = 0;
        bool mma_pending = false;
        int issued_out = 0;  // OUT-pre commits issued by this group
        int raw_issued = 0, raw_done = 0, v_issued = 0, v_done = 0;  // TMA loads (chunks) of this group
        constexpr uint32_t WB = sizeof(WT);
        // one thread each; `which`: 0 = w_log, 1 = r and k, 2 = a and b
        auto issue_raw = [&](int cc, const Pos& pc, int which) {
            const int t0 = static_cast<int>(pos_t0(cc, pc));
            const int h = pos_h(pc), hk = pos_hk(pc);
            if (which == 0) {
                // the first chunk's tile completes on rl (the group waits); later ones on rls,
                // whose only waiter is the serial group, in chunk order
                uint64_t* bl = (SERIAL_P1 && cc >= 2) ? &bars.rls[g] : &bars.rl[g];
                mbar_arrive_expect_tx(bl, 4096u * WB);
                tma_load_3d(gt + RAW_L, &maps.wl, bl, 0, h, t0);
            } else if (which == 1) {
                mbar_arrive_expect_tx(&bars.rrk[g], 2u * 8192u);
                tma_load_3d(gt + RAW_R, &maps.r, &bars.rrk[g], 0, h, t0);
                tma_load_3d(gt + RAW_K, &maps.k, &bars.rrk[g], 0, hk, t0);
            } else if constexpr (PRO) {
                mbar_arrive_expect_tx(&bars.rab[g], 8192u);
                tma_load_3d(gt + RAW_A, &maps.a, &bars.rab[g], 0, h, t0);
            } else {
                mbar_arrive_expect_tx(&bars.rab[g], 2u * 8192u);
                tma_load_3d(gt + RAW_A, &maps.a, &bars.rab[g], 0, h, t0);
                tma_load_3d(gt + RAW_B, &maps.b, &bars.rab[g], 0, h, t0);
            }
        };
        auto issue_v = [&](int cc, const Pos& pc) {  // one thread
            mbar_arrive_expect_tx(&bars.vld[g], 8192u);
            tma_load_3d(Vt, &maps.v, &bars.vld[g], 0, pos_hk(pc), static_cast<int>(pos_t0(cc, pc)));
        };
        Pos pcur = pos_of(g);          // this group's chunk c
        Pos pnext = advance2(pcur);    // and its chunk c + 2
        const bool zero_v = (map_flags & kMapZeroV) != 0;
        if (zero_v) {
            // v = 0: the V tile is cleared once and never loaded
            for (int i = tg; i < 512; i += static_cast<int>(GROUP))
                reinterpret_cast<uint4*>(Vt)[i] = make_uint4(0u, 0u, 0u, 0u);
            fence_proxy_async_smem();
        }
        if (g < nchunks) {
            if (tg == 0) {
                issue_raw(g, pcur, 0);
                issue_raw(g, pcur, 1);
                issue_raw(g, pcur, 2);
                if (!zero_v) issue_v(g, pcur);
            }
            raw_issued = 1;
            v_issued = zero_v ? 0 : 1;
        }

        // matrix descriptors of K-step 0; K-step s adds 2 s (K-major) or 128 s (MN-major)
        const uint64_t dRAM = kmajor_desc<false>(RAM, 128, 0), dBKt = kmajor_desc<false>(gt + OFF_NQ, 128, 0);
        const uint64_t dBH = kmajor_desc<false>(BH, 128, 0), dMK = kmajor_desc<false>(MK, 128, 0);
        const uint64_t dQt = kmajor_desc<false>(Qt, 128, 0);
        const uint64_t dTb = mnmajor_desc<false>(Tb, 64, 0), dAZ = mnmajor_desc<false>(RAM + 8192, 64, 0);
        const uint64_t dV = mnmajor_desc<false>(Vt, 64, 0);
        // p1 work split: thread (jp, tq) owns key channels 2jp, 2jp+1 of tokens 16tq .. 16tq+15
        const int jp = tg & 31, tq = tg >> 5, j0 = 2 * jp;
        float2 rkv = make_float2(0.f, 0.f);  // rk of key channels j0, j0 + 1 (gated read-out)
        if constexpr (GATED) rkv = make_float2(rk[h * kHead + j0], rk[h * kHead + j0 + 1]);
        const WT* rawl = reinterpret_cast<const WT*>(gt + RAW_L);
        WT* rawl_w = reinterpret_cast<WT*>(gt + RAW_L);
        uint8_t* BKt = gt + OFF_NQ;  // [Bt; Kt], written over the raw r, k rows
        const uint32_t* rawr = reinterpret_cast<const uint32_t*>(gt + RAW_R);
        const uint32_t* rawk = reinterpret_cast<const uint32_t*>(gt + RAW_K);
        const uint32_t* rawa = reinterpret_cast<const uint32_t*>(gt + RAW_A);
        const uint32_t* rawb = reinterpret_cast<const uint32_t*>(gt + RAW_B);

        for (int c = g; c < nchunks; c += 2) {
            const int kk_ = c >> 1;
            const int nv = pos_nv(c, pcur);

            // ---- p1: decay products and the scaled operand tiles
            const bool ragged = nv < L;  // group-uniform
            if (!SERIAL_P1 || kk_ == 0) {
                // pass 1 here (with SERIAL_P1 only for the group's first chunk)
                ok = group_sync_and(bar_id, GROUP,
                                    (tg == 0) ? mbar_wait(&bars.rl[g], static_cast<uint32_t>(kk_) & 1u, WAIT_NS)
                                              : true);
                if (!ok) break;
                if (ragged) {
                    // tokens past the end of the sequence are identity steps: w_log = -inf (w = 1)
                    for (int i = nv * 64 + tg; i < L * 64; i += static_cast<int>(GROUP)) rawl_w[i] = neg_inf_of<WT>();
                    group_sync(bar_id, GROUP);
                }
                decay_pass<WT>(rawl_w, red, tq, j0);
            } else {
                ok = group_sync_and(bar_id, GROUP,
                                    (tg == 0) ? mbar_wait(&bars.p1done[g], static_cast<uint32_t>(kk_ - 1) & 1u, WAIT_NS)
                                              : true);
                if (!ok) break;
            }
            {
                // pass 2 rewrites BH and MK and V is reloaded: the previous OUT product of this
                // group (chunk c-2) must have read them
                bool w_ok = true;
                if (tg == 0) {
                    if (kk_ >= 1) {
                        w_ok = mbar_wait(&bars.ready[g], static_cast<uint32_t>(kk_ - 1) & 1u, WAIT_NS);
                        if (w_ok && !zero_v) issue_v(c, pcur);
                    }
                    w_ok = w_ok && mbar_wait(&bars.rrk[g], static_cast<uint32_t>(kk_) & 1u, WAIT_NS) &&
                           mbar_wait(&bars.rab[g], static_cast<uint32_t>(kk_) & 1u, WAIT_NS);
                }
                if (kk_ >= 1 && !zero_v) ++v_issued;
                ok = group_sync_and(bar_id, GROUP, w_ok);
                if (!ok) break;
                ++raw_done;
            }
            if (ragged) {
                // ... and r = k = a = b = 0
                const int nrow = L - nv;
                for (int i = tg; i < 4 * nrow * 8; i += static_cast<int>(GROUP)) {
                    const int tile = i / (nrow * 8), rem = i - tile * nrow * 8;
                    const uint32_t off = tile == 0 ? RAW_R : tile == 1 ? RAW_K : tile == 2 ? RAW_A : RAW_B;
                    *reinterpret_cast<uint4*>(gt + off + (nv + (rem >> 3)) * 128 + (rem & 7) * 16) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
                group_sync(bar_id, GROUP);
            }
            float pre0 = 1.f, pre1 = 1.f, GL0 = 1.f, GL1 = 1.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float x0 = red[q * 64 + j0], x1 = red[q * 64 + j0 + 1];
                if (q < tq) { pre0 *= x0; pre1 *= x1; }
                GL0 *= x0;
                GL1 *= x1;
            }
            if (tq == 3) {
                gam[(kk_ & 1) * 64 + j0] = GL0;
                gam[(kk_ & 1) * 64 + j0 + 1] = GL1;
            }
            // pass 2, eight tokens at a time: Gamma_t (from the stored running products, or
            // from w again for bf16 w_log), then
            //   Rt = r Gamma_t, At = a Gamma_{t-1}, Bt = b / Gamma_t, Kt = k / Gamma_t  (token rows)
            //   Bh^T, Kh^T = (b, k) Gamma_L / Gamma_t                                    (key rows)
            // Rt and At overwrite the raw a, b rows of the same tokens in RAM, Bt and Kt the raw r, k
            // rows in NQ; each warp owns its 16 token rows and reads them before writing.
            {
                const float2 pre = make_float2(pre0, pre1), GL = make_float2(GL0, GL1);
                float2 gp = pre;  // Gamma_{t-1}
                const uint32_t cb = static_cast<uint32_t>(j0) * 2u;
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    const int t0 = 16 * tq + 8 * half;
                    uint32_t rr[8], kv[8], av[8], bv[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int idx = (t0 + e) * 32 + jp;  // 32-bit word of (t, j0)
                        rr[e] = rawr[idx];
                        kv[e] = rawk[idx];
                        av[e] = rawa[idx];
                        if constexpr (!PRO) bv[e] = rawb[idx];
                    }
                    __syncwarp();
                    float rn[8];  // prologue: 1 / max(||k_t||, 1e-12) of the 8 tokens, in every lane
                    if constexpr (PRO) {
                        float ss[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float2 kf = unpack_bf16x2(kv[e]);
                            ss[e] = kf.x * kf.x + kf.y * kf.y;
                        }
                        const float inv = 1.f / fmaxf(sqrtf(sum8_scatter(ss, jp)), 1e-12f);
#pragma unroll
                        for (int e = 0; e < 8; ++e) rn[e] = __shfl_sync(0xffffffffu, inv, 4 * e);
                    }
                    uint32_t bh0[4], bh1[4], kh0[4], kh1[4];  // 8 tokens of Bh^T / Kh^T rows j0, j0 + 1
                    float pd[8];                              // this thread's part of u for 8 tokens
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int t = t0 + e;
                        float2 G, wv;  // Gamma_t and (prologue) w_t
                        if constexpr (sizeof(WT) == 4) {
                            G = __fmul2_rn(pre, *reinterpret_cast<const float2*>(rawl + t * 64 + j0));
                            if constexpr (PRO) wv = make_float2(__fdividef(G.x, gp.x), __fdividef(G.y, gp.y));
                        } else {
                            wv = decay2(ld_wlog2(rawl, t * 64 + j0));
                            G = __fmul2_rn(gp, wv);
                        }
                        const float2 iv = make_float2(rcp_ftz(G.x), rcp_ftz(G.y));
                        const float2 l = __fmul2_rn(iv, GL);
                        const float2 rf = unpack_bf16x2(rr[e]);
                        float2 kf = unpack_bf16x2(kv[e]), af, bf;
                        if constexpr (PRO) {
                            const float2 alr = unpack_bf16x2(av[e]);
                            const float2 kn = make_float2(kf.x * rn[e], kf.y * rn[e]);  // kk
                            af = make_float2(-kn.x, -kn.y);
                            bf = __fmul2_rn(kn, alr);
                            kf = __fmul2_rn(kf, make_float2(1.f - wv.x + alr.x, 1.f - wv.y + alr.y));
                        } else {
                            af = unpack_bf16x2(av[e]);
                            bf = unpack_bf16x2(bv[e]);
                        }
                        if constexpr (GATED) pd[e] = rf.x * kf.x * rkv.x + rf.y * kf.y * rkv.y;
                        *reinterpret_cast<uint32_t*>(RAM + swz(t, cb, 128)) = pack2(__fmul2_rn(rf, G));
                        *reinterpret_cast<uint32_t*>(RAM + swz(64 + t, cb, 128)) = pack2(__fmul2_rn(af, gp));
                        *reinterpret_cast<uint32_t*>(BKt + swz(t, cb, 128)) = pack2(__fmul2_rn(bf, iv));
                        *reinterpret_cast<uint32_t*>(BKt + swz(64 + t, cb, 128)) = pack2(__fmul2_rn(kf, iv));
                        const float2 bhv = __fmul2_rn(bf, l), khv = __fmul2_rn(kf, l);
                        if ((e & 1) == 0) {
                            bh0[e >> 1] = __float_as_uint(bhv.x);
                            bh1[e >> 1] = __float_as_uint(bhv.y);
                            kh0[e >> 1] = __float_as_uint(khv.x);
                            kh1[e >> 1] = __float_as_uint(khv.y);
                        } else {
                            bh0[e >> 1] = pack_bf16x2(__uint_as_float(bh0[e >> 1]), bhv.x);
                            bh1[e >> 1] = pack_bf16x2(__uint_as_float(bh1[e >> 1]), bhv.y);
                            kh0[e >> 1] = pack_bf16x2(__uint_as_float(kh0[e >> 1]), khv.x);
                            kh1[e >> 1] = pack_bf16x2(__uint_as_float(kh1[e >> 1]), khv.y);
                        }
                        gp = G;
                    }
                    if constexpr (GATED) {
                        // u of the 8 tokens: the warp's 32 lanes cover the 64 key channels
                        const float q1 = sum8_scatter(pd, jp);
                        if ((jp & 3) == 0)
                            reinterpret_cast<float*>(sm + OFF_U)[g * 128 + (kk_ & 1) * 64 + t0 + ((jp >> 2) & 7)] = q1;
                    }
                    const uint32_t tb8 = static_cast<uint32_t>(t0) * 2u;  // byte of the first token
                    *reinterpret_cast<uint4*>(BH + swz(64 + j0, tb8, 128)) = make_uint4(bh0[0], bh0[1], bh0[2], bh0[3]);
                    *reinterpret_cast<uint4*>(BH + swz(64 + j0 + 1, tb8, 128)) = make_uint4(bh1[0], bh1[1], bh1[2], bh1[3]);
                    *reinterpret_cast<uint4*>(MK + swz(64 + j0, tb8, 128)) = make_uint4(kh0[0], kh0[1], kh0[2], kh0[3]);
                    *reinterpret_cast<uint4*>(MK + swz(64 + j0 + 1, tb8, 128)) = make_uint4(kh1[0], kh1[1], kh1[2], kh1[3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            group_sync(bar_id, GROUP);

            // ---- G = [Rt; At] [Bt; Kt]^T
            if (tg == 0) {
                tc_fence_after();
#pragma unroll
                for (uint32_t s = 0; s < 4; ++s)
                    mma_ss<false>(tm_gp, dRAM + 2 * s, dBKt + 2 * s, ID_G16, s > 0);
                mma_commit(&bars.mma[g]);
            }
            mma_pending = true;
            ok = group_sync_and(bar_id, GROUP, tg == 0 ? mbar_wait(&bars.mma[g], mma_phase, WAIT_NS) : true);
            if (!ok) break;
            mma_pending = false;
            mma_phase ^= 1u;
            tc_fence_after();

            // ---- masks.  Lanes 0..63 hold token rows of G: Mrb -> BH rows 0..63 and Mrk -> MK
            //      rows 0..63 (columns up to the diagonal).  Lanes 64..127 hold At rows: Nab ->
            //      fp32 row-major Nr and Mak -> the MN-major tile next to At (strictly lower).
            {
                const bool tok = tg < 64;
                const int t = tok ? tg : tg - 64;
                // gated read-out: u_t v_t joins y_t through the diagonal of Mrk, as 8 u_t (the
                // serial group scales the row by 1 / sqrt(D) = 1 / 8)
                float du = 0.f;
                if constexpr (GATED)
                    if (tok) du = 8.f * reinterpret_cast<const float*>(sm + OFF_U)[g * 128 + (kk_ & 1) * 64 + t];
#pragma unroll 1
                for (int qq = 0; qq < 4; ++qq) {
                    float x[32];
                    tmem_load32(tm_gp + lane_base + 32 * qq, x);
                    const int c0 = 32 * (qq & 1);
                    const int lim = t - c0 - (tok ? 0 : 1);  // columns c0 + i with i <= lim are kept
                    const float dd = qq >= 2 ? du : 0.f;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        if (i > lim) x[i] = 0.f;
                        if constexpr (GATED)
                            if (i == lim) x[i] += dd;
                    }
                    if (!tok && qq < 2) {
#pragma unroll
                        for (int i = 0; i < 32; i += 4)
                            *reinterpret_cast<float4*>(Nr + tf_idx(t, c0 + i)) = make_float4(
                                round_tf32(x[i]), round_tf32(x[i + 1]), round_tf32(x[i + 2]), round_tf32(x[i + 3]));
                    } else {
                        st_op_row32<false>(tok ? (qq < 2 ? BH : MK) : RAM + 16384, 128, t, c0, x);
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            group_sync(bar_id, GROUP);

            // ---- T = (I - Nab)^{-1} in fp32 (tf32-rounded), built in 16 x 16 blocks:
            //  (1) the diagonal blocks D_b = (I - Nab_bb)^{-1}: warp b, lane c (mod 16) computes
            //      column c by forward substitution over the rows of Nab;
            //  (2) T_{b+1,b} = D_{b+1} (Nab_{b+1,b} D_b) for b = 0, 2 (the inner product by warp b
            //      straight after its own block);
            //  (3) T_hl = T_hi (Nab_hl T_lo) for the 32 x 32 halves.
            //  Steps (2) and (3) are warp-level tf32 tensor-core products (m16n8k8); their
            //  intermediate products live in the upper-right 32 x 32 quadrant of Tf, which is zero
            //  in T.  T goes to the bf16 MN-major tile Tb as its blocks are final (Tb covers the
            //  first 8 KB of NQ, whose rows of Nab are no longer read from step (2) on).
            {
                const int w = tg >> 5, lane = tg & 31, gq = lane >> 2, t4 = lane & 3;
                {
                    const int c = lane & 15, r0 = 16 * w;
                    float x[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float p = (i == c) ? 1.f : 0.f;
#pragma unroll
                        for (int q = 0; q < i; q += 4) {
                            const float4 n4 = *reinterpret_cast<const float4*>(Nr + tf_idx(r0 + i, r0 + q));
                            p = fmaf(n4.x, x[q], p);
                            if (q + 1 < i) p = fmaf(n4.y, x[q + 1], p);
                            if (q + 2 < i) p = fmaf(n4.z, x[q + 2], p);
                            if (q + 3 < i) p = fmaf(n4.w, x[q + 3], p);
                        }
                        x[i] = p;
                    }
                    if (lane < 16) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) Tf[tf_idx(r0 + i, r0 + c)] = round_tf32(x[i]);
                    }
                }
                if ((w & 1) == 0) {
                    // Y_w = Nab_{w+1,w} D_w -> scratch rows 8w .. 8w+15, columns 32 .. 47
                    __syncwarp();
                    tf32_tile16(Nr, 16 * (w + 1), 16 * w, Tf, 16 * w, 16 * w, 0, 2, Tf, nullptr, 8 * w, 32, gq, t4);
                }
                group_sync(bar_id, GROUP);
                if (w & 1) {
                    // T_{w,w-1} = D_w Y_{w-1} -> Tf and Tb
                    tf32_tile16(Tf, 16 * w, 16 * w, Tf, 8 * (w - 1), 32, 0, 2, Tf, Tb, 16 * w, 16 * (w - 1), gq, t4);
                } else {
                    const int i0 = (w >> 1) * 32 + lane;  // 0 .. 63 over warps 0 and 2
                    // diagonal blocks -> Tb (64 rows x two 8-column chunks)
#pragma unroll
                    for (int m = 0; m < 2; ++m) {
                        const int q = i0 + 64 * m;
                        const int row = q >> 1, ch = 2 * (row >> 4) + (q & 1);
                        const float4 f0 = *reinterpret_cast<const float4*>(Tf + tf_idx(row, 8 * ch));
                        const float4 f1 = *reinterpret_cast<const float4*>(Tf + tf_idx(row, 8 * ch + 4));
                        *reinterpret_cast<uint4*>(Tb + swz(row, ch * 16, 64)) =
                            make_uint4(pack_bf16x2(f0.x, f0.y), pack_bf16x2(f0.z, f0.w), pack_bf16x2(f1.x, f1.y),
                                       pack_bf16x2(f1.z, f1.w));
                    }
                    // blocks above the diagonal are zero: rows 0-15 chunks 2-7, rows 16-31 chunks
                    // 4-7, rows 32-47 chunks 6-7 (192 chunks)
#pragma unroll
                    for (int m = 0; m < 3; ++m) {
                        const int q = i0 + 64 * m;
                        int row, ch;
                        if (q < 96) {
                            row = q / 6;
                            ch = 2 + q % 6;
                        } else if (q < 160) {
                            row = 16 + ((q - 96) >> 2);
                            ch = 4 + ((q - 96) & 3);
                        } else {
                            row = 32 + ((q - 160) >> 1);
                            ch = 6 + ((q - 160) & 1);
                        }
                        *reinterpret_cast<uint4*>(Tb + swz(row, ch * 16, 64)) = make_uint4(0u, 0u, 0u, 0u);
                    }
                }
                group_sync(bar_id, GROUP);
                const int mt = w >> 1, np = w & 1;
                // X = Nab_hl T_lo -> scratch rows 0 .. 31, columns 32 .. 63 (T_lo is zero in rows
                // 0 .. 15 of columns 16 .. 31, so those columns start at k = 16)
                tf32_tile16(Nr, 32 + 16 * mt, 0, Tf, 0, 16 * np, np ? 2 : 0, 4, Tf, nullptr, 16 * mt, 32 + 16 * np, gq, t4);
                group_sync(bar_id, GROUP);
                // T_hl = T_hi X -> Tb (rows 32 .. 47 of T_hi are zero beyond column 47)
                tf32_tile16(Tf, 32 + 16 * mt, 32, Tf, 0, 32 + 16 * np, 0, mt ? 4 : 2, nullptr, Tb, 32 + 16 * mt, 16 * np,
                            gq, t4);
            }
            fence_proxy_async_smem();
            group_sync(bar_id, GROUP);
            // BK (the fp32 T) is dead: load the w_log tile of this group's next chunk
            if (c + 2 < nchunks) {
                if (tg == 0) issue_raw(c + 2, pnext, 0);
                ++raw_issued;  // counted at the first of the chunk's three raw loads
            }

            // ---- Q = [Mrb; Bh^T] T
            if (tg == 0) {
                tc_fence_after();
#pragma unroll
                for (uint32_t s = 0; s < 4; ++s)
                    mma_ss<false>(tm_q, dBH + 2 * s, dTb + 128 * s, ID_KM64, s > 0);
                mma_commit(&bars.mma[g]);
            }
            mma_pending = true;
            ok = group_sync_and(bar_id, GROUP, tg == 0 ? mbar_wait(&bars.mma[g], mma_phase, WAIT_NS) : true);
            if (!ok) break;
            mma_pending = false;
            mma_phase ^= 1u;
            tc_fence_after();
            {
                float x[32];
#pragma unroll
                for (int qq = 0; qq < 2; ++qq) {
                    tmem_load32(tm_q + lane_base + 32 * qq, x);
                    st_op_row32<false>(Qt, 128, tg, 32 * qq, x);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            group_sync(bar_id, GROUP);

            // ---- P = Q [At | Mak]
            if (tg == 0) {
                tc_fence_after();
#pragma unroll
                for (uint32_t s = 0; s < 4; ++s)
                    mma_ss<false>(tm_gp, dQt + 2 * s, dAZ + 128 * s, ID_KM128, s > 0);
                mma_commit(&bars.mma[g]);
            }
            // the shared [R'; Bh^T W] tile is free once the serial product of chunk c-1 has read it
            mma_pending = true;
            {
                bool w1 = true;
                if (tg == 0) {
                    w1 = mbar_wait(&bars.mma[g], mma_phase, WAIT_NS);
                    // chunk c - 1 belongs to the other group; it is that group's ((c - 1) >> 1)-th
                    if (c >= 1)
                        w1 = w1 && mbar_wait(&bars.asfree[(c - 1) & 1], static_cast<uint32_t>((c - 1) >> 1) & 1u, WAIT_NS);
                }
                ok = group_sync_and(bar_id, GROUP, w1);
            }
            if (!ok) break;
            mma_pending = false;
            mma_phase ^= 1u;
            tc_fence_after();
            // NQ (Q) has been consumed by P: load r and k of this group's next chunk
            if (c + 2 < nchunks && tg == 0) issue_raw(c + 2, pnext, 1);
            {
                // P columns 0..63 -> AS (token rows get Rt added: R' = Rt + Mrb W; key rows Bh^T W),
                // columns 64..127 -> BH ([Mrb Z; Bh^T Z])
                const int row = tg;
#pragma unroll 1
                for (int q = 0; q < 4; ++q) {
                    float x[32];
                    tmem_load32(tm_gp + lane_base + 32 * q, x);
                    const int c0 = 32 * (q & 1);
                    if (q < 2 && tg < 64) {
                        float rt[32];
                        ld_op_row32<false>(RAM, 128, row, c0, rt);
#pragma unroll
                        for (int i = 0; i < 32; ++i) x[i] += rt[i];
                    }
                    st_op_row32<false>(q < 2 ? AS : BH, 128, row, c0, x);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            group_sync(bar_id, GROUP);

            // RAM (Rt, At, Mak) is dead: load a and b of this group's next chunk
            if (c + 2 < nchunks && tg == 0) issue_raw(c + 2, pnext, 2);
            // ---- OUT = [Mrb Z; Bh^T Z] V + [Mrk; Kh^T] V   (the serial group adds [R'; Bh^T W] S0^T)
            {
                // ... and the serial group must have read this group's OUT columns of its previous chunk
                bool vok = (tg == 0 && !zero_v) ? mbar_wait(&bars.vld[g], static_cast<uint32_t>(kk_) & 1u, WAIT_NS) : true;
                if (tg == 0 && kk_ >= 1)
                    vok = vok && mbar_wait(&bars.freeg[g], static_cast<uint32_t>(kk_ - 1) & 1u, WAIT_NS);
                ok = group_sync_and(bar_id, GROUP, vok);
                if (!ok) break;
                if (!zero_v) ++v_done;
            }
            if (tg == 0) {
                tc_fence_after();
#pragma unroll
                for (uint32_t s = 0; s < 4; ++s)
                    mma_ss<false>(tm_out, dBH + 2 * s, dV + 128 * s, ID_KM64, s > 0);
#pragma unroll
                for (uint32_t s = 0; s < 4; ++s)
                    mma_ss<false>(tm_out, dMK + 2 * s, dV + 128 * s, ID_KM64, 1);
                mma_commit(&bars.ready[g]);
                mbar_arrive(&bars.ready[g]);  // this chunk's [R'; Bh^T W] and Gamma_L are published
            }
            ++issued_out;
            pcur = pnext;
            pnext = advance2(pnext);
        }
        if (!ok && tg == 0) report_status(status, WKV7_ERR_DEVICE_TIMEOUT);
        // drain: an unwaited G/Q/P product, and the last OUT-pre product
        if (tg == 0) {
            if (mma_pending) mbar_wait(&bars.mma[g], mma_phase, WAIT_NS);
            if (issued_out > 0) mbar_wait(&bars.ready[g], static_cast<uint32_t>(issued_out - 1) & 1u, WAIT_NS);
            // a chunk's raw loads are issued in three batches; wait for every one that may be in flight
            for (int i = raw_done; i < raw_issued; ++i) {
                if (!SERIAL_P1 || i == 0) mbar_wait(&bars.rl[g], static_cast<uint32_t>(i) & 1u, WAIT_NS);
                else mbar_wait(&bars.rls[g], static_cast<uint32_t>(i - 1) & 1u, WAIT_NS);
                mbar_wait(&bars.rrk[g], static_cast<uint32_t>(i) & 1u, WAIT_NS);
                mbar_wait(&bars.rab[g], static_cast<uint32_t>(i) & 1u, WAIT_NS);
            }
            for (int i = v_done; i < v_issued; ++i) mbar_wait(&bars.vld[g], static_cast<uint32_t>(i) & 1u, WAIT_NS);
        }
    } else if constexpr (EXPORT) {
        // =========================================================== export group
        const int ts = tid - 256;
        const uint32_t bar_id = 3;
        const float* gam_all = reinterpret_cast<const float*>(sm + OFF_GAMMA);
        for (int c = 0; c < nchunks; ++c) {
            const int g = c & 1, kk_ = c >> 1;
            const uint32_t tm_out = tmem + 256u * g + TM_OUT;
            if (SERIAL_P1 && c + 2 < nchunks && !(ok = serial_pass1(c + 2, ts))) break;  // as in the serial group
            ok = group_sync_and(bar_id, GROUP,
                                ts == 0 ? mbar_wait(&bars.ready[g], static_cast<uint32_t>(kk_) & 1u, WAIT_NS) : true);
            if (!ok) break;
            tc_fence_after();
            const long slot = slot_of(c);
            if (ts == 0) {
                // the shared tile as it is, by one bulk copy (the prep group fenced it for the
                // async proxy before publishing the chunk)
                bulk_store(ex_as + slot * 16384, sm + OFF_AS, 16384u);
                bulk_commit();
            }
            if (ts < 64) ex_gam[slot * 64 + ts] = gam_all[g * 128 + (kk_ & 1) * 64 + ts];
            if (ts == 0) {
                // the other group's next conversion waits for the shared tile: release it
                // before the OUT columns are read
                bulk_wait_read<0>();                        // the copy has read the shared tile
                mbar_arrive(&bars.asfree[g]);
            }
            float* orow = ex_out + slot * 8192 + ts * 4;
#pragma unroll 1
            for (int q = 0; q < 2; ++q) {
                float o[32];
                tmem_load32(tm_out + lane_base + 32 * q, o);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    *reinterpret_cast<float4*>(orow + (8 * q + i) * 512) =
                        make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
            }
            tc_fence_before();
            group_sync(bar_id, GROUP);
            if (ts == 0) mbar_arrive(&bars.freeg[g]);
        }
        if (ts == 0) bulk_wait_all();  // every tile copy has landed before the block exits
        if (!ok && ts == 0) report_status(status, WKV7_ERR_DEVICE_TIMEOUT);
    } else {
        // =========================================================== serial group
        const int ts = tid - 256;
        const uint32_t bar_id = 3;
        uint8_t* St = sm + OFF_S;
        const float* gam_all = reinterpret_cast<const float*>(sm + OFF_GAMMA);
        const uint64_t dAS = kmajor_desc<false>(sm + OFF_AS, 128, 0), dSt = mnmajor_desc<false>(St, 64, 0);
        float S[64];
        const int x = ts - 64;  // key channel owned by lanes 64..127
        if (ts >= 64) {
#pragma unroll
            for (int i = 0; i < 64; ++i)
                S[i] = (map_flags & kMapIdentity) ? (i == x ? 1.f : 0.f) : (s0 ? s0[sbase + i * kHead + x] : 0.f);
            st_op_row32<false>(St, 64, x, 0, S);
            st_op_row32<false>(St, 64, x, 32, S + 32);
        }
        fence_proxy_async_smem();
        group_sync(bar_id, GROUP);
        uint32_t ser_phase = 0;
        bool ser_pending = false;
        for (int c = 0; c < nchunks; ++c) {
            const int g = c & 1, kk_ = c >> 1;
            const long row0 = tb + static_cast<long>(c) * L;
            const int nv = chunk_nv(c);
            const uint32_t tm_out = tmem + 256u * g + TM_OUT;
            // gated read-out: this token row of g (128 B) is brought into L2 before waiting
            // for the chunk, and read where it is used
            long goff = 0;
            if constexpr (GATED) {
                goff = (row0 + ts) * tstride + hoff;
                if (ts < nv) prefetch_line_l2(gte + goff);
            }
            // while group g finishes chunk c: pass 1 of its chunk c + 2 (its w_log tile lands
            // once that group's inverse of chunk c is done)
            if (SERIAL_P1 && c + 2 < nchunks && !(ok = serial_pass1(c + 2, ts))) break;
            ok = group_sync_and(bar_id, GROUP,
                                ts == 0 ? mbar_wait(&bars.ready[g], static_cast<uint32_t>(kk_) & 1u, WAIT_NS) : true);
            if (!ok) break;
            tc_fence_after();
            if (ts == 0) {
#pragma unroll
                for (uint32_t s = 0; s < 4; ++s)
                    mma_ss<false>(tm_out, dAS + 2 * s, dSt + 128 * s, ID_KM64, 1);
                mma_commit(bars.ser);
            }
            ser_pending = true;
            ok = group_sync_and(bar_id, GROUP, ts == 0 ? mbar_wait(bars.ser, ser_phase, WAIT_NS) : true);
            if (!ok) break;
            if (ts == 0) mbar_arrive(&bars.asfree[g]);  // the shared tile is free for the next chunk's conversion
            ser_pending = false;
            ser_phase ^= 1u;
            tc_fence_after();
            float o[32];
            if (ts < 64) {
                const int t = ts;
#pragma unroll(GATED ? 2 : 1)
                for (int q = 0; q < 2; ++q) {
                    tmem_load32(tm_out + lane_base + 32 * q, o);
                    if (t < nv && y != nullptr) {
                        const long off = (row0 + t) * tstride + hoff + 32 * q;
                        if constexpr (GATED) {
                            // z = (y + 8 u v) / 8 (.) g: the row already holds y + 8 u v (the
                            // diagonal of Mrk), so only g of this token row is read
#pragma unroll
                            for (int i = 0; i < 32; i += 8) {
                                const uint4 gq4 = *reinterpret_cast<const uint4*>(gte + goff + 32 * q + i);
                                const uint32_t gw[4] = {gq4.x, gq4.y, gq4.z, gq4.w};
#pragma unroll
                                for (int m = 0; m < 4; ++m) {
                                    const float2 gf = unpack_bf16x2(gw[m]);
                                    o[i + 2 * m] = o[i + 2 * m] * 0.125f * gf.x;
                                    o[i + 2 * m + 1] = o[i + 2 * m + 1] * 0.125f * gf.y;
                                }
                            }
                        }
                        __nv_bfloat16* dst = y + off;
#pragma unroll
                        for (int i = 0; i < 32; i += 8)
                            *reinterpret_cast<uint4*>(dst + i) =
                                make_uint4(pack_bf16x2(o[i], o[i + 1]), pack_bf16x2(o[i + 2], o[i + 3]),
                                           pack_bf16x2(o[i + 4], o[i + 5]), pack_bf16x2(o[i + 6], o[i + 7]));
                    }
                }
            } else {
                const float GL = gam_all[g * 128 + (kk_ & 1) * 64 + x];
                // 1 / Gamma_t must stay far inside the fp32 / bf16 range (false for NaN too)
                if (!(GL >= kMinGammaL)) report_status(status, WKV7_ERR_DECAY_RANGE);
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    tmem_load32(tm_out + lane_base + 32 * q, o);
#pragma unroll
                    for (int i = 0; i < 32; ++i) S[32 * q + i] = fmaf(GL, S[32 * q + i], o[i]);
                }
                st_op_row32<false>(St, 64, x, 0, S);
                st_op_row32<false>(St, 64, x, 32, S + 32);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            group_sync(bar_id, GROUP);
            if (ts == 0) mbar_arrive(&bars.freeg[g]);
        }
        if (!ok) {
            if (ts == 0) report_status(status, WKV7_ERR_DEVICE_TIMEOUT);
            if (ser_pending && ts == 0) mbar_wait(bars.ser, ser_phase, WAIT_NS);
        } else if (sT && ts >= 64) {
#pragma unroll
            for (int i = 0; i < 64; ++i) sT[sbase + i * kHead + x] = S[i];
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

template <typename WT, bool GATED, bool PRO, bool EXPORT = false>
cudaError_t launch_pipe_typed(const PrefillArgs& p, cudaStream_t stream) {
    auto kern = wkv7_prefill_pipe_kernel<WT, GATED, PRO, EXPORT>;
    static std::atomic<unsigned long long> configured{0};
    const cudaError_t e = configure_smem_once(kern, static_cast<int>(SMEM_BYTES), configured);
    if (e != cudaSuccess) return e;
    TmaMaps maps;
    const uint64_t ntok = p.seq_offsets ? static_cast<uint64_t>(p.T) : static_cast<uint64_t>(p.B) * p.T;
    const int H_kv = PRO ? p.H_kv : p.H;
    if (!make_prefill_maps(&maps, p.r, p.w_log, p.k, p.v, p.a, PRO ? nullptr : p.b, p.H, H_kv, ntok, sizeof(WT)))
        return cudaErrorInvalidValue;
    long units = static_cast<long>(p.B) * p.H;
    if (EXPORT) {  // persistent: one block per SM, or one per chunk when there are fewer
        int dev = 0, sms = 0;
        cudaError_t e2 = cudaGetDevice(&dev);
        if (e2 == cudaSuccess) e2 = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e2 != cudaSuccess) return e2;
        const long total = static_cast<long>(p.B) * ((static_cast<long>(p.T) + L - 1) / L) * p.H;
        units = total < sms ? total : sms;
    }
    kern<<<static_cast<unsigned>(units), NTHR, SMEM_BYTES, stream>>>(
        static_cast<const __nv_bfloat16*>(p.r), static_cast<const WT*>(p.w_log),
        static_cast<const __nv_bfloat16*>(p.k), static_cast<const __nv_bfloat16*>(p.v),
        static_cast<const __nv_bfloat16*>(p.a), static_cast<const __nv_bfloat16*>(p.b), p.s0,
        static_cast<__nv_bfloat16*>(p.y), p.sT, p.T, p.H, p.seq_offsets, p.status, p.rk,
        static_cast<const __nv_bfloat16*>(p.g), H_kv, (p.zero_v ? kMapZeroV : 0) | (p.s0_identity ? kMapIdentity : 0),
        p.B, p.ex_as, p.ex_out, p.ex_gam, maps);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_pipe_export(const PrefillArgs& p, int w_dtype, cudaStream_t stream) {
    return w_dtype == WKV7_BF16 ? launch_pipe_typed<__nv_bfloat16, false, false, true>(p, stream)
                                : launch_pipe_typed<float, false, false, true>(p, stream);
}

cudaError_t launch_prefill_pipe(const PrefillArgs& p, int w_dtype, cudaStream_t stream) {
    if (p.prologue) {
        if (p.rk)
            return w_dtype == WKV7_BF16 ? launch_pipe_typed<__nv_bfloat16, true, true>(p, stream)
                                        : launch_pipe_typed<float, true, true>(p, stream);
        return w_dtype == WKV7_BF16 ? launch_pipe_typed<__nv_bfloat16, false, true>(p, stream)
                                    : launch_pipe_typed<float, false, true>(p, stream);
    }
    if (p.rk)
        return w_dtype == WKV7_BF16 ? launch_pipe_typed<__nv_bfloat16, true, false>(p, stream)
                                    : launch_pipe_typed<float, true, false>(p, stream);
    return w_dtype == WKV7_BF16 ? launch_pipe_typed<__nv_bfloat16, false, false>(p, stream)
                                : launch_pipe_typed<float, false, false>(p, stream);
}

}  // namespace wkv7
