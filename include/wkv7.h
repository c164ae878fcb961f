/*
 * wkv7.h — C ABI of the B200 (sm_100a) WKV-7 library, libwkv7.so.
 *
 * The operator is the RWKV-7 "Goose" time-mixing recurrence.  Per sequence n
 * and head h it keeps a D x D fp32 state S (S[i][j]: i = value channel, j = key
 * channel) and, for every token t,
 *
 *     w_t = exp(-exp(w_log_t))                              (per key channel)
 *     S_t = S_{t-1} diag(w_t) + (S_{t-1} a_t) b_t^T + v_t k_t^T
 *     y_t = S_t r_t
 *
 * Sources: the state update is the generalized delta rule of the note
 * "RWKV-7 Goose: Expressive Dynamic State Evolution" (section "Generalized
 * Delta rule", full state-update formula), S_t = S_{t-1}(diag(w_t) -
 * kk^T (a (.) kk)) + v^T k, written here with a = -kk and b = kk (.) a_lr as in
 * the WKV call of the forward listing of "RWKV hxa07D architecture explainer"
 * (zenn.dev/openmose), which hands the kernel (r, log_neglog_w, k, v, -kk,
 * kk*a) as B,T,C tensors; w_log is that listing's log_neglog_w.  The output is
 * read from the updated state ("RWKV-7 Goose architecture analysis",
 * youngju.dev, section "Dynamic State Evolution").  Constant-size state and
 * token-by-token decoding: the same page's RNN-mode section.
 *
 * Conventions shared by every entry point
 *  - All tensor arguments are caller-owned DEVICE memory, contiguous, with the
 *    fastest index last.  The library allocates no device memory and keeps no
 *    handle between calls; it only launches kernels on `stream` (a
 *    cudaStream_t; NULL is the legacy default stream) and never synchronizes
 *    the host, except in wkv7_get_device_status.
 *  - Element types are passed as codes (enum wkv7_dtype): `io_dtype` for r, k,
 *    v, a, b and y; `w_dtype` for w_log.  States are always fp32.
 *  - D must be 64 (the head size of the RWKV-7 layers the pages describe);
 *    other head sizes return WKV7_ERR_UNSUPPORTED.
 *  - Every pointer must be 16-byte aligned (WKV7_ERR_MISALIGNED otherwise).
 *  - Decay range.  The hxa07D decay parametrisation -softplus(-x) - 0.5 gives
 *    w_log <= -0.5, i.e. w in [exp(-exp(-0.5)), 1] ~= [0.545, 1]; w_log = -inf
 *    gives w = 1 exactly (used for padding).  The prefill works on 64-token
 *    chunks and scales the operands by the decay accumulated inside a chunk,
 *    Gamma_t = prod_{s<=t} w_s per key channel, and by 1 / Gamma_t.  It is exact
 *    (to the stated tolerances) whenever every chunk keeps Gamma_64 >= 1e-30 in
 *    every channel, i.e. sum of exp(w_log) over the chunk <= 69: always true in
 *    the parametrised range (Gamma_64 >= e^-38.8) and for any w_log <= 0.
 *    A chunk that decays further (e.g. w_log > 0.08 on all 64 tokens) is
 *    detected on the device and reported as WKV7_ERR_DECAY_RANGE through
 *    wkv7_get_device_status; y and sT of that call are then unspecified.  The
 *    decode step works token by token and has no such limit.
 *  - Errors in the arguments are detected on the host before anything is
 *    launched and returned as a negative status; nothing is written then.
 *    Errors that only the device can see (a bounded wait that expired, packed
 *    offsets out of range) are recorded in a per-device status word and
 *    reported by wkv7_get_device_status.  No kernel traps or asserts.
 */
#ifndef WKV7_H
#define WKV7_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    WKV7_F32 = 0,  /* IEEE binary32 */
    WKV7_BF16 = 1  /* bfloat16 */
} wkv7_dtype;

typedef enum {
    WKV7_OK = 0,
    WKV7_ERR_INVALID_ARG = -1,    /* null pointer, bad size, bad dtype code, aliasing */
    WKV7_ERR_UNSUPPORTED = -2,    /* D != 64, or no sm_100 device */
    WKV7_ERR_MISALIGNED = -3,     /* a pointer not 16-byte aligned */
    WKV7_ERR_CUDA = -4,           /* a CUDA runtime call or a launch failed */
    WKV7_ERR_DEVICE_TIMEOUT = -5, /* a bounded device-side wait expired */
    WKV7_ERR_DEVICE_BOUNDS = -6,  /* packed offsets not monotone or beyond T */
    WKV7_ERR_SCRATCH_LIMIT = -7,  /* wkv7_backward_noalloc: problem needs more than its fixed scratch */
    WKV7_ERR_DECAY_RANGE = -8     /* device: a 64-token chunk decays below the exact range (see above) */
} wkv7_status;

/*
 * wkv7_forward — chunked prefill over whole sequences.
 *
 * Dense batch (seq_offsets == NULL):
 *   r, w_log, k, v, a, b, y : [B][T][H][D]  (the B,T,C layout with C = H*D)
 * Packed variable-length batch (seq_offsets != NULL):
 *   r, w_log, k, v, a, b, y : [T][H][D] with T the packed token count;
 *   seq_offsets: DEVICE int32[B+1], non-decreasing, seq_offsets[0] = 0,
 *   seq_offsets[B] = T; sequence n owns tokens [seq_offsets[n], seq_offsets[n+1]).
 *   Pad tokens are ordinary tokens carrying w_log = -inf and k = v = a = b = 0,
 *   which leave the state unchanged (the "attention_mask ... for variable length
 *   and padding" of the hxa07D WKV call).
 * s0 : [B][H][D][D] fp32 initial states, or NULL for zero states.
 * sT : [B][H][D][D] fp32 final states, or NULL to skip writing them.  sT == s0
 *      (state carried in place) is allowed; any other overlap is not.
 * y  : output, same shape and dtype code as r; must not overlap any input.
 * T == 0 is valid: y is empty and sT receives s0 (or zeros).
 * Returns WKV7_OK once the work is enqueued on `stream`.
 */
int wkv7_forward(const void* r, const void* w_log, const void* k, const void* v,
                 const void* a, const void* b, const float* s0, void* y, float* sT,
                 int B, int T, int H, int D, const int32_t* seq_offsets,
                 int io_dtype, int w_dtype, void* stream);

/*
 * wkv7_forward_gated — wkv7_forward followed by the read-out that the forward
 * listing of "RWKV hxa07D architecture explainer" (zenn.dev/openmose) applies
 * to the WKV result before its output projection (the lines after the WKV call;
 * section 9 of that page: scaling, the r-k-v term, the output gate):
 *
 *     u_t = sum_d r_t[d] k_t[d] r_k[h][d]
 *     z_t = (y_t / sqrt(D) + u_t v_t) (.) g_t          (per sequence, token, head)
 *
 * with y_t the WKV output of wkv7_forward, which is not written.
 *   r_k : [H][D] fp32 per-head weights (DEVICE).
 *   g   : gate, same shape and dtype code as r (DEVICE).
 *   z   : output, same shape and dtype code as r; must not overlap any input.
 * Every other argument, layout and rule as in wkv7_forward.  With bf16 inputs
 * the read-out is applied to the output rows inside the prefill kernel; with
 * fp32 inputs it runs as a second pass over z.
 */
int wkv7_forward_gated(const void* r, const void* w_log, const void* k, const void* v,
                       const void* a, const void* b, const float* s0, const float* r_k,
                       const void* g, void* z, float* sT, int B, int T, int H, int D,
                       const int32_t* seq_offsets, int io_dtype, int w_dtype, void* stream);

/*
 * wkv7_forward_fused — the prologue that the forward listing of "RWKV hxa07D
 * architecture explainer" (zenn.dev/openmose) runs between its projections and
 * the WKV call, fused into the prefill, then the recurrence of wkv7_forward and,
 * optionally, the read-out of wkv7_forward_gated.  Per token and head, with k
 * and v taken from kv head h / (H / H_kv) (the listing's repeat of k/v heads when
 * there are fewer kv heads than heads, done by indexing instead of a copy):
 *
 *     w  = exp(-exp(w_log))
 *     kk = k / max(||k||_2, 1e-12)        (normalised over the head)
 *     k' = k (1 - w + a_lr),   a = -kk,   b = kk (.) a_lr
 *
 * and the recurrence runs on (r, w_log, k', v, a, b).  No a, b, k' or repeated
 * k, v is materialised.
 *   k, v : [.., H_kv][D] rows of the kv heads (layouts as in wkv7_forward with
 *          H_kv in place of H); H must be a multiple of H_kv (H_kv == H: no
 *          sharing).
 *   a_lr : in-context learning rate, same shape and dtype code as r.
 *   r_k, g : both NULL (out = y, the WKV output) or both given (out = z of
 *          wkv7_forward_gated, whose r-k-v term then uses k' and the kv head's v).
 * r, w_log, s0, sT, seq_offsets, the dtype codes and the rules on overlap and
 * T == 0 as in wkv7_forward; `out` must not overlap any input.  Pad tokens of a
 * packed batch carry w_log = -inf and k = v = 0 (kk is then 0).  With bf16
 * inputs everything runs inside the prefill kernel; with fp32 inputs the
 * read-out (when asked for) is a second pass over out.
 */
int wkv7_forward_fused(const void* r, const void* w_log, const void* k, const void* v,
                       const void* a_lr, const float* s0, const float* r_k, const void* g,
                       void* out, float* sT, int B, int T, int H, int H_kv, int D,
                       const int32_t* seq_offsets, int io_dtype, int w_dtype, void* stream);

/*
 * wkv7_forward_long — wkv7_forward for dense batches with few (sequence, head)
 * units and long sequences, in two phases through a caller workspace.  Same
 * result as wkv7_forward (the same chunk algebra; "RWKV-7 Goose architecture
 * analysis", its Q5 on chunk-wise parallel WKV and its inference-cost table by
 * sequence length, up to 1M tokens).  Every 64-token chunk's output splits into a
 * part that does not depend on the chunk's start state and one product with
 * that state, so
 *   phase 1 forms the state-independent part of every chunk of every sequence
 *           (one block per SM, each taking every SM-th chunk and head, so all
 *           SMs stay busy even when B x H is small) and writes it to the
 *           workspace;
 *   phase 2 carries the state through the chunks of each (sequence, head), with
 *           one tensor-core product per chunk (a (sequence, head) split over up
 *           to four blocks by columns of the state).
 *   r, w_log, k, v, a, b, s0, y, sT, B, T, H, D : as in wkv7_forward for a
 *          dense batch (no seq_offsets); bf16 inputs only (io_dtype WKV7_BF16;
 *          WKV7_F32 returns WKV7_ERR_UNSUPPORTED: use wkv7_forward), w_log fp32
 *          or bf16.  B x T and B x ceil(T / 64) x H must be below 2^31
 *          (WKV7_ERR_UNSUPPORTED otherwise).
 *   workspace : DEVICE scratch of at least wkv7_forward_long_workspace_bytes(B,
 *          T, H, D) bytes (49,408 per 64-token chunk and head), owned by the
 *          caller, 16-byte aligned, not read before it is written; it must not
 *          overlap any input or output.  wkv7_forward_long_workspace_bytes
 *          returns 0 for invalid sizes (B <= 0, T < 0, H <= 0, D != 64).
 * Decay range and status codes as in wkv7_forward.  T == 0: sT receives s0 (or
 * zeros) and the workspace is not touched.
 */
size_t wkv7_forward_long_workspace_bytes(int B, int T, int H, int D);
int wkv7_forward_long(const void* r, const void* w_log, const void* k, const void* v,
                      const void* a, const void* b, const float* s0, void* y, float* sT,
                      void* workspace, size_t workspace_bytes, int B, int T, int H, int D,
                      int io_dtype, int w_dtype, void* stream);

/*
 * wkv7_state_map — the affine map that a token range applies to the state, for
 * splitting long sequences into ranges (across devices or launches).  Each step
 * S <- S (diag(w_t) + a_t b_t^T) + v_t k_t^T of the generalized delta rule ("RWKV-7
 * Goose: Expressive Dynamic State Evolution", section "Generalized Delta rule")
 * is affine in S, so over a range
 *
 *     S_end = S_start M + Q      for every start state S_start,
 *
 * with M = prod_t (diag(w_t) + a_t b_t^T) (key x key, the tokens in order) and Q
 * the end state from a zero start.  A range's start state then follows from the
 * maps of the ranges before it (wkv7_state_apply), and each range runs
 * wkv7_forward from it; this is what lets the recurrence serve the very long
 * contexts of the inference-cost table of "RWKV-7 Goose architecture analysis"
 * (youngju.dev) on several devices, each holding one range.
 *   r, w_log, k, v, a, b, B, T, H, D, seq_offsets, dtype codes : as in
 *       wkv7_forward (dense or packed; one map per sequence and head; r is not
 *       read for the result, but must be a valid tensor of its shape).
 *   M, Q : [B][H][D][D] fp32 outputs (M[j'][j] key x key; Q[i][j] value x key as
 *       the state); either may be NULL (not computed), not both.  They must not
 *       overlap any input or each other.  T == 0 gives M = I, Q = 0.
 * Cost: two passes of the prefill kernel over the range (Q from a zero state;
 * M from the identity state with v taken as zero), neither writing y.
 */
int wkv7_state_map(const void* r, const void* w_log, const void* k, const void* v,
                   const void* a, const void* b, float* M, float* Q,
                   int B, int T, int H, int D, const int32_t* seq_offsets,
                   int io_dtype, int w_dtype, void* stream);

/*
 * wkv7_state_apply — S_out = S_in M + Q for n_units (sequence, head) states of
 * D x D fp32 (layouts as wkv7_state_map's outputs; S_in == NULL means a zero
 * state, so S_out = Q).  S_out == S_in (in place) is allowed; any other overlap
 * of S_out with an input is not.  Computed in fp32.
 */
int wkv7_state_apply(const float* S_in, const float* M, const float* Q, float* S_out,
                     int n_units, int D, void* stream);

/*
 * wkv7_decode_step — one token per sequence (RNN mode).
 *   r, w_log, k, v, a, b, y : [B][H][D]
 *   s_in, s_out            : [B][H][D][D] fp32; s_in == s_out (in place) is
 *                            allowed, any other overlap is not.  s_in == NULL
 *                            means a zero state.
 * Returns WKV7_OK once the step is enqueued on `stream`.
 */
int wkv7_decode_step(const void* r, const void* w_log, const void* k, const void* v,
                     const void* a, const void* b, const float* s_in, void* y, float* s_out,
                     int B, int H, int D, int io_dtype, int w_dtype, void* stream);

/*
 * wkv7_decode_step_fused — one token per sequence with the prologue of
 * wkv7_forward_fused (kk, a = -kk, b = kk a_lr and the key scaled by
 * (1 - w + a_lr) formed inside the kernel; k and v from kv head h / (H / H_kv))
 * and, when r_k and g are both given, the gated read-out of wkv7_forward_gated
 * (whose r-k-v term uses the scaled key) written to `out` instead of y.
 *   r, w_log, a_lr, g, out : [B][H][D];  k, v : [B][H_kv][D];  r_k : [H][D] fp32
 *   s_in, s_out            : as in wkv7_decode_step.
 * H must be a multiple of H_kv; r_k and g are both NULL or both given; `out`
 * must not overlap any input.
 */
int wkv7_decode_step_fused(const void* r, const void* w_log, const void* k, const void* v,
                           const void* a_lr, const float* s_in, const float* r_k, const void* g,
                           void* out, float* s_out, int B, int H, int H_kv, int D,
                           int io_dtype, int w_dtype, void* stream);

/*
 * wkv7_backward — gradient of the recurrence of wkv7_forward (training).  For
 * the scalar L = sum over tokens of <dy_t, y_t> + <dsT, S_T>, writes
 * dL/dr, dL/dw_log, dL/dk, dL/dv, dL/da, dL/db and dL/ds0 (the chain rule
 * through each step of the generalized delta rule of "RWKV-7 Goose: Expressive
 * Dynamic State Evolution", section "Generalized Delta rule"; the pages print no
 * backward).
 *   r .. b, s0, seq_offsets, B, T, H, D, dtype codes : as in wkv7_forward.
 *   dy  : gradient of y, same shape and dtype code as r.
 *   dsT : [B][H][D][D] fp32 gradient of the final state, or NULL (zero).
 *   dr, dk, dv, da, db : outputs, same shape and dtype code as r;
 *   dw_log : output, same shape and dtype code as w_log; ds0 : [B][H][D][D] fp32
 *          (written even when s0 is NULL: the gradient of a zero initial state).
 *   workspace : DEVICE scratch of at least
 *          wkv7_backward_workspace_bytes(B, T, H, D, seq_offsets != NULL) bytes,
 *          owned by the caller and not read before it is written.
 *          wkv7_backward_workspace_bytes returns 0 for invalid sizes (B <= 0,
 *          T < 0, H <= 0, D != 64).
 * Every output and the workspace must be disjoint from every input and from
 * each other.
 * Chunked form: per 64-token chunk the maps between the chunk's end and start
 * state are formed in parallel, two scans over the chunks give the state and
 * its gradient at every chunk boundary, and every chunk's gradients follow in
 * parallel from the WY products of the chunk (tf32 tensor-core products, fp32
 * accumulation; fp32 inputs enter as tf32 high and low parts, three products
 * each, which keeps fp32 accuracy).  Its decay range is the prefill's: a chunk
 * whose Gamma falls below 1e-30 sets WKV7_ERR_DECAY_RANGE.
 */
size_t wkv7_backward_workspace_bytes(int B, int T, int H, int D, int packed);
int wkv7_backward(const void* r, const void* w_log, const void* k, const void* v,
                  const void* a, const void* b, const float* s0, const void* dy,
                  const float* dsT, void* dr, void* dw_log, void* dk, void* dv,
                  void* da, void* db, float* ds0, void* workspace, size_t workspace_bytes,
                  int B, int T, int H, int D, const int32_t* seq_offsets,
                  int io_dtype, int w_dtype, void* stream);

/*
 * wkv7_backward_noalloc — wkv7_backward with the library's own fixed scratch in
 * place of a caller workspace, for callers that cannot allocate device memory
 * at the point of the call (a device-memory budget that forbids new
 * allocations, runtimes that pass kernels only preallocated buffers, paths that
 * must not call cudaMalloc because it can synchronise the device).  Nothing is
 * allocated by the call.  The pages have no counterpart: this is an interface
 * convenience around the same kernel.
 *   Arguments, layouts and results as in wkv7_backward, without the workspace.
 *   Limit: wkv7_backward_workspace_bytes(B, T, H, D, packed) must not exceed
 *   WKV7_NOALLOC_SCRATCH_BYTES (16 MiB); otherwise WKV7_ERR_SCRATCH_LIMIT is
 *   returned and nothing is launched.  (For example B = 2, H = 3 and T up to
 *   3520 tokens fit; use wkv7_backward for larger problems.)
 *   Nothing in the scratch has to start at zero (every element is written
 *   before it is read), so the call clears nothing.
 *   There is one scratch per device: calls whose kernels may overlap on the
 *   same device (unordered streams, several host threads) race on it; the
 *   caller must order them.
 *   Every call looks up the scratch's address on the current device with
 *   cudaGetSymbolAddress (no allocation); the first call on a device may load
 *   the library's module there, so make that first call before any stream
 *   capture.
 */
#define WKV7_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
int wkv7_backward_noalloc(const void* r, const void* w_log, const void* k, const void* v,
                          const void* a, const void* b, const float* s0, const void* dy,
                          const float* dsT, void* dr, void* dw_log, void* dk, void* dv,
                          void* da, void* db, float* ds0, int B, int T, int H, int D,
                          const int32_t* seq_offsets, int io_dtype, int w_dtype, void* stream);

/* Human-readable text for a status code (static storage, never NULL). */
const char* wkv7_status_string(int status);

/*
 * Synchronizes `stream`, then reads and clears the status word of the current
 * device.  Returns WKV7_OK, WKV7_ERR_DEVICE_TIMEOUT, WKV7_ERR_DEVICE_BOUNDS,
 * WKV7_ERR_DECAY_RANGE, or WKV7_ERR_CUDA if the synchronization itself failed.
 */
int wkv7_get_device_status(void* stream);

/*
 * Test hook for the bounded-wait path: launches one block that waits on a
 * barrier nothing ever completes, with a limit of `spins` polls, then records
 * WKV7_ERR_DEVICE_TIMEOUT in the status word and returns.  Nothing else runs
 * and nothing is left in flight.  spins must be in [1, 1<<20].
 */
int wkv7_debug_expire_wait(int spins, void* stream);

/* Library version as major*10000 + minor*100 + patch. */
int wkv7_version(void);

#ifdef __cplusplus
}
#endif

#endif /* WKV7_H */
