// wkv7_api.cu — the C ABI declared in include/wkv7.h: argument validation on
// the host, dispatch to the kernels, and the per-device status word.
#include <atomic>
#include <cstdint>
#include <cstring>

#include "wkv7_internal.cuh"

namespace {

// One status word per device that loads the library: kernels record the first
// device-side error here (atomicCAS from 0); wkv7_get_device_status reads and
// clears it.
__device__ int g_status = 0;

constexpr int kMaxDevices = 64;

// Address of the current device's status word.  Looked up on every call
// (cudaGetSymbolAddress allocates nothing), so that no cached address can
// outlive a device reset and nothing is shared between host threads.
int status_ptr(int** out) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess || !p) return WKV7_ERR_CUDA;
    *out = static_cast<int*>(p);
    return WKV7_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool dtype_ok(int d) { return d == WKV7_F32 || d == WKV7_BF16; }
size_t dtype_bytes(int d) { return d == WKV7_F32 ? 4 : 2; }

bool overlaps(const void* p, size_t pn, const void* q, size_t qn) {
    if (!p || !q || pn == 0 || qn == 0) return false;
    const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(q);
    return a < b + qn && b < a + pn;
}

int check_device() {
    int dev = 0;
    cudaDeviceProp prop;
    if (cudaGetDevice(&dev) != cudaSuccess) return WKV7_ERR_CUDA;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return WKV7_ERR_CUDA;
    if (prop.major != 10) return WKV7_ERR_UNSUPPORTED;
    return WKV7_OK;
}

// The device check, remembered per device ordinal (0 unknown, 1 ok, else the
// status); entries are atomics because host threads may call concurrently.
int cached_device_check() {
    static std::atomic<int> cache[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return WKV7_ERR_CUDA;
    if (dev >= kMaxDevices) return check_device();
    int c = cache[dev].load(std::memory_order_acquire);
    if (c == 0) {
        const int s = check_device();
        c = (s == WKV7_OK) ? 1 : s;
        cache[dev].store(c, std::memory_order_release);
    }
    return c == 1 ? WKV7_OK : c;
}

// Zero-token call: sT <- s0 (or zeros).
__global__ void copy_or_zero_states(const float* __restrict__ s0, float* __restrict__ sT, long n) {
    const long i = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const long stride = static_cast<long>(gridDim.x) * blockDim.x;
    for (long e = i; e < n; e += stride) sT[e] = s0 ? s0[e] : 0.f;
}

}  // namespace

extern "C" {

int wkv7_version(void) { return 1 * 10000 + 0 * 100 + 0; }

const char* wkv7_status_string(int status) {
    switch (status) {
        case WKV7_OK: return "ok";
        case WKV7_ERR_INVALID_ARG: return "invalid argument";
        case WKV7_ERR_UNSUPPORTED: return "unsupported (head size must be 64 on an sm_100 device)";
        case WKV7_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case WKV7_ERR_CUDA: return "CUDA runtime error";
        case WKV7_ERR_DEVICE_TIMEOUT: return "device-side bounded wait expired";
        case WKV7_ERR_DEVICE_BOUNDS: return "packed sequence offsets out of range";
        case WKV7_ERR_SCRATCH_LIMIT: return "problem needs more than the fixed scratch of wkv7_backward_noalloc";
        case WKV7_ERR_DECAY_RANGE: return "a 64-token chunk decays below the prefill's exact range (Gamma < 1e-30)";
        default: return "unknown status";
    }
}

// wkv7_forward, wkv7_forward_gated and wkv7_forward_fused; rk and g are null
// without the gated read-out.  With `prologue`, `a` is a_lr, b is unused and k,
// v have H_kv heads; otherwise H_kv is H.
static int forward_impl(const void* r, const void* w_log, const void* k, const void* v, const void* a, const void* b,
                        const float* s0, const float* rk, const void* g, void* y, float* sT, int B, int T, int H,
                        int D, const int32_t* seq_offsets, int io_dtype, int w_dtype, void* stream,
                        bool prologue = false, int H_kv = 0) {
    const bool gated = rk != nullptr;
    if (!prologue) H_kv = H;
    // ---- host-side validation; nothing is launched on failure
    if (B <= 0 || T < 0 || H <= 0 || D <= 0) return WKV7_ERR_INVALID_ARG;
    if (H_kv <= 0 || H % H_kv != 0) return WKV7_ERR_INVALID_ARG;
    if (!dtype_ok(io_dtype) || !dtype_ok(w_dtype)) return WKV7_ERR_INVALID_ARG;
    if (D != wkv7::kHead) return WKV7_ERR_UNSUPPORTED;
    if (T > 0 && (!r || !w_log || !k || !v || !a || (!prologue && !b) || !y)) return WKV7_ERR_INVALID_ARG;
    if (gated && T > 0 && !g) return WKV7_ERR_INVALID_ARG;
    if (prologue) b = nullptr;
    const void* ptrs[] = {r, w_log, k, v, a, b, s0, y, sT, seq_offsets, rk, g};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return WKV7_ERR_MISALIGNED;
    const long tokens = seq_offsets ? static_cast<long>(T) : static_cast<long>(B) * T;
    const size_t n_act = static_cast<size_t>(tokens) * H * D;
    const size_t n_kv = static_cast<size_t>(tokens) * H_kv * D;  // k and v
    const size_t n_state = static_cast<size_t>(B) * H * D * D;
    const size_t io_b = dtype_bytes(io_dtype), w_b = dtype_bytes(w_dtype);
    const void* ins[] = {r, k, v, a, b};
    const size_t in_n[] = {n_act, n_kv, n_kv, n_act, n_act};
    for (int i = 0; i < 5; ++i)
        if (overlaps(y, n_act * io_b, ins[i], in_n[i] * io_b)) return WKV7_ERR_INVALID_ARG;
    if (overlaps(y, n_act * io_b, w_log, n_act * w_b) || overlaps(y, n_act * io_b, s0, n_state * 4) ||
        overlaps(y, n_act * io_b, sT, n_state * 4))
        return WKV7_ERR_INVALID_ARG;
    if (gated && (overlaps(y, n_act * io_b, g, n_act * io_b) ||
                  overlaps(y, n_act * io_b, rk, static_cast<size_t>(H) * D * 4) ||
                  overlaps(sT, n_state * 4, g, n_act * io_b) ||
                  overlaps(sT, n_state * 4, rk, static_cast<size_t>(H) * D * 4)))
        return WKV7_ERR_INVALID_ARG;
    // sT == s0 is allowed: each (sequence, head) block reads its own initial state
    // before it writes its own final state.  Any other overlap is rejected.
    if (sT && sT != s0 && overlaps(sT, n_state * 4, s0, n_state * 4)) return WKV7_ERR_INVALID_ARG;
    if (n_act > 0) {
        for (int i = 0; i < 5; ++i)
            if (overlaps(sT, n_state * 4, ins[i], in_n[i] * io_b)) return WKV7_ERR_INVALID_ARG;
        if (overlaps(sT, n_state * 4, w_log, n_act * w_b)) return WKV7_ERR_INVALID_ARG;
    }

    int dev_ok = cached_device_check();
    if (dev_ok != WKV7_OK) return dev_ok;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        if (!sT) return WKV7_OK;
        const long n = static_cast<long>(n_state);
        const int blocks = static_cast<int>((n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184);
        copy_or_zero_states<<<blocks, 256, 0, st>>>(s0, sT, n);
        return cudaGetLastError() == cudaSuccess ? WKV7_OK : WKV7_ERR_CUDA;
    }
    int* status = nullptr;
    if (status_ptr(&status) != WKV7_OK) return WKV7_ERR_CUDA;
    wkv7::PrefillArgs p{r, w_log, k, v, a, b, s0, y, sT, B, T, H, seq_offsets, status};
    if (gated) {
        p.rk = rk;
        p.g = g;
    }
    p.prologue = prologue;
    p.H_kv = H_kv;
    if (wkv7::launch_prefill(p, io_dtype, w_dtype, st) != cudaSuccess) return WKV7_ERR_CUDA;
    // the bf16 kernel writes the gated rows directly; the fp32 path applies the read-out in place
    if (gated && io_dtype == WKV7_F32 &&
        wkv7::launch_gate(y, r, k, v, rk, g, tokens, H, io_dtype, st, prologue ? w_log : nullptr,
                          prologue ? a : nullptr, H_kv, w_dtype) != cudaSuccess)
        return WKV7_ERR_CUDA;
    return WKV7_OK;
}

int wkv7_forward(const void* r, const void* w_log, const void* k, const void* v, const void* a, const void* b,
                 const float* s0, void* y, float* sT, int B, int T, int H, int D, const int32_t* seq_offsets,
                 int io_dtype, int w_dtype, void* stream) {
    return forward_impl(r, w_log, k, v, a, b, s0, nullptr, nullptr, y, sT, B, T, H, D, seq_offsets, io_dtype,
                        w_dtype, stream);
}

int wkv7_forward_gated(const void* r, const void* w_log, const void* k, const void* v, const void* a,
                       const void* b, const float* s0, const float* r_k, const void* g, void* z, float* sT, int B,
                       int T, int H, int D, const int32_t* seq_offsets, int io_dtype, int w_dtype, void* stream) {
    if (!r_k) return WKV7_ERR_INVALID_ARG;
    return forward_impl(r, w_log, k, v, a, b, s0, r_k, g, z, sT, B, T, H, D, seq_offsets, io_dtype, w_dtype,
                        stream);
}

int wkv7_forward_fused(const void* r, const void* w_log, const void* k, const void* v, const void* a_lr,
                       const float* s0, const float* r_k, const void* g, void* out, float* sT, int B, int T, int H,
                       int H_kv, int D, const int32_t* seq_offsets, int io_dtype, int w_dtype, void* stream) {
    if ((r_k == nullptr) != (g == nullptr)) return WKV7_ERR_INVALID_ARG;
    return forward_impl(r, w_log, k, v, a_lr, nullptr, s0, r_k, g, out, sT, B, T, H, D, seq_offsets, io_dtype,
                        w_dtype, stream, true, H_kv);
}


// wkv7_decode_step and wkv7_decode_step_fused (`prologue`: a is a_lr, b unused,
// k and v have H_kv heads; rk and g both null or both given).
static int decode_impl(const void* r, const void* w_log, const void* k, const void* v, const void* a, const void* b,
                       const float* s_in, const float* rk, const void* g, void* y, float* s_out, int B, int H,
                       int H_kv, int D, int io_dtype, int w_dtype, void* stream, bool prologue) {
    if (!prologue) H_kv = H;
    if (B <= 0 || H <= 0 || D <= 0 || H_kv <= 0 || H % H_kv != 0) return WKV7_ERR_INVALID_ARG;
    if (!dtype_ok(io_dtype) || !dtype_ok(w_dtype)) return WKV7_ERR_INVALID_ARG;
    if (D != wkv7::kHead) return WKV7_ERR_UNSUPPORTED;
    if (!r || !w_log || !k || !v || !a || (!prologue && !b) || !y || !s_out) return WKV7_ERR_INVALID_ARG;
    if ((rk == nullptr) != (g == nullptr)) return WKV7_ERR_INVALID_ARG;
    if (prologue) b = nullptr;
    const void* ptrs[] = {r, w_log, k, v, a, b, s_in, y, s_out, rk, g};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return WKV7_ERR_MISALIGNED;
    const size_t n_act = static_cast<size_t>(B) * H * D;
    const size_t n_kv = static_cast<size_t>(B) * H_kv * D;
    const size_t n_state = static_cast<size_t>(B) * H * D * D;
    const size_t io_b = dtype_bytes(io_dtype), w_b = dtype_bytes(w_dtype);
    const void* ins[] = {r, k, v, a, b, g};
    const size_t in_n[] = {n_act, n_kv, n_kv, n_act, n_act, n_act};
    for (int i = 0; i < 6; ++i) {
        if (overlaps(y, n_act * io_b, ins[i], in_n[i] * io_b)) return WKV7_ERR_INVALID_ARG;
        if (overlaps(s_out, n_state * 4, ins[i], in_n[i] * io_b)) return WKV7_ERR_INVALID_ARG;
    }
    const size_t rk_b = static_cast<size_t>(H) * D * 4;
    if (overlaps(y, n_act * io_b, w_log, n_act * w_b) || overlaps(y, n_act * io_b, s_in, n_state * 4) ||
        overlaps(y, n_act * io_b, s_out, n_state * 4) || overlaps(s_out, n_state * 4, w_log, n_act * w_b) ||
        overlaps(y, n_act * io_b, rk, rk_b) || overlaps(s_out, n_state * 4, rk, rk_b))
        return WKV7_ERR_INVALID_ARG;
    if (s_in && s_in != s_out && overlaps(s_in, n_state * 4, s_out, n_state * 4)) return WKV7_ERR_INVALID_ARG;

    int dev_ok = cached_device_check();
    if (dev_ok != WKV7_OK) return dev_ok;
    int* status = nullptr;
    if (status_ptr(&status) != WKV7_OK) return WKV7_ERR_CUDA;
    wkv7::DecodeArgs p{r, w_log, k, v, a, b, s_in, y, s_out, B, H};
    p.prologue = prologue;
    p.H_kv = H_kv;
    p.rk = rk;
    p.g = g;
    return wkv7::launch_decode(p, io_dtype, w_dtype, status, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? WKV7_OK
               : WKV7_ERR_CUDA;
}

int wkv7_decode_step(const void* r, const void* w_log, const void* k, const void* v, const void* a, const void* b,
                     const float* s_in, void* y, float* s_out, int B, int H, int D, int io_dtype, int w_dtype,
                     void* stream) {
    return decode_impl(r, w_log, k, v, a, b, s_in, nullptr, nullptr, y, s_out, B, H, H, D, io_dtype, w_dtype, stream,
                       false);
}

int wkv7_decode_step_fused(const void* r, const void* w_log, const void* k, const void* v, const void* a_lr,
                           const float* s_in, const float* r_k, const void* g, void* out, float* s_out, int B, int H,
                           int H_kv, int D, int io_dtype, int w_dtype, void* stream) {
    return decode_impl(r, w_log, k, v, a_lr, nullptr, s_in, r_k, g, out, s_out, B, H, H_kv, D, io_dtype, w_dtype,
                       stream, true);
}

size_t wkv7_forward_long_workspace_bytes(int B, int T, int H, int D) {
    if (B <= 0 || T < 0 || H <= 0 || D != wkv7::kHead) return 0;
    return wkv7::prefill_long_workspace_bytes(B, T, H);
}

int wkv7_forward_long(const void* r, const void* w_log, const void* k, const void* v, const void* a, const void* b,
                      const float* s0, void* y, float* sT, void* workspace, size_t workspace_bytes, int B, int T,
                      int H, int D, int io_dtype, int w_dtype, void* stream) {
    // ---- host-side validation; nothing is launched on failure
    if (B <= 0 || T < 0 || H <= 0 || D <= 0) return WKV7_ERR_INVALID_ARG;
    if (!dtype_ok(io_dtype) || !dtype_ok(w_dtype)) return WKV7_ERR_INVALID_ARG;
    if (D != wkv7::kHead || io_dtype != WKV7_BF16) return WKV7_ERR_UNSUPPORTED;
    // the first phase numbers token rows and (sequence, chunk, head) slots in 32 bits
    if (static_cast<long long>(B) * T >= (1LL << 31) ||
        static_cast<long long>(B) * ((static_cast<long long>(T) + 63) / 64) * H >= (1LL << 31))
        return WKV7_ERR_UNSUPPORTED;
    if (T > 0 && (!r || !w_log || !k || !v || !a || !b || !y || !workspace)) return WKV7_ERR_INVALID_ARG;
    const void* ptrs[] = {r, w_log, k, v, a, b, s0, y, sT, workspace};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return WKV7_ERR_MISALIGNED;
    const size_t need = wkv7::prefill_long_workspace_bytes(B, T, H);
    if (T > 0 && workspace_bytes < need) return WKV7_ERR_INVALID_ARG;
    const size_t n_act = static_cast<size_t>(B) * T * H * D;
    const size_t n_state = static_cast<size_t>(B) * H * D * D;
    const size_t io_b = dtype_bytes(io_dtype), w_b = dtype_bytes(w_dtype);
    const void* ins[] = {r, k, v, a, b, w_log, s0};
    const size_t in_b[] = {n_act * io_b, n_act * io_b, n_act * io_b, n_act * io_b, n_act * io_b, n_act * w_b,
                           n_state * 4};
    // outputs and workspace: disjoint from every input and from each other (sT may be s0)
    const void* outs[] = {y, sT, T > 0 ? workspace : nullptr};
    const size_t out_b[] = {n_act * io_b, n_state * 4, need};
    for (int o = 0; o < 3; ++o) {
        for (int i = 0; i < 7; ++i) {
            if (o == 1 && i == 6 && sT == s0) continue;
            if (overlaps(outs[o], out_b[o], ins[i], in_b[i])) return WKV7_ERR_INVALID_ARG;
        }
        for (int o2 = o + 1; o2 < 3; ++o2)
            if (overlaps(outs[o], out_b[o], outs[o2], out_b[o2])) return WKV7_ERR_INVALID_ARG;
    }

    int dev_ok = cached_device_check();
    if (dev_ok != WKV7_OK) return dev_ok;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        if (!sT) return WKV7_OK;
        const long n = static_cast<long>(n_state);
        const int blocks = static_cast<int>((n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184);
        copy_or_zero_states<<<blocks, 256, 0, st>>>(s0, sT, n);
        return cudaGetLastError() == cudaSuccess ? WKV7_OK : WKV7_ERR_CUDA;
    }
    int* status = nullptr;
    if (status_ptr(&status) != WKV7_OK) return WKV7_ERR_CUDA;
    wkv7::PrefillArgs p{r, w_log, k, v, a, b, s0, y, sT, B, T, H, nullptr, status};
    return wkv7::launch_prefill_long(p, w_dtype, workspace, st) == cudaSuccess ? WKV7_OK : WKV7_ERR_CUDA;
}

int wkv7_state_map(const void* r, const void* w_log, const void* k, const void* v, const void* a, const void* b,
                   float* M, float* Q, int B, int T, int H, int D, const int32_t* seq_offsets, int io_dtype,
                   int w_dtype, void* stream) {
    // ---- host-side validation; nothing is launched on failure
    if (B <= 0 || T < 0 || H <= 0 || D <= 0) return WKV7_ERR_INVALID_ARG;
    if (!dtype_ok(io_dtype) || !dtype_ok(w_dtype)) return WKV7_ERR_INVALID_ARG;
    if (D != wkv7::kHead) return WKV7_ERR_UNSUPPORTED;
    if (!M && !Q) return WKV7_ERR_INVALID_ARG;
    if (T > 0 && (!r || !w_log || !k || !v || !a || !b)) return WKV7_ERR_INVALID_ARG;
    const void* ptrs[] = {r, w_log, k, v, a, b, M, Q, seq_offsets};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return WKV7_ERR_MISALIGNED;
    const long tokens = seq_offsets ? static_cast<long>(T) : static_cast<long>(B) * T;
    const size_t n_act = static_cast<size_t>(tokens) * H * D;
    const size_t n_state = static_cast<size_t>(B) * H * D * D;
    const size_t io_b = dtype_bytes(io_dtype), w_b = dtype_bytes(w_dtype);
    if (overlaps(M, n_state * 4, Q, n_state * 4)) return WKV7_ERR_INVALID_ARG;
    const void* ins[] = {r, k, v, a, b, w_log};
    for (int i = 0; i < 6; ++i) {
        const size_t nb = n_act * (i == 5 ? w_b : io_b);
        if (overlaps(M, n_state * 4, ins[i], nb) || overlaps(Q, n_state * 4, ins[i], nb)) return WKV7_ERR_INVALID_ARG;
    }

    int dev_ok = cached_device_check();
    if (dev_ok != WKV7_OK) return dev_ok;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const long units = static_cast<long>(B) * H;
    if (T == 0) return wkv7::launch_state_identity(M, Q, units, st) == cudaSuccess ? WKV7_OK : WKV7_ERR_CUDA;
    int* status = nullptr;
    if (status_ptr(&status) != WKV7_OK) return WKV7_ERR_CUDA;
    // Q: the end state from a zero start; M: the end state from the identity with v = 0
    // (the product of the transitions); neither writes y
    wkv7::PrefillArgs p{r, w_log, k, v, a, b, nullptr, nullptr, Q, B, T, H, seq_offsets, status};
    if (Q && wkv7::launch_prefill(p, io_dtype, w_dtype, st) != cudaSuccess) return WKV7_ERR_CUDA;
    p.sT = M;
    p.zero_v = true;
    p.s0_identity = true;
    if (M && wkv7::launch_prefill(p, io_dtype, w_dtype, st) != cudaSuccess) return WKV7_ERR_CUDA;
    return WKV7_OK;
}

int wkv7_state_apply(const float* S_in, const float* M, const float* Q, float* S_out, int n_units, int D,
                     void* stream) {
    if (n_units <= 0 || D <= 0) return WKV7_ERR_INVALID_ARG;
    if (D != wkv7::kHead) return WKV7_ERR_UNSUPPORTED;
    if (!M || !Q || !S_out) return WKV7_ERR_INVALID_ARG;
    const void* ptrs[] = {S_in, M, Q, S_out};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return WKV7_ERR_MISALIGNED;
    const size_t nb = static_cast<size_t>(n_units) * D * D * 4;
    // S_out may be S_in (in place); any other overlap of the output is rejected
    if (overlaps(S_out, nb, M, nb) || overlaps(S_out, nb, Q, nb)) return WKV7_ERR_INVALID_ARG;
    if (S_in && S_in != S_out && overlaps(S_out, nb, S_in, nb)) return WKV7_ERR_INVALID_ARG;
    int dev_ok = cached_device_check();
    if (dev_ok != WKV7_OK) return dev_ok;
    return wkv7::launch_state_apply(S_in, M, Q, S_out, n_units, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? WKV7_OK
               : WKV7_ERR_CUDA;
}

size_t wkv7_backward_workspace_bytes(int B, int T, int H, int D, int packed) {
    if (B <= 0 || T < 0 || H <= 0 || D != wkv7::kHead) return 0;
    return wkv7::backward_workspace_floats(B, T, H, packed ? 1 : 0) * sizeof(float);
}

int wkv7_backward(const void* r, const void* w_log, const void* k, const void* v, const void* a, const void* b,
                  const float* s0, const void* dy, const float* dsT, void* dr, void* dw_log, void* dk, void* dv,
                  void* da, void* db, float* ds0, void* workspace, size_t workspace_bytes, int B, int T, int H,
                  int D, const int32_t* seq_offsets, int io_dtype, int w_dtype, void* stream) {
    // ---- host-side validation; nothing is launched on failure
    if (B <= 0 || T < 0 || H <= 0 || D <= 0) return WKV7_ERR_INVALID_ARG;
    if (!dtype_ok(io_dtype) || !dtype_ok(w_dtype)) return WKV7_ERR_INVALID_ARG;
    if (D != wkv7::kHead) return WKV7_ERR_UNSUPPORTED;
    if (!ds0 || !workspace) return WKV7_ERR_INVALID_ARG;
    if (T > 0 && (!r || !w_log || !k || !v || !a || !b || !dy || !dr || !dw_log || !dk || !dv || !da || !db))
        return WKV7_ERR_INVALID_ARG;
    const void* ptrs[] = {r, w_log, k, v, a, b, s0, dy, dsT, dr, dw_log, dk, dv, da, db, ds0, workspace, seq_offsets};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return WKV7_ERR_MISALIGNED;
    const int packed = seq_offsets ? 1 : 0;
    if (workspace_bytes < wkv7::backward_workspace_floats(B, T, H, packed) * sizeof(float))
        return WKV7_ERR_INVALID_ARG;
    const long tokens = packed ? static_cast<long>(T) : static_cast<long>(B) * T;
    const size_t n_act = static_cast<size_t>(tokens) * H * D;
    const size_t n_state = static_cast<size_t>(B) * H * D * D;
    const size_t io_b = dtype_bytes(io_dtype), w_b = dtype_bytes(w_dtype);
    // every output (and the workspace) is disjoint from every input and from the others
    const void* outs[] = {dr, dk, dv, da, db, dw_log, ds0, workspace};
    const size_t out_b[] = {n_act * io_b, n_act * io_b, n_act * io_b, n_act * io_b,
                            n_act * io_b, n_act * w_b,  n_state * 4,  workspace_bytes};
    const void* ins[] = {r, k, v, a, b, dy, w_log, s0, dsT};
    const size_t in_b[] = {n_act * io_b, n_act * io_b, n_act * io_b, n_act * io_b, n_act * io_b,
                           n_act * io_b, n_act * w_b,  n_state * 4,  n_state * 4};
    for (int i = 0; i < 8; ++i) {
        for (int j = 0; j < 9; ++j)
            if (overlaps(outs[i], out_b[i], ins[j], in_b[j])) return WKV7_ERR_INVALID_ARG;
        for (int j = i + 1; j < 8; ++j)
            if (overlaps(outs[i], out_b[i], outs[j], out_b[j])) return WKV7_ERR_INVALID_ARG;
    }

    int dev_ok = cached_device_check();
    if (dev_ok != WKV7_OK) return dev_ok;
    int* status = nullptr;
    if (status_ptr(&status) != WKV7_OK) return WKV7_ERR_CUDA;
    wkv7::BackwardArgs p{r, w_log, k, v, a, b, s0, dy, dsT, dr, dw_log, dk, dv, da, db, ds0,
                         static_cast<float*>(workspace), B, T, H, seq_offsets,
                         wkv7::backward_ckpt_chunks(B, T, packed), status};
    return wkv7::launch_backward(p, io_dtype, w_dtype, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? WKV7_OK
               : WKV7_ERR_CUDA;
}

int wkv7_get_device_status(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return WKV7_ERR_CUDA;
    int* dptr = nullptr;
    if (status_ptr(&dptr) != WKV7_OK) return WKV7_ERR_CUDA;
    int host = 0;
    if (cudaMemcpy(&host, dptr, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return WKV7_ERR_CUDA;
    if (host != 0) {
        const int zero = 0;
        if (cudaMemcpy(dptr, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return WKV7_ERR_CUDA;
    }
    return host;
}

int wkv7_debug_expire_wait(int spins, void* stream) {
    if (spins < 1 || spins > (1 << 20)) return WKV7_ERR_INVALID_ARG;
    int dev_ok = cached_device_check();
    if (dev_ok != WKV7_OK) return dev_ok;
    int* status = nullptr;
    if (status_ptr(&status) != WKV7_OK) return WKV7_ERR_CUDA;
    return wkv7::launch_expire_wait(spins, status, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? WKV7_OK
               : WKV7_ERR_CUDA;
}

}  // extern "C"
