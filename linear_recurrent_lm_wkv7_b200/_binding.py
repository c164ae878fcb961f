"""ctypes binding of libwkv7.so (include/wkv7.h).

Argument marshalling only: tensors are passed as raw device pointers, dtype
codes are derived from the tensors, and the current torch CUDA stream is used
unless one is given.  Every call runs in the CUDA library; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libwkv7.so")

WKV7_F32 = 0
WKV7_BF16 = 1

STATUS = {
    0: "WKV7_OK",
    -1: "WKV7_ERR_INVALID_ARG",
    -2: "WKV7_ERR_UNSUPPORTED",
    -3: "WKV7_ERR_MISALIGNED",
    -4: "WKV7_ERR_CUDA",
    -5: "WKV7_ERR_DEVICE_TIMEOUT",
    -6: "WKV7_ERR_DEVICE_BOUNDS",
    -7: "WKV7_ERR_SCRATCH_LIMIT",
    -8: "WKV7_ERR_DECAY_RANGE",
}
# every symbol include/wkv7.h declares
EXPORTS = (
    "wkv7_forward",
    "wkv7_forward_gated",
    "wkv7_forward_fused",
    "wkv7_forward_long",
    "wkv7_forward_long_workspace_bytes",
    "wkv7_decode_step",
    "wkv7_decode_step_fused",
    "wkv7_backward",
    "wkv7_backward_workspace_bytes",
    "wkv7_backward_noalloc",
    "wkv7_state_map",
    "wkv7_state_apply",
    "wkv7_status_string",
    "wkv7_get_device_status",
    "wkv7_debug_expire_wait",
    "wkv7_version",
)


class Wkv7Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({_lib().wkv7_status_string(status).decode()})")


_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python linear_recurrent_lm_wkv7_b200/build.py`")
        lib = ctypes.CDLL(LIB_PATH)
        vp, i = ctypes.c_void_p, ctypes.c_int
        lib.wkv7_forward.argtypes = [vp] * 9 + [i] * 4 + [vp, i, i, vp]
        lib.wkv7_forward.restype = i
        lib.wkv7_forward_gated.argtypes = [vp] * 11 + [i] * 4 + [vp, i, i, vp]
        lib.wkv7_forward_gated.restype = i
        lib.wkv7_forward_fused.argtypes = [vp] * 10 + [i] * 5 + [vp, i, i, vp]
        lib.wkv7_forward_fused.restype = i
        lib.wkv7_decode_step_fused.argtypes = [vp] * 10 + [i] * 4 + [i, i, vp]
        lib.wkv7_decode_step_fused.restype = i
        lib.wkv7_backward.argtypes = [vp] * 17 + [ctypes.c_size_t] + [i] * 4 + [vp, i, i, vp]
        lib.wkv7_backward.restype = i
        lib.wkv7_backward_workspace_bytes.argtypes = [i] * 5
        lib.wkv7_backward_workspace_bytes.restype = ctypes.c_size_t
        lib.wkv7_backward_noalloc.argtypes = [vp] * 16 + [i] * 4 + [vp, i, i, vp]
        lib.wkv7_backward_noalloc.restype = i
        lib.wkv7_forward_long.argtypes = [vp] * 10 + [ctypes.c_size_t] + [i] * 4 + [i, i, vp]
        lib.wkv7_forward_long.restype = i
        lib.wkv7_forward_long_workspace_bytes.argtypes = [i] * 4
        lib.wkv7_forward_long_workspace_bytes.restype = ctypes.c_size_t
        lib.wkv7_state_map.argtypes = [vp] * 8 + [i] * 4 + [vp, i, i, vp]
        lib.wkv7_state_map.restype = i
        lib.wkv7_state_apply.argtypes = [vp] * 4 + [i, i, vp]
        lib.wkv7_state_apply.restype = i
        lib.wkv7_decode_step.argtypes = [vp] * 9 + [i] * 3 + [i, i, vp]
        lib.wkv7_decode_step.restype = i
        lib.wkv7_status_string.argtypes = [i]
        lib.wkv7_status_string.restype = ctypes.c_char_p
        lib.wkv7_get_device_status.argtypes = [vp]
        lib.wkv7_get_device_status.restype = i
        lib.wkv7_debug_expire_wait.argtypes = [i, vp]
        lib.wkv7_debug_expire_wait.restype = i
        lib.wkv7_version.argtypes = []
        lib.wkv7_version.restype = i
        _LIB = lib
    return _LIB


def _dtype_code(t):
    import torch

    if t.dtype == torch.float32:
        return WKV7_F32
    if t.dtype == torch.bfloat16:
        return WKV7_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def wkv7_forward(r, w_log, k, v, a, b, s0, y, sT, B, T, H, D, seq_offsets=None, stream=None):
    """Enqueue the chunked prefill (see include/wkv7.h).  Raises Wkv7Error on a
    non-OK status."""
    st = _lib().wkv7_forward(_ptr(r), _ptr(w_log), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(s0), _ptr(y),
                             _ptr(sT), int(B), int(T), int(H), int(D), _ptr(seq_offsets), _dtype_code(r),
                             _dtype_code(w_log), _stream(stream))
    if st != 0:
        raise Wkv7Error(st, "wkv7_forward")


def wkv7_forward_gated(r, w_log, k, v, a, b, s0, r_k, g, z, sT, B, T, H, D, seq_offsets=None, stream=None):
    """Enqueue the prefill with the gated read-out (see include/wkv7.h)."""
    st = _lib().wkv7_forward_gated(_ptr(r), _ptr(w_log), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(s0), _ptr(r_k),
                                   _ptr(g), _ptr(z), _ptr(sT), int(B), int(T), int(H), int(D), _ptr(seq_offsets),
                                   _dtype_code(r), _dtype_code(w_log), _stream(stream))
    if st != 0:
        raise Wkv7Error(st, "wkv7_forward_gated")


def wkv7_forward_fused(r, w_log, k, v, a_lr, s0, r_k, g, out, sT, B, T, H, H_kv, D, seq_offsets=None, stream=None):
    """Enqueue the prefill with the fused prologue (and the gated read-out when
    r_k and g are given); see include/wkv7.h."""
    st = _lib().wkv7_forward_fused(_ptr(r), _ptr(w_log), _ptr(k), _ptr(v), _ptr(a_lr), _ptr(s0), _ptr(r_k), _ptr(g),
                                   _ptr(out), _ptr(sT), int(B), int(T), int(H), int(H_kv), int(D), _ptr(seq_offsets),
                                   _dtype_code(r), _dtype_code(w_log), _stream(stream))
    if st != 0:
        raise Wkv7Error(st, "wkv7_forward_fused")


def wkv7_decode_step_fused(r, w_log, k, v, a_lr, s_in, r_k, g, out, s_out, B, H, H_kv, D, stream=None):
    """Enqueue one decoding step with the fused prologue (and the gated read-out
    when r_k and g are given); see include/wkv7.h."""
    st = _lib().wkv7_decode_step_fused(_ptr(r), _ptr(w_log), _ptr(k), _ptr(v), _ptr(a_lr), _ptr(s_in), _ptr(r_k),
                                       _ptr(g), _ptr(out), _ptr(s_out), int(B), int(H), int(H_kv), int(D),
                                       _dtype_code(r), _dtype_code(w_log), _stream(stream))
    if st != 0:
        raise Wkv7Error(st, "wkv7_decode_step_fused")


def wkv7_forward_long_workspace_bytes(B, T, H, D) -> int:
    return int(_lib().wkv7_forward_long_workspace_bytes(int(B), int(T), int(H), int(D)))


def wkv7_forward_long(r, w_log, k, v, a, b, s0, y, sT, workspace, B, T, H, D, stream=None):
    """Enqueue the two-phase prefill for long sequences (see include/wkv7.h)."""
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = _lib().wkv7_forward_long(_ptr(r), _ptr(w_log), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(s0), _ptr(y),
                                  _ptr(sT), _ptr(workspace), int(nbytes), int(B), int(T), int(H), int(D),
                                  _dtype_code(r), _dtype_code(w_log), _stream(stream))
    if st != 0:
        raise Wkv7Error(st, "wkv7_forward_long")


def wkv7_backward_workspace_bytes(B, T, H, D, packed) -> int:
    return int(_lib().wkv7_backward_workspace_bytes(int(B), int(T), int(H), int(D), 1 if packed else 0))


def wkv7_backward(r, w_log, k, v, a, b, s0, dy, dsT, dr, dw_log, dk, dv, da, db, ds0, workspace, B, T, H, D,
                  seq_offsets=None, stream=None):
    """Enqueue the backward of the recurrence (see include/wkv7.h)."""
    nbytes = workspace.numel() * workspace.element_size()
    st = _lib().wkv7_backward(_ptr(r), _ptr(w_log), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(s0), _ptr(dy),
                              _ptr(dsT), _ptr(dr), _ptr(dw_log), _ptr(dk), _ptr(dv), _ptr(da), _ptr(db), _ptr(ds0),
                              _ptr(workspace), int(nbytes), int(B), int(T), int(H), int(D), _ptr(seq_offsets),
                              _dtype_code(r), _dtype_code(w_log), _stream(stream))
    if st != 0:
        raise Wkv7Error(st, "wkv7_backward")


def wkv7_backward_noalloc(r, w_log, k, v, a, b, s0, dy, dsT, dr, dw_log, dk, dv, da, db, ds0, B, T, H, D,
                          seq_offsets=None, stream=None):
    """Enqueue the backward with the library's fixed scratch: for callers that
    cannot allocate device memory at the call (see include/wkv7.h for the 16 MiB
    limit and the rule that overlapping calls must be ordered)."""
    st = _lib().wkv7_backward_noalloc(_ptr(r), _ptr(w_log), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(s0), _ptr(dy),
                                      _ptr(dsT), _ptr(dr), _ptr(dw_log), _ptr(dk), _ptr(dv), _ptr(da), _ptr(db),
                                      _ptr(ds0), int(B), int(T), int(H), int(D), _ptr(seq_offsets), _dtype_code(r),
                                      _dtype_code(w_log), _stream(stream))
    if st != 0:
        raise Wkv7Error(st, "wkv7_backward_noalloc")


def wkv7_state_map(r, w_log, k, v, a, b, M, Q, B, T, H, D, seq_offsets=None, stream=None):
    """Enqueue the affine map of a token range (see include/wkv7.h): S_end = S_start M + Q.
    M or Q may be None (not computed)."""
    st = _lib().wkv7_state_map(_ptr(r), _ptr(w_log), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(M), _ptr(Q), int(B),
                               int(T), int(H), int(D), _ptr(seq_offsets), _dtype_code(r), _dtype_code(w_log),
                               _stream(stream))
    if st != 0:
        raise Wkv7Error(st, "wkv7_state_map")


def wkv7_state_apply(S_in, M, Q, S_out, n_units, D, stream=None):
    """Enqueue S_out = S_in M + Q over n_units states (S_in None: a zero state)."""
    st = _lib().wkv7_state_apply(_ptr(S_in), _ptr(M), _ptr(Q), _ptr(S_out), int(n_units), int(D), _stream(stream))
    if st != 0:
        raise Wkv7Error(st, "wkv7_state_apply")


def wkv7_decode_step(r, w_log, k, v, a, b, s_in, y, s_out, B, H, D, stream=None):
    """Enqueue one decoding step (see include/wkv7.h)."""
    st = _lib().wkv7_decode_step(_ptr(r), _ptr(w_log), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(s_in), _ptr(y),
                                 _ptr(s_out), int(B), int(H), int(D), _dtype_code(r), _dtype_code(w_log),
                                 _stream(stream))
    if st != 0:
        raise Wkv7Error(st, "wkv7_decode_step")


def wkv7_get_device_status(stream=None) -> int:
    return int(_lib().wkv7_get_device_status(_stream(stream)))


def wkv7_debug_expire_wait(spins: int, stream=None) -> None:
    st = _lib().wkv7_debug_expire_wait(int(spins), _stream(stream))
    if st != 0:
        raise Wkv7Error(st, "wkv7_debug_expire_wait")


def wkv7_status_string(status: int) -> str:
    return _lib().wkv7_status_string(int(status)).decode()


def wkv7_version() -> int:
    return int(_lib().wkv7_version())


def raw_call_forward(*args):
    """Direct C call with raw integer pointers (used by host-validation tests)."""
    return int(_lib().wkv7_forward(*args))


def raw_call_forward_long(*args):
    return int(_lib().wkv7_forward_long(*args))


def raw_call_forward_gated(*args):
    return int(_lib().wkv7_forward_gated(*args))


def raw_call_forward_fused(*args):
    return int(_lib().wkv7_forward_fused(*args))


def raw_call_decode_fused(*args):
    return int(_lib().wkv7_decode_step_fused(*args))


def raw_call_backward(*args):
    return int(_lib().wkv7_backward(*args))


def raw_call_backward_noalloc(*args):
    return int(_lib().wkv7_backward_noalloc(*args))


def raw_call_state_map(*args):
    return int(_lib().wkv7_state_map(*args))


def raw_call_state_apply(*args):
    return int(_lib().wkv7_state_apply(*args))


def raw_call_decode(*args):
    return int(_lib().wkv7_decode_step(*args))
