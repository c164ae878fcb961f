"""WKV-7 oracle: plain fp64 CPU recurrence (test infrastructure only).

Only the test suite, the smoke check and the benchmark's CPU-baseline leg may
import this package.  It loads ``libwkv7_oracle.so`` built from
``wkv7_oracle.c`` (see :func:`build`), which shares no code with the CUDA
library.  Inputs are taken as float64 numpy arrays holding the values *after*
rounding to their storage dtype (bf16 or fp32); the oracle upcasts nothing else
and rounds nothing.

What is computed, and the passages it follows, is documented in the header of
``wkv7_oracle.c``.  Every function here is argument marshalling only.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wkv7_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libwkv7_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle shared object with gcc (no fast-math: the evaluation
    order is the one written in the C source)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-o", _LIB_PATH, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int32)
        lib.wkv7_oracle_forward.argtypes = [dp] * 9 + [ctypes.c_int] * 4 + [ip, ctypes.c_int]
        lib.wkv7_oracle_forward.restype = ctypes.c_int
        lib.wkv7_oracle_decode_step.argtypes = [dp] * 9 + [ctypes.c_int] * 4
        lib.wkv7_oracle_decode_step.restype = ctypes.c_int
        lib.wkv7_oracle_gate.argtypes = [dp] * 7 + [ctypes.c_long, ctypes.c_int, ctypes.c_int]
        lib.wkv7_oracle_gate.restype = ctypes.c_int
        lib.wkv7_oracle_prologue.argtypes = [dp] * 8 + [ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_int]
        lib.wkv7_oracle_prologue.restype = ctypes.c_int
        lib.wkv7_oracle_backward.argtypes = [dp] * 16 + [ctypes.c_int] * 4 + [ip, ctypes.c_int]
        lib.wkv7_oracle_backward.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor (CPU)
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(x):
    if x is None:
        return None
    return x.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def forward(r, w_log, k, v, a, b, s0=None, seq_offsets=None, n_threads=None, want_y=True):
    """Run the recurrence over whole sequences.

    Dense: r, w_log, k, v, a, b are [B, T, H, D]; packed (``seq_offsets`` given,
    B+1 int32 entries): they are [T, H, D].  ``s0`` is [B, H, D, D] or None.
    Returns ``(y, sT)`` as float64 arrays (``y`` is None when ``want_y`` is false).
    """
    lib = _load()
    r, w_log, k, v, a, b = (_f64(t) for t in (r, w_log, k, v, a, b))
    if seq_offsets is not None:
        offs = np.ascontiguousarray(np.asarray(seq_offsets, dtype=np.int32))
        T, H, D = r.shape
        B = offs.shape[0] - 1
        offs_p = offs.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    else:
        B, T, H, D = r.shape
        offs_p = None
    for t in (w_log, k, v, a, b):
        if t.shape != r.shape:
            raise ValueError("input shapes differ")
    s0 = _f64(s0)
    if s0 is not None and s0.shape != (B, H, D, D):
        raise ValueError("s0 must be [B, H, D, D]")
    y = np.empty_like(r) if want_y else None
    sT = np.empty((B, H, D, D), dtype=np.float64)
    nt = default_threads() if n_threads is None else n_threads
    rc = lib.wkv7_oracle_forward(_ptr(r), _ptr(w_log), _ptr(k), _ptr(v), _ptr(a), _ptr(b),
                                 _ptr(s0), _ptr(y), _ptr(sT), B, T, H, D, offs_p, nt)
    if rc != 0:
        raise RuntimeError(f"wkv7_oracle_forward failed with status {rc}")
    return y, sT


def state_map(w_log, k, v, a, b, seq_offsets=None, n_threads=None):
    """The affine map of each sequence's token range, S_end = S_start M + Q.

    Each step S <- S (diag(w_t) + a_t b_t^T) + v_t k_t^T of the generalized delta
    rule is affine in S, so the whole range is too: M = prod_t (diag(w_t) + a_t
    b_t^T) in token order, which is the end state of the recurrence started from
    the identity with v = 0, and Q is the end state started from zero.  Both are
    computed by :func:`forward` exactly so.  Returns ``(M, Q)``, [B, H, D, D]."""
    v = _f64(v)
    zeros = np.zeros_like(v)
    if seq_offsets is not None:
        B = len(seq_offsets) - 1
        H, D = v.shape[1], v.shape[2]
    else:
        B, _, H, D = v.shape
    eye = np.broadcast_to(np.eye(D), (B, H, D, D)).copy()
    _, M = forward(zeros, w_log, k, zeros, a, b, eye, seq_offsets=seq_offsets, n_threads=n_threads, want_y=False)
    _, Q = forward(zeros, w_log, k, v, a, b, None, seq_offsets=seq_offsets, n_threads=n_threads, want_y=False)
    return M, Q


def decode_step(r, w_log, k, v, a, b, s_in, n_threads=None):
    """One token per sequence: inputs [B, H, D], state [B, H, D, D].
    Returns ``(y, s_out)`` as float64 arrays."""
    lib = _load()
    r, w_log, k, v, a, b = (_f64(t) for t in (r, w_log, k, v, a, b))
    B, H, D = r.shape
    s = _f64(s_in)
    s_out = np.array(s, dtype=np.float64, copy=True) if s is not None else np.zeros((B, H, D, D))
    y = np.empty_like(r)
    nt = default_threads() if n_threads is None else n_threads
    rc = lib.wkv7_oracle_decode_step(_ptr(r), _ptr(w_log), _ptr(k), _ptr(v), _ptr(a), _ptr(b),
                                     _ptr(s_out), _ptr(y), _ptr(s_out), B, H, D, nt)
    if rc != 0:
        raise RuntimeError(f"wkv7_oracle_decode_step failed with status {rc}")
    return y, s_out


def gate(y, r, k, v, rk, g):
    """Gated read-out z = (y / sqrt(D) + (sum_d r k rk) v) * g.  y, r, k, v, g
    share one shape [..., H, D]; rk is [H, D].  Returns z as a float64 array."""
    lib = _load()
    y, r, k, v, g = (_f64(t) for t in (y, r, k, v, g))
    rk = _f64(rk)
    for t in (r, k, v, g):
        if t.shape != y.shape:
            raise ValueError("input shapes differ")
    H, D = y.shape[-2], y.shape[-1]
    if rk.shape != (H, D):
        raise ValueError("rk must be [H, D]")
    ntok = int(np.prod(y.shape[:-2])) if y.ndim > 2 else 1
    z = np.empty_like(y)
    rc = lib.wkv7_oracle_gate(_ptr(y), _ptr(r), _ptr(k), _ptr(v), _ptr(rk), _ptr(g), _ptr(z), ntok, H, D)
    if rc != 0:
        raise RuntimeError(f"wkv7_oracle_gate failed with status {rc}")
    return z


def forward_gated(r, w_log, k, v, a, b, rk, g, s0=None, seq_offsets=None, n_threads=None):
    """The recurrence followed by the gated read-out.  Returns ``(z, sT)``."""
    y, sT = forward(r, w_log, k, v, a, b, s0, seq_offsets, n_threads)
    return gate(y, r, k, v, rk, g), sT


def prologue(k, v, w_log, a_lr):
    """The steps between the projections and the WKV call: k, v [..., H_kv, D] of
    the kv heads, w_log and a_lr [..., H, D].  Returns ``(k', v_rep, a, b)``, each
    [..., H, D] float64: k' = k (1 - w + a_lr), v_rep the kv head's v,
    a = -kk and b = kk a_lr with kk = k / max(||k||, 1e-12)."""
    lib = _load()
    k, v, w_log, a_lr = (_f64(t) for t in (k, v, w_log, a_lr))
    if k.shape != v.shape or w_log.shape != a_lr.shape or k.shape[:-2] != w_log.shape[:-2]:
        raise ValueError("input shapes differ")
    H, D = w_log.shape[-2], w_log.shape[-1]
    H_kv = k.shape[-2]
    if k.shape[-1] != D or H % H_kv != 0:
        raise ValueError("H must be a multiple of H_kv and the head sizes must match")
    ntok = int(np.prod(w_log.shape[:-2])) if w_log.ndim > 2 else 1
    outs = [np.empty(w_log.shape, dtype=np.float64) for _ in range(4)]
    rc = lib.wkv7_oracle_prologue(_ptr(k), _ptr(v), _ptr(w_log), _ptr(a_lr), *(_ptr(o) for o in outs), ntok, H,
                                  H_kv, D)
    if rc != 0:
        raise RuntimeError(f"wkv7_oracle_prologue failed with status {rc}")
    return tuple(outs)


def forward_fused(r, w_log, k, v, a_lr, s0=None, seq_offsets=None, rk=None, g=None, n_threads=None):
    """Prologue, recurrence and (when rk and g are given) the gated read-out.
    Returns ``(y or z, sT)``."""
    kp, vr, a, b = prologue(k, v, w_log, a_lr)
    y, sT = forward(r, w_log, kp, vr, a, b, s0, seq_offsets, n_threads)
    if rk is None and g is None:
        return y, sT
    return gate(y, r, kp, vr, rk, g), sT


def decode_step_fused(r, w_log, k, v, a_lr, s_in, rk=None, g=None, n_threads=None):
    """One decode step with the prologue (and the gated read-out when rk and g
    are given).  Returns ``(y or z, s_out)``."""
    kp, vr, a, b = prologue(k, v, w_log, a_lr)
    y, s_out = decode_step(r, w_log, kp, vr, a, b, s_in, n_threads)
    if rk is None and g is None:
        return y, s_out
    return gate(y, r, kp, vr, rk, g), s_out


def backward(r, w_log, k, v, a, b, dy, s0=None, dsT=None, seq_offsets=None, n_threads=None):
    """Gradient of L = sum <dy, y> + <dsT, sT> with respect to r, w_log, k, v, a, b
    and s0.  Layouts as for ``forward``.  Returns ``(dr, dw_log, dk, dv, da, db, ds0)``
    as float64 arrays."""
    lib = _load()
    r, w_log, k, v, a, b, dy = (_f64(t) for t in (r, w_log, k, v, a, b, dy))
    for t in (w_log, k, v, a, b, dy):
        if t.shape != r.shape:
            raise ValueError("input shapes differ")
    if seq_offsets is not None:
        offs = np.ascontiguousarray(seq_offsets, dtype=np.int32)
        T, H, D = r.shape
        B = offs.size - 1
        offs_p = offs.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    else:
        B, T, H, D = r.shape
        offs, offs_p = None, None
    s0 = _f64(s0) if s0 is not None else None
    dsT = _f64(dsT) if dsT is not None else None
    grads = [np.zeros(r.shape, dtype=np.float64) for _ in range(6)]
    ds0 = np.zeros((B, H, D, D), dtype=np.float64)
    nt = default_threads() if n_threads is None else n_threads
    rc = lib.wkv7_oracle_backward(_ptr(r), _ptr(w_log), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(s0), _ptr(dy),
                                  _ptr(dsT), *(_ptr(g) for g in grads), _ptr(ds0), B, T, H, D, offs_p, nt)
    if rc != 0:
        raise RuntimeError(f"wkv7_oracle_backward failed with status {rc}")
    return tuple(grads) + (ds0,)
