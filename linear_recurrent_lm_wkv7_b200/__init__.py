"""B200 (sm_100a) WKV-7 operator: chunked tensor-core prefill and streaming
decode step behind a C ABI (``include/wkv7.h``, ``libwkv7.so``).

The Python layer only marshals arguments to the CUDA library; importing the
package loads ``libwkv7.so`` and fails loudly if it has not been built.
Convenience wrappers ``forward``, ``forward_long``, ``forward_gated``, ``forward_fused``,
``decode_step``, ``decode_step_fused`` and ``backward`` allocate outputs with
torch and call the C entry points; ``forward_host`` runs the prefill on inputs
and outputs that live in pinned host memory, overlapping the copies with the
kernels.
"""
from __future__ import annotations

from ._binding import (  # noqa: F401
    EXPORTS,
    LIB_PATH,
    STATUS,
    WKV7_BF16,
    WKV7_F32,
    Wkv7Error,
    _lib,
    wkv7_backward,
    wkv7_backward_noalloc,
    wkv7_backward_workspace_bytes,
    wkv7_debug_expire_wait,
    wkv7_decode_step,
    wkv7_decode_step_fused,
    wkv7_forward,
    wkv7_forward_fused,
    wkv7_forward_gated,
    wkv7_forward_long,
    wkv7_forward_long_workspace_bytes,
    wkv7_get_device_status,
    wkv7_state_apply,
    wkv7_state_map,
    wkv7_status_string,
    wkv7_version,
)

_lib()  # load now: a missing or broken library is an import error, never a silent fallback


def forward(r, w_log, k, v, a, b, s0=None, seq_offsets=None, want_state=True, stream=None):
    """Chunked prefill.  Dense inputs are [B, T, H, D]; packed inputs are
    [T, H, D] with int32 ``seq_offsets`` [B+1] on the device.  Returns
    ``(y, sT)`` (``sT`` is None when ``want_state`` is false)."""
    import torch

    if seq_offsets is not None:
        T, H, D = r.shape
        B = seq_offsets.numel() - 1
    else:
        B, T, H, D = r.shape
    y = torch.empty_like(r)
    sT = torch.empty((B, H, D, D), dtype=torch.float32, device=r.device) if want_state else None
    wkv7_forward(r, w_log, k, v, a, b, s0, y, sT, B, T, H, D, seq_offsets, stream)
    return y, sT


def forward_long(r, w_log, k, v, a, b, s0=None, want_state=True, workspace=None, stream=None):
    """Two-phase prefill of a dense batch [B, T, H, D] (bf16 inputs) for few,
    long sequences: every chunk's state-independent work in parallel, then one
    state pass per (sequence, head).  ``workspace`` (a device tensor of at least
    ``wkv7_forward_long_workspace_bytes`` bytes) is allocated when not given.
    Returns ``(y, sT)`` like ``forward``."""
    import torch

    B, T, H, D = r.shape
    if workspace is None:
        nbytes = wkv7_forward_long_workspace_bytes(B, T, H, D)
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=r.device)
    y = torch.empty_like(r)
    sT = torch.empty((B, H, D, D), dtype=torch.float32, device=r.device) if want_state else None
    wkv7_forward_long(r, w_log, k, v, a, b, s0, y, sT, workspace, B, T, H, D, stream)
    return y, sT


_HOST_STREAMS = {}
_INPUTS = ("r", "w_log", "k", "v", "a", "b")


def host_pieces(B, T, parts=4, t_parts=1):
    """How ``forward_host`` cuts a dense [B, T, ...] batch: returns ``(groups, bounds)``,
    sequence groups [b0, b1) and token bounds, so that each piece (group, [t0, t1))
    is contiguous in memory.  With ``t_parts`` > 1 every sequence is its own group
    and the token bounds are multiples of 64 (the chunk length), so a range
    continues exactly where the previous one stopped; otherwise there are ``parts``
    groups of whole sequences.  T = 0 gives one empty range."""
    t_parts = max(1, int(t_parts))
    nck = (T + 63) // 64
    bounds = sorted({min(T, 64 * (nck * j // t_parts)) for j in range(t_parts)} | {T})
    if T == 0:
        bounds = [0, 0]  # one empty piece: sT receives s0 (or zeros)
    if len(bounds) > 2:
        groups = [(b, b + 1) for b in range(B)]
    else:
        n = max(1, min(int(parts), B))
        groups = [(B * p // n, B * (p + 1) // n) for p in range(n)]
    return groups, bounds


def forward_host(host, dev, y_host, sT_host, s0=None, parts=4, t_parts=1, stream=None):
    """Prefill of a dense batch whose inputs and outputs live in pinned host memory.

    ``host``: pinned CPU tensors r, w_log, k, v, a, b of shape [B, T, H, D];
    ``dev``: device staging tensors of the same names and shapes plus ``y`` and
    ``sT`` ([B, H, D, D] fp32), allocated once by the caller; ``y_host``,
    ``sT_host``: pinned CPU outputs; ``s0``: optional device initial states.
    The batch is cut into pieces, each contiguous in memory: ``parts`` groups of
    whole sequences, or, with ``t_parts`` > 1 (for batches of few long
    sequences), every sequence cut into that many token ranges whose bounds are
    multiples of 64, a range continuing from the state the previous one left in
    ``dev["sT"]`` (updated in place).  Every piece costs a few host-side calls, so
    a handful of large pieces is best.
    The upload of one piece, the prefill of the previous and the download of the
    one before run on three CUDA streams at once, and the results equal one call
    over the whole batch.  Everything is ordered after ``stream`` (default: the
    current stream), which then waits for all of it: the call is asynchronous
    like a kernel launch on ``stream``.
    The three side streams are created once per device and shared by every call
    on that device.  Calls from several host threads at once are correct but
    their copies and kernels serialise on those streams; such calls must not
    share ``dev`` buffers (nothing orders one call's use of them against
    another's)."""
    import torch

    device = dev["r"].device
    st = stream if stream is not None else torch.cuda.current_stream(device)
    idx = device.index if device.index is not None else torch.cuda.current_device()
    if idx not in _HOST_STREAMS:
        _HOST_STREAMS[idx] = tuple(torch.cuda.Stream(device) for _ in range(3))
    s_up, s_run, s_down = _HOST_STREAMS[idx]
    B, T, H, D = host["r"].shape
    groups, tb = host_pieces(B, T, parts, t_parts)
    start = torch.cuda.Event()
    start.record(st)
    for s_ in (s_up, s_run, s_down):
        s_.wait_event(start)
    for b0, b1 in groups:
        if b1 == b0:
            continue
        for j in range(len(tb) - 1):
            t0, t1 = tb[j], tb[j + 1]
            with torch.cuda.stream(s_up):
                for n in _INPUTS:
                    dev[n][b0:b1, t0:t1].copy_(host[n][b0:b1, t0:t1], non_blocking=True)
            up = torch.cuda.Event()
            up.record(s_up)
            s_run.wait_event(up)
            init = (s0[b0:b1] if s0 is not None else None) if j == 0 else dev["sT"][b0:b1]
            wkv7_forward(*(dev[n][b0:b1, t0:t1] for n in _INPUTS), init, dev["y"][b0:b1, t0:t1],
                         dev["sT"][b0:b1], b1 - b0, t1 - t0, H, D, None, s_run)
            ran = torch.cuda.Event()
            ran.record(s_run)
            s_down.wait_event(ran)
            with torch.cuda.stream(s_down):
                y_host[b0:b1, t0:t1].copy_(dev["y"][b0:b1, t0:t1], non_blocking=True)
                if j == len(tb) - 2:
                    sT_host[b0:b1].copy_(dev["sT"][b0:b1], non_blocking=True)
    done = torch.cuda.Event()
    done.record(s_down)
    st.wait_event(done)


def forward_gated(r, w_log, k, v, a, b, r_k, g, s0=None, seq_offsets=None, want_state=True, stream=None):
    """Chunked prefill with the gated read-out z = (y / sqrt(D) + (sum r k r_k) v) * g.
    ``r_k`` is [H, D] fp32, ``g`` has the shape and dtype of ``r``.  Returns
    ``(z, sT)``."""
    import torch

    if seq_offsets is not None:
        T, H, D = r.shape
        B = seq_offsets.numel() - 1
    else:
        B, T, H, D = r.shape
    z = torch.empty_like(r)
    sT = torch.empty((B, H, D, D), dtype=torch.float32, device=r.device) if want_state else None
    wkv7_forward_gated(r, w_log, k, v, a, b, s0, r_k, g, z, sT, B, T, H, D, seq_offsets, stream)
    return z, sT


def forward_fused(r, w_log, k, v, a_lr, s0=None, seq_offsets=None, r_k=None, g=None, want_state=True, stream=None):
    """Chunked prefill with the fused prologue: ``k`` and ``v`` are the raw rows
    of the kv heads ([.., H_kv, D]), ``a_lr`` the in-context learning rate; the
    kernel forms kk, a = -kk, b = kk a_lr and k (1 - w + a_lr) itself.  With
    ``r_k`` and ``g`` the output is the gated read-out z.  Returns ``(y or z, sT)``."""
    import torch

    if seq_offsets is not None:
        T, H, D = r.shape
        B = seq_offsets.numel() - 1
    else:
        B, T, H, D = r.shape
    H_kv = k.shape[-2]
    out = torch.empty_like(r)
    sT = torch.empty((B, H, D, D), dtype=torch.float32, device=r.device) if want_state else None
    wkv7_forward_fused(r, w_log, k, v, a_lr, s0, r_k, g, out, sT, B, T, H, H_kv, D, seq_offsets, stream)
    return out, sT


def decode_step_fused(r, w_log, k, v, a_lr, state, r_k=None, g=None, out=None, stream=None):
    """One decoding step with the fused prologue (and the gated read-out when
    ``r_k`` and ``g`` are given), updating ``state`` in place.  ``k``, ``v`` are
    [B, H_kv, D].  Returns the output rows [B, H, D]."""
    import torch

    B, H, D = r.shape
    if out is None:
        out = torch.empty_like(r)
    wkv7_decode_step_fused(r, w_log, k, v, a_lr, state, r_k, g, out, state, B, H, k.shape[-2], D, stream)
    return out


def backward(r, w_log, k, v, a, b, dy, s0=None, dsT=None, seq_offsets=None, workspace=None, stream=None):
    """Gradient of <dy, y> + <dsT, sT> with respect to r, w_log, k, v, a, b and s0.
    Layouts as for ``forward``.  ``workspace`` (a device tensor of at least
    ``wkv7_backward_workspace_bytes`` bytes) is allocated when not given.
    Returns ``(dr, dw_log, dk, dv, da, db, ds0)``."""
    import torch

    if seq_offsets is not None:
        T, H, D = r.shape
        B = seq_offsets.numel() - 1
    else:
        B, T, H, D = r.shape
    if workspace is None:
        nbytes = wkv7_backward_workspace_bytes(B, T, H, D, seq_offsets is not None)
        workspace = torch.empty(nbytes // 4, dtype=torch.float32, device=r.device)
    grads = [torch.empty_like(x) for x in (r, w_log, k, v, a, b)]
    ds0 = torch.empty((B, H, D, D), dtype=torch.float32, device=r.device)
    wkv7_backward(r, w_log, k, v, a, b, s0, dy, dsT, grads[0], grads[1], grads[2], grads[3], grads[4], grads[5], ds0,
                  workspace, B, T, H, D, seq_offsets, stream)
    return tuple(grads) + (ds0,)


def decode_step(r, w_log, k, v, a, b, state, y=None, stream=None):
    """One decoding step, updating ``state`` ([B, H, D, D] fp32) in place.
    Returns y ([B, H, D])."""
    import torch

    B, H, D = r.shape
    if y is None:
        y = torch.empty_like(r)
    wkv7_decode_step(r, w_log, k, v, a, b, state, y, state, B, H, D, stream)
    return y
