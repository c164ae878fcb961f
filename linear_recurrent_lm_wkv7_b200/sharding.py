"""Splitting work across ranks: whole sequences, or one sequence's tokens.

Every (sequence, head) unit of the WKV-7 recurrence is independent of every
other one (the state is per sequence and head), so a batch shards across GPUs
without any exchange on the data path: each rank runs ``wkv7_forward`` on its
own sequences and owns their outputs and final states.  The only host-side
decision is which sequences go where; for packed variable-length batches the
assignment balances token counts (longest sequences first, each to the least
loaded rank).

A long sequence can also be cut along its tokens (``token_ranges``): the
recurrence is affine in its start state over any token range, S_end =
S_start M + Q (``wkv7_state_map``), so each range's start state follows from
the maps of the ranges before it by an exclusive scan (``start_states``), after
which every range runs ``wkv7_forward`` on its own.  ``forward_sequence_parallel``
does this across ranks (the maps, B x H x 64 x 64 fp32 each, are all-gathered
over the process group; nothing else crosses ranks); ``forward_split`` does the
same on one device.  The arithmetic of every step runs in the CUDA library; the
functions here only order the calls.
"""
from __future__ import annotations

from typing import List, Sequence


def assign_sequences(lengths: Sequence[int], world_size: int) -> List[List[int]]:
    """Indices of the sequences each rank owns, balanced by length.

    Greedy longest-processing-time assignment; ties go to the lower rank and
    each rank's list is returned in ascending sequence order, so the result is
    deterministic and identical on every rank."""
    if world_size <= 0:
        raise ValueError("world_size must be positive")
    loads = [0] * world_size
    owned: List[List[int]] = [[] for _ in range(world_size)]
    order = sorted(range(len(lengths)), key=lambda i: (-int(lengths[i]), i))
    for i in order:
        rk = min(range(world_size), key=lambda q: (loads[q], q))
        owned[rk].append(i)
        loads[rk] += int(lengths[i])
    return [sorted(o) for o in owned]


def packed_shard(offsets: Sequence[int], owned: Sequence[int]):
    """Token ranges and new offsets for a rank's sequences of a packed batch.

    Returns ``(ranges, new_offsets)``: ``ranges`` lists the (start, end) token
    slices of the original packed axis in the order of ``owned``, and
    ``new_offsets`` (len(owned) + 1 entries) describes the rank's own packed
    batch made by concatenating those slices."""
    ranges = [(int(offsets[i]), int(offsets[i + 1])) for i in owned]
    new = [0]
    for s, e in ranges:
        new.append(new[-1] + (e - s))
    return ranges, new


def dense_shard(batch: int, world_size: int, rank: int) -> range:
    """Contiguous block of sequences of a dense [B, T, H, D] batch for one rank
    (sizes differ by at most one)."""
    base, extra = divmod(batch, world_size)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def token_ranges(T: int, n_parts: int, chunk: int = 64) -> List[tuple]:
    """Cut T tokens into ``n_parts`` contiguous ranges ``(t0, t1)`` whose inner
    bounds are multiples of ``chunk`` (so every range but the last starts a
    fresh chunk) and whose chunk counts differ by at most one; ranges past the
    end are empty."""
    if n_parts <= 0:
        raise ValueError("n_parts must be positive")
    nck = (T + chunk - 1) // chunk
    bounds = [min(T, chunk * (nck * j // n_parts)) for j in range(n_parts)] + [T]
    return [(bounds[j], bounds[j + 1]) for j in range(n_parts)]


def start_states(maps, s0, apply):
    """Start state of every range from the maps of the ranges before it:
    S_0 = s0 and S_{j+1} = apply(S_j, M_j, Q_j), the end state of range j.
    ``maps`` lists (M_j, Q_j) in token order; the last one is not needed.
    ``apply(S, M, Q)`` returns S M + Q (S may be None for a zero state)."""
    starts = [s0]
    S = s0
    for M, Q in list(maps)[:-1]:
        S = apply(S, M, Q)
        starts.append(S)
    return starts


def _device_apply(wk, stream):
    import torch

    def apply(S, M, Q):
        out = torch.empty_like(Q)
        n = Q.numel() // (64 * 64)
        wk.wkv7_state_apply(S, M, Q, out, n, 64, stream)
        return out

    return apply


def _range_map(wk, x, B, T, H, stream, out=None):
    """(M, Q) of a dense range [B, T, H, 64] by wkv7_state_map, written into
    ``out`` ([2, B, H, 64, 64] fp32) when given."""
    import torch

    if out is None:
        out = torch.empty((2, B, H, 64, 64), dtype=torch.float32, device=x["r"].device)
    wk.wkv7_state_map(x["r"], x["w_log"], x["k"], x["v"], x["a"], x["b"], out[0], out[1], B, T, H, 64, None,
                      stream)
    return out[0], out[1]


def gather_maps(mine, group=None):
    """Every rank's map, in rank order: ``mine`` is this rank's [2, ...] stack of
    (M, Q); returns the list of all ranks' stacks (one all-gather over the
    group, on any backend)."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    out = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(out, mine.contiguous(), group=group)
    return out


def forward_split(r, w_log, k, v, a, b, s0=None, n_parts=2, stream=None):
    """One device, a dense batch [B, T, H, D] cut along its tokens into
    ``n_parts`` ranges: the map of every range but the last, the scan for the
    start states, then one wkv7_forward per range.  Returns ``(y, sT)`` as one
    call over the whole batch would (within the kernels' tolerance)."""
    import torch

    import linear_recurrent_lm_wkv7_b200 as wk

    B, T, H, D = r.shape
    ranges = [rg for rg in token_ranges(T, n_parts) if rg[1] > rg[0]]
    if not ranges:
        ranges = [(0, 0)]
    parts = []
    for t0, t1 in ranges:
        parts.append({n: x[:, t0:t1].contiguous() for n, x in
                      dict(r=r, w_log=w_log, k=k, v=v, a=a, b=b).items()})
    maps = [_range_map(wk, p, B, t1 - t0, H, stream) for p, (t0, t1) in zip(parts[:-1], ranges[:-1])]
    maps.append(None)
    starts = start_states(maps, s0, _device_apply(wk, stream))
    ys = []
    sT = torch.empty((B, H, D, D), dtype=torch.float32, device=r.device)
    for p, (t0, t1), S in zip(parts, ranges, starts):
        y = torch.empty_like(p["r"])
        wk.wkv7_forward(p["r"], p["w_log"], p["k"], p["v"], p["a"], p["b"], S, y, sT, B, t1 - t0, H, D, None,
                        stream)
        ys.append(y)
    return torch.cat(ys, dim=1), sT


def forward_sequence_parallel(r, w_log, k, v, a, b, s0=None, group=None, stream=None):
    """Sequence parallelism across the ranks of ``group``: rank j holds token
    range j (in rank order) of the same dense batch, [B, T_j, H, D] on its own
    device, and ``s0`` (the batch's initial states, or None) is given on every
    rank.  Every rank but the last computes its range's map; the maps are
    all-gathered (one collective of 2 x B x H x 64 x 64 fp32 per rank); rank j
    folds the maps of ranks < j into its start state and runs wkv7_forward from
    it.  Returns ``(y_j, sT_j)``: this rank's outputs and the state at the end of
    its range (the last rank's is the batch's final state)."""
    import torch
    import torch.distributed as dist

    import linear_recurrent_lm_wkv7_b200 as wk

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, T, H, D = r.shape
    x = dict(r=r, w_log=w_log, k=k, v=v, a=a, b=b)
    mine = torch.zeros((2, B, H, D, D), dtype=torch.float32, device=r.device)
    if rank < world - 1:  # nobody starts after the last range
        _range_map(wk, x, B, T, H, stream, out=mine)
    stacks = gather_maps(mine, group)
    maps = [(m[0], m[1]) for m in stacks[:rank]] + [None]
    S = start_states(maps, s0, _device_apply(wk, stream))[-1]
    y = torch.empty_like(r)
    sT = torch.empty((B, H, D, D), dtype=torch.float32, device=r.device)
    wk.wkv7_forward(r, w_log, k, v, a, b, S, y, sT, B, T, H, D, None, stream)
    return y, sT


_SIDE_STREAMS = {}


def _side_streams(device, n):
    import torch

    idx = device.index if device.index is not None else torch.cuda.current_device()
    have = _SIDE_STREAMS.setdefault(idx, [])
    while len(have) < n:
        have.append(torch.cuda.Stream(device))
    return have[:n]


def forward_long(r, w_log, k, v, a, b, s0=None, n_parts=3, stream=None):
    """One long sequence (a dense batch with B = 1) on one device, cut into
    ``n_parts`` token ranges that run side by side.  A single sequence has only
    H (sequence, head) units, fewer than the SMs; cutting it multiplies the
    units that run at once.  Phase 1, concurrently: range 0 from s0 (which
    gives y of range 0 and the start state of range 1) and the map of every
    middle range (its Q and its M as two separate launches); then the start
    states by the scan; phase 2, concurrently: ranges 1 .. n_parts-1 from their
    start states.  Work on the side streams is ordered after ``stream``
    (default: the current stream), which then waits for all of it.  Returns
    ``(y, sT)`` as one wkv7_forward call would (within the kernels' tolerance);
    with H = 40 heads and 148 SMs, n_parts = 3 keeps each phase within one wave
    of blocks (3 x 40 in phase 1, 2 x 40 in phase 2)."""
    import torch

    import linear_recurrent_lm_wkv7_b200 as wk

    B, T, H, D = r.shape
    if B != 1:
        raise ValueError("forward_long takes one sequence (B = 1)")
    ranges = [rg for rg in token_ranges(T, n_parts) if rg[1] > rg[0]]
    y = torch.empty_like(r)
    sT = torch.empty((1, H, D, D), dtype=torch.float32, device=r.device)
    st = stream if stream is not None else torch.cuda.current_stream(r.device)
    if len(ranges) <= 1:
        wk.wkv7_forward(r, w_log, k, v, a, b, s0, y, sT, B, T, H, D, None, st)
        return y, sT
    P = len(ranges)
    view = lambda x, rg: x[:, rg[0]:rg[1]]  # contiguous for B = 1
    part = lambda rg: [view(x, rg) for x in (r, w_log, k, v, a, b)]
    state = lambda: torch.empty((1, H, D, D), dtype=torch.float32, device=r.device)
    # every buffer is allocated on the caller's stream before the side streams start
    starts = [None] + [state() for _ in range(1, P)]
    maps = [(state(), state()) for _ in range(1, P - 1)]
    ends = [state() for _ in range(1, P - 1)] + [sT]
    side = _side_streams(r.device, max(1 + 2 * (P - 2), P - 1))
    start = torch.cuda.Event()
    start.record(st)
    for s_ in side:
        s_.wait_event(start)
    # ---- phase 1: range 0 from s0; the maps (Q and M as two launches) of the middle ranges
    t_of = lambda j: ranges[j][1] - ranges[j][0]
    wk.wkv7_forward(*part(ranges[0]), s0, view(y, ranges[0]), starts[1], B, t_of(0), H, D, None, side[0])
    for j in range(1, P - 1):
        Mj, Qj = maps[j - 1]
        wk.wkv7_state_map(*part(ranges[j]), None, Qj, B, t_of(j), H, D, None, side[2 * j - 1])
        wk.wkv7_state_map(*part(ranges[j]), Mj, None, B, t_of(j), H, D, None, side[2 * j])
    for s_ in side[:1 + 2 * (P - 2)]:
        e = torch.cuda.Event()
        e.record(s_)
        st.wait_event(e)
    # ---- the scan, on the caller's stream: S_{j+1} = S_j M_j + Q_j
    for j in range(2, P):
        Mj, Qj = maps[j - 2]
        wk.wkv7_state_apply(starts[j - 1], Mj, Qj, starts[j], H, D, st)
    scan = torch.cuda.Event()
    scan.record(st)
    # ---- phase 2: ranges 1 .. P-1 from their start states
    for j in range(1, P):
        s_ = side[j - 1]
        s_.wait_event(scan)
        wk.wkv7_forward(*part(ranges[j]), starts[j], view(y, ranges[j]), ends[j - 1], B, t_of(j), H, D, None, s_)
        e = torch.cuda.Event()
        e.record(s_)
        st.wait_event(e)
    return y, sT
