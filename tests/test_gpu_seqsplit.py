"""GPU: the affine maps of token ranges (wkv7_state_map, wkv7_state_apply) and
one sequence cut into ranges, against the fp64 oracle.

A range's map is S_end = S_start M + Q; the oracle's M and Q are the end states
of its recurrence from the identity with v = 0 and from zero (pinned on the CPU
against materialised transition products).  Bounds as for the states of the
prefill: max|out - ref| / max|ref| <= 2e-3 (fp32 inputs) and 2e-2 (bf16)."""
import numpy as np
import pytest
import torch

import wkv7_inputs as W

pytestmark = pytest.mark.gpu

TOL = {"f32": 2e-3, "bf16": 2e-2}


@pytest.fixture(scope="module")
def wk():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_recurrent_lm_wkv7_b200 as wk

    return wk


def relerr(out, ref):
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(out)), "non-finite output"
    return float(np.max(np.abs(out - ref)) / max(np.max(np.abs(ref)), 1e-30))


def f64(t):
    return t.double().numpy()


@pytest.mark.parametrize("io,wdt,T", [("bf16", "f32", 200), ("bf16", "bf16", 64), ("f32", "f32", 130),
                                      ("bf16", "f32", 1)])
def test_state_map_dense(wk, oracle_mod, io, wdt, T):
    inp = W.make_prefill(2, T, 3, io=io, wdt=wdt, seed=140 + T)
    t = inp.tensors()
    d = {n: x.cuda() for n, x in t.items()}
    M = torch.empty((2, 3, 64, 64), device="cuda")
    Q = torch.empty_like(M)
    wk.wkv7_state_map(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], M, Q, 2, T, 3, 64)
    assert wk.wkv7_get_device_status() == 0
    Mr, Qr = oracle_mod.state_map(*(f64(t[n]) for n in ("w_log", "k", "v", "a", "b")))
    assert relerr(M.cpu(), Mr) <= TOL[io]
    assert relerr(Q.cpu(), Qr) <= TOL[io]


def test_state_map_packed_and_empty(wk, oracle_mod):
    """Packed batch with pads and an empty sequence (whose map is the identity),
    and T == 0 (every map the identity)."""
    inp = W.make_packed([70, 0, 129, 5], [3, 2, 0, 60], 2, io="bf16", wdt="f32", seed=150)
    t = inp.tensors()
    d = {n: x.cuda() for n, x in t.items()}
    offs = inp.seq_offsets.cuda()
    M = torch.full((4, 2, 64, 64), float("nan"), device="cuda")
    Q = torch.full_like(M, float("nan"))
    wk.wkv7_state_map(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], M, Q, 4, inp.T, 2, 64, offs)
    assert wk.wkv7_get_device_status() == 0
    Mr, Qr = oracle_mod.state_map(*(f64(t[n]) for n in ("w_log", "k", "v", "a", "b")),
                                  seq_offsets=inp.seq_offsets.numpy())
    assert relerr(M.cpu(), Mr) <= TOL["bf16"] and relerr(Q.cpu(), Qr) <= TOL["bf16"]
    dummy = torch.empty(8, device="cuda", dtype=torch.bfloat16)
    wk.wkv7_state_map(dummy, torch.empty(8, device="cuda"), dummy, dummy, dummy, dummy, M, Q, 4, 0, 2, 64)
    torch.cuda.synchronize()
    assert torch.equal(M.cpu(), torch.eye(64).expand(4, 2, 64, 64)) and torch.equal(Q.cpu(), torch.zeros_like(Q.cpu()))


def test_state_apply(wk):
    """S_out = S_in M + Q in fp32, in place and from a zero state."""
    g = torch.Generator().manual_seed(160)
    S, M, Q = (torch.randn((3, 64, 64), generator=g) for _ in range(3))
    ref = (S.double() @ M.double() + Q.double()).numpy()
    Sd, Md, Qd = S.cuda(), M.cuda(), Q.cuda()
    out = torch.empty_like(Sd)
    wk.wkv7_state_apply(Sd, Md, Qd, out, 3, 64)
    torch.cuda.synchronize()
    assert relerr(out.cpu(), ref) <= 1e-5
    wk.wkv7_state_apply(Sd, Md, Qd, Sd, 3, 64)  # in place
    torch.cuda.synchronize()
    assert relerr(Sd.cpu(), ref) <= 1e-5
    wk.wkv7_state_apply(None, Md, Qd, out, 3, 64)
    torch.cuda.synchronize()
    assert torch.equal(out.cpu(), Q)


@pytest.mark.parametrize("n_parts", [2, 4, 8])
def test_long_prefill_cut_into_ranges(wk, oracle_mod, n_parts):
    """B1 T16384 H40 (the long-context workload, N(0, 0.1^2) initial state) cut
    into ranges: maps, scan, and one prefill per range; y and the final state
    against the oracle on three sampled heads."""
    from linear_recurrent_lm_wkv7_b200 import sharding

    inp = W.make_workload("prefill_2p9b_long")
    t = inp.tensors()
    d = {n: x.cuda() for n, x in t.items()}
    y, sT = sharding.forward_split(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], inp.s0.cuda(), n_parts)
    assert wk.wkv7_get_device_status() == 0
    heads = [0, 19, 39]
    hs = lambda x: f64(x[..., heads, :].contiguous())
    yr, sr = oracle_mod.forward(*(hs(t[n]) for n in ("r", "w_log", "k", "v", "a", "b")),
                                f64(inp.s0[:, heads].contiguous()))
    assert relerr(y.float().cpu()[..., heads, :], yr) <= TOL["bf16"]
    assert relerr(sT.cpu()[:, heads], sr) <= TOL["bf16"]


def test_sequence_parallel_single_rank_group(wk):
    """forward_sequence_parallel through a one-rank NCCL group (the all-gather
    path on one device) equals wkv7_forward on the same range."""
    import os

    import torch.distributed as dist

    from linear_recurrent_lm_wkv7_b200 import sharding

    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29531")
    inp = W.make_prefill(2, 200, 3, io="bf16", wdt="f32", s0_std=0.1, seed=170)
    d = {n: x.cuda() for n, x in inp.tensors().items()}
    s0 = inp.s0.cuda()
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        y, sT = sharding.forward_sequence_parallel(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], s0)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    y_ref, s_ref = wk.forward(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], s0)
    assert torch.equal(y, y_ref) and torch.equal(sT, s_ref)


@pytest.mark.parametrize("n_parts", [2, 3, 5])
def test_long_prefill_overlapped_ranges(wk, oracle_mod, n_parts):
    """forward_long: one sequence (B1 T16384 H40, N(0, 0.1^2) initial state) whose
    ranges run side by side on several streams (range 0 with the maps of the
    middle ranges, then the other ranges from their scanned start states); y and
    the final state against the oracle on three sampled heads."""
    from linear_recurrent_lm_wkv7_b200 import sharding

    inp = W.make_workload("prefill_2p9b_long")
    t = inp.tensors()
    d = {n: x.cuda() for n, x in t.items()}
    y, sT = sharding.forward_long(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], inp.s0.cuda(), n_parts)
    torch.cuda.synchronize()
    assert wk.wkv7_get_device_status() == 0
    heads = [0, 19, 39]
    hs = lambda x: f64(x[..., heads, :].contiguous())
    yr, sr = oracle_mod.forward(*(hs(t[n]) for n in ("r", "w_log", "k", "v", "a", "b")),
                                f64(inp.s0[:, heads].contiguous()))
    assert relerr(y.float().cpu()[..., heads, :], yr) <= TOL["bf16"]
    assert relerr(sT.cpu()[:, heads], sr) <= TOL["bf16"]
