"""GPU parity of wkv7_forward_long (two-phase prefill: every chunk's
state-independent part in parallel, then one state pass per (sequence, head))
against the fp64 oracle, through the C ABI.  Same metric and bound as the
prefill: max|out - ref| / max|ref| <= 2e-2 for bf16 inputs."""
import numpy as np
import pytest
import torch

import wkv7_inputs as W

pytestmark = pytest.mark.gpu

TOL = 2e-2


@pytest.fixture(scope="module")
def wk():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_recurrent_lm_wkv7_b200 import build

    build.build()
    import linear_recurrent_lm_wkv7_b200 as wk

    return wk


def relerr(out, ref):
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(out)), "non-finite output"
    return float(np.max(np.abs(out - ref)) / max(np.max(np.abs(ref)), 1e-30))


def run_long(wk, inp):
    d = {k: t.cuda() for k, t in inp.tensors().items()}
    s0 = inp.s0.cuda() if inp.s0 is not None else None
    y, sT = wk.forward_long(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], s0)
    assert wk.wkv7_get_device_status() == 0
    return y.float().cpu().numpy(), sT.cpu().numpy()


def oracle_forward(oracle_mod, inp, heads=None):
    t = inp.tensors()
    s0 = inp.s0
    if heads is not None:
        t = {k: v[..., heads, :].contiguous() for k, v in t.items()}
        s0 = s0[:, heads].contiguous() if s0 is not None else None
    f64 = lambda x: x.double().numpy()
    return oracle_mod.forward(*(f64(t[n]) for n in ("r", "w_log", "k", "v", "a", "b")),
                              f64(s0) if s0 is not None else None)


def check(wk, oracle_mod, inp, heads=None):
    y, sT = run_long(wk, inp)
    yr, sr = oracle_forward(oracle_mod, inp, heads)
    if heads is not None:
        y, sT = y[..., heads, :], sT[:, heads]
    ey, es = relerr(y, yr), relerr(sT, sr)
    assert ey <= TOL and es <= TOL, (ey, es)


@pytest.mark.parametrize("T", [1, 63, 130, 512, 1100])
@pytest.mark.parametrize("wdt", ["f32", "bf16"])
def test_long_dense_lengths(wk, oracle_mod, T, wdt):
    """One partial chunk, a ragged chunk, and 3, 8 and 18 chunks per sequence: the
    first phase's blocks take chunks of different sequences, heads and positions
    in turn (fewer slots than SMs for the short cases)."""
    check(wk, oracle_mod, W.make_prefill(2, T, 3, io="bf16", wdt=wdt, s0_std=0.1, seed=800 + T))


@pytest.mark.parametrize("B,T,H", [(4, 200, 10), (8, 130, 20)])
def test_long_wider_batches(wk, oracle_mod, B, T, H):
    """40 and 160 (sequence, head) units: the state pass splits each unit over
    four blocks of 16 value columns, or runs it whole (64 columns) when four
    blocks per unit would not stay resident."""
    check(wk, oracle_mod, W.make_prefill(B, T, H, io="bf16", wdt="f32", s0_std=0.1, seed=820 + B))


def test_long_no_initial_state(wk, oracle_mod):
    check(wk, oracle_mod, W.make_prefill(3, 700, 2, io="bf16", wdt="f32", s0_std=None, seed=811))


def test_long_decay_at_the_bound(wk, oracle_mod):
    """w_log = -0.5 on every token: each chunk decays by e^-38.8, over 21 chunks."""
    inp = W.make_prefill(1, 1300, 2, io="bf16", wdt="f32", s0_std=0.1, seed=812)
    inp.w_log = torch.full_like(inp.w_log, -0.5)
    check(wk, oracle_mod, inp)


def test_long_decay_beyond_exact_range_is_reported(wk):
    inp = W.make_prefill(1, 600, 2, io="bf16", wdt="f32", s0_std=0.1, seed=813)
    inp.w_log = torch.full_like(inp.w_log, 1.0)
    d = {k: t.cuda() for k, t in inp.tensors().items()}
    wk.forward_long(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], inp.s0.cuda())
    assert wk.wkv7_get_device_status() == -8
    assert wk.wkv7_get_device_status() == 0


@pytest.mark.parametrize("mu_z", [1.0, -3.0])
def test_long_2p9b_sampled(wk, oracle_mod, mu_z):
    """B1 T16384 H40 with N(0, 0.1^2) initial states (both decay draws), the
    oracle on three sampled heads; also against the one-pass prefill."""
    inp = W.make_workload("prefill_2p9b_long", mu_z=mu_z)
    y, sT = run_long(wk, inp)
    heads = [0, 19, 39]
    yr, sr = oracle_forward(oracle_mod, inp, heads)
    ey, es = relerr(y[..., heads, :], yr), relerr(sT[:, heads], sr)
    assert ey <= TOL and es <= TOL, (ey, es)
    d = {k: t.cuda() for k, t in inp.tensors().items()}
    y1, s1 = wk.forward(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], inp.s0.cuda())
    assert relerr(y, y1.float().cpu().numpy()) <= 1e-2
    assert relerr(sT, s1.cpu().numpy()) <= 1e-2


def test_long_state_in_place_and_zero_tokens(wk):
    inp = W.make_prefill(2, 200, 2, io="bf16", wdt="f32", s0_std=0.1, seed=814)
    d = {k: t.cuda() for k, t in inp.tensors().items()}
    s0 = inp.s0.cuda()
    y, sT = wk.forward_long(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], s0)
    s = s0.clone()
    y2 = torch.empty_like(d["r"])
    ws = torch.empty(wk.wkv7_forward_long_workspace_bytes(2, 200, 2, 64), dtype=torch.uint8, device="cuda")
    wk.wkv7_forward_long(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], s, y2, s, ws, 2, 200, 2, 64)
    torch.testing.assert_close(y2, y, rtol=0, atol=0)
    torch.testing.assert_close(s, sT, rtol=0, atol=0)
    e = {k: t[:, :0].contiguous() for k, t in d.items()}
    out = torch.empty((2, 2, 64, 64), device="cuda")
    wk.wkv7_forward_long(e["r"], e["w_log"], e["k"], e["v"], e["a"], e["b"], s0, e["r"].clone(), out, ws, 2, 0, 2,
                         64)
    torch.cuda.synchronize()
    torch.testing.assert_close(out, s0, rtol=0, atol=0)


def test_long_is_deterministic(wk):
    inp = W.make_prefill(1, 1500, 3, io="bf16", wdt="f32", s0_std=0.1, seed=815)
    d = {k: t.cuda() for k, t in inp.tensors().items()}
    args = (d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], inp.s0.cuda())
    a = wk.forward_long(*args)
    b = wk.forward_long(*args)
    for x, z in zip(a, b):
        assert torch.equal(x, z)


def test_million_token_context(wk, oracle_mod):
    """B1 T1048576 H1 with the long-memory decay draw (median w 0.97) and a
    non-zero initial state: 16,384 chunks of state carried through both prefill
    forms (the pages' long-context claim reaches 1M tokens).  Every output is
    compared with the oracle's."""
    inp = W.make_prefill(1, 1 << 20, 1, io="bf16", wdt="f32", s0_std=0.1, mu_z=-3.0, seed=902)
    yr, sr = oracle_forward(oracle_mod, inp)
    y, sT = run_long(wk, inp)
    ey, es = relerr(y, yr), relerr(sT, sr)
    assert ey <= TOL and es <= TOL, (ey, es)
    d = {k: t.cuda() for k, t in inp.tensors().items()}
    y1, s1 = wk.forward(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], inp.s0.cuda())
    assert wk.wkv7_get_device_status() == 0
    e1y, e1s = relerr(y1.float().cpu().numpy(), yr), relerr(s1.cpu().numpy(), sr)
    assert e1y <= TOL and e1s <= TOL, (e1y, e1s)
