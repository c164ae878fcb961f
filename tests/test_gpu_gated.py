"""GPU parity of wkv7_forward_gated (prefill with the gated read-out
z = (y / sqrt(D) + (sum_d r k r_k) v) * g) against the fp64 oracle, through the
C ABI.  Same metric and bounds as the plain prefill: max|out - ref| / max|ref|
<= 2e-3 for fp32 inputs and <= 2e-2 for bf16 inputs, for z and for sT."""
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
    from linear_recurrent_lm_wkv7_b200 import build

    build.build()
    import linear_recurrent_lm_wkv7_b200 as wk

    return wk


def relerr(out, ref):
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(out)), "non-finite output"
    return float(np.max(np.abs(out - ref)) / max(np.max(np.abs(ref)), 1e-30))


def run_both(wk, oracle_mod, inp, seed):
    rk, g = W.make_gate(inp.r.shape, inp.H, inp.D, io=inp.io, seed=seed)
    t = inp.tensors()
    d = {k: x.cuda() for k, x in t.items()}
    s0 = inp.s0.cuda() if inp.s0 is not None else None
    offs = inp.seq_offsets.cuda() if inp.seq_offsets is not None else None
    z, sT = wk.forward_gated(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], rk.cuda(), g.cuda(), s0, offs)
    assert wk.wkv7_get_device_status() == 0
    f64 = lambda x: x.double().numpy()
    zr, sr = oracle_mod.forward_gated(*(f64(t[n]) for n in ("r", "w_log", "k", "v", "a", "b")), f64(rk), f64(g),
                                      f64(inp.s0) if inp.s0 is not None else None,
                                      inp.seq_offsets.numpy() if inp.seq_offsets is not None else None)
    return z.float().cpu().numpy(), sT.cpu().numpy(), zr, sr


def check(wk, oracle_mod, inp, seed=0):
    z, sT, zr, sr = run_both(wk, oracle_mod, inp, seed)
    tol = TOL[inp.io]
    ez, es = relerr(z, zr), relerr(sT, sr)
    assert ez <= tol and es <= tol, (ez, es)


def test_gated_tiny_f32(wk, oracle_mod):
    """fp32 inputs: the recurrence kernel followed by the separate read-out pass."""
    check(wk, oracle_mod, W.make_workload("tiny_f32"), seed=1)


@pytest.mark.parametrize("T", [1, 63, 64, 130, 200])
@pytest.mark.parametrize("wdt", ["f32", "bf16"])
def test_gated_dense_bf16(wk, oracle_mod, T, wdt):
    """bf16 inputs: the read-out applied inside the prefill kernel; ragged tails."""
    check(wk, oracle_mod, W.make_prefill(2, T, 3, io="bf16", wdt=wdt, s0_std=0.1, seed=300 + T), seed=T)


@pytest.mark.parametrize("T", [7, 130])
def test_gated_dense_f32(wk, oracle_mod, T):
    check(wk, oracle_mod, W.make_prefill(2, T, 2, io="f32", wdt="f32", s0_std=0.1, seed=400 + T), seed=T)


def test_gated_packed_with_pads(wk, oracle_mod):
    lengths = [0, 5, 64, 100, 1, 190]
    pads = [3, 0, 7, 1, 0, 63]
    check(wk, oracle_mod, W.make_packed(lengths, pads, 2, io="bf16", wdt="f32", s0_std=0.1, seed=55), seed=5)


def test_gated_prefill_1p5b_full(wk, oracle_mod):
    """The benchmark workload (B4 T1024 H32, zero initial state), every head."""
    check(wk, oracle_mod, W.make_workload("prefill_1p5b"), seed=9)


def test_gated_matches_plain_forward(wk):
    """z equals the read-out applied in fp32 to the plain forward's y (which is
    bf16-rounded, hence the bf16-level bound), and sT agrees with the plain
    forward's."""
    inp = W.make_prefill(2, 200, 4, io="bf16", wdt="f32", s0_std=0.1, seed=77)
    rk, g = W.make_gate(inp.r.shape, inp.H, inp.D, io="bf16", seed=78)
    d = {k: x.cuda() for k, x in inp.tensors().items()}
    s0 = inp.s0.cuda()
    y, s1 = wk.forward(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], s0)
    z, s2 = wk.forward_gated(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], rk.cuda(), g.cuda(), s0)
    assert wk.wkv7_get_device_status() == 0
    assert relerr(s2.cpu().numpy(), s1.cpu().numpy()) <= 1e-6
    r, k, v = (d[n].float() for n in ("r", "k", "v"))
    u = (r * k * rk.cuda()[None, None]).sum(-1, keepdim=True)
    zref = (y.float() * 0.125 + u * v) * g.cuda().float()
    assert relerr(z.float().cpu().numpy(), zref.cpu().numpy()) <= 1e-2
