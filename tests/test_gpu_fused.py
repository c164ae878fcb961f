"""GPU parity of the fused prologue (wkv7_forward_fused, wkv7_decode_step_fused)
against the fp64 oracle, through the C ABI: raw k, v rows of H_kv kv heads and
a_lr in, the normalised key, a = -kk, b = kk a_lr and the scaled key formed
inside the kernels, optionally followed by the gated read-out.  Same metric and
bounds as the plain prefill: max|out - ref| / max|ref| <= 2e-3 for fp32 inputs
and <= 2e-2 for bf16 inputs, for the output rows and for the final state."""
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


def f64(x):
    return x.double().numpy() if x is not None else None


def check_prefill(wk, oracle_mod, inp, gated, seed=0):
    rk = g = None
    if gated:
        rk, g = W.make_gate(inp.r.shape, inp.H, inp.D, io=inp.io, seed=seed)
    t = inp.tensors()
    d = {k: x.cuda() for k, x in t.items()}
    s0 = inp.s0.cuda() if inp.s0 is not None else None
    offs = inp.seq_offsets.cuda() if inp.seq_offsets is not None else None
    out, sT = wk.forward_fused(d["r"], d["w_log"], d["k"], d["v"], d["a_lr"], s0, offs,
                               rk.cuda() if gated else None, g.cuda() if gated else None)
    assert wk.wkv7_get_device_status() == 0
    ref, sref = oracle_mod.forward_fused(*(f64(t[n]) for n in ("r", "w_log", "k", "v", "a_lr")), f64(inp.s0),
                                         inp.seq_offsets.numpy() if inp.seq_offsets is not None else None,
                                         f64(rk), f64(g))
    eo, es = relerr(out.float().cpu().numpy(), ref), relerr(sT.cpu().numpy(), sref)
    tol = TOL[inp.io]
    assert eo <= tol and es <= tol, (eo, es)


def test_fused_tiny_f32(wk, oracle_mod):
    """fp32 inputs, one 64-token chunk, two heads sharing one kv head."""
    check_prefill(wk, oracle_mod, W.make_fused(1, 64, 2, 1, io="f32", wdt="f32", seed=1), gated=False)


@pytest.mark.parametrize("gated", [False, True])
@pytest.mark.parametrize("wdt", ["f32", "bf16"])
def test_fused_dense_f32(wk, oracle_mod, gated, wdt):
    """fp32 inputs: prologue in the fp32 kernel; the read-out as a second pass."""
    inp = W.make_fused(2, 130, 4, 2, io="f32", wdt=wdt, s0_std=0.1, seed=600 + gated)
    check_prefill(wk, oracle_mod, inp, gated, seed=7)


@pytest.mark.parametrize("T", [1, 63, 64, 130, 200])
@pytest.mark.parametrize("wdt", ["f32", "bf16"])
def test_fused_dense_bf16(wk, oracle_mod, T, wdt):
    """bf16 inputs: the prologue in the prefill kernel's element-wise stage; ragged tails;
    4 heads over 2 kv heads."""
    check_prefill(wk, oracle_mod, W.make_fused(2, T, 4, 2, io="bf16", wdt=wdt, s0_std=0.1, seed=700 + T), False)


@pytest.mark.parametrize("H_kv", [1, 2, 4])
def test_fused_gated_bf16(wk, oracle_mod, H_kv):
    """Prologue and read-out both inside the bf16 kernel, for every kv sharing of 4 heads."""
    inp = W.make_fused(2, 130, 4, H_kv, io="bf16", wdt="f32", s0_std=0.1, seed=800 + H_kv)
    check_prefill(wk, oracle_mod, inp, gated=True, seed=H_kv)


@pytest.mark.parametrize("gated", [False, True])
def test_fused_packed_with_pads(wk, oracle_mod, gated):
    """Packed sequences with pad tokens (zero k and v rows: kk must come out 0)."""
    lengths = [0, 5, 64, 100, 1, 190]
    pads = [3, 0, 7, 1, 0, 63]
    inp = W.make_fused(0, 0, 4, 2, io="bf16", wdt="f32", s0_std=0.1, seed=66, lengths=lengths, pads=pads)
    check_prefill(wk, oracle_mod, inp, gated, seed=9)


@pytest.mark.parametrize("wdt", ["f32", "bf16"])
@pytest.mark.parametrize("gated", [False, True])
def test_fused_many_chunks_ragged(wk, oracle_mod, wdt, gated):
    """11 chunks per sequence with a ragged tail: the serial group runs pass 1 (the decay
    products) of each prep group's chunks after the first, handed over chunk by chunk."""
    inp = W.make_fused(2, 700, 4, 2, io="bf16", wdt=wdt, s0_std=0.1, seed=900 + gated)
    check_prefill(wk, oracle_mod, inp, gated, seed=12)


def test_fused_gated_full_size(wk, oracle_mod):
    """The 1.5B-class prefill (B4 T1024 H32) with 8 kv heads and the read-out, in
    the launch configuration of the benchmark."""
    inp = W.make_fused(4, 1024, 32, 8, io="bf16", wdt="f32", seed=11)
    check_prefill(wk, oracle_mod, inp, gated=True, seed=12)


@pytest.mark.parametrize("io,wdt", [("bf16", "bf16"), ("bf16", "f32"), ("f32", "f32")])
@pytest.mark.parametrize("gated", [False, True])
def test_fused_decode_steps(wk, oracle_mod, io, wdt, gated):
    """12 chained decode steps (state carried in place) against the oracle's fused
    decode step, 6 heads over 3 kv heads, one unit per block and several units
    per block (B = 40 gives 240 units)."""
    for B in (3, 40):
        H, H_kv, D = 6, 3, 64
        state = W.make_state(B, H, std=0.1, seed=B).cuda()
        sref = state.double().cpu().numpy()
        rk = g = None
        if gated:
            rk, _ = W.make_gate((B, H, D), H, D, io=io, seed=B)
        for step in range(12):
            inp = W.make_fused(B, 1, H, H_kv, io=io, wdt=wdt, seed=1000 * B + step)
            t = {n: x[:, 0].contiguous() for n, x in inp.tensors().items()}
            if gated:
                _, g = W.make_gate((B, H, D), H, D, io=io, seed=50 + step)
            d = {n: x.cuda() for n, x in t.items()}
            out = wk.decode_step_fused(d["r"], d["w_log"], d["k"], d["v"], d["a_lr"], state,
                                       rk.cuda() if gated else None, g.cuda() if gated else None)
            assert wk.wkv7_get_device_status() == 0
            ref, sref = oracle_mod.decode_step_fused(*(f64(t[n]) for n in ("r", "w_log", "k", "v", "a_lr")), sref,
                                                     f64(rk), f64(g))
            eo = relerr(out.float().cpu().numpy(), ref)
            assert eo <= TOL[io], (B, step, eo)
        es = relerr(state.cpu().numpy(), sref)
        assert es <= TOL[io], (B, es)


def test_fused_decode_matches_fused_prefill(wk):
    """T decode steps with the state carried equal a T-token fused prefill of the
    same inputs (both on the GPU)."""
    B, T, H, H_kv = 3, 20, 4, 2
    inp = W.make_fused(B, T, H, H_kv, io="bf16", wdt="f32", s0_std=0.1, seed=77)
    d = {n: x.cuda() for n, x in inp.tensors().items()}
    y, sT = wk.forward_fused(d["r"], d["w_log"], d["k"], d["v"], d["a_lr"], inp.s0.cuda())
    state = inp.s0.clone().cuda()
    ys = []
    for t in range(T):
        ys.append(wk.decode_step_fused(*(d[n][:, t].contiguous() for n in ("r", "w_log", "k", "v", "a_lr")), state))
    yd = torch.stack(ys, 1)
    assert wk.wkv7_get_device_status() == 0
    assert relerr(yd.float().cpu().numpy(), y.float().cpu().numpy()) <= 2e-2
    assert relerr(state.cpu().numpy(), sT.cpu().numpy()) <= 2e-2


def test_fused_decode_full_size(wk, oracle_mod):
    """The 2.9B-class decode batch (B256 H40) with 8 kv heads and the read-out, two
    chained steps, in the launch configuration of the benchmark."""
    B, H, H_kv, D = 256, 40, 8, 64
    state = W.make_state(B, H, std=0.1, seed=5).cuda()
    sref = state.double().cpu().numpy()
    rk, _ = W.make_gate((B, H, D), H, D, io="bf16", seed=6)
    for step in range(2):
        inp = W.make_fused(B, 1, H, H_kv, io="bf16", wdt="bf16", seed=2000 + step)
        t = {n: x[:, 0].contiguous() for n, x in inp.tensors().items()}
        _, g = W.make_gate((B, H, D), H, D, io="bf16", seed=70 + step)
        d = {n: x.cuda() for n, x in t.items()}
        out = wk.decode_step_fused(d["r"], d["w_log"], d["k"], d["v"], d["a_lr"], state, rk.cuda(), g.cuda())
        assert wk.wkv7_get_device_status() == 0
        ref, sref = oracle_mod.decode_step_fused(*(f64(t[n]) for n in ("r", "w_log", "k", "v", "a_lr")), sref,
                                                 f64(rk), f64(g))
        assert relerr(out.float().cpu().numpy(), ref) <= TOL["bf16"]
    assert relerr(state.cpu().numpy(), sref) <= TOL["bf16"]
