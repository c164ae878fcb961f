"""GPU parity of wkv7_backward (gradient of <dy, y> + <dsT, sT> with respect to
r, w_log, k, v, a, b and s0) against the fp64 oracle's backward, through the C
ABI.  Same metric and bounds as the forward: max|out - ref| / max|ref| <= 2e-3
for a gradient stored in fp32 and <= 2e-2 for one stored in bf16 (each gradient
takes its input's storage type; bf16 rounding alone is 2^-9 relative)."""
import numpy as np
import pytest
import torch

import wkv7_inputs as W

pytestmark = pytest.mark.gpu

TOL = {"f32": 2e-3, "bf16": 2e-2}
NAMES = ("dr", "dw_log", "dk", "dv", "da", "db", "ds0")


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


def check(wk, oracle_mod, inp, seed=0, with_dsT=True):
    dy, dsT = W.make_upstream(inp.r.shape, inp.B, inp.H, io=inp.io, seed=seed, with_dsT=with_dsT)
    t = inp.tensors()
    d = {n: x.cuda() for n, x in t.items()}
    s0 = inp.s0.cuda() if inp.s0 is not None else None
    offs = inp.seq_offsets.cuda() if inp.seq_offsets is not None else None
    got = wk.backward(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], dy.cuda(), s0,
                      dsT.cuda() if dsT is not None else None, offs)
    assert wk.wkv7_get_device_status() == 0
    f64 = lambda x: x.double().numpy() if x is not None else None
    ref = oracle_mod.backward(*(f64(t[n]) for n in ("r", "w_log", "k", "v", "a", "b")), f64(dy), f64(inp.s0),
                              f64(dsT), inp.seq_offsets.numpy() if inp.seq_offsets is not None else None)
    errs = {n: relerr(g.float().cpu().numpy(), rf) for n, g, rf in zip(NAMES, got, ref)}
    # each gradient is stored in its input's type: dw_log in w_log's, ds0 in fp32
    tol = {n: TOL[inp.wdt] if n == "dw_log" else TOL[inp.io] for n in NAMES}
    assert all(errs[n] <= tol[n] for n in NAMES), errs


def test_backward_tiny_f32(wk, oracle_mod):
    check(wk, oracle_mod, W.make_prefill(1, 64, 2, io="f32", wdt="f32", s0_std=0.1, seed=1), seed=1)


@pytest.mark.parametrize("T", [1, 63, 64, 130])
@pytest.mark.parametrize("wdt", ["f32", "bf16"])
def test_backward_dense_bf16(wk, oracle_mod, T, wdt):
    """bf16 inputs, ragged tails, a partial and several chunks."""
    check(wk, oracle_mod, W.make_prefill(2, T, 3, io="bf16", wdt=wdt, s0_std=0.1, seed=500 + T), seed=T)


def test_backward_dense_f32_no_state(wk, oracle_mod):
    """fp32 inputs, no initial state and no gradient on the final state."""
    check(wk, oracle_mod, W.make_prefill(2, 130, 2, io="f32", wdt="f32", s0_std=None, seed=9), seed=9,
          with_dsT=False)


@pytest.mark.parametrize("T", [1, 63, 200])
def test_backward_dense_f32_bf16_decay(wk, oracle_mod, T):
    """fp32 inputs with bf16 decay logits (the mixed pair of storage types)."""
    check(wk, oracle_mod, W.make_prefill(2, T, 3, io="f32", wdt="bf16", s0_std=0.1, seed=700 + T), seed=T)


def test_backward_packed_f32(wk, oracle_mod):
    """fp32 inputs in a packed batch with pads and a sequence of one token."""
    check(wk, oracle_mod, W.make_packed([70, 1, 129, 64], [5, 0, 17, 3], 2, io="f32", wdt="f32", s0_std=0.1,
                                        seed=710), seed=711)


def test_backward_packed_with_pads(wk, oracle_mod):
    lengths = [0, 5, 64, 100, 1, 130]
    pads = [3, 0, 7, 1, 0, 63]
    check(wk, oracle_mod, W.make_packed(lengths, pads, 2, io="bf16", wdt="f32", s0_std=0.1, seed=56), seed=6)


def test_backward_prefill_1p5b_full(wk, oracle_mod):
    """The 1.5B-class prefill (B4 T1024 H32), in the launch configuration of the benchmark."""
    check(wk, oracle_mod, W.make_workload("prefill_1p5b"), seed=21)


def test_backward_zero_tokens(wk):
    """T = 0: no token to differentiate; ds0 is dsT itself, or zero without dsT."""
    B, H = 2, 3
    r = torch.empty((B, 0, H, 64), dtype=torch.bfloat16, device="cuda")
    wl = torch.empty((B, 0, H, 64), dtype=torch.float32, device="cuda")
    _, dsT = W.make_upstream((B, 0, H, 64), B, H, io="bf16", seed=3)
    got = wk.backward(r, wl, r, r, r, r, r, None, dsT.cuda())
    assert wk.wkv7_get_device_status() == 0
    assert torch.equal(got[6].cpu(), dsT)
    got = wk.backward(r, wl, r, r, r, r, r)
    assert torch.count_nonzero(got[6]).item() == 0


def _constant_decay(inp, value):
    """The same inputs with every decay logit set to `value` (pad tokens of a
    packed batch keep their -inf)."""
    w = inp.w_log
    pad = torch.isneginf(w.float())
    inp.w_log = torch.where(pad, w, torch.full_like(w, value)).contiguous()
    return inp


@pytest.mark.parametrize("io,wdt", [("bf16", "f32"), ("bf16", "bf16"), ("f32", "f32")])
def test_backward_decay_at_the_bound(wk, oracle_mod, io, wdt):
    """w_log = -0.5 on every token (w = 0.545): a 64-token chunk decays by e^-38.8,
    the extreme the chunked form's 1 / Gamma scaling carries through every product
    of the adjoint.  Four chunks, the last ragged, non-zero initial state and dsT."""
    inp = _constant_decay(W.make_prefill(2, 200, 3, io=io, wdt=wdt, s0_std=0.1, seed=130), -0.5)
    check(wk, oracle_mod, inp, seed=131)


def test_backward_decay_bound_packed_with_pads(wk, oracle_mod):
    """The bound on every real token of a packed batch whose pads carry -inf (w = 1)."""
    inp = _constant_decay(W.make_packed([150, 64, 7, 130], [13, 63, 0, 40], 3, io="bf16", wdt="f32",
                                        s0_std=0.1, seed=132), -0.5)
    check(wk, oracle_mod, inp, seed=133)


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_backward_decay_beyond_exact_range_is_reported(wk, io):
    """w_log = 1 (w = e^-e): Gamma of a 64-token chunk falls below 1e-30, outside the
    chunked form's exact range; the backward reports WKV7_ERR_DECAY_RANGE (-8) like
    the prefill, instead of returning inf or NaN with status OK."""
    inp = _constant_decay(W.make_prefill(1, 130, 2, io=io, wdt="f32", s0_std=0.1, seed=134), 1.0)
    dy, dsT = W.make_upstream(inp.r.shape, inp.B, inp.H, io=inp.io, seed=135)
    d = {n: x.cuda() for n, x in inp.tensors().items()}
    wk.backward(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], dy.cuda(), inp.s0.cuda(), dsT.cuda())
    assert wk.wkv7_get_device_status() == -8
    assert wk.wkv7_get_device_status() == 0  # read and cleared


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_backward_long_sequence(wk, oracle_mod, io):
    """B1 T4096 H2: 64 chunks, so both boundary scans run 64 steps; their fp32
    accuracy (tf32 high and low parts of the carried state) keeps the first
    chunk's gradients and ds0 within the bound."""
    check(wk, oracle_mod, W.make_prefill(1, 4096, 2, io=io, wdt="f32", s0_std=0.1, seed=136), seed=137)


def test_backward_many_short_packed(wk, oracle_mod):
    """40 packed sequences of 1 .. 70 tokens with pads: the persistent map kernel's
    items include chunk slots past the last real chunk (the packed workspace bound
    is ceil(T / 64) + B chunks per head), and most sequences are one ragged chunk."""
    g = torch.Generator().manual_seed(140)
    lengths = torch.randint(1, 71, (40,), generator=g).tolist()
    pads = torch.randint(0, 4, (40,), generator=g).tolist()
    check(wk, oracle_mod, W.make_packed(lengths, pads, 2, io="bf16", wdt="f32", s0_std=0.1, seed=141), seed=142)


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_backward_is_deterministic(wk, io):
    """No atomics anywhere: two calls on the same inputs give the same bits."""
    inp = W.make_prefill(2, 300, 3, io=io, wdt="f32", s0_std=0.1, seed=143)
    dy, dsT = W.make_upstream(inp.r.shape, inp.B, inp.H, io=inp.io, seed=144)
    d = {n: x.cuda() for n, x in inp.tensors().items()}
    args = (d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], dy.cuda(), inp.s0.cuda(), dsT.cuda())
    first = wk.backward(*args)
    second = wk.backward(*args)
    assert wk.wkv7_get_device_status() == 0
    for x, y in zip(first, second):
        assert torch.equal(x, y)
