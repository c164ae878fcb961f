"""GPU parity: the CUDA library (called through the C ABI) against the fp64
oracle on the same seeded inputs.

Metric: max|out - ref| / max|ref| over the whole compared tensor, for y and for
the final state.  Bounds: 2e-3 when the inputs are fp32 (tf32 tensor-core
operands) and 2e-2 when they are bf16 (bf16 operands, fp32 state).
"""
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


def to_dev(inp):
    d = {k: t.cuda() for k, t in inp.tensors().items()}
    s0 = inp.s0.cuda() if inp.s0 is not None else None
    offs = inp.seq_offsets.cuda() if inp.seq_offsets is not None else None
    return d, s0, offs


def gpu_forward(wk, inp, heads=None):
    d, s0, offs = to_dev(inp)
    y, sT = wk.forward(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], s0, offs)
    assert wk.wkv7_get_device_status() == 0
    y, sT = y.float().cpu().numpy(), sT.cpu().numpy()
    return y, sT


def oracle_forward(oracle_mod, inp, heads=None):
    t = inp.tensors()
    s0 = inp.s0
    if heads is not None:
        hsel = lambda x: x[..., heads, :].contiguous()
        t = {k: hsel(v) for k, v in t.items()}
        s0 = s0[:, heads].contiguous() if s0 is not None else None
    f64 = lambda x: x.double().numpy()
    return oracle_mod.forward(*(f64(t[n]) for n in ("r", "w_log", "k", "v", "a", "b")),
                              f64(s0) if s0 is not None else None,
                              seq_offsets=inp.seq_offsets.numpy() if inp.seq_offsets is not None else None)


def check_prefill(wk, oracle_mod, inp, heads=None, tol=None):
    y, sT = gpu_forward(wk, inp)
    yr, sr = oracle_forward(oracle_mod, inp, heads)
    if heads is not None:
        y, sT = y[..., heads, :], sT[:, heads]
    tol = tol or TOL[inp.io]
    ey, es = relerr(y, yr), relerr(sT, sr)
    assert ey <= tol and es <= tol, (ey, es)
    return ey, es


# ------------------------------------------------------------------ prefill
def test_tiny_f32_workload(wk, oracle_mod):
    """B1 T64 H2 D64, all fp32, zero initial state."""
    check_prefill(wk, oracle_mod, W.make_workload("tiny_f32"))


@pytest.mark.parametrize("T", [1, 7, 63, 64, 65, 130, 200])
@pytest.mark.parametrize("io,wdt", [("bf16", "f32"), ("bf16", "bf16"), ("f32", "f32"), ("f32", "bf16")])
def test_dense_ragged_lengths(wk, oracle_mod, T, io, wdt):
    """Several chunks and a ragged tail, with a non-zero initial state."""
    inp = W.make_prefill(2, T, 3, io=io, wdt=wdt, s0_std=0.1, seed=100 + T)
    check_prefill(wk, oracle_mod, inp)


def test_zero_initial_state_pointer(wk, oracle_mod):
    inp = W.make_prefill(1, 150, 2, io="bf16", wdt="f32", s0_std=None, seed=7)
    check_prefill(wk, oracle_mod, inp)


def test_long_memory_decay(wk, oracle_mod):
    """Decay close to one (z ~ N(-3, 1), median w ~ 0.97) over 8 chunks."""
    inp = W.make_prefill(1, 512, 2, io="bf16", wdt="f32", s0_std=0.1, mu_z=-3.0, seed=8)
    check_prefill(wk, oracle_mod, inp)


def _constant_decay(inp, value):
    """The same inputs with every decay logit set to `value` (pad tokens of a
    packed batch keep their -inf)."""
    w = inp.w_log
    pad = torch.isneginf(w.float())
    inp.w_log = torch.where(pad, w, torch.full_like(w, value)).contiguous()
    return inp


@pytest.mark.parametrize("io,wdt", [("bf16", "f32"), ("bf16", "bf16"), ("f32", "f32")])
def test_decay_at_the_parametrised_bound(wk, oracle_mod, io, wdt):
    """w_log = -0.5 on every token (w = 0.545, the fastest decay the hxa07D
    parametrisation produces): a 64-token chunk decays by e^-38.8 in every
    channel, the extreme the chunked algebra's 1 / Gamma scaling must carry.
    Four chunks, the last one ragged, non-zero initial state."""
    inp = _constant_decay(W.make_prefill(2, 200, 3, io=io, wdt=wdt, s0_std=0.1, seed=120), -0.5)
    check_prefill(wk, oracle_mod, inp)


def test_decay_bound_packed_with_pads(wk, oracle_mod):
    """w_log = -0.5 on every real token of a packed batch whose pad tokens carry
    -inf (w = 1): chunks mix the fastest decay with identity steps, and the
    sequence starts are not chunk aligned."""
    inp = _constant_decay(W.make_packed([150, 64, 7, 130], [13, 63, 0, 40], 3, io="bf16", wdt="f32",
                                        s0_std=0.1, seed=121), -0.5)
    check_prefill(wk, oracle_mod, inp)


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_decay_inside_exact_range_beyond_bound(wk, oracle_mod, io):
    """w_log = 0 on every token (w = 0.368, faster than the parametrisation
    allows): each chunk decays by e^-64, still inside the exact range
    (Gamma_64 >= 1e-30), so results stay within the parity bounds."""
    inp = _constant_decay(W.make_prefill(1, 200, 2, io=io, wdt="f32", s0_std=0.1, seed=122), 0.0)
    check_prefill(wk, oracle_mod, inp)
    assert wk.wkv7_get_device_status() == 0


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_decay_beyond_exact_range_is_reported(wk, io):
    """w_log = 1 on every token (w = 0.066): a 64-token chunk would decay by
    e^-174, below the exact range; the call reports WKV7_ERR_DECAY_RANGE in the
    device status instead of returning silently."""
    inp = _constant_decay(W.make_prefill(1, 130, 2, io=io, wdt="f32", s0_std=0.1, seed=123), 1.0)
    d, s0, _ = to_dev(inp)
    assert wk.wkv7_get_device_status() == 0
    wk.forward(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], s0)
    assert wk.wkv7_get_device_status() == -8
    assert wk.wkv7_get_device_status() == 0  # cleared by the read


def test_packed_with_pads_and_empty(wk, oracle_mod):
    """Packed batch: empty sequence, sub-chunk sequences, chunk-straddling
    starts, pad tokens (w_log = -inf, k = v = a = b = 0)."""
    lengths = [0, 5, 64, 100, 1, 190]
    pads = [3, 0, 7, 63, 0, 17]
    inp = W.make_packed(lengths, pads, 3, io="bf16", wdt="f32", s0_std=0.1, seed=9)
    check_prefill(wk, oracle_mod, inp)


def test_packed_f32(wk, oracle_mod):
    inp = W.make_packed([70, 3, 129], [2, 9, 0], 2, io="f32", wdt="f32", s0_std=0.1, seed=10)
    check_prefill(wk, oracle_mod, inp)


def test_prefill_1p5b_full(wk, oracle_mod):
    """B4 T1024 H32, bf16 inputs, fp32 decay logits, zero initial state: every head compared."""
    check_prefill(wk, oracle_mod, W.make_workload("prefill_1p5b"))


@pytest.mark.parametrize("mu_z", [1.0, -3.0])
def test_prefill_2p9b_long_sampled(wk, oracle_mod, mu_z):
    """B1 T16384 H40 with N(0, 0.1^2) initial state, full length; the oracle
    runs on three sampled heads (first, middle, last).  mu_z = 1 is the
    workload's literal decay formula; mu_z = -3 is the long-memory variant."""
    inp = W.make_workload("prefill_2p9b_long", mu_z=mu_z)
    check_prefill(wk, oracle_mod, inp, heads=[0, 19, 39])


def test_packed_1p5b_sampled(wk, oracle_mod):
    """16 packed sequences, lengths U{512..8192}, pads U{0..63}, H32; oracle on
    two sampled heads over every sequence."""
    inp = W.make_workload("packed_1p5b")
    check_prefill(wk, oracle_mod, inp, heads=[0, 31])


def test_chaining_through_states(wk):
    """forward(T) == forward(T1) then forward(T2, s0 = sT1), within tolerance;
    the split (T1 = 100) is not chunk-aligned."""
    inp = W.make_prefill(2, 300, 2, io="bf16", wdt="f32", s0_std=0.1, seed=11)
    d, s0, _ = to_dev(inp)
    y, sT = wk.forward(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], s0)
    T1 = 100
    p1 = {k: v[:, :T1].contiguous() for k, v in d.items()}
    p2 = {k: v[:, T1:].contiguous() for k, v in d.items()}
    y1, s1 = wk.forward(p1["r"], p1["w_log"], p1["k"], p1["v"], p1["a"], p1["b"], s0)
    y2, s2 = wk.forward(p2["r"], p2["w_log"], p2["k"], p2["v"], p2["a"], p2["b"], s1)
    yc = torch.cat([y1, y2], dim=1)
    assert relerr(yc.float().cpu(), y.float().cpu()) <= 2e-2
    assert relerr(s2.cpu(), sT.cpu()) <= 2e-2


def test_state_in_place(wk):
    """sT == s0 (state carried in place) gives the same result as separate buffers."""
    inp = W.make_prefill(2, 90, 2, io="bf16", wdt="f32", s0_std=0.1, seed=12)
    d, s0, _ = to_dev(inp)
    y, sT = wk.forward(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], s0)
    s = s0.clone()
    y2 = torch.empty_like(d["r"])
    wk.wkv7_forward(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], s, y2, s, 2, 90, 2, 64)
    torch.testing.assert_close(y2, y, rtol=0, atol=0)
    torch.testing.assert_close(s, sT, rtol=0, atol=0)


def test_zero_tokens_copies_state(wk):
    s0 = torch.randn(2, 3, 64, 64, device="cuda")
    sT = torch.empty_like(s0)
    e = torch.empty(0, device="cuda", dtype=torch.bfloat16)
    # T == 0: no token data is read; any aligned pointer may be passed
    dummy = torch.empty(8, device="cuda", dtype=torch.bfloat16)
    wk.wkv7_forward(dummy, torch.empty(8, device="cuda"), dummy, dummy, dummy, dummy, s0, dummy.clone(), sT,
                    2, 0, 3, 64)
    torch.cuda.synchronize()
    torch.testing.assert_close(sT, s0, rtol=0, atol=0)
    del e


# ------------------------------------------------------------------ decode
def test_decode_small(wk, oracle_mod):
    B, H = 3, 2
    s = W.make_state(B, H, seed=1)
    sd = s.cuda()
    ref = s.double().numpy()
    for step in range(5):
        inp = W.make_decode_step(B, H, io="bf16", wdt="bf16", seed=21, step=step)
        d = {k: t.cuda() for k, t in inp.tensors().items()}
        y = wk.decode_step(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], sd)
        yr, ref = oracle_mod.decode_step(*(inp.tensors()[n].double().numpy()
                                           for n in ("r", "w_log", "k", "v", "a", "b")), ref)
        assert relerr(y.float().cpu().numpy(), yr) <= 2e-2
    assert relerr(sd.cpu().numpy(), ref) <= 2e-2


@pytest.mark.parametrize("io,wdt", [("f32", "f32"), ("bf16", "f32")])
def test_decode_dtypes_out_of_place(wk, oracle_mod, io, wdt):
    B, H = 4, 3
    s = W.make_state(B, H, seed=2)
    inp = W.make_decode_step(B, H, io=io, wdt=wdt, seed=22)
    d = {k: t.cuda() for k, t in inp.tensors().items()}
    s_in = s.cuda()
    s_out = torch.empty_like(s_in)
    y = torch.empty_like(d["r"])
    wk.wkv7_decode_step(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], s_in, y, s_out, B, H, 64)
    yr, sr = oracle_mod.decode_step(*(inp.tensors()[n].double().numpy() for n in ("r", "w_log", "k", "v", "a", "b")),
                                    s.double().numpy())
    assert relerr(y.float().cpu().numpy(), yr) <= TOL[io]
    assert relerr(s_out.cpu().numpy(), sr) <= TOL[io]
    torch.testing.assert_close(s_in.cpu(), s, rtol=0, atol=0)  # input state untouched


def test_decode_2p9b_128_steps(wk, oracle_mod):
    """B256 H40, fp32 state carried through 128 steps of fresh bf16 inputs;
    y compared at every step, the state after the last step."""
    cfg = W.WORKLOADS["decode_2p9b"]
    B, H = cfg["B"], cfg["H"]
    s = W.make_state(B, H, std=cfg["s0_std"], seed=cfg["seed"])
    sd = s.cuda()
    ref = s.double().numpy()
    worst = 0.0
    for step in range(cfg["steps"]):
        inp = W.make_decode_step(B, H, io=cfg["io"], wdt=cfg["wdt"], seed=cfg["seed"], step=step)
        d = {k: t.cuda() for k, t in inp.tensors().items()}
        y = wk.decode_step(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], sd)
        yr, ref = oracle_mod.decode_step(*(inp.tensors()[n].double().numpy()
                                           for n in ("r", "w_log", "k", "v", "a", "b")), ref)
        worst = max(worst, relerr(y.float().cpu().numpy(), yr))
    assert worst <= 2e-2
    assert relerr(sd.cpu().numpy(), ref) <= 2e-2


def test_decode_equals_prefill(wk):
    """128 decode steps on the GPU equal a T = 128 prefill on the same inputs."""
    inp = W.make_prefill(2, 128, 2, io="bf16", wdt="bf16", s0_std=0.1, seed=13)
    d, s0, _ = to_dev(inp)
    y, sT = wk.forward(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], s0)
    s = s0.clone()
    ys = []
    for t in range(128):
        dt = {k: v[:, t].contiguous() for k, v in d.items()}
        ys.append(wk.decode_step(dt["r"], dt["w_log"], dt["k"], dt["v"], dt["a"], dt["b"], s))
    yd = torch.stack(ys, dim=1)
    assert relerr(yd.float().cpu(), y.float().cpu()) <= 2e-2
    assert relerr(s.cpu(), sT.cpu()) <= 2e-2


# ------------------------------------------------------------------ device-side errors
def test_bounded_wait_expiry_is_reported(wk):
    assert wk.wkv7_get_device_status() == 0
    wk.wkv7_debug_expire_wait(64)
    assert wk.wkv7_get_device_status() == -5
    assert wk.wkv7_get_device_status() == 0  # cleared by the read


def test_bad_offsets_reported_not_read(wk):
    """Non-monotone offsets are caught on the device before any token is read."""
    inp = W.make_packed([10, 10], [0, 0], 1, io="bf16", wdt="f32", s0_std=None, seed=14)
    d, _, _ = to_dev(inp)
    offs = torch.tensor([0, 15, 5], dtype=torch.int32, device="cuda")
    y = torch.zeros_like(d["r"])
    sT = torch.zeros(2, 1, 64, 64, device="cuda")
    wk.wkv7_forward(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], None, y, sT, 2, 20, 1, 64, offs)
    assert wk.wkv7_get_device_status() == -6
    assert wk.wkv7_get_device_status() == 0


def test_forward_host_pipeline(wk, oracle_mod):
    """forward_host (pinned host inputs and outputs, pieces whose copies overlap
    the prefill on three streams) equals one device-side call bit for bit and the
    oracle within the bf16 bound: 3 sequences in 2 groups, and every sequence in
    3 token ranges chained through the state."""
    inp = W.make_prefill(3, 130, 3, io="bf16", wdt="f32", s0_std=0.1, seed=91)
    t = inp.tensors()
    host = {n: x.pin_memory() for n, x in t.items()}
    dev = {n: torch.empty_like(x, device="cuda") for n, x in t.items()}
    dev["y"] = torch.empty(tuple(inp.r.shape), dtype=torch.bfloat16, device="cuda")
    dev["sT"] = torch.empty((3, 3, 64, 64), dtype=torch.float32, device="cuda")
    y_h = torch.empty(tuple(inp.r.shape), dtype=torch.bfloat16).pin_memory()
    sT_h = torch.empty((3, 3, 64, 64), dtype=torch.float32).pin_memory()
    s0 = inp.s0.cuda()
    # whole sequences in 2 groups, then token ranges [0, 64), [64, 128), [128, 130) of every
    # sequence with the state carried between ranges; the calls reuse buffers and streams
    for kw in (dict(parts=2), dict(t_parts=3), dict(parts=2)):
        y_h.fill_(float("nan"))
        sT_h.fill_(float("nan"))
        wk.forward_host(host, dev, y_h, sT_h, s0=s0, **kw)
        torch.cuda.synchronize()
        assert wk.wkv7_get_device_status() == 0
        d = {n: x.cuda() for n, x in t.items()}
        y_ref, s_ref = wk.forward(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], s0)
        assert torch.equal(y_h, y_ref.cpu()) and torch.equal(sT_h, s_ref.cpu())
    f64 = lambda x: x.double().numpy()
    yr, sr = oracle_mod.forward(*(f64(t[n]) for n in ("r", "w_log", "k", "v", "a", "b")), f64(inp.s0))
    assert relerr(y_h.float().numpy(), yr) <= TOL["bf16"] and relerr(sT_h.numpy(), sr) <= TOL["bf16"]
