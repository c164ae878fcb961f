"""wkv7_backward_noalloc (the backward with the library's fixed scratch, for
callers that cannot allocate device memory at the call) against wkv7_backward
with a caller workspace, through the C ABI: two calls in a row, each within the
backward's parity bound (max|out - ref| / max|ref| <= 2e-2 for bf16 inputs)."""
import numpy as np
import pytest
import torch

import wkv7_inputs as W

pytestmark = pytest.mark.gpu


def relerr(out, ref):
    out = out.double().cpu().numpy()
    ref = ref.double().cpu().numpy()
    assert np.all(np.isfinite(out)), "non-finite output"
    return float(np.max(np.abs(out - ref)) / max(np.max(np.abs(ref)), 1e-30))


def test_backward_noalloc_matches_workspace_entry_point():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_recurrent_lm_wkv7_b200 import build

    build.build()
    import linear_recurrent_lm_wkv7_b200 as wk

    inp = W.make_prefill(2, 130, 3, io="bf16", wdt="f32", s0_std=0.1, seed=77)
    assert wk.wkv7_backward_workspace_bytes(2, 130, 3, 64, False) <= 16 << 20
    dy, dsT = W.make_upstream(inp.r.shape, inp.B, inp.H, io="bf16", seed=78)
    d = {n: x.cuda() for n, x in inp.tensors().items()}
    s0, dy, dsT = inp.s0.cuda(), dy.cuda(), dsT.cuda()
    ref = wk.backward(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], dy, s0, dsT)
    for _ in range(2):
        grads = [torch.full_like(d[n], float("nan")) for n in ("r", "w_log", "k", "v", "a", "b")]
        ds0 = torch.full((2, 3, 64, 64), float("nan"), device="cuda")
        wk.wkv7_backward_noalloc(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], s0, dy, dsT, *grads, ds0,
                                 2, 130, 3, 64)
        torch.cuda.synchronize()
        assert wk.wkv7_get_device_status() == 0
        for g, rf in zip(grads + [ds0], ref):
            assert relerr(g, rf) <= 2e-2
