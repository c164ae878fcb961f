"""wkv7_backward_noalloc: the backward for callers that cannot allocate device
memory at the call, run on the library's own fixed scratch instead of a caller
workspace.  Checked through the C ABI against wkv7_backward with a caller
workspace: the same kernel on the same inputs, so the gradients must agree bit
for bit (a race or a stale value in the shared scratch would show up as a
difference).  Two calls in a row per case; a dense case, a packed case (whose
chunk count is B + ceil(T/64) per head), and the longest sequence whose
workspace fits the 16 MiB scratch.  One token more is refused on the host.

This file sorts last so that a run stopping at its first failure has run every
other test before it; it also passes on its own in a fresh process."""
import pytest
import torch

import wkv7_inputs as W

pytestmark = pytest.mark.gpu

LIMIT = 16 << 20  # WKV7_NOALLOC_SCRATCH_BYTES


@pytest.fixture(scope="module")
def wk():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_recurrent_lm_wkv7_b200 as wk

    return wk


def _run_both(wk, inp, seed):
    B, T, H = inp.B, inp.T, inp.H
    packed = inp.seq_offsets is not None
    need = wk.wkv7_backward_workspace_bytes(B, T, H, 64, packed)
    assert 0 < need <= LIMIT
    shape = inp.r.shape
    dy, dsT = W.make_upstream(shape, B, H, io=inp.io, seed=seed)
    d = {n: x.cuda() for n, x in inp.tensors().items()}
    s0 = inp.s0.cuda() if inp.s0 is not None else None
    offs = inp.seq_offsets.cuda() if packed else None
    dy, dsT = dy.cuda(), dsT.cuda()
    ref = wk.backward(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], dy, s0, dsT, seq_offsets=offs)
    torch.cuda.synchronize()
    assert wk.wkv7_get_device_status() == 0
    for _ in range(2):
        grads = [torch.full_like(d[n], float("nan")) for n in ("r", "w_log", "k", "v", "a", "b")]
        ds0 = torch.full((B, H, 64, 64), float("nan"), device="cuda")
        wk.wkv7_backward_noalloc(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], s0, dy, dsT, *grads, ds0,
                                 B, T, H, 64, offs)
        torch.cuda.synchronize()
        assert wk.wkv7_get_device_status() == 0
        for g, rf in zip(grads + [ds0], ref):
            assert torch.equal(g, rf), "no-alloc gradients differ from the workspace entry point"


def test_backward_noalloc_dense(wk):
    inp = W.make_prefill(2, 130, 3, io="bf16", wdt="f32", s0_std=0.1, seed=77)
    _run_both(wk, inp, seed=78)


def test_backward_noalloc_packed(wk):
    """Three sequences of uneven length with pad tokens, packed along T."""
    inp = W.make_packed([70, 5, 131], [2, 0, 17], 2, io="bf16", wdt="f32", s0_std=0.1, seed=79)
    _run_both(wk, inp, seed=80)


def test_backward_noalloc_at_the_limit(wk):
    """B1 H1 T21760 (340 chunks), the longest sequence that fits: the chunked
    form's 3 x (340 + 1) states of 16 KiB take 16 MiB less one state; T + 1
    needs a chunk more (three states) and is refused before anything is launched."""
    B, T, H = 1, 21760, 1
    assert wk.wkv7_backward_workspace_bytes(B, T, H, 64, False) == LIMIT - 16384
    inp = W.make_prefill(B, T, H, io="bf16", wdt="f32", s0_std=0.1, seed=81)
    _run_both(wk, inp, seed=82)

    assert wk.wkv7_backward_workspace_bytes(B, T + 1, H, 64, False) > LIMIT
    lib = wk._lib()
    x = torch.empty(16, device="cuda")
    p = x.data_ptr()
    st = lib.wkv7_backward_noalloc(p, p, p, p, p, p, None, p, None, p, p, p, p, p, p, p, B, T + 1, H, 64, None,
                                   1, 0, None)
    assert st == -7  # WKV7_ERR_SCRATCH_LIMIT
