"""Seeded synthetic inputs for the WKV-7 operator (shared by tests and benchmark).

This module only draws random numbers and casts them to their storage dtype.
It holds none of the operator's arithmetic, and both the oracle and the CUDA
path receive exactly the tensors it returns.

Distributions (one torch CPU ``Generator`` per call, seeded explicitly; draw
order r, k, v, kappa, a_lr logit, decay logit, s0):

* r, k, v ~ N(0, 1)
* kappa = x / ||x||_2 over the head dimension, x ~ N(0, 1)  (unit removal key)
* a_lr = sigmoid(N(0, 1)) in (0, 1); a = -kappa, b = kappa * a_lr
  (the argument pair handed to the WKV kernel in the hxa07D forward listing)
* log_neglog_w = -softplus(-z) - 0.5 with z ~ N(mu_z, 1), so that
  w = exp(-exp(log_neglog_w)) lies in (exp(-exp(-0.5)), 1) ~= (0.545, 1)
* s0 ~ N(0, s0_std^2) in fp32 when an initial state is requested
* gated read-out (make_gate, its own generator): r_k ~ N(0, rk_std^2) [H, D]
  fp32, gate g ~ N(0, 1) in the io dtype
* fused prologue (make_fused, its own generator; draw order r, k, v, a_lr logit,
  decay logit, s0): r ~ N(0, 1) [.., H, D]; raw k, v ~ N(0, 1) over the H_kv
  kv heads [.., H_kv, D]; a_lr = sigmoid(N(0, 1)) [.., H, D]; log_neglog_w as
  above.  The prologue (normalised kk, a, b and the scaled key) happens inside
  the path under test.
* backward upstream gradients (make_upstream, its own generator): dy ~ N(0, 1)
  in the io dtype with the shape of r, dsT ~ N(0, 0.1^2) fp32 [B, H, D, D]
* packed batches: lengths ~ U{len_lo..len_hi} and pad counts ~ U{0..pad_hi};
  pad tokens carry log_neglog_w = -inf (w = 1) and k = v = a = b = 0, so they
  leave the state unchanged; r stays drawn at pads.

Storage dtypes: ``io`` for r, k, v, a, b; ``wdt`` for log_neglog_w; states fp32.
Values are computed in fp32 and rounded once (round-to-nearest-even) to the
storage dtype.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch

_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclass
class PrefillInputs:
    r: torch.Tensor
    w_log: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    a: torch.Tensor
    b: torch.Tensor
    s0: Optional[torch.Tensor]
    seq_offsets: Optional[torch.Tensor]  # int32 [B+1] for packed batches
    B: int
    T: int  # per-sequence T (dense) or packed length (packed)
    H: int
    D: int
    io: str
    wdt: str
    n_real_tokens: int
    lengths: Optional[list] = None  # real tokens per sequence (packed)
    pads: Optional[list] = None  # pad tokens per sequence (packed)

    def tensors(self):
        return dict(r=self.r, w_log=self.w_log, k=self.k, v=self.v, a=self.a, b=self.b)


def _draw(g, shape, io, wdt, mu_z):
    r = torch.randn(shape, generator=g)
    k = torch.randn(shape, generator=g)
    v = torch.randn(shape, generator=g)
    x = torch.randn(shape, generator=g)
    kappa = x / x.norm(dim=-1, keepdim=True)
    a_lr = torch.sigmoid(torch.randn(shape, generator=g))
    z = torch.randn(shape, generator=g) + mu_z
    w_log = -torch.nn.functional.softplus(-z) - 0.5
    a = -kappa
    b = kappa * a_lr
    cast = lambda t, d: t.to(_DT[d]).contiguous()
    return (cast(r, io), cast(w_log, wdt), cast(k, io), cast(v, io), cast(a, io), cast(b, io))


def make_prefill(B, T, H, D=64, io="bf16", wdt="f32", s0_std=None, mu_z=0.0, seed=0):
    """Dense batch: tensors [B, T, H, D]."""
    g = torch.Generator().manual_seed(seed)
    r, w_log, k, v, a, b = _draw(g, (B, T, H, D), io, wdt, mu_z)
    s0 = None
    if s0_std is not None:
        s0 = (torch.randn((B, H, D, D), generator=g) * s0_std).contiguous()
    return PrefillInputs(r, w_log, k, v, a, b, s0, None, B, T, H, D, io, wdt, B * T)


def make_packed(lengths, pads, H, D=64, io="bf16", wdt="f32", s0_std=0.1, mu_z=0.0, seed=0):
    """Packed batch: tensors [T_total, H, D]; sequence n holds lengths[n] real
    tokens followed by pads[n] pad tokens."""
    lengths = [int(x) for x in lengths]
    pads = [int(x) for x in pads]
    slots = [l + p for l, p in zip(lengths, pads)]
    offs = [0]
    for s in slots:
        offs.append(offs[-1] + s)
    T_total = offs[-1]
    B = len(lengths)
    g = torch.Generator().manual_seed(seed)
    r, w_log, k, v, a, b = _draw(g, (T_total, H, D), io, wdt, mu_z)
    s0 = None
    if s0_std is not None:
        s0 = (torch.randn((B, H, D, D), generator=g) * s0_std).contiguous()
    pad_mask = torch.zeros(T_total, dtype=torch.bool)
    for n in range(B):
        pad_mask[offs[n] + lengths[n]: offs[n + 1]] = True
    if bool(pad_mask.any()):
        w_log[pad_mask] = float("-inf")
        for t in (k, v, a, b):
            t[pad_mask] = 0
    seq_offsets = torch.tensor(offs, dtype=torch.int32)
    return PrefillInputs(r, w_log, k, v, a, b, s0, seq_offsets, B, T_total, H, D, io, wdt,
                         sum(lengths), lengths, pads)


def make_gate(shape, H, D=64, io="bf16", rk_std=0.5, seed=0):
    """Inputs of the gated read-out: per-head weights r_k [H, D] fp32 ~ N(0, rk_std^2)
    and a gate of the given activation shape ~ N(0, 1), rounded to the io dtype."""
    g = torch.Generator().manual_seed(seed)
    rk = (torch.randn((H, D), generator=g) * rk_std).contiguous()
    gate = torch.randn(tuple(shape), generator=g).to(_DT[io]).contiguous()
    return rk, gate


@dataclass
class FusedInputs:
    r: torch.Tensor
    w_log: torch.Tensor
    k: torch.Tensor  # [.., H_kv, D]
    v: torch.Tensor  # [.., H_kv, D]
    a_lr: torch.Tensor
    s0: Optional[torch.Tensor]
    seq_offsets: Optional[torch.Tensor]
    B: int
    T: int
    H: int
    H_kv: int
    D: int
    io: str
    wdt: str
    n_real_tokens: int

    def tensors(self):
        return dict(r=self.r, w_log=self.w_log, k=self.k, v=self.v, a_lr=self.a_lr)


def make_fused(B, T, H, H_kv, D=64, io="bf16", wdt="f32", s0_std=None, mu_z=0.0, seed=0, lengths=None, pads=None):
    """Inputs of the fused-prologue path.  Dense [B, T, .., D] when ``lengths`` is
    None, else packed [T_total, .., D] with sequence n holding lengths[n] real
    tokens followed by pads[n] pad tokens (w_log = -inf, k = v = 0)."""
    g = torch.Generator().manual_seed(seed)
    seq_offsets = None
    if lengths is None:
        lead = (B, T)
        n_real = B * T
    else:
        offs = [0]
        for l, p_ in zip(lengths, pads):
            offs.append(offs[-1] + int(l) + int(p_))
        B, T = len(lengths), offs[-1]
        lead = (T,)
        n_real = int(sum(lengths))
        seq_offsets = torch.tensor(offs, dtype=torch.int32)
    r = torch.randn(lead + (H, D), generator=g)
    k = torch.randn(lead + (H_kv, D), generator=g)
    v = torch.randn(lead + (H_kv, D), generator=g)
    a_lr = torch.sigmoid(torch.randn(lead + (H, D), generator=g))
    z = torch.randn(lead + (H, D), generator=g) + mu_z
    w_log = -torch.nn.functional.softplus(-z) - 0.5
    s0 = None
    if s0_std is not None:
        s0 = (torch.randn((B, H, D, D), generator=g) * s0_std).contiguous()
    if lengths is not None:
        pad_mask = torch.zeros(T, dtype=torch.bool)
        for n in range(B):
            pad_mask[offs[n] + int(lengths[n]): offs[n + 1]] = True
        if bool(pad_mask.any()):
            w_log[pad_mask] = float("-inf")
            k[pad_mask] = 0
            v[pad_mask] = 0
    cast = lambda t, d: t.to(_DT[d]).contiguous()
    return FusedInputs(cast(r, io), cast(w_log, wdt), cast(k, io), cast(v, io), cast(a_lr, io), s0, seq_offsets,
                       B, T, H, H_kv, D, io, wdt, n_real)


def make_upstream(shape, B, H, D=64, io="bf16", seed=0, with_dsT=True, dsT_std=0.1):
    """Upstream gradients for the backward: dy of the activation shape (io dtype)
    and dsT [B, H, D, D] fp32 (None when with_dsT is false)."""
    g = torch.Generator().manual_seed(seed)
    dy = torch.randn(tuple(shape), generator=g).to(_DT[io]).contiguous()
    dsT = (torch.randn((B, H, D, D), generator=g) * dsT_std).contiguous() if with_dsT else None
    return dy, dsT


def draw_lengths(n_seq, len_lo, len_hi, pad_hi, seed):
    """Sequence lengths U{len_lo..len_hi} and pad counts U{0..pad_hi}."""
    g = torch.Generator().manual_seed(seed)
    lengths = torch.randint(len_lo, len_hi + 1, (n_seq,), generator=g).tolist()
    pads = torch.randint(0, pad_hi + 1, (n_seq,), generator=g).tolist()
    return lengths, pads


@dataclass
class DecodeInputs:
    r: torch.Tensor
    w_log: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    a: torch.Tensor
    b: torch.Tensor
    B: int
    H: int
    D: int

    def tensors(self):
        return dict(r=self.r, w_log=self.w_log, k=self.k, v=self.v, a=self.a, b=self.b)


def make_decode_step(B, H, D=64, io="bf16", wdt="bf16", mu_z=0.0, seed=0, step=0):
    """Fresh per-step inputs [B, H, D]; step s uses seed (seed * 1_000_003 + s)."""
    g = torch.Generator().manual_seed(seed * 1_000_003 + step)
    r, w_log, k, v, a, b = _draw(g, (B, H, D), io, wdt, mu_z)
    return DecodeInputs(r, w_log, k, v, a, b, B, H, D)


def make_state(B, H, D=64, std=0.1, seed=0):
    g = torch.Generator().manual_seed(seed * 7919 + 1)
    return (torch.randn((B, H, D, D), generator=g) * std).contiguous()


# The five workloads: sizes, dtypes and distributions of the RWKV-7 layers the
# pages describe (head size 64; C = 2048 for a 1.5B-class layer, C = 2560 for a
# 2.9B-class layer).
WORKLOADS = {
    "tiny_f32": dict(kind="prefill", B=1, T=64, H=2, io="f32", wdt="f32", s0_std=None, mu_z=0.0, seed=0),
    "prefill_1p5b": dict(kind="prefill", B=4, T=1024, H=32, io="bf16", wdt="f32", s0_std=None, mu_z=0.0, seed=1),
    "prefill_2p9b_long": dict(kind="prefill", B=1, T=16384, H=40, io="bf16", wdt="f32", s0_std=0.1, mu_z=1.0, seed=2),
    "decode_2p9b": dict(kind="decode", B=256, H=40, io="bf16", wdt="bf16", s0_std=0.1, mu_z=0.0, seed=3, steps=128),
    "packed_1p5b": dict(kind="packed", n_seq=16, len_lo=512, len_hi=8192, pad_hi=63, H=32, io="bf16", wdt="f32",
                        s0_std=0.1, mu_z=0.0, seed=4),
}


def make_workload(name, **override):
    cfg = dict(WORKLOADS[name])
    cfg.update(override)
    kind = cfg.pop("kind")
    if kind == "prefill":
        return make_prefill(cfg["B"], cfg["T"], cfg["H"], io=cfg["io"], wdt=cfg["wdt"], s0_std=cfg["s0_std"],
                            mu_z=cfg["mu_z"], seed=cfg["seed"])
    if kind == "packed":
        lengths, pads = draw_lengths(cfg["n_seq"], cfg["len_lo"], cfg["len_hi"], cfg["pad_hi"], cfg["seed"])
        return make_packed(lengths, pads, cfg["H"], io=cfg["io"], wdt=cfg["wdt"], s0_std=cfg["s0_std"],
                           mu_z=cfg["mu_z"], seed=cfg["seed"])
    raise ValueError(f"{name} is a decode workload: use make_decode_step / make_state")
