"""WKV-7 benchmark: chunked prefill tokens/s (headline) and decode steps/s on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One JSON line on rank 0.  `value` is prefill tokens/s of the whole job for the
B4 T1024 H32 D64 prefill (bf16 inputs, fp32 decay logits, zero initial state),
timed with CUDA events per launch on the launching stream.  Consecutive
launches alternate between two resident copies of the inputs (2 x 136 MB,
more than the 126 MB L2), so no launch finds its inputs in L2 and no flush
kernel has to run between them.  `long` and `packed` time the same entry
point on the long-context prefill (B1 T16384 H40, N(0, 0.1^2) initial state;
the literal decay formula and the long-memory variant) and on the packed
variable-length prefill (16 sequences, lengths U{512..8192}, pad tokens),
each with its own roofline.  `e2e` is the same metric through the
public API from pinned host buffers (host->device copies of the inputs and
device->host copies of y and sT inside the timed region).  `gated` times the
same prefill with the gated read-out (wkv7_forward_gated, z instead of y; the
gate adds its bf16 bytes to the roofline).  `decode` reports
the B256 H40 decode step with the fp32 state carried through 128 steps, timed as
128 back-to-back launches between one event pair (the state, 2 x 168 MB, exceeds
L2 on its own); the mean of per-launch event pairs is reported beside it.
Multi-GPU: every rank runs the same per-GPU workload on its own device
(independent (sequence, head) units, no collective on the data path); the job
time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "WKV7 prefill tokens/s and decode steps/s on 1 B200; % of roofline"
PREFILL_WORKLOAD = "prefill_1p5b"
DECODE_WORKLOAD = "decode_2p9b"
FUSED_HKV = 8  # kv heads of the fused-prologue measurement (4 query heads per kv head)
D = 64
L2_FLUSH_BYTES = 256 << 20


# DRAM traffic of one prefill launch (dram__bytes_read.sum + dram__bytes_write.sum)
# from an ncu capture of this workload, valid only for the kernel sources it was
# taken on (SHA-256 over the files below); any change makes it null until the
# capture is repeated.
NCU_TRAFFIC = {"sha256": "cd625ceb3a69fe5b2b460e6c49410ca036493dfc4bf99b7ca7ce3c9bc6c97c77",
               "bytes": 123425536, "workload": "prefill_1p5b"}
KERNEL_SOURCES = ("linear_recurrent_lm_wkv7_b200/csrc/wkv7_prefill_pipe.cu",
                  "linear_recurrent_lm_wkv7_b200/csrc/prefill_common.cuh",
                  "linear_recurrent_lm_wkv7_b200/csrc/sm100_ptx.cuh")


def measured_traffic():
    import hashlib

    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return NCU_TRAFFIC["bytes"] if h.hexdigest() == NCU_TRAFFIC["sha256"] else None


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), "measured"
    return 6650.0, 1590.0, "fallback"


def prefill_bytes(n_tokens_heads, io_b, w_b, n_states, with_s0):
    """Algorithmic HBM bytes: r, k, v, a, b read and y written once (io_b each),
    w_log read once (w_b), sT written once (and s0 read once when given)."""
    per = D * (6 * io_b + w_b)
    return n_tokens_heads * per + n_states * D * D * 4 * (2 if with_s0 else 1)


def prefill_config(B, T, H, world):
    """`config` of the headline line, shared by both arms of the benchmark."""
    return {"workload": PREFILL_WORKLOAD, "B": B, "T": T, "H": H, "D": D, "io": "bf16", "w_log": "f32",
            "s0": "zero", "chunk": 64,
            "l2": "inputs larger than L2: two input copies (2 x 136 MB) alternated between launches",
            "parallelism": f"replicas{world}" if world > 1 else "single"}


def prefill_flops(n_tokens_heads, L=64):
    return n_tokens_heads * (15 * L * D + 8 * D * D)


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (FileNotFoundError, OSError):
            self.proc = None
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def time_launches(fn, steps, stream, flush=None):
    """Per-launch CUDA-event times (ms) on `stream`; `flush` runs between launches, untimed."""
    import torch

    times = []
    for _ in range(steps):
        if flush is not None:
            flush()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        fn()
        e.record(stream)
        times.append((s, e))
    torch.cuda.synchronize()
    return [s.elapsed_time(e) for s, e in times]


def oracle_baseline(budget_s=20.0):
    """The oracle, as it stands, on a bounded sample of the prefill workload:
    whole sequences of a subset of heads, grown until ~budget_s of CPU work."""
    import numpy as np

    import oracle
    import wkv7_inputs as W

    oracle.build()
    inp = W.make_workload(PREFILL_WORKLOAD)
    t = inp.tensors()
    threads = oracle.default_threads()
    full = {k: v.double().numpy() for k, v in t.items()}
    total_tokens, total_s, passes = 0, 0.0, 0
    while total_s < budget_s and passes < 1000:
        t0 = time.perf_counter()
        oracle.forward(full["r"], full["w_log"], full["k"], full["v"], full["a"], full["b"], None, n_threads=threads)
        total_s += time.perf_counter() - t0
        total_tokens += inp.B * inp.T
        passes += 1
    tok_s = total_tokens / total_s
    return {"value": tok_s, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"prefill_1p5b (B4 T1024 H32, all heads) repeated {passes} times: "
                      f"{total_tokens} tokens in {total_s:.1f} s of fp64 CPU work"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cb = oracle_baseline(budget_s=max(5.0, min(60.0, 3.0 * args.steps)))
    line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * 4 * 1024 / cb["value"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": prefill_config(4, 1024, 32, 1),
            "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    import linear_recurrent_lm_wkv7_b200 as wk
    import wkv7_inputs as W

    hbm_peak, bf16_peak, peak_src = measured_peaks()
    stream = torch.cuda.current_stream()
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    flush = lambda: flush_buf.zero_()

    # ---------------- prefill (headline)
    inp = W.make_workload(PREFILL_WORKLOAD, seed=1 + 1000 * rank)
    B, T, H = inp.B, inp.T, inp.H
    host = {k: v.pin_memory() for k, v in inp.tensors().items()}
    dev = {k: v.cuda() for k, v in host.items()}
    # a second resident copy of the inputs: launches alternate between the two, so the
    # working set (2 x 136 MB) exceeds L2 and every launch reads its inputs from HBM
    dev2 = {k: v.clone() for k, v in dev.items()}
    copies = (dev, dev2)
    alt = {"i": 0}

    def cur():
        alt["i"] += 1
        return copies[alt["i"] & 1]

    y = torch.empty_like(dev["r"])
    sT = torch.empty((B, H, D, D), dtype=torch.float32, device="cuda")

    def step():
        x = cur()
        wk.wkv7_forward(x["r"], x["w_log"], x["k"], x["v"], x["a"], x["b"], None, y, sT, B, T, H, D, None, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if wk.wkv7_get_device_status() != 0:
        raise RuntimeError("device status set during warm-up")
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk = ClockSampler(local)
    clk.start()
    times = time_launches(step, args.steps, stream)
    clocks = clk.stop()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = sum(times) / len(times)
    if world > 1:
        t = torch.tensor([ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    tokens = B * T
    value = world * tokens / (ms * 1e-3)
    bytes_alg = prefill_bytes(B * T * H, 2, 4, B * H, with_s0=False)
    achieved = bytes_alg / (ms * 1e-3) / 1e9
    flops = prefill_flops(B * T * H)

    def max_over_ranks(x):
        if world > 1:
            t_ = torch.tensor([x], device="cuda")
            dist.all_reduce(t_, op=dist.ReduceOp.MAX)
            x = float(t_.item())
        return x

    def prefill_section(name, inp_, label, s0_kind):
        """Times wkv7_forward on one more prefill workload: per-launch CUDA events,
        inputs far larger than L2 (no flush needed); tokens/s counts real tokens (pads excluded);
        the roofline bytes are the workload's own (s0 read and sT written)."""
        d_ = {k_: v_.cuda() for k_, v_ in inp_.tensors().items()}
        s0_ = inp_.s0.cuda() if inp_.s0 is not None else None
        offs_ = inp_.seq_offsets.cuda() if inp_.seq_offsets is not None else None
        y_ = torch.empty_like(d_["r"])
        sT_ = torch.empty((inp_.B, inp_.H, D, D), dtype=torch.float32, device="cuda")

        def st_():
            wk.wkv7_forward(d_["r"], d_["w_log"], d_["k"], d_["v"], d_["a"], d_["b"], s0_, y_, sT_, inp_.B, inp_.T,
                            inp_.H, D, offs_, stream)

        for _ in range(max(3, args.warmup)):
            st_()
        torch.cuda.synchronize()
        tt = time_launches(st_, args.steps, stream)
        if wk.wkv7_get_device_status() != 0:
            raise RuntimeError(f"device status set during the {name} run")
        ms_ = max_over_ranks(sum(tt) / len(tt))
        slots = inp_.T if inp_.seq_offsets is not None else inp_.B * inp_.T  # tokens in the tensors, pads included
        io_b_, w_b_ = (4 if inp_.io == "f32" else 2), (4 if inp_.wdt == "f32" else 2)
        bytes_ = prefill_bytes(slots * inp_.H, io_b_, w_b_, inp_.B * inp_.H, with_s0=inp_.s0 is not None)
        ach = bytes_ / (ms_ * 1e-3) / 1e9
        out = {"workload": name, "variant": label, "B": inp_.B, "H": inp_.H, "tokens": inp_.n_real_tokens,
               "token_slots": slots, "s0": s0_kind, "tokens_per_s": world * inp_.n_real_tokens / (ms_ * 1e-3),
               "ms_per_step": ms_,
               "roofline": {"bound": "hbm", "achieved": ach, "peak": hbm_peak, "unit": "GB/s", "frac": ach / hbm_peak,
                            "algorithmic_bytes_per_launch": bytes_,
                            "hbm_time_floor_us": bytes_ / (hbm_peak * 1e9) * 1e6}}
        if inp_.seq_offsets is not None:
            out["lengths"] = inp_.lengths
        del d_, y_, sT_
        return out

    # ---------------- long-context prefill B1 T16384 H40 (the workload's literal decay formula,
    # and the labelled long-memory variant), N(0, 0.1^2) initial state
    long_sections = []
    for mu_z, label in ((1.0, "decay z ~ N(1,1) (literal formula)"), (-3.0, "decay z ~ N(-3,1) (long memory)")):
        linp = W.make_workload("prefill_2p9b_long", mu_z=mu_z, seed=2 + 1000 * rank)
        long_sections.append(prefill_section("prefill_2p9b_long", linp, label, "N(0, 0.1^2)"))
        del linp
    # ---------------- the same long sequence cut into 3 token ranges that run side by side
    # (sharding.forward_long: range 0 with the map of range 1, then ranges 1 and 2)
    from linear_recurrent_lm_wkv7_b200 import sharding

    linp = W.make_workload("prefill_2p9b_long", seed=2 + 1000 * rank)
    ld_ = {k_: v_.cuda() for k_, v_ in linp.tensors().items()}
    ls0 = linp.s0.cuda()

    def lsplit():
        sharding.forward_long(ld_["r"], ld_["w_log"], ld_["k"], ld_["v"], ld_["a"], ld_["b"], ls0, 3, stream)

    for _ in range(max(3, args.warmup)):
        lsplit()
    torch.cuda.synchronize()
    lt = time_launches(lsplit, args.steps, stream)
    if wk.wkv7_get_device_status() != 0:
        raise RuntimeError("device status set during the long split run")
    lms = max_over_ranks(sum(lt) / len(lt))
    lbytes = prefill_bytes(linp.T * linp.H, 2, 4, linp.H, with_s0=True)
    lach = lbytes / (lms * 1e-3) / 1e9
    long_split = {"workload": "prefill_2p9b_long", "variant": "decay z ~ N(1,1); 3 token ranges side by side",
                  "tokens_per_s": world * linp.T / (lms * 1e-3), "ms_per_step": lms,
                  "launches_per_step": 6,
                  "roofline": {"bound": "hbm", "achieved": lach, "peak": hbm_peak, "unit": "GB/s",
                               "frac": lach / hbm_peak, "algorithmic_bytes_per_launch": lbytes,
                               "hbm_time_floor_us": lbytes / (hbm_peak * 1e9) * 1e6}}
    # ---------------- the same long sequence through the two-phase prefill (wkv7_forward_long):
    # every chunk's state-independent part in parallel, then one state pass per head
    lws = torch.empty(wk.wkv7_forward_long_workspace_bytes(1, linp.T, linp.H, 64), dtype=torch.uint8, device="cuda")
    ly = torch.empty_like(ld_["r"])
    lsT = torch.empty_like(ls0)

    def ltwo():
        wk.wkv7_forward_long(ld_["r"], ld_["w_log"], ld_["k"], ld_["v"], ld_["a"], ld_["b"], ls0, ly, lsT, lws, 1,
                             linp.T, linp.H, 64, stream)

    for _ in range(max(3, args.warmup)):
        ltwo()
    torch.cuda.synchronize()
    l2t = time_launches(ltwo, args.steps, stream)
    if wk.wkv7_get_device_status() != 0:
        raise RuntimeError("device status set during the two-phase long run")
    l2ms = max_over_ranks(sum(l2t) / len(l2t))
    l2ach = lbytes / (l2ms * 1e-3) / 1e9
    long_two_phase = {"workload": "prefill_2p9b_long", "variant": "decay z ~ N(1,1); two-phase (wkv7_forward_long)",
                      "tokens_per_s": world * linp.T / (l2ms * 1e-3), "ms_per_step": l2ms,
                      "launches_per_step": 2, "workspace_bytes": lws.numel(),
                      "roofline": {"bound": "hbm", "achieved": l2ach, "peak": hbm_peak, "unit": "GB/s",
                                   "frac": l2ach / hbm_peak, "algorithmic_bytes_per_launch": lbytes,
                                   "hbm_time_floor_us": lbytes / (hbm_peak * 1e9) * 1e6}}
    del ld_, linp, ls0, lws, ly, lsT
    # ---------------- packed variable-length prefill: 16 sequences, lengths U{512..8192}, pads U{0..63}
    # the same packed draw on every rank: the lengths (and so the real-token count and the bytes)
    # are equal across ranks, so world x tokens is the job's count
    pinp = W.make_workload("packed_1p5b", seed=4)
    packed_section = prefill_section("packed_1p5b", pinp, "16 sequences, pads U{0..63} (w = 1, k = v = a = b = 0)",
                                     "N(0, 0.1^2)")
    del pinp

    # ---------------- the headline shape with fp32 inputs (the tf32 kernel; fp32 y)
    finp = W.make_prefill(B, T, H, io="f32", wdt="f32", s0_std=None, seed=1 + 1000 * rank)
    f32_section = prefill_section("prefill_1p5b_f32", finp, "fp32 inputs and outputs", "zero")
    del finp

    # ---------------- the same prefill with the gated read-out (wkv7_forward_gated)
    rk_h, gate_h = W.make_gate(tuple(dev["r"].shape), H, D, io="bf16", seed=2 + 1000 * rank)
    rk_d, gate_d = rk_h.cuda(), gate_h.cuda()
    z = torch.empty_like(dev["r"])

    def gstep():
        x = cur()
        wk.wkv7_forward_gated(x["r"], x["w_log"], x["k"], x["v"], x["a"], x["b"], None, rk_d, gate_d, z,
                              sT, B, T, H, D, None, stream)

    for _ in range(max(3, args.warmup)):
        gstep()
    torch.cuda.synchronize()
    gtimes = time_launches(gstep, args.steps, stream, flush)  # gate, r_k and the fused inputs have one copy
    if wk.wkv7_get_device_status() != 0:
        raise RuntimeError("device status set during the gated run")
    gms = sum(gtimes) / len(gtimes)
    if world > 1:
        t = torch.tensor([gms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        gms = float(t.item())
    gbytes = bytes_alg + B * T * H * D * 2 + H * D * 4  # + the bf16 gate and r_k
    gach = gbytes / (gms * 1e-3) / 1e9
    del z

    # ---------------- the fused layer path (wkv7_forward_fused): raw k, v of FUSED_HKV kv heads
    # and a_lr in, the prologue and the gated read-out inside the kernel
    fin = W.make_fused(B, T, H, FUSED_HKV, io="bf16", wdt="f32", seed=3 + 1000 * rank)
    fd = {k_: v_.cuda() for k_, v_ in fin.tensors().items()}
    del fin
    zf = torch.empty_like(dev["r"])

    def fstep():
        wk.wkv7_forward_fused(fd["r"], fd["w_log"], fd["k"], fd["v"], fd["a_lr"], None, rk_d, gate_d, zf, sT, B, T,
                              H, FUSED_HKV, D, None, stream)

    for _ in range(max(3, args.warmup)):
        fstep()
    torch.cuda.synchronize()
    ftimes = time_launches(fstep, args.steps, stream, flush)
    if wk.wkv7_get_device_status() != 0:
        raise RuntimeError("device status set during the fused run")
    fms = sum(ftimes) / len(ftimes)
    if world > 1:
        t = torch.tensor([fms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        fms = float(t.item())
    # r, a_lr, g, z (bf16) and w_log (fp32) per token-head; k, v (bf16) per token-kv-head; sT; r_k
    fbytes = B * T * H * D * (2 + 2 + 2 + 2 + 4) + B * T * FUSED_HKV * D * 2 * 2 + B * H * D * D * 4 + H * D * 4
    fach = fbytes / (fms * 1e-3) / 1e9
    del zf, fd, gate_d

    # ---------------- backward of the recurrence (wkv7_backward), same workload
    dy_h, _ = W.make_upstream(tuple(dev["r"].shape), B, H, D, io="bf16", seed=4 + 1000 * rank, with_dsT=False)
    dyd = dy_h.cuda()
    del dy_h
    bgrads = [torch.empty_like(dev[n]) for n in ("r", "w_log", "k", "v", "a", "b")]
    bds0 = torch.empty((B, H, D, D), dtype=torch.float32, device="cuda")
    bws = torch.empty(wk.wkv7_backward_workspace_bytes(B, T, H, D, False) // 4, dtype=torch.float32, device="cuda")

    def bstep():
        x = cur()
        wk.wkv7_backward(x["r"], x["w_log"], x["k"], x["v"], x["a"], x["b"], None, dyd, None,
                         *bgrads, bds0, bws, B, T, H, D, None, stream)

    for _ in range(3):
        bstep()
    torch.cuda.synchronize()
    btimes = time_launches(bstep, max(3, args.steps // 5), stream, flush)
    if wk.wkv7_get_device_status() != 0:
        raise RuntimeError("device status set during the backward run")
    bms = sum(btimes) / len(btimes)
    if world > 1:
        t = torch.tensor([bms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        bms = float(t.item())
    # inputs (r, k, v, a, b, dy bf16; w_log fp32) in, gradients (bf16; dw_log fp32) out, ds0 out
    bbytes = B * T * H * D * (6 * 2 + 4) + B * T * H * D * (5 * 2 + 4) + B * H * D * D * 4
    bach = bbytes / (bms * 1e-3) / 1e9
    del bgrads, bds0, bws, dyd

    # ---------------- end to end through the public API from pinned host memory
    y_h = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    sT_h = torch.empty(sT.shape, dtype=sT.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = y_h.numel() * y_h.element_size() + sT_h.numel() * sT_h.element_size()

    # the public host-memory entry point: per-sequence groups whose upload, prefill and
    # download overlap on three streams, ordered after and waited for by `stream`
    staging = dict(dev, y=y, sT=sT)

    def e2e_step():
        wk.forward_host(host, staging, y_h, sT_h, parts=B, stream=stream)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    e2e_times = time_launches(e2e_step, max(3, args.steps // 4), stream, flush)
    e2e_ms = sum(e2e_times) / len(e2e_times)
    if world > 1:
        t = torch.tensor([e2e_ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    e2e_value = world * tokens / (e2e_ms * 1e-3)
    del dev, dev2, copies, host

    # ---------------- decode step (B256 H40, state carried through 128 steps)
    cfg = W.WORKLOADS[DECODE_WORKLOAD]
    dB, dH, nsteps = cfg["B"], cfg["H"], cfg["steps"]
    state = W.make_state(dB, dH, std=cfg["s0_std"], seed=cfg["seed"]).cuda()
    dsteps = [{k: v.cuda() for k, v in W.make_decode_step(dB, dH, io=cfg["io"], wdt=cfg["wdt"], seed=cfg["seed"],
                                                          step=s).tensors().items()} for s in range(nsteps)]
    dy = torch.empty((dB, dH, D), dtype=torch.bfloat16, device="cuda")
    it = {"i": 0}

    def dstep():
        d = dsteps[it["i"] % nsteps]
        it["i"] += 1
        wk.wkv7_decode_step(d["r"], d["w_log"], d["k"], d["v"], d["a"], d["b"], state, dy, state, dB, dH, D, stream)

    for _ in range(max(3, args.warmup)):
        dstep()
    torch.cuda.synchronize()
    it["i"] = 0
    dtimes = time_launches(dstep, nsteps, stream, None)  # state (168 MB x2) exceeds L2 by itself
    dms_launch = sum(dtimes) / len(dtimes)
    # steps back to back: one event pair around the whole sequence of nsteps launches
    it["i"] = 0
    torch.cuda.synchronize()
    ls, le = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ls.record(stream)
    for _ in range(nsteps):
        dstep()
    le.record(stream)
    torch.cuda.synchronize()
    if wk.wkv7_get_device_status() != 0:
        raise RuntimeError("device status set during the run")
    dms = ls.elapsed_time(le) / nsteps
    if world > 1:
        t = torch.tensor([dms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dms = float(t.item())
    dbytes = 2 * dB * dH * D * D * 4 + dB * dH * D * (6 * 2 + 2)
    dach = dbytes / (dms * 1e-3) / 1e9

    # ---------------- fused decode step: raw k, v of FUSED_HKV kv heads, a_lr, gated read-out
    fsteps = []
    for s_ in range(4):
        fi = W.make_fused(dB, 1, dH, FUSED_HKV, io=cfg["io"], wdt=cfg["wdt"], seed=cfg["seed"] + 100 * s_)
        fsteps.append({k_: v_[:, 0].contiguous().cuda() for k_, v_ in fi.tensors().items()})
    drk, _ = W.make_gate((dB, dH, D), dH, D, io=cfg["io"], seed=cfg["seed"])
    _, dg = W.make_gate((dB, dH, D), dH, D, io=cfg["io"], seed=cfg["seed"] + 1)
    drk, dg = drk.cuda(), dg.cuda()
    fit = {"i": 0}

    def dfstep():
        d = fsteps[fit["i"] % len(fsteps)]
        fit["i"] += 1
        wk.wkv7_decode_step_fused(d["r"], d["w_log"], d["k"], d["v"], d["a_lr"], state, drk, dg, dy, state, dB, dH,
                                  FUSED_HKV, D, stream)

    for _ in range(max(3, args.warmup)):
        dfstep()
    torch.cuda.synchronize()
    ls.record(stream)
    for _ in range(nsteps):
        dfstep()
    le.record(stream)
    torch.cuda.synchronize()
    if wk.wkv7_get_device_status() != 0:
        raise RuntimeError("device status set during the fused decode run")
    dfms = ls.elapsed_time(le) / nsteps
    if world > 1:
        t = torch.tensor([dfms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dfms = float(t.item())
    # state in and out; r, w_log, a_lr, g, out per head row; k, v per kv-head row; r_k
    dfbytes = 2 * dB * dH * D * D * 4 + dB * dH * D * 2 * 5 + dB * FUSED_HKV * D * 2 * 2 + dH * D * 4
    dfach = dfbytes / (dfms * 1e-3) / 1e9
    del fsteps

    if rank == 0:
        cb = oracle_baseline(budget_s=20.0) if (world == 1 and not args.no_cpu_baseline) else None
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": prefill_config(B, T, H, world),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                         "frac": achieved / hbm_peak, "traffic": measured_traffic(), "peak_source": peak_src,
                         "algorithmic_bytes_per_launch": bytes_alg,
                         "tensor_flop_per_launch": flops,
                         "tensor_time_floor_us": flops / (bf16_peak * 1e12) * 1e6,
                         "hbm_time_floor_us": bytes_alg / (hbm_peak * 1e9) * 1e6},
            "cpu_baseline": cb,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms, "api": "forward_host (per-sequence upload / prefill / download overlapped)"},
            "gpu_launches": args.steps,
            "clocks": clocks,
            "long": long_sections,
            "long_split": long_split,
            "long_two_phase": long_two_phase,
            "packed": packed_section,
            "prefill_f32": f32_section,
            "gated": {"workload": PREFILL_WORKLOAD, "tokens_per_s": world * tokens / (gms * 1e-3),
                      "ms_per_step": gms,
                      "roofline": {"bound": "hbm", "achieved": gach, "peak": hbm_peak, "unit": "GB/s",
                                   "frac": gach / hbm_peak, "algorithmic_bytes_per_launch": gbytes}},
            "fused": {"workload": PREFILL_WORKLOAD, "H_kv": FUSED_HKV, "read_out": "gated",
                      "tokens_per_s": world * tokens / (fms * 1e-3), "ms_per_step": fms,
                      "roofline": {"bound": "hbm", "achieved": fach, "peak": hbm_peak, "unit": "GB/s",
                                   "frac": fach / hbm_peak, "algorithmic_bytes_per_launch": fbytes}},
            "backward": {"workload": PREFILL_WORKLOAD, "tokens_per_s": world * tokens / (bms * 1e-3),
                         "ms_per_step": bms, "form": "chunked (WY): chunk maps, boundary scans, per-chunk gradients on tf32 tensor cores",
                         "roofline": {"bound": "hbm", "achieved": bach, "peak": hbm_peak, "unit": "GB/s",
                                      "frac": bach / hbm_peak, "algorithmic_bytes_per_launch": bbytes}},
            "decode": {"workload": DECODE_WORKLOAD, "B": dB, "H": dH, "steps_per_s": 1000.0 / dms,
                       "tokens_per_s": world * dB / (dms * 1e-3), "ms_per_step": dms,
                       "timing": f"{nsteps} steps back to back, one event pair around them",
                       "ms_per_step_single_launch": dms_launch,
                       "roofline": {"bound": "hbm", "achieved": dach, "peak": hbm_peak, "unit": "GB/s",
                                    "frac": dach / hbm_peak, "algorithmic_bytes_per_launch": dbytes}},
            "decode_fused": {"workload": DECODE_WORKLOAD, "H_kv": FUSED_HKV, "read_out": "gated",
                             "steps_per_s": 1000.0 / dfms, "ms_per_step": dfms,
                             "timing": f"{nsteps} steps back to back, one event pair around them",
                             "roofline": {"bound": "hbm", "achieved": dfach, "peak": hbm_peak, "unit": "GB/s",
                                          "frac": dfach / hbm_peak, "algorithmic_bytes_per_launch": dfbytes}},
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
