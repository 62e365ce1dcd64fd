#!/usr/bin/env python
"""Benchmark of the HSTU jagged layer stack on B200 through the C ABI.

One step = one forward pass of the 4-layer bf16 HSTU stack over one synthetic jagged batch
(8 users, lengths U{2048..8192}, d_model 512, 8 heads of width 64, interleaved item/action
tokens): per layer the f1 GEMM + SiLU, the jagged causal pointwise attention with relative
position/time bias, LayerNorm(AV) ⊙ U and the f2 GEMM + residual.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun, one process per GPU): every rank runs its own batch (a different seed of
the same workload, weak scaling); no collective sits on the data path, only the timing barrier
and the max-over-ranks reduction of the measured time.

Prints one JSON line on rank 0.  ``value`` is layer-tokens/s (tokens x layers / device time);
the attention kernel's TFLOP/s (unmasked causal FLOPs only) and its roofline fraction are in
``attn_tflops`` and ``roofline``.  The reference arm (``--impl reference``) times the fp64
CPU oracle on the host cores.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from hstu_sequential_transducer_jagged_b200 import workloads as W  # noqa: E402

WORKLOAD = "stack4_bf16_b8_inter"
NOMINAL_BF16_TFLOPS = 2250.0  # dense bf16 tensor-core peak of a B200 (vendor figure, context)
METRIC = "HSTU jagged causal attention TFLOP/s & layer tokens/s on 1 B200 (% of peak)"
UNIT = "layer-tokens/s"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


def attention_pairs(wl) -> int:
    pairs = 0
    for L in wl.lengths.tolist():
        if wl.mask == W.MASK_MFALCON:
            n = max(L - wl.num_candidates, 0)
            m = L - n
            pairs += n * (n + 1) // 2 + m * (n + 1)
        else:
            pairs += L * (L + 1) // 2
    return pairs


def attention_flops(wl) -> float:
    return 4.0 * wl.d_qk * wl.num_heads * attention_pairs(wl)


def gemm_flops(wl) -> float:
    n1 = 2 * wl.num_heads * (wl.d_qk + wl.d_v)
    hv = wl.num_heads * wl.d_v
    return 2.0 * wl.total_tokens * wl.d_model * n1 + 2.0 * wl.total_tokens * hv * wl.d_model


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


def attn_traffic_bytes():
    """DRAM bytes per attention launch from the committed ncu summary (its `traffic_record`
    line), if the kernel source is unchanged since the counters were taken (else None)."""
    summ = os.path.join(ROOT, "profiles", "attn_fwd_pair_stack4_b2.md")
    src = os.path.join(ROOT, "hstu_sequential_transducer_jagged_b200", "csrc", "attn_fwd_pair.cu")
    if not os.path.exists(summ):
        return None
    rec = {}
    with open(summ) as f:
        for line in f:
            if line.strip().startswith("traffic_record "):
                rec = dict(kv.split("=", 1) for kv in line.split()[1:])
    with open(src, "rb") as f:
        digest = hashlib.sha256(f.read()).hexdigest()
    if rec.get("kernel_source_sha256") != digest or "dram_bytes_per_launch" not in rec:
        return None
    return int(rec["dram_bytes_per_launch"])


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20", "-i", str(gpu_index)], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "samples": len(sm),
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------- CPU oracle
def _oracle_layer_once(wl, b, O):
    s, e = int(wl.seq_offsets[b]), int(wl.seq_offsets[b + 1])
    lp = wl.layers[0]
    kw = dict(num_heads=wl.num_heads, d_qk=wl.d_qk, d_v=wl.d_v, max_pos_dist=wl.max_pos_dist,
              num_time_buckets=wl.num_time_buckets, alpha=wl.alpha, mask=wl.mask,
              num_candidates=wl.num_candidates)
    t0 = time.perf_counter()
    O.layer_forward(wl.x[s:e], lp.w1, lp.w2, np.array([0, e - s]), wl.timestamps[s:e],
                    lp.rab_pos, lp.rab_time, **kw)
    return time.perf_counter() - t0


def oracle_cost_model(wl):
    """The fp64 oracle's cost of one layer over the whole workload, scaled from a sample.

    The oracle's layer costs a L + b L^2 seconds for a sequence of L tokens (the two linear
    layers and the LayerNorm grow with L, the attention with its L(L+1)/2 pairs).  It is timed on
    the workload's shortest and its median-length sequence, a and b are fitted through the two
    points, and the fit is summed over every sequence.  Returns (seconds per layer over the
    whole workload, fit, sample description, threads)."""
    from oracle import hstu_oracle as O
    order = np.argsort(wl.lengths)
    b_short, b_mid = int(order[0]), int(order[len(order) // 2])
    t_short = _oracle_layer_once(wl, b_short, O)
    t_mid = _oracle_layer_once(wl, b_mid, O)
    l1, l2 = float(wl.lengths[b_short]), float(wl.lengths[b_mid])
    if l2 > l1:
        # t = a L + b L^2 through (l1, t_short) and (l2, t_mid)
        bq = (t_mid / l2 - t_short / l1) / (l2 - l1)
        a = t_short / l1 - bq * l1
        if a < 0 or bq < 0:  # noisy timings: fall back to pure pair scaling
            a, bq = 0.0, t_mid / (l2 * l2)
    else:
        a, bq = 0.0, t_short / (l1 * l1)
    Ls = wl.lengths.astype(np.float64)
    full = float(np.sum(a * Ls + bq * Ls * Ls))
    sample = (f"fp64 oracle, one layer over sequences {b_short} ({int(l1)} tokens) and {b_mid} "
              f"({int(l2)} tokens) of {wl.name} seed 0 ({t_short + t_mid:.1f} s of CPU work); "
              f"t(L) = a L + b L^2 fitted through them and summed over all {wl.num_seqs} "
              f"sequences ({wl.total_tokens} tokens): {full:.0f} s per layer")
    return full, (a, bq), sample, len(os.sched_getaffinity(0))


def reduce_over_ranks(values_max, values_sum, device):
    """Across the ranks of the default process group: the maximum of each of values_max (the
    ranks' device times: the job is as slow as its slowest rank) and the sum of each of
    values_sum (tokens: weak scaling, every rank its own batch).  Every rank calls it in the
    same order with lists of the same lengths."""
    import torch
    import torch.distributed as dist
    vmax = torch.tensor(list(values_max), device=device, dtype=torch.float64)
    vsum = torch.tensor(list(values_sum), device=device, dtype=torch.float64)
    if vmax.numel():
        dist.all_reduce(vmax, op=dist.ReduceOp.MAX)
    if vsum.numel():
        dist.all_reduce(vsum, op=dist.ReduceOp.SUM)
    return [float(v) for v in vmax.tolist()], [float(v) for v in vsum.tolist()]


def run_reference(args, rank):
    """The reference arm: the fp64 CPU oracle (the pages give no implementation to run).  The
    warm-up fits the oracle's cost model (oracle_cost_model); each timed step runs one oracle layer
    over the workload's shortest sequence and is scaled to the whole workload by that model."""
    if rank != 0:
        return
    wl = W.make(WORKLOAD, seed=args.seed)
    from oracle import hstu_oracle as O
    full, (a, bq), fit_sample, cores = oracle_cost_model(wl)
    b = int(np.argmin(wl.lengths))
    Lb = float(wl.lengths[b])
    scale = full / (a * Lb + bq * Lb * Lb)
    for _ in range(max(args.warmup - 2, 0)):
        _oracle_layer_once(wl, b, O)
    el = 0.0
    for _ in range(args.steps):
        el += _oracle_layer_once(wl, b, O)
    # one step = one layer over the whole workload, predicted from the timed sample
    step_s = el / args.steps * scale
    value = wl.total_tokens / step_s
    sample = (f"each step: one fp64 oracle layer over sequence {b} ({int(Lb)} tokens, the "
              f"shortest), scaled x{scale:.1f} to all {wl.num_seqs} sequences by the cost model "
              f"of the warm-up ({fit_sample})")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * step_s, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "description": wl.description, "seed": args.seed},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------- our arm
def truncate_batch(wl, b):
    """The first b sequences of a workload (a smaller case of the same shapes)."""
    T = int(wl.seq_offsets[b])
    wl.lengths = wl.lengths[:b]
    wl.seq_offsets = wl.seq_offsets[:b + 1]
    wl.timestamps = wl.timestamps[:T]
    wl.x = wl.x[:T]
    return wl


def run_attention_only(args, lib, Bd, desc, ly, x, y, ws, stream, wl):
    """Time the attention stage of layer 0 alone (f1 runs once first to fill Q/K/V)."""
    import torch
    sp = ctypes.c_void_p(stream.cuda_stream)

    def stage(k):
        st = lib.hstu_layer_forward_stage(
            ctypes.byref(desc), k, ctypes.c_void_p(x.data_ptr()),
            ctypes.c_void_p(ly["w1"].data_ptr()), None, ctypes.c_void_p(ly["w2"].data_ptr()),
            None, ctypes.c_void_p(y.data_ptr()), ws.ptr, ws.nbytes, sp)
        if st != 0:
            raise Bd.HstuError(st, f"stage {k}")

    stage(1)
    for _ in range(args.warmup):
        stage(2)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    for a, b in ev:
        a.record(stream)
        stage(2)
        b.record(stream)
    torch.cuda.synchronize()
    if ws.sync_status() != 0:
        raise RuntimeError("device status word set")
    ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    fl = attention_flops(wl)
    print(json.dumps({"mode": "attn", "workload": wl.name, "seqs": wl.num_seqs,
                      "tokens": wl.total_tokens, "attn_ms": ms,
                      "attn_tflops": fl / (ms / 1e3) / 1e12}), flush=True)


def time_attention_fwd_bwd(lib, Bd, dev, steps, warmup, seed=0, batch=0):
    """The attention forward and backward alone on the attention forward+backward workload
    (B=64, L~U{512..2048}, H=8, d=64) through the C ABI with preallocated buffers, L2 flushed
    between timed calls.  FLOPs are the unmasked pairs' algorithmic work: 4 d per pair forward,
    8 d per pair backward (the backward's recomputation of S is reported apart)."""
    import torch
    wl = W.make("attn_fwdbwd_bf16_b64", seed=seed)
    if batch > 0:  # the first `batch` sequences only (profiling aid)
        T = int(wl.seq_offsets[batch])
        wl.lengths, wl.seq_offsets = wl.lengths[:batch], wl.seq_offsets[:batch + 1]
        wl.timestamps, wl.q, wl.k, wl.v, wl.d_o = (a[:T] for a in (wl.timestamps, wl.q, wl.k,
                                                                   wl.v, wl.d_o))
    bf = torch.bfloat16
    q, k, v, d_o = (torch.from_numpy(a).to(bf).to(dev) for a in (wl.q, wl.k, wl.v, wl.d_o))
    off = torch.from_numpy(wl.seq_offsets).to(dev)
    ts = torch.from_numpy(wl.timestamps).to(dev)
    rp = torch.from_numpy(wl.rab_pos).to(dev)
    rt = torch.from_numpy(wl.rab_time).to(dev)
    o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    d_pos, d_time = torch.empty_like(rp), torch.empty_like(rt)
    desc = Bd.attn_desc(seq_offsets=off, total_tokens=wl.total_tokens,
                        max_seq_len=int(wl.lengths.max()), timestamps=ts,
                        num_heads=wl.num_heads, d_qk=wl.d_qk, d_v=wl.d_v, ld_q=q.stride(0),
                        ld_k=k.stride(0), ld_v=v.stride(0), ld_o=o.stride(0), rab_pos=rp,
                        max_pos_dist=wl.max_pos_dist, rab_time=rt,
                        num_time_buckets=wl.num_time_buckets, alpha=wl.alpha)
    ws = Bd.Workspace(lib.hstu_attention_backward_workspace_size(ctypes.byref(desc)), dev)
    stream = torch.cuda.current_stream()
    sp = ctypes.c_void_p(stream.cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def fwd():
        st = lib.hstu_attention_forward(ctypes.byref(desc), P(q), P(k), P(v), P(o), ws.ptr,
                                        ws.nbytes, sp)
        if st != 0:
            raise Bd.HstuError(st, "hstu_attention_forward")

    def bwd():
        st = lib.hstu_attention_backward(ctypes.byref(desc), P(q), P(k), P(v), P(d_o), P(dq),
                                         P(dk), P(dv), P(d_pos), P(d_time), ws.ptr, ws.nbytes, sp)
        if st != 0:
            raise Bd.HstuError(st, "hstu_attention_backward")

    res = {}
    for name, fn in (("fwd", fwd), ("bwd", bwd)):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for a, b in ev:
            flush.zero_()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        res[name] = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    if ws.sync_status() != 0:
        raise RuntimeError("device status word set")
    pairs = attention_pairs(wl) * wl.num_heads
    return {"workload": wl.name, "tokens": wl.total_tokens, "steps": steps,
            "fwd_ms": res["fwd"], "fwd_tflops": 4.0 * wl.d_qk * pairs / (res["fwd"] / 1e3) / 1e12,
            "bwd_ms": res["bwd"], "bwd_tflops": 8.0 * wl.d_qk * pairs / (res["bwd"] / 1e3) / 1e12,
            "bwd_recompute_gflop": 2.0 * wl.d_qk * pairs / 1e9,
            "bwd_tflops_incl_recompute": 10.0 * wl.d_qk * pairs / (res["bwd"] / 1e3) / 1e12,
            "tokens_per_s_fwd_bwd": wl.total_tokens / ((res["fwd"] + res["bwd"]) / 1e3),
            "l2": "256 MB buffer written before each timed call (outside its events)"}


def run_attention_bwd(args, lib, Bd, dev):
    r = time_attention_fwd_bwd(lib, Bd, dev, args.steps, args.warmup, args.seed, args.batch)
    r["mode"] = "attn_bwd"
    print(json.dumps(r), flush=True)


def time_layer_stack(lib, Bd, dev, name, steps, warmup, seed=0):
    """A layer-stack workload through hstu_layer_forward_stage, with CUDA events around every
    attention stage; L2 flushed between steps.  Returns tokens/s and the attention's TFLOP/s."""
    import torch
    wl = W.make(name, seed=seed)
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    x = torch.from_numpy(wl.x).to(dt).to(dev)
    off = torch.from_numpy(wl.seq_offsets).to(dev)
    ts = torch.from_numpy(wl.timestamps).to(dev)
    layers = [dict(w1=torch.from_numpy(lp.w1).to(dt).to(dev), w2=torch.from_numpy(lp.w2).to(dt).to(dev),
                   rp=torch.from_numpy(lp.rab_pos).to(dev), rt=torch.from_numpy(lp.rab_time).to(dev))
              for lp in wl.layers]
    descs = [Bd.layer_desc(seq_offsets=off, total_tokens=wl.total_tokens,
                           max_seq_len=wl.max_seq_len, timestamps=ts, d_model=wl.d_model,
                           num_heads=wl.num_heads, d_qk=wl.d_qk, d_v=wl.d_v, mask=wl.mask,
                           num_candidates=wl.num_candidates, microbatch=wl.microbatch or 1,
                           rab_pos=ly["rp"], max_pos_dist=wl.max_pos_dist, rab_time=ly["rt"],
                           num_time_buckets=wl.num_time_buckets, alpha=wl.alpha,
                           ln_eps=wl.ln_eps, dtype=Bd._dtype_code(x)) for ly in layers]
    ws = Bd.Workspace(lib.hstu_layer_workspace_size(ctypes.byref(descs[0])), dev)
    bufs = [torch.empty_like(x), torch.empty_like(x)]
    stream = torch.cuda.current_stream()
    sp = ctypes.c_void_p(stream.cuda_stream)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    L = len(layers)

    def run(attn_ev=None):
        cur = x
        for l in range(L):
            out = bufs[l % 2]
            for stage in (1, 2, 3):
                if attn_ev is not None and stage == 2:
                    attn_ev[l][0].record(stream)
                st = lib.hstu_layer_forward_stage(
                    ctypes.byref(descs[l]), stage, ctypes.c_void_p(cur.data_ptr()),
                    ctypes.c_void_p(layers[l]["w1"].data_ptr()), None,
                    ctypes.c_void_p(layers[l]["w2"].data_ptr()), None,
                    ctypes.c_void_p(out.data_ptr()), ws.ptr, ws.nbytes, sp)
                if st != 0:
                    raise Bd.HstuError(st, f"{name} layer {l} stage {stage}")
                if attn_ev is not None and stage == 2:
                    attn_ev[l][1].record(stream)
            cur = out

    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
    attn_ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(L)] for _ in range(steps)]
    for k in range(steps):
        flush.zero_()
        step_ev[k][0].record(stream)
        run(attn_ev[k])
        step_ev[k][1].record(stream)
    torch.cuda.synchronize()
    if ws.sync_status() != 0:
        raise RuntimeError(f"{name}: device status word set")
    ms = float(np.mean([a.elapsed_time(b) for a, b in step_ev]))
    attn_ms = float(np.mean([a.elapsed_time(b) for row in attn_ev for a, b in row]))
    aflops = attention_flops(wl)
    return {"workload": wl.name, "dtype": wl.dtype, "tokens": wl.total_tokens, "layers": L,
            "steps": steps, "ms_per_step": ms,
            "layer_tokens_per_s": wl.total_tokens * L / (ms / 1e3),
            "attn_ms_per_layer": attn_ms, "attn_tflops": aflops / (attn_ms / 1e3) / 1e12,
            "stack_tflops": L * (aflops + gemm_flops(wl)) / (ms / 1e3) / 1e12,
            "l2": "256 MB buffer written between steps (outside the step events)"}


def time_layer_backward(lib, Bd, dev, steps, warmup, seed=0, batch=0):
    """One layer's backward (hstu_layer_backward, forward recomputed inside) on layer 0 of the
    4-layer workload, next to that layer's forward; L2 flushed between timed calls.  FLOPs:
    forward f1 + attention + f2, backward 2x the GEMMs and 8 d per attention pair (plus the
    recomputed forward, reported apart)."""
    import torch
    wl = W.make(WORKLOAD, seed=seed)
    if batch > 0:
        wl = truncate_batch(wl, batch)
    bf = torch.bfloat16
    lp = wl.layers[0]
    x = torch.from_numpy(wl.x).to(bf).to(dev)
    w1 = torch.from_numpy(lp.w1).to(bf).to(dev)
    w2 = torch.from_numpy(lp.w2).to(bf).to(dev)
    off = torch.from_numpy(wl.seq_offsets).to(dev)
    ts = torch.from_numpy(wl.timestamps).to(dev)
    rp, rt = torch.from_numpy(lp.rab_pos).to(dev), torch.from_numpy(lp.rab_time).to(dev)
    d_y = torch.randn(x.shape, generator=torch.Generator().manual_seed(seed)).to(bf).to(dev)
    kw = dict(num_heads=wl.num_heads, d_qk=wl.d_qk, d_v=wl.d_v, max_pos_dist=wl.max_pos_dist,
              num_time_buckets=wl.num_time_buckets, alpha=wl.alpha)
    desc = Bd.layer_desc(seq_offsets=off, total_tokens=wl.total_tokens, max_seq_len=wl.max_seq_len,
                         timestamps=ts, d_model=wl.d_model, rab_pos=rp, rab_time=rt,
                         ln_eps=wl.ln_eps, **kw)
    ws = Bd.Workspace(lib.hstu_layer_backward_workspace_size(ctypes.byref(desc)), dev)
    y = torch.empty_like(x)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def fwd():
        Bd.layer_forward(x, w1, w2, off, wl.max_seq_len, ts, rp, rt, out=y, ws=ws, **kw)

    def bwd():
        Bd.layer_backward(x, w1, w2, d_y, off, wl.max_seq_len, ts, rp, rt, ws=ws, **kw)

    res = {}
    for name, fn in (("fwd", fwd), ("bwd", bwd)):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for a, b in ev:
            flush.zero_()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        res[name] = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    if ws.sync_status() != 0:
        raise RuntimeError("device status word set")
    aflops, gflops = attention_flops(wl), gemm_flops(wl)
    bwd_alg = 2 * gflops + 2 * aflops  # dX, dW per GEMM; 8 d per pair for the attention
    return {"workload": wl.name + " layer 0", "tokens": wl.total_tokens, "steps": steps,
            "fwd_ms": res["fwd"], "bwd_ms": res["bwd"],
            "fwd_bwd_tokens_per_s": wl.total_tokens / ((res["fwd"] + res["bwd"]) / 1e3),
            "bwd_tflops_algorithmic": bwd_alg / (res["bwd"] / 1e3) / 1e12,
            "bwd_recompute_gflop": (aflops + gflops) / 1e9,
            "l2": "256 MB buffer written before each timed call (outside its events)"}


def measure_other_configs(lib, Bd, dev, peaks):
    """The other four workloads, each timed on its own (they are parity cases of the same
    kernels; the headline line is the 4-layer stack)."""
    pk = peaks["bf16_tflops"]
    out = {}
    for name, steps in (("layer_fp32_b4", 200), ("layer_bf16_b32_geo", 200),
                        ("mfalcon_bf16_b16", 30)):
        r = time_layer_stack(lib, Bd, dev, name, steps, 5)
        if r["dtype"] == "bf16":
            r["attn_frac_of_bf16_peak"] = r["attn_tflops"] / pk
        out[name] = r
    r = time_attention_fwd_bwd(lib, Bd, dev, 30, 3)
    r["fwd_frac_of_bf16_peak"] = r["fwd_tflops"] / pk
    r["bwd_frac_of_bf16_peak"] = r["bwd_tflops"] / pk
    out[r["workload"]] = r
    r = time_layer_backward(lib, Bd, dev, 10, 3)
    r["bwd_frac_of_bf16_peak"] = r["bwd_tflops_algorithmic"] / pk
    out["layer_backward"] = r
    return out


def run_e2e_pipelined(K, L, layers, wl, xh, offh, tsh, yh_serial, x, off, ts, stream, ws, world,
                      dev):
    """End to end through binding.layer_forward with the copies of neighbouring steps overlapped:
    step i's inputs go host-to-device on one copy stream and its output device-to-host on a
    second, into double buffers, while the compute stream runs the layers of the step between.
    Every step still copies its inputs in and its result out inside the timed region.  Returns
    (elapsed ms over K steps, check) or None; the last output is compared with the serial step's
    (the kernels are deterministic, so the two must be identical)."""
    import torch
    import torch.distributed as dist
    from hstu_sequential_transducer_jagged_b200 import binding as Bd
    if K < 2:
        return None
    h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    xd = [torch.empty_like(x) for _ in range(2)]
    offd = [torch.empty_like(off) for _ in range(2)]
    tsd = [torch.empty_like(ts) for _ in range(2)]
    yd = [torch.empty_like(x) for _ in range(2)]
    mid = [torch.empty_like(x) for _ in range(2)]
    yh = [torch.empty_like(yh_serial).pin_memory() for _ in range(2)]
    ev = lambda: torch.cuda.Event()  # noqa: E731
    h2d_done, comp_done, d2h_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def step(i):
        sl = i % 2
        if i >= 2:
            h2d_s.wait_event(comp_done[sl])  # step i-2 has finished reading this slot's inputs
        with torch.cuda.stream(h2d_s):
            xd[sl].copy_(xh, non_blocking=True)
            offd[sl].copy_(offh, non_blocking=True)
            tsd[sl].copy_(tsh, non_blocking=True)
            h2d_done[sl].record(h2d_s)
        stream.wait_event(h2d_done[sl])
        if i >= 2:
            stream.wait_event(d2h_done[sl])  # step i-2's result has left this slot's output
        cur = xd[sl]
        for l in range(L):
            ly = layers[l]
            out = yd[sl] if l == L - 1 else mid[l % 2]
            cur = Bd.layer_forward(cur, ly["w1"], ly["w2"], offd[sl], wl.max_seq_len, tsd[sl],
                                   ly["rp"], ly["rt"], num_heads=wl.num_heads, d_qk=wl.d_qk,
                                   d_v=wl.d_v, max_pos_dist=wl.max_pos_dist,
                                   num_time_buckets=wl.num_time_buckets, alpha=wl.alpha,
                                   mask=wl.mask, num_candidates=wl.num_candidates, out=out,
                                   ws=ws, stream=stream)
        comp_done[sl].record(stream)
        d2h_s.wait_event(comp_done[sl])
        with torch.cuda.stream(d2h_s):
            yh[sl].copy_(yd[sl], non_blocking=True)
            d2h_done[sl].record(d2h_s)

    def drain():
        for e in d2h_done:
            stream.wait_event(e)

    for i in range(2):  # warm-up
        step(i)
    drain()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d_s.wait_event(e0)
    d2h_s.wait_event(e0)
    for i in range(K):
        step(i)
    drain()
    e1.record(stream)
    torch.cuda.synchronize()
    p_ms = e0.elapsed_time(e1)
    if world > 1:
        (p_ms,), _ = reduce_over_ranks([p_ms], [], dev)
    same = torch.equal(yh[(K - 1) % 2], yh_serial)
    return p_ms, ("output identical to the serial step" if same else "output differs: not used")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)  # about 1 s of device time
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other four workloads (timed after the headline line)")
    ap.add_argument("--mode", default="stack", choices=["stack", "attn", "attn_bwd", "layer_bwd"],
                    help="attn: time only the attention stage of layer 0 (profiling aid); "
                         "attn_bwd: attention forward and backward on the B=64 workload")
    ap.add_argument("--batch", type=int, default=0,
                    help="use only the first B sequences of the workload (profiling aid)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return

    import torch
    import torch.distributed as dist
    from hstu_sequential_transducer_jagged_b200 import binding as Bd

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    lib = Bd.lib()
    if args.mode == "attn_bwd":
        run_attention_bwd(args, lib, Bd, dev)
        return
    if args.mode == "layer_bwd":
        r = time_layer_backward(lib, Bd, dev, args.steps, args.warmup, args.seed, args.batch)
        r["mode"] = "layer_bwd"
        print(json.dumps(r), flush=True)
        return

    # CPU oracle baseline first (rank 0, one GPU), before any other GPU work
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        wl0 = W.make(WORKLOAD, seed=args.seed)
        full, _, sample, cores = oracle_cost_model(wl0)
        cpu = {"value": wl0.total_tokens / full, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": sample}
        del wl0

    wl = W.make(WORKLOAD, seed=args.seed + rank)
    if args.batch > 0:
        wl = truncate_batch(wl, args.batch)
    T, L = wl.total_tokens, len(wl.layers)
    bf = torch.bfloat16
    x = torch.from_numpy(wl.x).to(bf).to(dev)
    off = torch.from_numpy(wl.seq_offsets).to(dev)
    ts = torch.from_numpy(wl.timestamps).to(dev)
    layers = []
    for lp in wl.layers:
        layers.append(dict(w1=torch.from_numpy(lp.w1).to(bf).to(dev),
                           w2=torch.from_numpy(lp.w2).to(bf).to(dev),
                           rp=torch.from_numpy(lp.rab_pos).to(dev),
                           rt=torch.from_numpy(lp.rab_time).to(dev)))
    bufs = [torch.empty_like(x), torch.empty_like(x)]
    descs = [Bd.layer_desc(seq_offsets=off, total_tokens=T, max_seq_len=wl.max_seq_len,
                           timestamps=ts, d_model=wl.d_model, num_heads=wl.num_heads,
                           d_qk=wl.d_qk, d_v=wl.d_v, mask=wl.mask,
                           num_candidates=wl.num_candidates, microbatch=wl.microbatch or 1,
                           rab_pos=ly["rp"], max_pos_dist=wl.max_pos_dist, rab_time=ly["rt"],
                           num_time_buckets=wl.num_time_buckets, alpha=wl.alpha,
                           ln_eps=wl.ln_eps) for ly in layers]
    ws_bytes = lib.hstu_layer_workspace_size(ctypes.byref(descs[0]))
    ws = Bd.Workspace(ws_bytes, dev)
    stream = torch.cuda.current_stream()
    sp = ctypes.c_void_p(stream.cuda_stream)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def run_stack(attn_events=None):
        cur = x
        for l in range(L):
            out = bufs[l % 2]
            ly = layers[l]
            for stage in (1, 2, 3):
                if attn_events is not None and stage == 2:
                    attn_events[l][0].record(stream)
                st = lib.hstu_layer_forward_stage(
                    ctypes.byref(descs[l]), stage, ctypes.c_void_p(cur.data_ptr()),
                    ctypes.c_void_p(ly["w1"].data_ptr()), None,
                    ctypes.c_void_p(ly["w2"].data_ptr()), None,
                    ctypes.c_void_p(out.data_ptr()), ws.ptr, ws.nbytes, sp)
                if st != 0:
                    raise Bd.HstuError(st, f"layer {l} stage {stage}")
                if attn_events is not None and stage == 2:
                    attn_events[l][1].record(stream)
            cur = out
        return cur

    if args.mode == "attn":
        run_attention_only(args, lib, Bd, descs[0], layers[0], x, bufs[0], ws, stream, wl)
        return

    for _ in range(args.warmup):
        run_stack()
    torch.cuda.synchronize()
    if ws.sync_status() != 0:
        raise RuntimeError("device status word set during warm-up")

    K = args.steps
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)]
    attn_ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(L)] for _ in range(K)]
    sampler = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    for k in range(K):
        flush.zero_()  # L2 flush between steps, outside the step events
        step_ev[k][0].record(stream)
        run_stack(attn_ev[k])
        step_ev[k][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    wall = time.perf_counter() - wall0
    clocks = sampler.stop() if sampler is not None else None
    status = ws.sync_status()
    if status != 0:
        raise RuntimeError(f"device status word {status} after the timed region")

    step_ms = [a.elapsed_time(b) for a, b in step_ev]
    attn_ms = [a.elapsed_time(b) for row in attn_ev for a, b in row]
    total_ms = float(sum(step_ms))
    if world > 1:
        (total_ms,), (tokens_all,) = reduce_over_ranks([total_ms], [float(T)], dev)
    else:
        tokens_all = float(T)
    ms_per_step = total_ms / K
    value = tokens_all * L * K / (total_ms / 1e3)

    # ---- L2-warm reference (informational): a few steps back to back with no flush between
    warm_k = min(K, 10)
    warm_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(warm_k)]
    warm_attn = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(L)] for _ in range(warm_k)]
    for k in range(warm_k):
        warm_ev[k][0].record(stream)
        run_stack(warm_attn[k])
        warm_ev[k][1].record(stream)
    torch.cuda.synchronize()
    l2_warm = {
        "ms_per_step": float(np.mean([a.elapsed_time(b) for a, b in warm_ev])),
        "attn_ms_per_layer": float(np.mean([a.elapsed_time(b) for row in warm_attn
                                            for a, b in row])),
        "steps": warm_k,
    }

    # ---- end to end through the public API with host buffers (pinned), copies timed
    e2e = None
    if args.e2e_steps > 0:
        xh = torch.from_numpy(wl.x).to(bf).pin_memory()
        offh = torch.from_numpy(wl.seq_offsets).pin_memory()
        tsh = torch.from_numpy(wl.timestamps).pin_memory()
        yh = torch.empty_like(xh).pin_memory()
        xd, offd, tsd = torch.empty_like(x), torch.empty_like(off), torch.empty_like(ts)
        e2e_ws = Bd.Workspace(ws_bytes, dev)

        def e2e_step():
            xd.copy_(xh, non_blocking=True)
            offd.copy_(offh, non_blocking=True)
            tsd.copy_(tsh, non_blocking=True)
            cur = xd
            for l in range(L):
                ly = layers[l]
                cur = Bd.layer_forward(cur, ly["w1"], ly["w2"], offd, wl.max_seq_len, tsd,
                                       ly["rp"], ly["rt"], num_heads=wl.num_heads, d_qk=wl.d_qk,
                                       d_v=wl.d_v, max_pos_dist=wl.max_pos_dist,
                                       num_time_buckets=wl.num_time_buckets, alpha=wl.alpha,
                                       mask=wl.mask, num_candidates=wl.num_candidates,
                                       out=bufs[l % 2], ws=e2e_ws)
            yh.copy_(cur, non_blocking=True)

        for _ in range(2):
            e2e_step()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1)
        if world > 1:
            (e2e_ms,), _ = reduce_over_ranks([e2e_ms], [], dev)
        h2d = xh.numel() * xh.element_size() + offh.numel() * 4 + tsh.numel() * 8
        d2h = yh.numel() * yh.element_size()
        serial_value = tokens_all * L * args.e2e_steps / (e2e_ms / 1e3)
        e2e = {"value": serial_value, "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "api": "binding.layer_forward (hstu_layer_forward) x layers, pinned host buffers",
               "pipelined": False}
        try:
            piped = run_e2e_pipelined(args.e2e_steps, L, layers, wl, xh, offh, tsh, yh, x, off,
                                      ts, stream, e2e_ws, world, dev)
        except Exception as exc:  # noqa: BLE001 -- keep the serial figure whatever went wrong
            piped = None
            e2e["pipeline_check"] = f"not run: {type(exc).__name__}: {exc}"[:200]
        if piped is not None:
            p_ms, check = piped
            e2e["serial_value"] = serial_value
            e2e["pipeline_check"] = check
            if check == "output identical to the serial step":
                e2e["value"] = tokens_all * L * args.e2e_steps / (p_ms / 1e3)
                e2e["pipelined"] = True
                e2e["api"] += ("; step i+1's host-to-device copy and step i-1's device-to-host "
                               "copy overlap step i's layers (two copy streams, double buffers)")

    peaks = load_peaks()
    configs = None
    if world == 1 and not args.no_configs:
        configs = measure_other_configs(lib, Bd, dev, peaks)

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    aflops = attention_flops(wl)
    attn_avg_ms = float(np.mean(attn_ms))
    attn_tflops = aflops / (attn_avg_ms / 1e3) / 1e12
    traffic = attn_traffic_bytes()
    # The SiLU's tanh costs one MUFU operation per score and the MUFU pipe takes 16 per clock per
    # SM, so the attention cannot exceed 16 x 4 d FLOP per clock per SM (at the sampled clock).
    sm_mhz = (clocks or {}).get("sm_mhz") or 1965.0
    n_sms = torch.cuda.get_device_properties(dev).multi_processor_count
    ceil_tflops = 16 * 4 * wl.d_qk * n_sms * sm_mhz * 1e6 / 1e12
    epi_ceiling = {"value": ceil_tflops, "unit": "TFLOP/s",
                   "basis": f"one MUFU tanh per score, 16 per clock per SM, {n_sms} SMs at "
                            f"{sm_mhz:.0f} MHz", "attn_frac": attn_tflops / ceil_tflops}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "description": wl.description, "tokens_per_rank": T,
                   "layers": L, "global_batch": wl.num_seqs * world,
                   "parallelism": f"independent batch per GPU x{world} (no collective)",
                   "l2": "256 MB buffer written between timed steps (outside step events)"},
        "attn_tflops": attn_tflops,
        "attn_ms_per_layer": attn_avg_ms,
        "stack_tflops": (L * (aflops + gemm_flops(wl))) / (ms_per_step / 1e3) / 1e12,
        "roofline": {"bound": "tensor", "kernel": "attn_fwd_pair_kernel (+ its work-list "
                     "kernel, inside the same events)", "achieved": attn_tflops,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": attn_tflops / peaks["bf16_tflops"],
                     "peak_source": f"{peaks['source']} bf16 (burst)",
                     "traffic": traffic,
                     "algorithmic_flops_per_launch": aflops},
        "attn_frac_of_nominal": attn_tflops / NOMINAL_BF16_TFLOPS,
        "epilogue_ceiling": epi_ceiling,
        "l2_warm": l2_warm,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "configs": configs,
        "clocks": clocks,
        # per layer: f1 GEMM, work list, attention (which also leaves the LayerNorm statistics),
        # and the fused Norm(AV) * U + f2 kernel (bf16 with H d_v and d_model <= 512), or
        # LayerNorm * U and the f2 GEMM
        "gpu_launches": (4 if wl.num_heads * wl.d_v <= 512 and wl.d_model <= 512 else 5) * L * K,
        "wall_s_timed_region": wall,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
