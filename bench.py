#!/usr/bin/env python
"""Benchmark of the FP8 vision-encoder attention path on B200.

One step = one dynamic-scaling forward of the 8192-token, 16-head,
head_dim-128 workload: amax ring update + per-tensor e4m3 quantize of Q/K/V
(one cooperative launch) -> varlen FP8 attention (BF16 out) -> per-token-group e4m3 quantize of
the attention output viewed as [8192, 2048].  Inputs are seeded synthetic
BF16 (N(0,1), 1% of channels x8) for 20 forwards, resident in HBM, rotated
step by step (2.0 GB > 126 MB L2).

Prints one JSON line: metric = counted attention TFLOP/s (4*S^2*D*H per
image), whole job over all ranks, plus the attention kernel's roofline, the
oracle's CPU baseline, an end-to-end number through host buffers, clocks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU: launched under torch.distributed.run, one rank per GPU; every
rank runs its own replica of the workload (weak scaling, no collective on
the data path); timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "FP8 varlen attention TFLOP/s (counted 4*S^2*D*H) over the full step"
UNIT = "TFLOP/s"
WORKLOAD = "1x8192_d128"


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def _source_sha(path):
    return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]


def _traffic(kernel_src: str, workload: str):
    """DRAM bytes per launch recorded from an ncu capture, if it was taken on
    the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        e = d.get(workload)
        if e and e.get("source_sha") == _source_sha(kernel_src):
            return float(e["dram_bytes_per_launch"])
    except Exception:
        return None
    return None


def _host_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def _oracle_rows_time_mt(w, codes, desc, budget_s: float, seed: int, threads: int):
    """The oracle's attention on seeded (token, head) rows from `threads`
    host threads at once (each thread runs the unchanged single-threaded
    oracle on rows of its own; the C call releases the GIL); returns
    (counted FLOPs, wall seconds, rows)."""
    import concurrent.futures as cf
    if threads <= 1:
        return _oracle_rows_time(w, codes, desc, budget_s, seed)
    t0 = time.perf_counter()
    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        parts = list(ex.map(lambda i: _oracle_rows_time(w, codes, desc, budget_s, seed * 1000 + i),
                            range(threads)))
    wall = time.perf_counter() - t0
    return sum(p[0] for p in parts), wall, sum(p[2] for p in parts)


def _oracle_rows_time(w, codes, desc, rows_budget_s: float, seed: int):
    """Time the oracle's attention on seeded (token, head) rows until the
    budget is spent; returns (counted FLOPs, seconds, rows)."""
    import oracle
    import synth
    cu = synth.cu_seqlens(w.seg_lens)
    rng = np.random.default_rng(seed)
    flops, secs, rows = 0.0, 0.0, 0
    batch = 8
    while secs < rows_budget_s:
        toks = rng.integers(0, w.tokens, size=batch).astype(np.int64)
        hs = rng.integers(0, w.heads, size=batch).astype(np.int32)
        t0 = time.perf_counter()
        oracle.attn_pairs(*codes, *desc, cu, w.heads, w.head_dim, w.softmax_scale, toks, hs)
        secs += time.perf_counter() - t0
        for t in toks:
            seg = int(np.searchsorted(cu, t, side="right") - 1)
            S = int(cu[seg + 1] - cu[seg])
            flops += 4.0 * S * w.head_dim
        rows += batch
    return flops, secs, rows


def _oracle_inputs(w):
    """The oracle's e4m3 codes and descales of forward 0: static scales from
    the margin x the exact amax, or a fresh ring's first update."""
    import oracle
    q, k, v = w.qkv(0)
    amax = [oracle.amax_bf16(x) for x in (q, k, v)]
    if w.mode == "static":
        desc = [oracle.descale_from_amax(np.float32(w.margin) * np.float32(a)) for a in amax]
    else:
        desc = list(oracle.Ring().update(amax))
    codes = [oracle.quantize_per_tensor(x, d).reshape(w.tokens, w.heads, w.head_dim)
             for x, d in zip((q, k, v), desc)]
    return codes, desc


def _sample_rows(cu: np.ndarray, heads: int, per_seg: int, seed: int):
    """(token, head) rows per image: its first and last rows, the rows on both
    sides of the first 128-row tile edge, its middle row and seeded random
    rows, with the heads cycling."""
    rng = np.random.default_rng(seed)
    toks, hs = [], []
    for i in range(len(cu) - 1):
        a, L = int(cu[i]), int(cu[i + 1] - cu[i])
        if L <= 0:
            continue
        fixed = sorted({0, L - 1, min(127, L - 1), min(128, L - 1), L // 2})
        rows = fixed + [int(r) for r in rng.integers(0, L, size=max(0, per_seg - len(fixed)))]
        for n, r in enumerate(rows):
            toks.append(a + r)
            hs.append((n + i) % heads)
    return np.array(toks, dtype=np.int64), np.array(hs, dtype=np.int32)


def _attn_error_stats(got: np.ndarray, ref: np.ndarray) -> dict:
    """Raw max-abs, mean-abs, the max excess over half a BF16 spacing of the
    exact value (the output format's own rounding) and the cosine."""
    got = got.astype(np.float64).ravel()
    ref = ref.astype(np.float64).ravel()
    d = np.abs(got - ref)
    a = np.abs(ref)
    half_ulp = np.where(a > 0, 0.5 * np.exp2(np.floor(np.log2(np.where(a > 0, a, 1.0))) - 7), 0.0)
    cos = float(np.dot(got, ref) / (np.linalg.norm(got) * np.linalg.norm(ref) + 1e-300))
    return {"max_abs": float(d.max()), "mean_abs": float(d.mean()),
            "max_excess_over_bf16_rounding": float(np.maximum(0.0, d - half_ulp).max()),
            "cos": cos}


def _parity_from_outputs(w, codes, desc, got_desc, got_codes, got_out_bits, per_seg=32,
                         seed=11):
    """Forward 0 of the workload, as the kernels computed it from a fresh ring,
    against the oracle: descales and e4m3 codes bit for bit, and the attention
    output on sampled (token, head) rows (fp64 oracle rows, computed one by
    one) against the gate max-abs 3e-2 over the BF16 rounding, mean-abs 3e-3,
    cosine 0.999."""
    import oracle
    import synth
    cu = synth.cu_seqlens(w.seg_lens)
    want_desc = np.asarray(desc, dtype=np.float32)
    desc_exact = bool((np.asarray(got_desc, dtype=np.float32).view(np.uint32) ==
                       want_desc.view(np.uint32)).all())
    codes_exact = bool(all(np.array_equal(np.asarray(g).reshape(-1), np.asarray(c).reshape(-1))
                           for g, c in zip(got_codes, codes)))
    toks, hs = _sample_rows(cu, w.heads, per_seg, seed)
    ref = oracle.attn_pairs(*codes, *desc, cu, w.heads, w.head_dim, w.softmax_scale, toks, hs)
    got = synth.bf16_to_float(np.ascontiguousarray(got_out_bits[toks, hs])).astype(np.float64)
    e = _attn_error_stats(got, ref)
    e.update({"rows": int(len(toks)), "descales_bit_exact": desc_exact,
              "codes_bit_exact": codes_exact,
              "within_gate": bool(desc_exact and codes_exact and
                                  e["max_excess_over_bf16_rounding"] <= 3e-2 and
                                  e["mean_abs"] <= 3e-3 and e["cos"] >= 0.999)})
    return e


def _parity_field(w, codes, desc, fwd0) -> dict:
    """The line's parity record; a failure of the check itself is reported in
    the record (with the exception) instead of costing the whole line."""
    if isinstance(fwd0, Exception):
        return {"error": repr(fwd0)}
    try:
        return _parity_from_outputs(w, codes, desc, *fwd0)
    except Exception as exc:  # reported, not dropped
        return {"error": repr(exc)}


def _forward0_outputs(fv, ctx, w, qkv0, cu_d, max_s, q8, k8, v8, out, dev, static_desc=None):
    """Runs forward 0 again (after the timed region; dynamic workloads from a
    fresh ring, static ones with their calibrated descales) and returns what
    the kernels produced: descales, e4m3 codes, BF16 output bits (host arrays;
    compared with the oracle by the CPU-baseline leg)."""
    import torch
    if static_desc is not None:
        desc0 = static_desc
        fv.fp8_quantize_qkv_per_tensor(*qkv0, desc0, q8, k8, v8, ctx=ctx)
    else:
        ring0 = fv.new_ring(dev)
        desc0 = torch.zeros(3, dtype=torch.float32, device=dev)
        fv.fp8_amax_ring_quantize_qkv(*qkv0, ring0, desc0, q8, k8, v8, ctx=ctx)
    fv.fp8_varlen_attn_fwd(q8, k8, v8, desc0[0:1], desc0[1:2], desc0[2:3], cu_d, max_s,
                           w.softmax_scale, out, ctx=ctx)
    st, site = ctx.check()
    if st != fv.OK:
        raise RuntimeError(f"device fault in the parity forward: {fv.status_string(st)} "
                           f"site {site}")
    got_out = out.view(torch.int16).cpu().numpy().view(np.uint16)
    got_codes = [t.cpu().numpy() for t in (q8, k8, v8)]
    return desc0.cpu().numpy(), got_codes, got_out


def run_reference(args):
    """The oracle (plain single-threaded C, run on rows of its own by every
    host thread) as the reference arm."""
    ws, rank, _ = _dist()
    if rank != 0:
        return 0
    import synth
    w = synth.WORKLOADS[args.workload]
    codes, desc = _oracle_inputs(w)
    # each step a bounded sample: the whole run stays within about two minutes
    per_step = min(args.ref_step_seconds, 120.0 / max(1, args.steps + args.warmup / 4))
    threads = _host_threads()
    for _ in range(args.warmup):
        _oracle_rows_time_mt(w, codes, desc, per_step / 4, seed=1, threads=threads)
    tot_f, tot_s, tot_rows = 0.0, 0.0, 0
    for s in range(args.steps):
        f, sec, rows = _oracle_rows_time_mt(w, codes, desc, per_step, seed=100 + s,
                                            threads=threads)
        tot_f += f
        tot_s += sec
        tot_rows += rows
    value = tot_f / tot_s / 1e12
    sample = (f"{tot_rows} seeded (token, head) query rows of forward 0's attention "
              f"({tot_rows / args.steps:.0f} per step, {per_step:.2f} s per step on each of "
              f"{threads} host threads; amax/quantize stages excluded)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_s / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": _config(w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _sdpa_comparator(w, inputs, dev, reps=10):
    """torch's BF16 scaled_dot_product_attention on the same BF16 inputs of a
    single-image workload: a library comparator for context, not the metric."""
    import torch
    import torch.nn.functional as F
    if len(w.seg_lens) != 1:
        return None
    T, H, D = w.tokens, w.heads, w.head_dim
    q, k, v = (x.view(1, T, H, D).transpose(1, 2) for x in inputs[0])
    try:
        for _ in range(2):
            F.scaled_dot_product_attention(q, k, v, scale=w.softmax_scale)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            F.scaled_dot_product_attention(q, k, v, scale=w.softmax_scale)
        e1.record()
        torch.cuda.synchronize()
    except Exception as exc:  # no fused BF16 kernel for this shape
        return {"unavailable": str(exc).splitlines()[0][:120]}
    ms = e0.elapsed_time(e1) / reps
    return {"impl": "torch.nn.functional.scaled_dot_product_attention, bf16",
            "ms": ms, "tflops": w.attn_flops() / (ms * 1e-3) / 1e12}


def _bf16_comparator(fv, ctx, w, inputs, dev, reps=10):
    """This library's BF16 attention kernel (same skeleton as the FP8 one,
    kind::f16 MMAs) on the same BF16 inputs: the BF16 side of the pages'
    BF16-vs-FP8 comparison, for context, not the metric."""
    import torch
    import synth
    T, H, D = w.tokens, w.heads, w.head_dim
    q, k, v = inputs[0]
    cu = torch.from_numpy(synth.cu_seqlens(w.seg_lens)).to(dev)
    out = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
    run = lambda: fv.bf16_varlen_attn_fwd(q, k, v, cu, max(w.seg_lens), w.softmax_scale, out,
                                          ctx=ctx)
    for _ in range(2):
        run()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        run()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    return {"impl": "bf16_varlen_attn_fwd (this library, kind::f16)", "ms": ms,
            "tflops": w.attn_flops() / (ms * 1e-3) / 1e12}


def _output_modes(fv, ctx, w, inputs, dev, reps=10, rounds=3):
    """The attention call's output epilogues on the same e4m3 inputs (static
    scales, 1.5 x the exact amax): BF16 output, FP8 output through an
    output_scale (the amax of the BF16 output / 448), and at head_dim 128 the
    fused group-128 quantizer.  Each mode is timed over `reps` launches
    between two events, in `rounds` alternating rounds; the best round
    counts."""
    import torch
    import synth
    T, H, D = w.tokens, w.heads, w.head_dim
    q, k, v = inputs[0]
    cu = torch.from_numpy(synth.cu_seqlens(w.seg_lens)).to(dev)
    amax3 = torch.zeros(3, dtype=torch.float32, device=dev)
    fv.fp8_amax3(q, k, v, amax3, ctx=ctx)
    desc = torch.tensor([fv.fp8_descale_from_amax(float(np.float32(1.5) * np.float32(a)))
                         for a in amax3.cpu().numpy()], dtype=torch.float32, device=dev)
    q8, k8, v8 = (torch.empty((T, H, D), dtype=torch.uint8, device=dev) for _ in range(3))
    fv.fp8_quantize_qkv_per_tensor(q, k, v, desc, q8, k8, v8, ctx=ctx)
    call = (q8, k8, v8, desc[0:1], desc[1:2], desc[2:3], cu, max(w.seg_lens), w.softmax_scale)
    out = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
    fv.fp8_varlen_attn_fwd(*call, out, ctx=ctx)
    oscale = (out.float().abs().max() / 448.0).reshape(1).contiguous()
    out8 = torch.empty((T, H, D), dtype=torch.uint8, device=dev)
    runs = {"bf16": lambda: fv.fp8_varlen_attn_fwd(*call, out, ctx=ctx),
            "fp8_output_scale": lambda: fv.fp8_varlen_attn_fwd(*call, out8, output_scale=oscale,
                                                               ctx=ctx)}
    if D == 128:
        xq = torch.empty((T, H * D), dtype=torch.uint8, device=dev)
        xs = torch.empty((T, H * D // 128), dtype=torch.float32, device=dev)
        runs["fused_group_quant"] = lambda: fv.fp8_varlen_attn_fwd_group_quant(*call, xq, xs,
                                                                               ctx=ctx)
    best = {name: float("inf") for name in runs}
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    for _ in range(rounds):
        for name, run in runs.items():
            run()
            e0.record()
            for _ in range(reps):
                run()
            e1.record()
            torch.cuda.synchronize()
            best[name] = min(best[name], e0.elapsed_time(e1) / reps)
    st, site = ctx.check()
    if st != fv.OK:
        raise RuntimeError(f"device fault in the output-mode timing: {fv.status_string(st)} "
                           f"site {site}")
    flops = w.attn_flops()
    return {name: {"ms": ms, "tflops": flops / (ms * 1e-3) / 1e12} for name, ms in best.items()}


# The shapes of atrex-bench "#025 per_token_group_quant_fp8" (token_count x
# hidden_size), with the pages' speed-of-light and production times on their
# hardware ("XPU-A"), in microseconds: context for the same kernel on B200.
GROUP_QUANT_TABLE = [
    (1, 2048, 0.00, 7.60), (37504, 2048, 43.93, 106.10), (75008, 2048, 87.86, 199.60),
    (85632, 2048, 100.30, 223.30), (128192, 2048, 150.15, 325.70),
    (256896, 2048, 300.91, 639.80), (500736, 2048, 586.52, 1260.0),
    (1029056, 2048, 1210.0, 2620.0), (2058112, 2048, 2410.0, 5330.0),
    (3087168, 2048, 3620.0, 7130.0), (1, 7168, 0.00, 7.60), (726, 7168, 2.98, 13.90),
    (969, 7168, 3.97, 15.60), (1933, 7168, 7.92, 23.10), (4192, 7168, 17.19, 47.60),
    (8667, 7168, 35.53, 91.50), (16768, 7168, 68.74, 154.10), (40448, 7168, 165.82, 355.80),
    (58688, 7168, 240.60, 515.10),
]


def _group_quant_table(fv, ctx, dev, hbm_gbs, reps=10):
    """per_token_group_quant_fp8 (group 128) on the table's shapes.  Inputs
    are seeded N(0,1) BF16 drawn on the device (the table's inputs are
    torch.randn); each shape rotates over enough input/output copies to pass
    256 MB, so that shapes above L2 stream from HBM (smaller ones stay
    latency-bound), and the launches are replayed from one CUDA graph.
    Bytes = 3 per element + 4 per group of 128."""
    import torch
    g = torch.Generator(device=dev)
    g.manual_seed(25)
    rows = []
    for m, n, t_sol, t_prod in GROUP_QUANT_TABLE:
        nbytes = m * n * 3 + (m * n // 128) * 4
        copies = max(1, min(16, (256 << 20) // max(1, m * n * 2)))
        xs = [torch.randn((m, n), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
              for _ in range(copies)]
        qs = [torch.empty((m, n), dtype=torch.uint8, device=dev) for _ in range(copies)]
        ss = [torch.empty((m, n // 128), dtype=torch.float32, device=dev) for _ in range(copies)]
        for i in range(3):
            fv.per_token_group_quant_fp8(xs[i % copies], 128, qs[i % copies], ss[i % copies], ctx=ctx)
        torch.cuda.synchronize()
        # the reps as one CUDA graph, so that small shapes time the device and
        # not the host's launch rate
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for i in range(reps):
                fv.per_token_group_quant_fp8(xs[i % copies], 128, qs[i % copies], ss[i % copies],
                                             ctx=ctx)
        graph.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) / reps * 1e3
        del graph
        rows.append({"tokens": m, "hidden": n, "us": us, "GBps": nbytes / (us * 1e-6) / 1e9,
                     "frac_of_hbm": nbytes / (us * 1e-6) / 1e9 / hbm_gbs,
                     "pages_t_sol_us": t_sol, "pages_t_prod_us": t_prod})
        del xs, qs, ss
    return {"kernel": "group_quant_kernel (group 128)", "peak_GBps": hbm_gbs, "rows": rows}


def _attn_sweep(fv, ctx, dev, reps=10):
    """The pages' attention tables, on this library's kernels: for the
    head_dim-72 sequence sweep (2304..16384 tokens, 16 heads; the FP8 call
    includes the Q/K/V quantization, as in the pages' AITER table) and the
    8192-token head_dim-128 image: the full FP8 call (dynamic amax + ring +
    quantize, then attention), the FP8 attention alone, this library's BF16
    attention and torch's BF16 SDPA, all on the same BF16 inputs; CUDA
    events over `reps` back-to-back calls."""
    import torch
    import torch.nn.functional as F
    import synth
    rows = []
    for name in ("1x2304_d72", "1x4096_d72", "1x8192_d72", "1x16384_d72", "1x8192_d128"):
        w = synth.WORKLOADS[name]
        T, H, D = w.tokens, w.heads, w.head_dim
        q, k, v = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).reshape(T, H, D)
                   .to(dev) for x in w.qkv(0))
        cu = torch.from_numpy(synth.cu_seqlens(w.seg_lens)).to(dev)
        ring = fv.new_ring(dev)
        desc = torch.zeros(3, dtype=torch.float32, device=dev)
        q8, k8, v8 = (torch.empty((T, H, D), dtype=torch.uint8, device=dev) for _ in range(3))
        out = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)

        def fp8_attn():
            fv.fp8_varlen_attn_fwd(q8, k8, v8, desc[0:1], desc[1:2], desc[2:3], cu, T,
                                   w.softmax_scale, out, ctx=ctx)

        def fp8_full():
            fv.fp8_amax_ring_quantize_qkv(q, k, v, ring, desc, q8, k8, v8, ctx=ctx)
            fp8_attn()

        qs, ks, vs = (x.view(1, T, H, D).transpose(1, 2) for x in (q, k, v))
        calls = {
            "fp8_with_quant": fp8_full,
            "fp8_attention": fp8_attn,
            "bf16_this_library": lambda: fv.bf16_varlen_attn_fwd(q, k, v, cu, T, w.softmax_scale,
                                                                 out, ctx=ctx),
            "bf16_torch_sdpa": lambda: F.scaled_dot_product_attention(qs, ks, vs,
                                                                      scale=w.softmax_scale),
        }
        row = {"tokens": T, "heads": H, "head_dim": D}
        for key, fn in calls.items():
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                fn()
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / reps
            row[key] = {"ms": ms, "tflops": w.attn_flops() / (ms * 1e-3) / 1e12}
        rows.append(row)
        del q, k, v, q8, k8, v8, out
    return rows


def _quant_rooflines(fv, ctx, src, dev, hbm_gbs, reps=10):
    """HBM roofline of the three quantizer kernels on 3 x 32400-token, 16-head,
    head_dim-72 tensors ([97200, 1152] BF16 each, 224 MB): the resident BF16
    inputs are tiled on the device to that size (same value distribution).
    Each kernel reads more than the 126 MB L2, so its bytes come from HBM."""
    import torch
    n = 97200 * 1152
    flat = [t.reshape(-1) for t in src]
    big = [f.repeat((n + f.numel() - 1) // f.numel())[:n].contiguous() for f in flat]
    ring = fv.new_ring(dev)
    desc = torch.zeros(3, dtype=torch.float32, device=dev)
    q8, k8, v8 = (torch.empty(n, dtype=torch.uint8, device=dev) for _ in range(3))
    xq = torch.empty((97200, 1152), dtype=torch.uint8, device=dev)
    xs = torch.empty((97200, 9), dtype=torch.float32, device=dev)
    x2 = big[0].view(97200, 1152)
    runs = {
        "amax_ring_kernel": (lambda: fv.fp8_amax_ring_update(*big, ring, desc, ctx=ctx),
                             3 * n * 2),
        "quant3_kernel": (lambda: fv.fp8_quantize_qkv_per_tensor(*big, desc, q8, k8, v8,
                                                                 ctx=ctx), 3 * n * 3),
        # the dynamic path's entry point (at this size it takes the two
        # kernels above): 2 B read for the amax, then 2 B read + 1 B written
        # for the codes per element
        "fp8_amax_ring_quantize_qkv": (lambda: fv.fp8_amax_ring_quantize_qkv(*big, ring, desc,
                                                                              q8, k8, v8,
                                                                              ctx=ctx),
                                       3 * n * 5),
        "group_quant_kernel": (lambda: fv.per_token_group_quant_fp8(x2, 128, xq, xs, ctx=ctx),
                               n * 3 + (n // 128) * 4),
    }
    out = {}
    stream = torch.cuda.current_stream(dev)
    for name, (fn, nbytes) in runs.items():
        for _ in range(3):
            fn()
        # sustained rate: `reps` back-to-back launches between one pair of
        # events (no event between launches), median of three such batches
        batches = []
        for _ in range(3):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                fn()
            b.record(stream)
            torch.cuda.synchronize()
            batches.append(a.elapsed_time(b) / reps)
        ms = statistics.median(batches)
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[name] = {"bytes": nbytes, "ms": ms, "achieved_GBps": gbs, "peak_GBps": hbm_gbs,
                     "frac": gbs / hbm_gbs}
    del big, q8, k8, v8, xq, xs
    return {"workload": "3x32400 tokens, 16 heads, head_dim 72 ([97200, 1152] per tensor)",
            "bound": "hbm", "kernels": out}


def _step_description(w) -> str:
    """What one timed step of workload w runs (the configuration's own path)."""
    if w.mode == "static":
        quant = "per-tensor quantize q/k/v with static scales (1.5 x the calibrated amax)"
    else:
        quant = "amax ring update + per-tensor quantize q/k/v (one launch)"
    out = ("attention (fp8 out, output_scale = amax(bf16 out)/448 from a calibration pass on "
           "the device)" if w.fp8_out else "attention (bf16 out)")
    tail = " + group quant (128)" if w.group_quant else ""
    return f"{quant} + {out}{tail}"


def _launches_per_step(w, l2_bytes: int, group_tail: bool = False) -> int:
    """Kernels one step launches: the quantizer (the dynamic entry point takes
    two kernels once the BF16 inputs exceed twice the L2), attention, and the
    group quantizer where the workload has it (none when it is the attention
    launch's tail)."""
    quant = 1
    if w.mode != "static" and 3 * w.tokens * w.hd * 2 > 2 * l2_bytes:
        quant = 2
    return quant + 1 + (1 if w.group_quant and not group_tail else 0)


def _config(w, n_fwd=None):
    n_fwd = len(w.seeds) if n_fwd is None else n_fwd
    gb = n_fwd * 3 * w.tokens * w.hd * 2 / 1e9
    return {"workload": w.name, "seq_lens": list(w.seg_lens), "heads": w.heads,
            "head_dim": w.head_dim, "forwards": n_fwd,
            "step": _step_description(w),
            "l2": f"inputs rotate over {n_fwd} forwards ({gb:.2f} GB; L2 is 126 MB)",
            "rings": (f"one amax ring per layer ({n_fwd} layers)" if w.per_layer_rings
                      else ("no ring (static scales)" if w.mode == "static"
                            else "one amax ring over the rotation")),
            "parallelism": "replicas"}


class _Path:
    """One workload's own step on the device: the scale state (static
    descales, or dynamic rings) and the buffers, built once; step(i) runs
    forward i on the current stream through the library's entry points."""

    def __init__(self, fv, ctx, w, inputs, dev, group_tail=False):
        import torch
        import synth
        self.fv, self.ctx, self.w = fv, ctx, w
        # group_tail: the group quantizer runs as the attention launch's tail
        # (fp8_varlen_attn_fwd_bf16_group_quant), timed inside the attention events
        self.group_tail = group_tail and w.group_quant
        T, H, D = w.tokens, w.heads, w.head_dim
        self.inputs = inputs
        self.cu = torch.from_numpy(synth.cu_seqlens(w.seg_lens)).to(dev)
        self.max_s = max(w.seg_lens)
        self.q8, self.k8, self.v8 = (torch.empty((T, H, D), dtype=torch.uint8, device=dev)
                                     for _ in range(3))
        self.out = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
        self.out8 = torch.empty((T, H, D), dtype=torch.uint8, device=dev) if w.fp8_out else None
        self.xq = torch.empty((T, H * D), dtype=torch.uint8, device=dev)
        self.xs = torch.empty((T, H * D // 128), dtype=torch.float32, device=dev)
        self.desc = torch.zeros(3, dtype=torch.float32, device=dev)
        self.d3 = (self.desc[0:1], self.desc[1:2], self.desc[2:3])  # views made once
        self.counters = (fv.new_tile_counters(T, len(w.seg_lens), H * D, dev)
                         if self.group_tail else None)
        self.oscale = None
        if w.mode == "static":
            # calibration (untimed): exact amax of forward 0 on the device,
            # saved with the margin; the static descales then stay fixed
            amax3 = torch.zeros(3, dtype=torch.float32, device=dev)
            fv.fp8_amax3(*inputs[0], amax3, ctx=ctx)
            self.desc.copy_(torch.tensor([fv.fp8_descale_from_amax_margin(float(a), w.margin)
                                          for a in amax3.cpu().numpy()], dtype=torch.float32))
            self.rings = []
        else:
            self.rings = [fv.new_ring(dev) for _ in range(len(inputs) if w.per_layer_rings
                                                             else 1)]
        if w.fp8_out:
            # output_scale = amax(bf16 output of forward 0) / 448, formed on the
            # device: the amax kernel on the output, then the ring rule of a
            # fresh ring (max over one entry / 448, floored at 1e-10)
            self._quantize(0)
            self._attend(self.out, None)
            amax3 = torch.zeros(3, dtype=torch.float32, device=dev)
            fv.fp8_amax3(self.out, self.out, self.out, amax3, ctx=ctx)
            os3 = torch.zeros(3, dtype=torch.float32, device=dev)
            fv.fp8_ring_push(amax3, fv.new_ring(dev), os3)
            self.oscale = os3[0:1].clone()
            for r in self.rings:
                fv.ring_init(r)

    def _quantize(self, i):
        fv, q, k, v = self.fv, *self.inputs[i % len(self.inputs)]
        if self.w.mode == "static":
            fv.fp8_quantize_qkv_per_tensor(q, k, v, self.desc, self.q8, self.k8, self.v8,
                                           ctx=self.ctx)
        else:
            fv.fp8_amax_ring_quantize_qkv(q, k, v, self.rings[i % len(self.rings)], self.desc,
                                          self.q8, self.k8, self.v8, ctx=self.ctx)

    def _attend(self, out, oscale):
        d = self.d3
        self.fv.fp8_varlen_attn_fwd(self.q8, self.k8, self.v8, d[0], d[1], d[2], self.cu,
                                    self.max_s, self.w.softmax_scale, out, output_scale=oscale,
                                    ctx=self.ctx)

    def attend_with_tail(self, xq, xs):
        d = self.d3
        self.fv.fp8_varlen_attn_fwd_bf16_group_quant(
            self.q8, self.k8, self.v8, d[0], d[1], d[2], self.cu, self.max_s,
            self.w.softmax_scale, self.out, xq, xs, self.counters, ctx=self.ctx)

    def step(self, i, ev_a=None, ev_b=None, stream=None):
        w = self.w
        self._quantize(i)
        if ev_a is not None:
            ev_a.record(stream)
        if self.group_tail:
            self.attend_with_tail(self.xq, self.xs)
        elif w.fp8_out:
            self._attend(self.out8, self.oscale)
        else:
            self._attend(self.out, None)
        if ev_b is not None:
            ev_b.record(stream)
        if w.group_quant and not self.group_tail:
            T, HD = w.tokens, w.heads * w.head_dim
            self.fv.per_token_group_quant_fp8(self.out.view(T, HD), 128, self.xq, self.xs,
                                              ctx=self.ctx)


def _graph_times(path, w, inputs, reps=20, rounds=5):
    """Launch-bound sizes: the workload's step and its attention launch alone,
    each captured reps times in a CUDA graph and replayed, so host issue
    gaps between launches drop out of the device time; torch's BF16 SDPA on
    the same inputs the same way (single images)."""
    import torch
    import torch.nn.functional as F
    cur = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    side.wait_stream(cur)
    with torch.cuda.stream(side):
        for i in range(3):
            path.step(i)
    cur.wait_stream(side)
    torch.cuda.synchronize()
    out = path.out8 if path.w.fp8_out else path.out

    def timed(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(reps):
                fn(i)
        g.replay()
        torch.cuda.synchronize()
        best = None
        for _ in range(rounds):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / reps
            best = ms if best is None else min(best, ms)
        del g
        return best

    rec = {"reps_per_graph": reps, "timing": f"best of {rounds} graph replays",
           "ms_per_step": timed(path.step),
           "attn_ms": timed(lambda i: path._attend(out, path.oscale))}
    rec["attn_tflops"] = w.attn_flops() / (rec["attn_ms"] * 1e-3) / 1e12
    if len(w.seg_lens) == 1:
        T, H, D = w.tokens, w.heads, w.head_dim
        q, k, v = (x.view(1, T, H, D).transpose(1, 2) for x in inputs[0])
        try:
            ms = timed(lambda i: F.scaled_dot_product_attention(q, k, v, scale=w.softmax_scale))
            rec["torch_bf16_sdpa"] = {"ms": ms, "tflops": w.attn_flops() / (ms * 1e-3) / 1e12}
        except Exception as exc:  # no capturable fused BF16 kernel for this shape
            rec["torch_bf16_sdpa"] = {"unavailable": str(exc).splitlines()[0][:120]}
    torch.cuda.synchronize()
    return rec


def _events_median(fn, reps, stream, warmup=3):
    """Median over reps of one call's device time (CUDA events on the stream)."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    per = []
    for _ in range(reps):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        per.append((a, b))
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in per)


def _time_path(path, steps, warmup, stream):
    """(ms per step, median and mean attention ms per launch) of a workload's
    own step, CUDA events on the launching stream."""
    import torch
    for i in range(warmup):
        path.step(i)
    torch.cuda.synchronize()
    ev_a = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ev_b = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        path.step(i, ev_a[i], ev_b[i], stream)
    t1.record(stream)
    torch.cuda.synchronize()
    per = [a.elapsed_time(b) for a, b in zip(ev_a, ev_b)]
    return t0.elapsed_time(t1) / steps, statistics.median(per), statistics.mean(per)


def _config_records(fv, ctx, dev, peaks, stream, steps=20, warmup=3):
    """Every target workload's own step, timed in the same run as the headline
    (attention TFLOP/s and its fraction of the FP8 denominator, step time), with
    torch's BF16 SDPA on the same inputs beside the single-image workloads."""
    import torch
    import synth
    fp8_peak = 2.0 * peaks["bf16"]
    recs = {}
    for name in ("1x1024_d72", "1x2304_d72", "1x4096_d72", "1x8192_d72", "1x16384_d72",
                 "3x14400_d72", "3x32400_d72"):
        w = synth.WORKLOADS[name]
        T, H, D = w.tokens, w.heads, w.head_dim
        n_in = len(w.seeds) if w.per_layer_rings else min(2, len(w.seeds))
        inputs = [[torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).reshape(T, H, D)
                   .to(dev) for x in w.qkv(f)] for f in range(n_in)]
        path = _Path(fv, ctx, w, inputs, dev)
        n_steps = n_in if w.per_layer_rings else steps  # one pass over all 27 layers
        ms, attn_ms, attn_mean = _time_path(path, n_steps, min(warmup, n_steps), stream)
        st, site = ctx.check()
        if st != fv.OK:
            raise RuntimeError(f"device fault in {name}: {fv.status_string(st)} site {site}")
        tf = w.attn_flops() / (attn_ms * 1e-3) / 1e12
        rec = {"workload": w.name, "step": _step_description(w), "ms_per_step": ms,
               "steps_timed": n_steps, "attn_ms": attn_ms, "attn_ms_mean": attn_mean,
               "attn_timing": "median of the steps' attention events", "attn_tflops": tf,
               "attn_frac_of_fp8_peak": tf / fp8_peak,
               "step_tflops": w.attn_flops() / (ms * 1e-3) / 1e12}
        if len(w.seg_lens) == 1:
            rec["torch_bf16_sdpa"] = _sdpa_comparator(w, inputs, dev)
        if w.fp8_out:
            # the same attention with BF16 output (the run before the FP8-out one)
            b_ms = _events_median(lambda: path._attend(path.out, None), steps, stream)
            rec["bf16_out"] = {"attn_ms": b_ms,
                               "attn_tflops": w.attn_flops() / (b_ms * 1e-3) / 1e12}
        if w.tokens <= 4096:
            rec["graph"] = _graph_times(path, w, inputs)
            st, site = ctx.check()
            if st != fv.OK:
                raise RuntimeError(f"device fault in {name} (graph replay): "
                                   f"{fv.status_string(st)} site {site}")
        if w.group_quant and D != 128:
            # the same step with the group quantizer as the attention launch's
            # tail: one launch instead of attention + per_token_group_quant_fp8
            del path
            path = _Path(fv, ctx, w, inputs, dev, group_tail=True)
            ms_t, attn_t, _ = _time_path(path, n_steps, min(warmup, n_steps), stream)
            st, site = ctx.check()
            if st != fv.OK:
                raise RuntimeError(f"device fault in {name} (group tail): "
                                   f"{fv.status_string(st)} site {site}")
            rec["group_tail"] = {"ms_per_step": ms_t, "attn_plus_tail_ms": attn_t,
                                 "step_speedup_vs_two_launches": ms / ms_t}
        recs[name] = rec
        del path, inputs
        torch.cuda.empty_cache()
    return {"fp8_peak_tflops": fp8_peak, "peak_source": f"{peaks['source']} bf16 burst x 2",
            "records": recs}


def run_ours(args):
    import torch
    import fp8_quantized_vit_b200 as fv
    import synth

    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    dist = None
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    w = synth.WORKLOADS[args.workload]
    T, H, D = w.tokens, w.heads, w.head_dim
    n_fwd = len(w.seeds) if args.forwards <= 0 else min(args.forwards, len(w.seeds))
    ctx = fv.Context(local)
    if args.p_terms != 2:
        ctx.set_attn_p_terms(args.p_terms)
    dev = torch.device("cuda", local)

    # inputs: all forwards resident in HBM
    inputs = []
    for f in range(n_fwd):
        qkv = w.qkv(f)
        inputs.append([torch.from_numpy(x.view(np.int16)).view(torch.bfloat16)
                       .reshape(T, H, D).to(dev) for x in qkv])
    stream = torch.cuda.current_stream(dev)
    # the workload's own step: static or dynamic scales (one ring per layer
    # when the seeds are the layers of one encoder forward), BF16 or FP8
    # output, group quantization of the output where the workload has it
    path = _Path(fv, ctx, w, inputs, dev, group_tail=args.group_tail)
    cu, max_s = path.cu, path.max_s
    q8, k8, v8, out, xq, xs = path.q8, path.k8, path.v8, path.out, path.xq, path.xs
    rings = path.rings
    ev_a = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev_b = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]

    def step(i, timed=False):
        if timed:
            path.step(i, ev_a[i], ev_b[i], stream)
        else:
            path.step(i)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    st, site = ctx.check()
    if st != fv.OK:
        raise RuntimeError(f"device fault during warm-up: {fv.status_string(st)} site {site}")

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        step(i, timed=True)
    t1.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clk = clocks.stop()
    elapsed_ms = t0.elapsed_time(t1)
    attn_ms = [a.elapsed_time(b) for a, b in zip(ev_a, ev_b)]
    st, site = ctx.check()
    if st != fv.OK:
        raise RuntimeError(f"device fault: {fv.status_string(st)} site {site}")

    if dist:
        t = torch.tensor([elapsed_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        elapsed_ms = float(t.item())

    flops_step = w.attn_flops()
    value = ws * flops_step * args.steps / (elapsed_ms * 1e-3) / 1e12
    attn_avg_s = statistics.mean(attn_ms) * 1e-3
    attn_tflops = flops_step / attn_avg_s / 1e12

    # end to end through host buffers: pinned BF16 q/k/v in, quantized
    # attention output (codes + group scales) back, every step's copies inside
    # the timing.  Copies overlap compute the way a serving loop would run
    # them: step i+1's inputs go up on a copy stream while step i computes,
    # step i's results come down on a third stream; device and pinned host
    # buffers are double-buffered and events order every reuse.
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    host_in = [[t.cpu().pin_memory() for t in inputs[f]] for f in range(min(n_fwd, e2e_steps))]
    dbuf = [[torch.empty((T, H, D), dtype=torch.bfloat16, device=dev) for _ in range(3)]
            for _ in range(2)]
    # the step's result, double-buffered on the device and in pinned host
    # memory: the group-quantized output (codes + scales), else the FP8 or
    # BF16 attention output
    if w.group_quant:
        dres = [[xq, xs], [torch.empty_like(xq), torch.empty_like(xs)]]
    elif w.fp8_out:
        dres = [[path.out8], [torch.empty_like(path.out8)]]
    else:
        dres = [[out], [torch.empty_like(out)]]
    hres = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in dres[0]] for _ in range(2)]
    up = torch.cuda.Stream(dev)
    down = torch.cuda.Stream(dev)
    ev_up = [torch.cuda.Event() for _ in range(e2e_steps)]
    ev_done = [torch.cuda.Event() for _ in range(e2e_steps)]
    ev_down = [torch.cuda.Event() for _ in range(e2e_steps)]

    def upload(i):
        with torch.cuda.stream(up):
            if i >= 2:
                up.wait_event(ev_done[i - 2])  # step i-2 has finished reading dbuf[i % 2]
            for d_t, h_t in zip(dbuf[i % 2], host_in[i % len(host_in)]):
                d_t.copy_(h_t, non_blocking=True)
            ev_up[i].record(up)

    def e2e_compute(i):
        r = dres[i % 2]
        path.inputs = [dbuf[i % 2]]
        path._quantize(i)
        if path.group_tail:
            path.attend_with_tail(r[0], r[1])
        elif w.group_quant:
            path._attend(out, None)
            fv.per_token_group_quant_fp8(out.view(T, H * D), 128, r[0], r[1], ctx=ctx)
        elif w.fp8_out:
            path._attend(r[0], path.oscale)
        else:
            path._attend(r[0], None)

    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    up.wait_stream(stream)
    upload(0)
    for i in range(e2e_steps):
        if i + 1 < e2e_steps:
            upload(i + 1)
        stream.wait_event(ev_up[i])
        if i >= 2:
            stream.wait_event(ev_down[i - 2])  # result buffers [i % 2] have been read back
        e2e_compute(i)
        ev_done[i].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(ev_done[i])
            for h_t, d_t in zip(hres[i % 2], dres[i % 2]):
                h_t.copy_(d_t, non_blocking=True)
            ev_down[i].record(down)
    stream.wait_stream(up)
    stream.wait_stream(down)
    e1.record(stream)
    torch.cuda.synchronize()
    path.inputs = inputs
    e2e_ms = e0.elapsed_time(e1)
    if dist:
        t = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    e2e_value = ws * flops_step * e2e_steps / (e2e_ms * 1e-3) / 1e12
    h2d = 3 * T * H * D * 2
    d2h = sum(t.numel() * t.element_size() for t in dres[0])

    # forward 0 once more from a fresh ring (untimed), for the CPU-baseline
    # leg's full-size parity check
    cpu_leg = rank == 0 and ws == 1 and not args.no_cpu_baseline
    fwd0 = None
    if cpu_leg:
        try:
            fwd0 = _forward0_outputs(fv, ctx, w, inputs[0], cu, max_s, q8, k8, v8, out, dev,
                                     static_desc=path.desc if w.mode == "static" else None)
        except Exception as exc:  # reported in the line's parity field, not dropped
            fwd0 = exc

    peaks = _peaks()
    fp8_peak = 2.0 * peaks["bf16"]  # dense FP8 = 2 x dense BF16 (nominal ratio)
    quant = None if args.no_quant_roofline else _quant_rooflines(fv, ctx, inputs[0], dev,
                                                                 peaks["hbm"])
    traffic = _traffic(os.path.join(ROOT, "fp8_quantized_vit_b200", "csrc", "attn.cu"),
                       args.workload + ("+group_tail" if path.group_tail else ""))
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp8_e4m3 (fp32 accumulate)",
        "data": "synthetic", "config": dict(_config(w, n_fwd), p_terms=args.p_terms,
                                            **({"group_tail": True} if path.group_tail else {})),
        "roofline": {"bound": "tensor", "kernel": f"attn_fwd_kernel<{D}>",
                     "achieved": attn_tflops, "peak": fp8_peak, "unit": "TFLOP/s",
                     "frac": attn_tflops / fp8_peak, "traffic": traffic,
                     "peak_source": f"{peaks['source']} bf16 burst {peaks['bf16']} x 2 (fp8/bf16)",
                     "kernel_ms": attn_avg_s * 1e3,
                     "kernel_ms_median": statistics.median(attn_ms)},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "copies": "pinned host buffers; uploads, compute and read-backs on three "
                          "streams, double-buffered, overlapping across steps"},
        "gpu_launches": _launches_per_step(
            w, torch.cuda.get_device_properties(dev).L2_cache_size,
            path.group_tail) * args.steps,
        "clocks": clk,
        "quantizers": quant,
    }
    if args.compare_sdpa:
        line["comparator"] = _sdpa_comparator(w, inputs, dev)
    if args.compare_bf16:
        line["comparator_bf16_same_skeleton"] = _bf16_comparator(fv, ctx, w, inputs, dev)
    if args.group_quant_table:
        line["group_quant_table"] = _group_quant_table(fv, ctx, dev, peaks["hbm"])
    if args.attn_sweep:
        line["attn_sweep"] = _attn_sweep(fv, ctx, dev)
    if args.output_modes:
        line["output_modes"] = _output_modes(fv, ctx, w, inputs, dev)
    if rank == 0 and ws == 1 and not args.no_configs:
        del path, inputs
        torch.cuda.empty_cache()
        line["configs"] = _config_records(fv, ctx, dev, peaks, stream)
    if cpu_leg:
        codes, dsc = _oracle_inputs(w)
        threads = _host_threads()
        per_thread = max(1.0, args.cpu_seconds / threads)
        f, sec, rows = _oracle_rows_time_mt(w, codes, dsc, per_thread, seed=7, threads=threads)
        line["cpu_baseline"] = {
            "value": f / sec / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{rows} seeded (token, head) query rows of forward 0's attention, "
                      f"{threads} host threads each running the single-threaded oracle on rows "
                      f"of its own for {per_thread:.1f} s ({sec:.1f} s wall; amax/quantize "
                      f"stages excluded)",
            # the same oracle, on the kernels' forward 0 at full size
            "parity_of_forward0": _parity_field(w, codes, dsc, fwd0)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    ctx.close()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--forwards", type=int, default=0,
                    help="distinct input sets kept resident (0 = all of the workload's)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-step-seconds", type=float, default=1.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--group-tail", action="store_true",
                    help="workloads with a group-quantized output at head_dim 72: run the "
                         "group quantizer as the attention launch's tail")
    ap.add_argument("--no-quant-roofline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-workload records (each target workload's own step "
                         "timed in the same run)")
    ap.add_argument("--p-terms", type=int, choices=[1, 2], default=2,
                    help="e4m3 terms of P in the PV product (2: hi + lo, the default that meets "
                         "the attention tolerance; 1: a single term, faster, less accurate)")
    ap.add_argument("--compare-sdpa", action="store_true",
                    help="also time torch BF16 SDPA on the same inputs (single-image workloads)")
    ap.add_argument("--compare-bf16", action="store_true",
                    help="also time this library's BF16 attention kernel on the same inputs")
    ap.add_argument("--output-modes", action="store_true",
                    help="also time the attention call with BF16 output, FP8 output "
                         "(output_scale) and, at head_dim 128, the fused group quantizer")
    ap.add_argument("--attn-sweep", action="store_true",
                    help="also time the pages' attention tables (head_dim-72 sequence sweep, "
                         "8192-token head_dim 128): FP8 with and without quantization, BF16")
    ap.add_argument("--group-quant-table", action="store_true",
                    help="also time the group quantizer on the shapes of the pages' table")
    args = ap.parse_args()
    ws = int(os.environ.get("WORLD_SIZE", "0"))
    if args.gpus > 1 and ws == 0:
        # not launched by torch.distributed.run: start one rank per GPU here
        return _launch_ranks(args.gpus)
    if ws and ws != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={ws}", file=sys.stderr)
        return 2
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


def _launch_ranks(n: int) -> int:
    """Re-run this command under torch.distributed.run with n ranks on this
    node (rendezvous on 127.0.0.1); rank 0 prints the line."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


if __name__ == "__main__":
    sys.exit(main())
