"""Benchmark of the exact-attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

The default workload is "B4 H16 N4096 d128 causal" (4 x 16 heads, 4096
tokens, head dim 128, bf16, synthetic N(0, 1) inputs from
exact_io_aware_42_b200.inputs).  Every row of the hot path runs in each timed
iteration of one of two loops of K steps:

  step (the metric's path): bf16 forward (O, LSE) -> bf16 backward (dQ, dK, dV)
  FP8 loop:                 E4M3 block quantisation of Q, K (rotated) and V
                            -> FP8 forward (key ``fp8`` of the JSON line)

``value`` is the whole job's BF16 attention TFLOPS: algorithmic FLOPs of the
step (forward 4 B H N^2 d, halved when causal; backward 2.5 x forward) over
the device time of the K timed steps, max over ranks; ``dtype`` is bf16.  The
FP8 forward has its own line and its own roofline against an FP8 peak.  Inputs
(4 x 64 MiB) exceed the 126 MB L2, so no flush is needed between steps.
Workloads whose inputs fit in L2 are latency-bound; their steps are submitted
as one CUDA graph (``config.submission``) so that the device time is the
kernels', not the host's launch rate.  ``e2e`` is the step through the public
API, eagerly, with the inputs copied from pinned host memory and every output
copied back inside the timed region.  Under torchrun every rank runs its own
copy of the workload on its own GPU (independent heads, no collective on the
data path): weak scaling.

``--impl reference`` times the fp64 CPU oracle (the only other code this
script may run) on a bounded sample of the same workload on the host cores.

``--bwd deterministic`` times the reproducible backward (dK, dV kernel plus
the query-block-major dQ kernel) in place of the atomic one; the ``gqa_`` /
``mqa_`` workloads have fewer K/V heads than query heads (grouped K/V).
``--fwd-poly-pairs`` / ``--fwd-poly-degree`` set the forward's exp2 split for
a measurement (fa_set_tuning); the default is the library's.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "attn_B4_H16_N4096_d128_causal"


def workloads():
    """Every timed configuration: the default (the one the headline metric is
    quoted on), the small and FP8 workloads and the sequence-length sweep,
    each causal and non-causal."""
    from exact_io_aware_42_b200 import inputs
    out = {DEFAULT_WORKLOAD: dict(B=4, H=16, N=4096, d=128, causal=True, seed=2),
           "attn_B4_H16_N4096_d128_noncausal": dict(B=4, H=16, N=4096, d=128, causal=False, seed=2)}
    for w in (inputs.TINY, inputs.SMALL, inputs.FP8) + inputs.sweep():
        for c in w.causal:
            name = w.name.replace("attn_fwd_", "attn_").replace("attn_fp8_", "attn_fp8_") + \
                ("_causal" if c else "_noncausal")
            out[name] = dict(B=w.B, H=w.H, N=w.N, d=w.d, causal=c, seed=w.seed)
    # grouped K/V heads: FLOPs as for H query heads, K/V (and dK, dV) of H_kv heads
    out["gqa_B4_H32_Hkv8_N4096_d128_causal"] = dict(B=4, H=32, H_kv=8, N=4096, d=128, causal=True, seed=5)
    out["gqa_B4_H32_Hkv8_N4096_d128_noncausal"] = dict(B=4, H=32, H_kv=8, N=4096, d=128, causal=False, seed=5)
    out["mqa_B4_H16_Hkv1_N4096_d128_causal"] = dict(B=4, H=16, H_kv=1, N=4096, d=128, causal=True, seed=6)
    # causal sliding window of 1024 keys at N = 16384: FLOPs counted over the visible pairs only
    out["window1024_B1_H16_N16384_d128"] = dict(B=1, H=16, N=16384, d=128, causal=True, seed=7, window=1024)
    # head dim 256 (its own forward kernel; backward by the d = 256 dK, dV and dQ kernels)
    out["attn_B4_H8_N4096_d256_causal"] = dict(B=4, H=8, N=4096, d=256, causal=True, seed=9)
    out["attn_B4_H8_N4096_d256_noncausal"] = dict(B=4, H=8, N=4096, d=256, causal=False, seed=9)
    # ALiBi with the geometric slopes 2^(-8 (h + 1) / H)
    out["alibi_B4_H16_N4096_d128_causal"] = dict(B=4, H=16, N=4096, d=128, causal=True, seed=8, alibi=True)
    for name, w in out.items():
        w["name"] = name
        w.setdefault("H_kv", w["H"])
        w.setdefault("window", None)
        w.setdefault("alibi", False)
        w.setdefault("fwd_only", False)
    return out


def alibi_slopes(H):
    """Geometric ALiBi slopes 2^(-8 (h + 1) / H), one per query head."""
    return [2.0 ** (-8.0 * (h + 1) / H) for h in range(H)]


WORKLOAD = None   # set in main()


def visible_pairs(N, causal, window=None):
    """(query, key) pairs the mask leaves visible."""
    if not causal:
        return N * N
    if window is None or window >= N - 1:
        return N * (N + 1) / 2
    w = window   # row i sees min(i, w) + 1 keys
    return (w + 1) * (w + 2) / 2 - (w + 1) + (N - w) * (w + 1) if N > w else N * (N + 1) / 2


def fwd_flops(B, H, N, d, causal, window=None):
    """4 B H d x visible pairs (x N^2 / 2 for plain causal, the usual count)."""
    if causal and window is None:
        return 4.0 * B * H * N * N * d / 2
    return 4.0 * B * H * d * visible_pairs(N, causal, window)


def fwd_bytes(B, H, N, d, H_kv=None):
    """Algorithmic bytes of the forward: Q, K, V read once, O written, LSE written."""
    H_kv = H if H_kv is None else H_kv
    return (B * H + 2 * B * H_kv) * N * d * 2 + B * H * N * d * 2 + B * H * N * 4


def bwd_bytes(B, H, N, d, H_kv=None):
    """Q, O, dO read and dQ written (query heads); K, V read and dK, dV
    written (K/V heads); L and D read."""
    H_kv = H if H_kv is None else H_kv
    return (3 * B * H + 2 * B * H_kv) * N * d * 2 + 2 * B * H * N * 4 + (B * H + 2 * B * H_kv) * N * d * 2


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


KERNEL_SOURCES = {
    "fwd_tile": ("fa_fwd_tile.cu",),
    "fwd_q1": ("fa_fwd_q1.cu",),
    "fwd256": ("fa_fwd_d256.cu",),
    "bwd": ("fa_bwd.cu",),
    "bwd_dq": ("fa_bwd_dq.cu",),
    "bwd_pair": ("fa_bwd_pair.cu",),
    "bwd256": ("fa_bwd_d256.cu",),
    "fp8": ("fa_fp8.cu",),
}


def kernel_source_hash(which: str):
    """Hash of the sources a kernel is built from (its own file and the shared
    headers), to tell whether a stored profile was taken on this code."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[which] + ("fa_ptx.cuh", "fa_exp2.cuh", "fa_exp2_poly.h", "fa_internal.h"):
        with open(os.path.join(ROOT, "exact_io_aware_42_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str, which: str):
    """DRAM bytes (read + write) per launch of ``kernel`` on ``workload`` from
    profiles/traffic.json, written from an ncu capture; None unless that
    capture was taken on the current source of the kernel (``which``)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        table = json.load(f)
    for e in table.get("entries", []):
        if e.get("kernel") == kernel and e.get("workload") == workload:
            if e.get("source_sha") != kernel_source_hash(which):
                return None
            return float(e["dram_bytes_per_launch"])
    return None


class ClockSampler:
    """nvidia-smi sampled every 200 ms while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def build_step(fa, torch, B, H, N, d, causal, q, k, v, do, signs, deterministic=False, window=None,
               alibi=None, fwd_only=False):
    """The hot path as two lists of (stage name, callable, FLOPs, kernel
    launches): the bf16 step the metric is quoted on, and the FP8 rows."""
    state = {}

    ws = torch.empty(max(1, fa.bwd_workspace_size(B, H, N, d, deterministic, k.shape[1])), dtype=torch.uint8,
                     device=q.device)
    bufs = {n: torch.empty_like(q) for n in ("o", "dq")}
    bufs.update({n: torch.empty_like(k) for n in ("dk", "dv")})
    bufs["lse"] = torch.empty((B, H, N), dtype=torch.float32, device=q.device)

    def s_fwd():
        state["o"], state["lse"] = fa.fwd(q, k, v, causal=causal, out=bufs["o"], lse=bufs["lse"],
                                          window=window, alibi=alibi)

    def s_bwd():
        state["dq"], state["dk"], state["dv"] = fa.bwd(
            q, k, v, bufs["o"], do, bufs["lse"], causal=causal, workspace=ws,
            dq=bufs["dq"], dk=bufs["dk"], dv=bufs["dv"], deterministic=deterministic, window=window,
            alibi=alibi)

    src = {"q": q, "k": k, "v": v}
    q8 = {n: torch.empty(t.shape, dtype=torch.uint8, device=q.device) for n, t in src.items()}
    sc8 = {n: torch.empty((B, t.shape[1], fa.n_blocks(N)), dtype=torch.float32, device=q.device)
           for n, t in src.items()}
    o8 = torch.empty_like(q)
    lse8 = torch.empty((B, H, N), dtype=torch.float32, device=q.device)

    def s_quant():
        fa.quant_fp8(q, signs, out=q8["q"], scales=sc8["q"])
        fa.quant_fp8(k, signs, out=q8["k"], scales=sc8["k"])
        fa.quant_fp8(v, None, out=q8["v"], scales=sc8["v"])

    def s_fwd8():
        fa.fwd_fp8(q8["q"], q8["k"], q8["v"], sc8["q"], sc8["k"], sc8["v"], causal=causal, out=o8, lse=lse8,
                   window=window, alibi=alibi)

    f = fwd_flops(B, H, N, d, causal, window)
    # backward launches: preprocess, main, and postprocess (atomic) or dQ
    # (deterministic), plus the split reduction when few K/V heads share out a group
    bwd_launches = 3 + (1 if fa.bwd_workspace_size(B, H, N, d, deterministic, k.shape[1]) >
                        fa.bwd_workspace_size(B, H, N, d, deterministic) else 0)
    step = [("fwd_bf16", s_fwd, f, 1)]
    if not fwd_only:
        step.append(("bwd_bf16", s_bwd, 2.5 * f, bwd_launches))
    fp8 = [("quant_fp8", s_quant, 0.0, 3), ("fwd_fp8", s_fwd8, f, 1)] if d == 128 else []
    return step, fp8, state


def time_stages(torch, stages, steps, stream, graph=False):
    """Device time of ``steps`` passes over the stages, plus per-stage event
    times.  With ``graph`` each stage's ``steps`` calls are captured into one
    CUDA graph first; the graphs are then replayed in stage order inside the
    timed region, each bracketed by events on the launching stream."""
    if graph:
        graphs = []
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        for _, fn, _, _ in stages:
            with torch.cuda.stream(side):
                fn()                   # one eager call on the capture stream first
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                for _ in range(steps):
                    fn()
            graphs.append(g)
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in stages]
        for (e0, e1), g in zip(ev, graphs):
            e0.record(stream)
            g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        per_stage = [e0.elapsed_time(e1) / steps for e0, e1 in ev]
        total_ms = ev[0][0].elapsed_time(ev[-1][1])
        del graphs
        return total_ms, per_stage
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in stages] for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(steps):
        for j, (_, fn, _, _) in enumerate(stages):
            ev[i][j][0].record(stream)
            fn()
            ev[i][j][1].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    total_ms = start.elapsed_time(end)
    per_stage = [sum(ev[i][j][0].elapsed_time(ev[i][j][1]) for i in range(steps)) / steps
                 for j in range(len(stages))]
    return total_ms, per_stage


_ORACLE_INPUTS = {}


def reduce_max(x: float, dist, device, world: int) -> float:
    """Max of a per-rank scalar over all ranks (the slowest rank's time)."""
    if world == 1:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world: int, step_flops: float, ms_per_step: float) -> float:
    """Weak scaling: every rank runs its own copy of the workload, so the job
    processes world x step_flops per (max-over-ranks) step time."""
    return world * step_flops / (ms_per_step * 1e-3) / 1e12


def oracle_sample(budget_s: float, B, H, N, d, causal, with_bwd: bool):
    """Time the fp64 oracle head by head on the host cores until ``budget_s``."""
    import numpy as np
    import oracle
    from exact_io_aware_42_b200 import inputs
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [os.cpu_count()])
    except Exception:  # noqa: BLE001
        cores = os.cpu_count()
    g = WORKLOAD["H"] // WORKLOAD.get("H_kv", WORKLOAD["H"])   # query heads per K/V head
    if H % g:
        g = 1                       # a smaller warm-up shape than the workload's
    H_kv = H // g
    key = (B, H, H_kv, N, d)
    if key not in _ORACLE_INPUTS:
        _ORACLE_INPUTS[key] = inputs.make_gqa(B, H, H_kv, N, d, WORKLOAD["seed"], with_do=True)
    q, k, v, do = _ORACLE_INPUTS[key]
    sc = 1.0 / math.sqrt(d)
    flops, heads, t0 = 0.0, 0, time.perf_counter()
    for idx in range(B * H):
        b, h = divmod(idx, H)
        sl = (slice(b, b + 1), slice(h, h + 1))
        kh = h // (H // H_kv)           # the K/V head of query head h
        kl = (slice(b, b + 1), slice(kh, kh + 1))
        win = WORKLOAD.get("window")
        sl_ = [alibi_slopes(H)[h]] if WORKLOAD.get("alibi") else None
        oracle.attn_fwd_gqa_ref(q[sl], k[kl], v[kl], sc, causal, window=win, alibi=sl_)
        flops += fwd_flops(1, 1, N, d, causal, win)
        if with_bwd:
            oracle.attn_bwd_gqa_ref(q[sl], k[kl], v[kl], do[sl], sc, causal, window=win, alibi=sl_)
            flops += 2.5 * fwd_flops(1, 1, N, d, causal, win)
        heads += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": "TFLOPS", "cores": int(cores), "kind": "oracle",
            "sample": f"{heads} of {B * H} heads of {WORKLOAD['name']}, fwd"
                      + ("+bwd" if with_bwd else "") + f", fp64 numpy, {dt:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = WORKLOAD
    with_bwd = not w["fwd_only"]
    for _ in range(args.warmup):
        oracle_sample(0.0, 1, 1, 256, w["d"], w["causal"], with_bwd)
    vals = []
    t_all = time.perf_counter()
    # each step a bounded sample: about 150 s of oracle work for the whole run at most
    per_step = min(args.ref_seconds, max(0.5, 150.0 / max(1, args.steps)))
    for _ in range(args.steps):
        vals.append(oracle_sample(per_step, w["B"], w["H"], w["N"], w["d"], w["causal"], with_bwd))
    dt = time.perf_counter() - t_all
    v = sum(x["value"] for x in vals) / len(vals)
    cpu = dict(vals[-1])
    cpu["value"] = v
    line = {"metric": METRIC, "value": v, "unit": "TFLOPS", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1000 * dt / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "config": config_block(False), "cpu_baseline": cpu,
            "e2e": {"value": v, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


METRIC = "attention fwd/bwd TFLOPS (BF16 causal+non-causal) and % of B200 tensor peak"
BWD_MODE = "atomic"   # set in main()


def latency_bound(w) -> bool:
    """Inputs (Q, K, V, dO) small enough to stay in the 126 MB L2."""
    return 2 * (w["H"] + w["H_kv"]) * w["B"] * w["N"] * w["d"] * 2 <= 126e6


def config_block(graph: bool):
    w = WORKLOAD
    in_bytes = 2 * (w["H"] + w["H_kv"]) * w["B"] * w["N"] * w["d"] * 2
    return {"workload": w["name"], "B": w["B"], "H": w["H"], "H_kv": w["H_kv"], "N": w["N"], "d": w["d"],
            "bwd": BWD_MODE, "window": w["window"], "alibi": "slopes 2^(-8(h+1)/H)" if w["alibi"] else None,
            "causal": w["causal"], "global_batch": w["B"], "seq_len": w["N"],
            "parallelism": "independent replicas per GPU (heads), no collective",
            "l2": (f"inputs (Q, K, V, dO) {in_bytes / 2**20:.0f} MiB > 126 MB L2, no flush"
                   if in_bytes > 126e6 else
                   "inputs smaller than L2: timed warm in L2 (latency-bound workload)"),
            "submission": ("one CUDA graph per stage of K calls (latency-bound: device time, not host launch rate)"
                           if graph else "eager launches through the public API"),
            "step": ("fwd_bf16 (head dim 256: forward only)" if w["fwd_only"] else "fwd_bf16 + bwd_bf16")
                    + " (value, ms_per_step, e2e)",
            "fp8_loop": ("quant_fp8 (Q, K rotated; V) + fwd_fp8 in a second loop of K steps, key fp8"
                         if w["d"] == 128 else "none (the FP8 forward is built for d = 128)"),
            "bwd_pair": TUNING.get("bwd_pair"),
            "fwd_persistent": TUNING.get("fwd_persistent"),
            "fwd_causal_group": TUNING.get("fwd_causal_group"), "fwd_q1": TUNING.get("fwd_q1"),
            "bwd_causal_group": TUNING.get("bwd_causal_group"),
            "exp2_split": {"fwd_poly_pairs": TUNING.get("fwd_poly_pairs"),
                           "fwd_poly_degree": TUNING.get("fwd_poly_degree"),
                           "fp8_poly_pairs": TUNING.get("fp8_poly_pairs")}}


TUNING = {}   # effective measurement controls, filled in run_ours


def run_ours(args):
    import torch
    import torch.distributed as dist
    import exact_io_aware_42_b200 as fa
    from exact_io_aware_42_b200 import inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    w = WORKLOAD
    B, H, N, d, causal, H_kv = w["B"], w["H"], w["N"], w["d"], w["causal"], w["H_kv"]
    if args.fwd_poly_pairs is not None:
        fa.set_tuning("fwd_poly_pairs", args.fwd_poly_pairs)
    if args.fwd_poly_degree is not None:
        fa.set_tuning("fwd_poly_degree", args.fwd_poly_degree)
    if args.fp8_poly_pairs is not None:
        fa.set_tuning("fp8_poly_pairs", args.fp8_poly_pairs)
    if args.bwd_pair is not None:
        fa.set_tuning("bwd_pair", args.bwd_pair)
    for knob in ("fwd_persistent", "fwd_causal_group", "fwd_q1", "bwd_causal_group"):
        if getattr(args, knob) is not None:
            fa.set_tuning(knob, getattr(args, knob))
    TUNING.update({k_: fa.get_tuning(k_, d) for k_ in ("fwd_poly_pairs", "fwd_poly_degree", "fp8_poly_pairs",
                                                       "bwd_pair", "fwd_persistent", "bwd_causal_group",
                                                       "fwd_causal_group", "fwd_q1")})
    graph = {"auto": latency_bound(w), "on": True, "off": False}[args.graph]
    hq, hk, hv, hdo = inputs.make_gqa(B, H, H_kv, N, d, w["seed"] + rank, with_do=True)
    signs = inputs.signs(d).to(dev)
    q, k, v, do = (t.to(dev) for t in (hq, hk, hv, hdo))
    stages, fp8_stages, state = build_step(
        fa, torch, B, H, N, d, causal, q, k, v, do, signs, deterministic=BWD_MODE == "deterministic",
        window=w["window"],
        alibi=torch.tensor(alibi_slopes(H), dtype=torch.float32, device=dev) if w["alibi"] else None,
        fwd_only=w["fwd_only"])
    step_flops = sum(s[2] for s in stages)
    launches_per_step = sum(s[3] for s in stages)

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def max_over_ranks(x: float) -> float:
        return reduce_max(x, dist, dev, world)

    for _ in range(args.warmup):
        for s in stages + fp8_stages:
            s[1]()
    barrier()
    with ClockSampler(local) as clk:
        total_ms, per_stage = time_stages(torch, stages, args.steps, stream, graph)
        barrier()
        fp8_total_ms, fp8_per_stage = (time_stages(torch, fp8_stages, args.steps, stream, graph)
                                       if fp8_stages else (0.0, []))
    barrier()
    fa_status = fa.get_status()
    total_ms = max_over_ranks(total_ms)
    per_stage = [max_over_ranks(x) for x in per_stage]
    fp8_total_ms = max_over_ranks(fp8_total_ms)
    fp8_per_stage = [max_over_ranks(x) for x in fp8_per_stage]
    ms_step = total_ms / args.steps
    value = whole_job_tflops(world, step_flops, ms_step)

    # End to end through the public API (eager), host buffers in and out.
    # Every step copies its inputs in from pinned host memory and its outputs
    # back.  With large copies two slots of device buffers let the copies of
    # step k + 1 (in) and step k - 1 (out) run on their own streams while
    # step k computes; small (launch-bound) steps run on one stream.
    pin = {n: t.pin_memory() for n, t in (("q", hq), ("k", hk), ("v", hv), ("do", hdo))}
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    pipelined = h2d >= (8 << 20)
    slot_in = [{"q": q, "k": k, "v": v, "do": do}]
    slot_stages, slot_state = [stages], [state]
    if pipelined:
        slot_in.append({n: torch.empty_like(t) for n, t in slot_in[0].items()})
        st2, _, state2 = build_step(
            fa, torch, B, H, N, d, causal, slot_in[1]["q"], slot_in[1]["k"], slot_in[1]["v"], slot_in[1]["do"],
            signs, deterministic=BWD_MODE == "deterministic", window=w["window"],
            alibi=torch.tensor(alibi_slopes(H), dtype=torch.float32, device=dev) if w["alibi"] else None,
            fwd_only=w["fwd_only"])
        slot_stages.append(st2)
        slot_state.append(state2)
    slot_out = [{}, {}]
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    ev = [{n: torch.cuda.Event() for n in ("in", "done", "read")} for _ in range(2)]

    def e2e_step(kk):
        if not pipelined:
            for n, t in pin.items():
                slot_in[0][n].copy_(t, non_blocking=True)
            for s in stages:
                s[1]()
            for n, t in state.items():
                if n not in slot_out[0]:
                    slot_out[0][n] = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                slot_out[0][n].copy_(t, non_blocking=True)
            return
        s_ = kk % 2
        e = ev[s_]
        if kk >= 2:
            h2d_s.wait_event(e["done"])      # step kk - 2 has finished with this slot's inputs
        with torch.cuda.stream(h2d_s):
            for n, t in pin.items():
                slot_in[s_][n].copy_(t, non_blocking=True)
            e["in"].record(h2d_s)
        stream.wait_event(e["in"])
        if kk >= 2:
            stream.wait_event(e["read"])     # step kk - 2's outputs have been read back
        for s in slot_stages[s_]:
            s[1]()
        e["done"].record(stream)
        d2h_s.wait_event(e["done"])
        with torch.cuda.stream(d2h_s):
            for n, t in slot_state[s_].items():
                if n not in slot_out[s_]:
                    slot_out[s_][n] = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                slot_out[s_][n].copy_(t, non_blocking=True)
            e["read"].record(d2h_s)

    for kk in range(2):
        e2e_step(kk)
    torch.cuda.synchronize()
    d2h = sum(t.numel() * t.element_size() for t in slot_out[0].values())
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d_s.wait_stream(stream)
    d2h_s.wait_stream(stream)
    for kk in range(args.steps):
        e2e_step(kk)
    stream.wait_stream(d2h_s)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1)) / args.steps
    barrier()

    peaks, peak_src = measured_peaks()
    burst = float(peaks["bf16_tflops"])
    sustained = float(peaks["bf16_tflops_sustained"])
    clocks = clk.summary()

    def roof(stage_list, times, name, kernel, nbytes, peak, peak_note, traffic):
        i = [st[0] for st in stage_list].index(name)
        ms = times[i]
        ach = stage_list[i][2] / (ms * 1e-3) / 1e12
        out = {"kernel": kernel, "bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
               "frac": ach / peak, "peak_source": peak_note, "algorithmic_bytes": nbytes,
               "ms_per_launch": ms, "traffic": traffic}
        return out

    burst_note = (f"{peak_src} bf16_tflops (burst: the timed region is short and the SM clock "
                  f"sampled during it is {clocks.get('sm_mhz')} of {clocks.get('sm_max_mhz')} MHz)")
    cz = "causal" if causal else "non-causal"
    if d == 256:
        # one path at d = 256 (both modes): the dK/dV and dQ kernels; traffic
        # is theirs summed while both captures match the current source
        bwd_kernel = f"bwd_kv256_kernel<{cz}> + bwd_dq256_kernel<{cz}> (+ preprocess) in the timed call"
        t_kv = profiled_traffic("bwd_kv256_kernel", w["name"], "bwd256")
        t_dq = profiled_traffic("bwd_dq256_kernel", w["name"], "bwd256")
        bwd_traffic = t_kv + t_dq if t_kv is not None and t_dq is not None else None
    elif BWD_MODE == "atomic":
        bwd_kernel = f"bwd_main_kernel<{d}, {cz}> (+ preprocess and dQ postprocess launches in the timed call)"
        bwd_traffic = profiled_traffic("bwd_main_kernel", w["name"], "bwd")
    else:
        main = "bwd_pair_kernel (CTA pairs)" if TUNING.get("bwd_pair") == 1 else f"bwd_main_kernel<{d}, {cz}, no dQ>"
        bwd_kernel = f"{main} + bwd_dq_kernel (+ preprocess) in the timed call"
        bwd_traffic = None
    roof_bwd = None
    if not w["fwd_only"]:
        roof_bwd = roof(stages, per_stage, "bwd_bf16", bwd_kernel, bwd_bytes(B, H, N, d, H_kv), burst, burst_note,
                        bwd_traffic)
        roof_bwd["frac_sustained"] = roof_bwd["achieved"] / sustained
        roof_bwd["frac_nominal_2250"] = roof_bwd["achieved"] / 2250.0
    # the two-tile forward's grid: set explicitly, or (-1) the library's
    # per-call default: persistent except for the FP8 non-causal forward, one
    # CTA per item with ALiBi or a polynomial exp2 share
    pk = TUNING.get("fwd_persistent")
    plain = not w["alibi"]
    pers = plain and TUNING.get("fwd_poly_pairs") == 0 and pk in (1, -1)
    pers8 = plain and TUNING.get("fp8_poly_pairs") == 0 and (pk == 1 or (pk == -1 and causal))
    # the one-tile kernel: chosen explicitly, or by the library when the
    # two-tile kernel would have fewer work items than SMs
    n_pairs = ((N + 127) // 128 + 1) // 2
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    q1 = d != 256 and (TUNING.get("fwd_q1") == 1 or (TUNING.get("fwd_q1") == -1 and n_pairs * B * H < sms))
    fwd_name, fwd_src = (("fwd256_kernel", "fwd256") if d == 256 else ("fwd_q1_kernel", "fwd_q1") if q1
                         else ("fwd_tile_kernel", "fwd_tile"))
    fwd_desc = f"{fwd_name}<{d}, {cz}, bf16>" + (
        " (persistent, one query tile per item)" if q1 else " (persistent)" if d == 256 or pers
        else " (one CTA per item)")
    roof_fwd = roof(stages, per_stage, "fwd_bf16", fwd_desc, fwd_bytes(B, H, N, d, H_kv), burst, burst_note,
                    profiled_traffic(fwd_name, w["name"], fwd_src))
    roof_fwd["frac_sustained"] = roof_fwd["achieved"] / sustained
    roof_fwd["frac_nominal_2250"] = roof_fwd["achieved"] / 2250.0
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config_block(graph),
        "pct_of_peak": {"measured_bf16_burst": value / world / burst,
                        "measured_bf16_sustained": value / world / sustained,
                        "nominal_2250": value / world / 2250.0},
        "stages": {s[0]: {"ms": per_stage[i], "tflops": s[2] / (per_stage[i] * 1e-3) / 1e12}
                   for i, s in enumerate(stages)},
        # the dominant kernel: the backward where the step has one, else the forward
        "roofline": roof_bwd if roof_bwd is not None else roof_fwd,
        "roofline_fwd": roof_fwd,
        "e2e": {"value": whole_job_tflops(world, step_flops, e2e_ms), "unit": "TFLOPS",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "submission": ("eager, two buffer slots: the copies in of step k + 1 and out of step k - 1 "
                               "overlap step k on their own streams") if pipelined else "eager, one stream"},
        "gpu_launches": launches_per_step * args.steps + sum(s[3] for s in fp8_stages) * args.steps,
        "clocks": clocks,
        "device_status": fa_status,
    }
    if fp8_stages:
        fp8_peak = 2.0 * burst
        fp8_flops = sum(s[2] for s in fp8_stages)
        rf = roof(fp8_stages, fp8_per_stage, "fwd_fp8",
                  f"fwd_tile_kernel<128, {cz}, e4m3> ({'persistent' if pers8 else 'one CTA per item'})", None, fp8_peak,
                  f"2 x {peak_src} bf16_tflops burst (nominal 2:1 ratio of dense E4M3 to bf16; no measured "
                  "FP8 peak)", None)
        rf["algorithmic_bytes"] = fwd_bytes(B, H, N, d, H_kv) - (B * H + 2 * B * H_kv) * N * d
        line["fp8"] = {
            "dtype": "e4m3 (Q, K, V, P) with fp32 accumulation", "ms_per_step": fp8_total_ms / args.steps,
            "tflops": world * fp8_flops / (fp8_total_ms / args.steps * 1e-3) / 1e12,
            "stages": {s[0]: {"ms": fp8_per_stage[i],
                              "tflops": (s[2] / (fp8_per_stage[i] * 1e-3) / 1e12) if s[2] else None}
                       for i, s in enumerate(fp8_stages)},
            "roofline_fp8": rf,
        }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_sample(args.ref_seconds, B, H, N, d, causal, not w["fwd_only"])
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0 if fa_status == 0 else 1


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--ref-seconds", type=float, default=12.0,
                    help="host-core seconds of oracle work per reference step / cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(workloads()),
                    help="configuration to time (default: the one the headline metric is quoted on)")
    ap.add_argument("--bwd", choices=["atomic", "deterministic"], default="atomic",
                    help="backward variant timed in the step (default: atomic dQ accumulation)")
    ap.add_argument("--graph", choices=["auto", "on", "off"], default="auto",
                    help="submit the timed calls as CUDA graphs (auto: for workloads whose inputs fit in L2)")
    ap.add_argument("--fwd-poly-pairs", type=int, choices=[0, 2, 4], default=None,
                    help="forward exp2 split for a measurement (default: the library's)")
    ap.add_argument("--fwd-poly-degree", type=int, choices=[3, 4], default=None)
    ap.add_argument("--bwd-pair", type=int, choices=[0, 1], default=None,
                    help="deterministic backward at d = 128: dK, dV on CTA pairs (1) or single CTAs (0)")
    ap.add_argument("--fwd-persistent", type=int, choices=[0, 1], default=None,
                    help="two-tile forward: persistent grid (1) or one CTA per work item (0)")
    ap.add_argument("--fwd-q1", type=int, choices=[0, 1], default=None,
                    help="bf16 forward, d <= 128: one query tile per item with two score buffers (1)")
    ap.add_argument("--bwd-causal-group", type=int, choices=[0, 1], default=None,
                    help="causal backward: CTAs longest first within L2-sized head groups (1) or head by head (0)")
    ap.add_argument("--fwd-causal-group", type=int, choices=[0, 1], default=None,
                    help="causal forward: longest first within L2-sized head groups (1) or over all heads (0)")
    ap.add_argument("--fp8-poly-pairs", type=int, choices=[0, 2, 4], default=None,
                    help="FP8 forward exp2 split for a measurement (default: the library's)")
    args = ap.parse_args()
    global WORKLOAD, BWD_MODE
    WORKLOAD = workloads()[args.workload]
    BWD_MODE = args.bwd
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
