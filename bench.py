#!/usr/bin/env python
"""Benchmark of one NVFP4 MoE FFN layer on B200 through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole layer (route -> permute -> gate/up GEMM +
SwiGLU -> down GEMM -> combine) over one batch of synthetic tokens.  Steps
rotate over R independent layers (own weights, activations and logits) so
that the expert weights a step reads are not in L2 from the step before.
Prints one JSON line on rank 0: the headline workload (--workload, default
decode_T64) at top level, and every workload of the task, the headline
included, under `workloads` (tokens/s, the median of individually timed
graph replays, the dominant kernel's roofline, the oracle on the host cores),
with the 48-layer back-to-back decode sweep of the wide layer as
`wide_decode_T1_48_layers`.  --only measures the headline workload alone.  With N > 1 (torchrun) every rank runs its
own independent batches (weak scaling; no data-path collective) and the time
is the maximum over ranks.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from moe_expert_layer_renorm_b200 import inputs  # noqa: E402

METRIC = "MoE-layer tokens/s; decode HBM GB/s and prefill TFLOP/s vs B200 peak"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decode_T64", choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--layers", type=int, default=4, help="independent layers the steps rotate over")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-sample-tokens", type=int, default=64)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", action="store_true",
                    help="measure the --workload alone (default: it, then every other workload and the "
                         "48-layer sweep, reported under `workloads`)")
    ap.add_argument("--fmt", default="nvfp4", choices=["nvfp4", "mxfp4"], help="expert weight format")
    ap.add_argument("--layout", default="rows", choices=["rows", "tiled"],
                    help="expert slot layout: row-major tensors, or stage-tiled (each weight box contiguous)")
    ap.add_argument("--ep", action="store_true",
                    help="expert parallelism: the experts split over the ranks, rows exchanged all-to-all "
                         "(each rank still brings its own tokens: weak scaling)")
    ap.add_argument("--whole", action="store_true",
                    help="run each layer through ft_moe_layer_nvfp4 (one launch for decode-sized batches)")
    ap.add_argument("--fused-front", action="store_true",
                    help="route and permute through ft_moe_route_permute (one launch for small batches)")
    ap.add_argument("--slot-churn", nargs="?", const="decode", default=None, choices=["decode", "prefill_stream"],
                    help="measure the expert-cache miss path (pinned host banks, LRU slot manager) instead: "
                         "domain-rotation decode steps, or prefill layers streamed through a two-layer pool")
    return ap.parse_args()


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def bytes_per_expert(H: int, I: int, fmt: str = "nvfp4") -> int:
    """Algorithmic bytes of one expert: codes + unpadded scales (+ 3 fp32
    globals for NVFP4; MXFP4 has one E8M0 byte per 32 values and no global)."""
    if fmt == "mxfp4":
        return 3 * (H * I // 2 + H * I // 32)
    return 3 * (H * I // 2 + H * I // 16) + 12


def gate_up_bytes_per_expert(H: int, I: int, fmt: str = "nvfp4") -> int:
    if fmt == "mxfp4":
        return 2 * (H * I // 2 + H * I // 32)
    return 2 * (H * I // 2 + H * I // 16) + 8


# ---------------------------------------------------------------- clocks ---

class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed region runs."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                                          "-i", str(self.idx), "-lms", "200"], stdout=self.out,
                                         stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.flush()
        self.out.seek(0)
        rows = [r for r in csv.reader(io.StringIO(self.out.read())) if len(r) >= 9]
        os.unlink(self.out.name)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------ our arm ---

def _code_only(text: str) -> str:
    """C++/CUDA source with comments and blank lines removed (the kernels'
    sources contain no string literal holding a comment marker)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*", "", ln).rstrip() for ln in text.splitlines())
    return "\n".join(ln for ln in lines if ln)


def kernel_source_hash() -> str:
    """Hash of the code (comments excluded) of the expert FFN kernels, the
    helpers they include and the host code that sizes their launches: a
    counter taken on other code no longer describes the launches that run."""
    d = os.path.join(ROOT, "moe_expert_layer_renorm_b200", "csrc")
    h = hashlib.sha256()
    for name in ("sm100.cuh", "ffn.cu", "decode.cu", "ffn_host.cu", "layer.cu"):
        with open(os.path.join(d, name), encoding="utf-8") as f:
            h.update(name.encode() + b"\0" + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


def traffic_record(key: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f).get(key)
    if not rec:
        return None
    return rec["bytes_per_launch"] if rec.get("src_sha256_16") == kernel_source_hash() else None


L2_BYTES = 126e6


def rank_layer_seed(w, rank: int, layer: int) -> int:
    """Seed of layer `layer` on rank `rank`: every rank draws its own batches
    and weights (weak scaling over independent problems)."""
    return inputs.layer_seed(w.seed + 1_000_003 * rank, layer)


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank number over all ranks (the value itself without
    a process group).  Every rank must call it at the same point."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rotation_layers(w, requested: int) -> int:
    """Independent layers the steps rotate over: at least `requested`, and
    enough that the weights the other layers read between two visits of a
    layer (about 3x L2) have evicted that layer's weights from L2."""
    per_step = inputs.expected_distinct_experts(w.T, w.E, w.k) * bytes_per_expert(w.H, w.I)
    need = int(np.ceil(3.0 * L2_BYTES / max(per_step, 1.0))) + 1
    return int(min(64, max(1, requested, need)))


def workload_config(w, R: int, S: int, world: int) -> dict:
    """The `config` object of a workload, the same in both arms' JSON lines
    (it depends only on the workload and the run's options, never on what a
    run measured)."""
    step_mb = inputs.expected_distinct_experts(w.T, w.E, w.k) * bytes_per_expert(w.H, w.I) / 1e6
    return {"workload": w.name, "T": w.T, "E": w.E, "k": w.k, "H": w.H, "I": w.I,
            "route": "softmax_renorm" if w.route_mode == 0 else "topk_softmax",
            "slots": w.slots, "layers_rotated": R, "pool_slots": S,
            "parallelism": f"dp{world} (independent batches)",
            "l2": "steps rotate over %d independent layers of ~%.0f MB of expert weights per step (uniform-routing "
                  "expectation); a layer's weights come back after ~%.0f MB of other layers' (L2 is 126 MB)"
                  % (R, step_mb, (R - 1) * step_mb)}


class E2EPipeline:
    """End-to-end steps with host buffers, overlapped across steps.

    nbuf buffer sets (device inputs, layer buffers, host result) alternate
    between steps.  Step i's inputs are copied in on the h2d stream while step
    i - 1 computes, and its result is copied out on the d2h stream while step
    i + 1 computes.  Every step still copies its own inputs in and its own
    result out.  Ordering (all by events, nothing on the host):
      copy_in(i)   waits until replay(i - nbuf) has read buffer i % nbuf;
      replay(i)    waits for copy_in(i) and for copy_out(i - nbuf), which
                   must have read the layer output that replay(i) overwrites;
      copy_out(i)  waits for replay(i).
    copy_in, replay and copy_out are callables (step, buffer, stream)."""

    def __init__(self, nbuf, h2d, compute, d2h, make_event, copy_in, replay, copy_out):
        self.nbuf, self.h2d, self.compute, self.d2h = nbuf, h2d, compute, d2h
        self.copy_in, self.replay, self.copy_out = copy_in, replay, copy_out
        self.in_ready = [make_event() for _ in range(nbuf)]
        self.computed = [make_event() for _ in range(nbuf)]
        self.out_done = [make_event() for _ in range(nbuf)]

    def _in(self, i):
        b = i % self.nbuf
        self.h2d.wait_event(self.computed[b])
        self.copy_in(i, b, self.h2d)
        self.in_ready[b].record(self.h2d)

    def _compute_out(self, i):
        b = i % self.nbuf
        self.compute.wait_event(self.in_ready[b])
        self.compute.wait_event(self.out_done[b])
        self.replay(i, b, self.compute)
        self.computed[b].record(self.compute)
        self.d2h.wait_event(self.computed[b])
        self.copy_out(i, b, self.d2h)
        self.out_done[b].record(self.d2h)

    def run(self, n, start_event=None):
        """Enqueue n steps; the compute stream ends after the last copy-out.
        start_event (recorded on the compute stream) gates the copy streams."""
        if start_event is not None:
            self.h2d.wait_event(start_event)
            self.d2h.wait_event(start_event)
        if n <= 0:
            return
        self._in(0)
        for i in range(n):
            if i + 1 < n:
                self._in(i + 1)
            self._compute_out(i)
        self.compute.wait_event(self.out_done[(n - 1) % self.nbuf])


def run_config(args, base: dict) -> dict:
    """The reported config: the workload's, plus the options that change what runs."""
    calls = ("ft_moe_layer_nvfp4" if getattr(args, "whole", False) else
             ("ft_moe_route_permute" if args.fused_front else "ft_moe_route + ft_moe_permute")
             + " + ft_moe_ffn_nvfp4 + ft_moe_combine")
    return dict(base, format=args.fmt, slot_layout=args.layout, calls=calls)


# Workloads reported in the `workloads` object of the JSON line, besides the
# headline one: every layer family of the task, at every batch size it names.
ALL_WORKLOADS = ("tiny", "decode_T1", "decode_T8", "decode_T32", "decode_T64", "prefill_zipf_T4096",
                 "slots512_T1", "slots512_T2048", "slots512_T8192", "wide_T8192")
SWEEP_WORKLOAD = "wide_decode_T1"
MEDIAN_REPLAYS = 60          # individually timed graph replays behind each median


def _roofline(dom_name, dom_ms, w, mean_distinct, fmt, clk, peaks):
    """Roofline of the dominant kernel: HBM GB/s on the algorithmic bytes for
    decode-shaped layers, tensor TFLOP/s on the real rows' FLOPs otherwise."""
    hbm, bf16, bf16_sus, peak_src = peaks
    P = w.T * w.k
    flops_step = 6.0 * w.H * w.I * P
    decode_like = flops_step / (mean_distinct * bytes_per_expert(w.H, w.I, fmt)) < 200
    if dom_name == "layer_decode":
        # the whole layer in one launch: the three weight tensors of every expert hit, the token rows
        # (bf16) and logits in, the expert outputs and y (fp32) out
        alg_bytes = (mean_distinct * bytes_per_expert(w.H, w.I, fmt) + w.T * w.H * 2 + w.T * w.E * 4
                     + P * w.H * 4 + w.T * w.H * 4)
        alg_flops = flops_step
    elif dom_name == "ffn_decode":
        # both GEMMs in one launch: the three weight tensors of every expert hit,
        # the token rows in (bf16) and the expert outputs out (fp32)
        alg_bytes = mean_distinct * bytes_per_expert(w.H, w.I, fmt) + w.T * w.H * 2 + P * w.H * 4
        alg_flops = flops_step
    elif dom_name == "gemm_gate_up":
        alg_bytes = mean_distinct * gate_up_bytes_per_expert(w.H, w.I, fmt) + w.T * w.H * 2 + P * w.I * 2
        alg_flops = 4.0 * w.H * w.I * P
    else:
        alg_bytes = mean_distinct * (w.H * w.I // 2 + w.H * w.I // 16 + 4) + P * w.I * 2 + P * w.H * 4
        alg_flops = 2.0 * w.H * w.I * P
    traffic = traffic_record(f"{dom_name}:{w.name}")
    if decode_like:
        achieved = alg_bytes / (dom_ms * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4), "traffic": traffic, "kernel": dom_name,
                "launch_ms": round(dom_ms, 5), "algorithmic_bytes": int(alg_bytes), "peak_source": peak_src}
    achieved = alg_flops / (dom_ms * 1e-3) / 1e12
    # the burst GEMM peak while the SMs held their maximum clock through the
    # timed region, the sustained (power-capped) one otherwise
    full_clock = bool(clk and clk.get("sm_mhz") and clk.get("sm_max_mhz") and clk["sm_mhz"] >= 0.95 * clk["sm_max_mhz"])
    peak = bf16 if full_clock else bf16_sus
    return {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "traffic": traffic, "kernel": dom_name,
            "launch_ms": round(dom_ms, 5), "algorithmic_flops": alg_flops,
            "peak_source": f"{peak_src} ({'burst' if full_clock else 'sustained'} bf16 GEMM)"}


class Timer:
    """CUDA-event timing on one stream, max over ranks."""

    def __init__(self, stream, world, dev):
        self.stream, self.world, self.dev = stream, world, dev

    def _sync_start(self):
        import torch
        import torch.distributed as dist
        if self.world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def block(self, fn, n):
        """Device time (ms) of n calls of fn(i) between two events, max over ranks."""
        import torch
        self._sync_start()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(self.stream):
            torch.cuda._sleep(2_000_000)          # let the host queue the steps ahead of the GPU
            a.record(self.stream)
            for i in range(n):
                fn(i)
            b.record(self.stream)
        self.stream.synchronize()
        return max_over_ranks(a.elapsed_time(b), self.dev)

    def median_each(self, fn, n):
        """Median over n calls of fn(i), each between its own pair of events
        (max over ranks of the median)."""
        import torch
        self._sync_start()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        with torch.cuda.stream(self.stream):
            torch.cuda._sleep(2_000_000)
            for i in range(n):
                ev[i][0].record(self.stream)
                fn(i)
                ev[i][1].record(self.stream)
        self.stream.synchronize()
        return max_over_ranks(statistics.median(a.elapsed_time(b) for a, b in ev), self.dev)


def measure_workload(args, name, rank, world, local, dev, peaks, headline, want_cpu):
    """Every number of one workload: graph-replay throughput (a K-step block
    and the median of individually timed replays), per-kernel device times
    from eager steps, the dominant kernel's roofline, the end-to-end figure
    with host buffers, and the oracle on the host cores."""
    import torch

    from moe_expert_layer_renorm_b200 import _lib
    from moe_expert_layer_renorm_b200.layer import ExpertPool, MoELayer

    w = inputs.WORKLOADS[name]
    R = rotation_layers(w, args.layers)
    T = w.T
    # per-rank, per-layer independent inputs; the R layers' experts share one
    # slot pool (disjoint slots, scattered over the pool when the workload's
    # slots are permuted), as the layers of a model share an expert cache
    S = max(w.slots, R * w.E)
    order = np.random.default_rng([w.seed, rank, 9]).permutation(S) if w.permuted_slots else np.arange(S)
    pool = ExpertPool(w.H, w.I, S, device=dev,
                      fmt=_lib.FT_SCALE_MXFP4 if args.fmt == "mxfp4" else _lib.FT_SCALE_NVFP4,
                      tiled=args.layout == "tiled")
    layers = []
    for l in range(R):
        s = rank_layer_seed(w, rank, l)
        li = inputs.make_layer_inputs(inputs.custom_workload(w, seed=s), 0)
        st = order[l * w.E:(l + 1) * w.E].astype(np.int32)
        for e in range(w.E):
            for mat in range(3):
                N, K = pool.shape(mat)
                pool.pack_into(int(st[e]), mat, inputs.make_weight_fp32_torch(N, K, s, e, mat, dev))
        x = torch.from_numpy(li.x_bits.view(np.int16)).view(torch.bfloat16).to(dev)
        lg = torch.from_numpy(li.logits).to(dev)
        layers.append(dict(li=li, pool=pool, st_host=st, st=torch.from_numpy(st).to(dev), x=x, lg=lg, seed=s))
    torch.cuda.synchronize()
    layer = MoELayer(T, w.E, w.k, w.H, w.I, mode=w.route_mode, device=dev, fused_front=args.fused_front,
                     whole=args.whole)
    stream = torch.cuda.Stream(device=dev)
    tm = Timer(stream, world, dev)

    # distinct experts per layer (routing is deterministic; used for the algorithmic bytes)
    distinct = []
    with torch.cuda.stream(stream):
        for L in layers:
            layer.forward(L["x"], L["lg"], L["st"], L["pool"], stream=stream)
            stream.synchronize()
            distinct.append(int(torch.unique(layer.ids).numel()))

    def step(i):
        L = layers[i % R]
        layer.forward(L["x"], L["lg"], L["st"], L["pool"], stream=stream)

    with torch.cuda.stream(stream):
        for i in range(max(3, args.warmup)):
            step(i)
    stream.synchronize()

    # one CUDA graph per layer: the whole layer (route -> ... -> combine)
    graphs = []
    for l in range(R):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                step(l)
        graphs.append(g)
    with torch.cuda.stream(stream):
        for i in range(max(3, args.warmup)):
            graphs[i % R].replay()
    stream.synchronize()
    replay = lambda i: graphs[i % R].replay()   # noqa: E731

    # -------- timed region 1: graph replays, device-resident inputs --------
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    reps = max(1, int(round(0.3 / max(1e-6, 1e-3 * tm.block(replay, args.steps))))) if headline else 1
    elapsed_ms = 0.0
    for _ in range(reps):   # repeat the K-step measurement so the clock sampler sees load
        elapsed_ms = tm.block(replay, args.steps)
    median_ms = tm.median_each(replay, max(MEDIAN_REPLAYS, args.steps))
    clk = clocks.stop()

    # -------- timed region 2: eager launches with per-kernel device timing --------
    _lib.profile_read(reset=True)
    _lib.profile_enable(True)
    eager_ms = tm.block(step, args.steps)
    _lib.profile_enable(False)
    prof = _lib.profile_read(reset=True)

    # -------- end to end: pinned host inputs, copies inside the timed region --------
    host = [(L["x"].cpu().pin_memory(), L["lg"].cpu().pin_memory()) for L in layers]
    bufs = []
    for _ in range(2):
        bufs.append(dict(lay=MoELayer(T, w.E, w.k, w.H, w.I, mode=w.route_mode, device=dev,
                                      fused_front=args.fused_front, whole=args.whole),
                         xd=torch.empty_like(layers[0]["x"]), lgd=torch.empty_like(layers[0]["lg"]),
                         y_host=torch.empty((T, w.H), dtype=torch.float32).pin_memory()))
    e2e_graphs = {}
    for bi, B in enumerate(bufs):
        for l in range(R):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(stream):
                with torch.cuda.graph(g, stream=stream):
                    B["lay"].forward(B["xd"], B["lgd"], layers[l]["st"], layers[l]["pool"], stream=stream)
            e2e_graphs[(l, bi)] = g
    h2d_stream = torch.cuda.Stream(device=dev)
    d2h_stream = torch.cuda.Stream(device=dev)

    def e2e_in(i, bi, s):
        hx, hl = host[i % R]
        with torch.cuda.stream(s):
            bufs[bi]["xd"].copy_(hx, non_blocking=True)
            bufs[bi]["lgd"].copy_(hl, non_blocking=True)

    def e2e_replay(i, bi, s):
        with torch.cuda.stream(s):
            e2e_graphs[(i % R, bi)].replay()

    def e2e_out(i, bi, s):
        with torch.cuda.stream(s):
            bufs[bi]["y_host"].copy_(bufs[bi]["lay"].y, non_blocking=True)

    pipe = E2EPipeline(2, h2d_stream, stream, d2h_stream, torch.cuda.Event, e2e_in, e2e_replay, e2e_out)

    def timed_e2e(n):
        """Like Timer.block: CUDA-event time of n pipelined end-to-end steps, max over ranks."""
        tm._sync_start()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            torch.cuda._sleep(2_000_000)
            a.record(stream)
        pipe.run(n, start_event=a)
        b.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(a.elapsed_time(b), dev)

    def serial_e2e_step(i):
        """One step with its copies on the compute stream, nothing overlapped."""
        e2e_in(i, 0, stream)
        e2e_replay(i, 0, stream)
        e2e_out(i, 0, stream)

    e2e_pipelined, e2e_note = True, None
    try:
        pipe.run(3)
        torch.cuda.synchronize()
        e2e_ms = timed_e2e(args.steps)
    except Exception as exc:   # report it, and measure the plain order instead
        e2e_pipelined, e2e_note = False, f"{type(exc).__name__}: {exc}"[:200]
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            for i in range(3):
                serial_e2e_step(i)
        stream.synchronize()
        e2e_ms = tm.block(serial_e2e_step, args.steps)
    for g in graphs + list(e2e_graphs.values()):
        g.reset()

    # -------- roofline of the dominant kernel --------
    cands = [("layer_decode", prof["layer_decode"]), ("ffn_decode", prof["ffn_decode"]),
             ("gemm_gate_up", prof["gemm_gate_up"]), ("gemm_down", prof["gemm_down"])]
    dom_name, dom = max(cands, key=lambda c: c[1][2])
    dom_ms = dom[2] / max(1, dom[1])
    steps_per_layer = [sum(1 for i in range(args.steps) if i % R == l) for l in range(R)]
    mean_distinct = sum(d * n for d, n in zip(distinct, steps_per_layer)) / args.steps
    roof = _roofline(dom_name, dom_ms, w, mean_distinct, args.fmt, clk, peaks)

    ms_per_step = elapsed_ms / args.steps
    flops_step = 6.0 * w.H * w.I * T * w.k
    weight_bytes = mean_distinct * bytes_per_expert(w.H, w.I, args.fmt)
    cpu = None
    if want_cpu and rank == 0 and world == 1:
        cpu = cpu_baseline(layers[0], w, T, args.cpu_sample_tokens, args.fmt, budget_s=10.0 if headline else 2.0)
    out = {
        "value": round(world * T * args.steps / (elapsed_ms * 1e-3), 1), "unit": "tokens/s",
        "ms_per_step": round(ms_per_step, 5),
        "median_ms_per_step": round(median_ms, 5),
        "median_tokens_per_s": round(world * T / (median_ms * 1e-3), 1),
        "median_of": max(MEDIAN_REPLAYS, args.steps),
        "eager_ms_per_step": round(eager_ms / args.steps, 5),
        "config": run_config(args, workload_config(w, R, S, world)),
        "layer": {"distinct_experts": round(mean_distinct, 2),
                  "weight_GBps": round(weight_bytes / (ms_per_step * 1e-3) / 1e9, 1),
                  "TFLOPs": round(flops_step / (ms_per_step * 1e-3) / 1e12, 2),
                  "hbm_frac_of_measured": round(weight_bytes / (ms_per_step * 1e-3) / 1e9 / peaks[0], 4)},
        "roofline": roof,
        "e2e": {"value": round(world * T * args.steps / (e2e_ms * 1e-3), 1), "unit": "tokens/s",
                "overlap": ("two buffer sets: step i+1's inputs copy in and step i-1's result copies out while "
                            "step i computes") if e2e_pipelined else f"none (pipelined order failed: {e2e_note})",
                "h2d_bytes_per_step": T * w.H * 2 + T * w.E * 4, "d2h_bytes_per_step": T * w.H * 4},
        "gpu_launches": sum(v[0] for v in prof.values()),
        "kernels": {k: {"launches": v[0], "avg_ms": round(v[2] / v[1], 5) if v[1] else None}
                    for k, v in prof.items() if v[0]},
        "clocks": clk,
        "cpu_baseline": cpu,
    }
    del graphs, e2e_graphs, layers, pool, bufs, host, layer
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def measure_sweep(args, rank, world, local, dev, peaks, want_cpu):
    """The wide layer's 48-layer decode sweep: one token through 48
    independent resident layers (E32 k4 H=I=2880, own seeded weights, inputs
    and logits per layer), launched back to back in one CUDA graph.  The
    layers' experts (48 x 32 x 14 MB) stay resident in HBM; one replay reads
    each layer's selected experts once, 2.7 GB per token, far beyond L2."""
    import torch

    from moe_expert_layer_renorm_b200 import _lib
    from moe_expert_layer_renorm_b200.layer import ExpertPool, MoELayer

    w = inputs.WORKLOADS[SWEEP_WORKLOAD]
    NL = inputs.WIDE_SWEEP_LAYERS
    pool = ExpertPool(w.H, w.I, NL * w.E, device=dev,
                      fmt=_lib.FT_SCALE_MXFP4 if args.fmt == "mxfp4" else _lib.FT_SCALE_NVFP4,
                      tiled=args.layout == "tiled")
    layers = []
    for l in range(NL):
        s = rank_layer_seed(w, rank, l)
        li = inputs.make_layer_inputs(inputs.custom_workload(w, seed=s), 0)
        st = np.arange(l * w.E, (l + 1) * w.E, dtype=np.int32)
        for e in range(w.E):
            for mat in range(3):
                N, K = pool.shape(mat)
                pool.pack_into(int(st[e]), mat, inputs.make_weight_fp32_torch(N, K, s, e, mat, dev))
        layers.append(dict(li=li, st_host=st, st=torch.from_numpy(st).to(dev), pool=pool,
                           x=torch.from_numpy(li.x_bits.view(np.int16)).view(torch.bfloat16).to(dev),
                           lg=torch.from_numpy(li.logits).to(dev),
                           lay=MoELayer(w.T, w.E, w.k, w.H, w.I, mode=w.route_mode, device=dev,
                                        fused_front=args.fused_front, whole=args.whole)))
    torch.cuda.synchronize()
    stream = torch.cuda.Stream(device=dev)
    tm = Timer(stream, world, dev)
    distinct = 0
    with torch.cuda.stream(stream):
        for L in layers:
            L["lay"].forward(L["x"], L["lg"], L["st"], pool, stream=stream)
        stream.synchronize()
        for L in layers:
            distinct += int(torch.unique(L["lay"].ids).numel())

    def token(_i=0):
        for L in layers:
            L["lay"].forward(L["x"], L["lg"], L["st"], pool, stream=stream)

    with torch.cuda.stream(stream):
        for i in range(max(3, args.warmup)):
            token(i)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            token()
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            g.replay()
    stream.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    n = max(MEDIAN_REPLAYS, args.steps)
    median_ms = tm.median_each(lambda i: g.replay(), n)
    block_ms = tm.block(lambda i: g.replay(), args.steps) / args.steps
    clk = clocks.stop()
    _lib.profile_read(reset=True)
    _lib.profile_enable(True)
    eager_ms = tm.block(token, 3) / 3
    _lib.profile_enable(False)
    prof = _lib.profile_read(reset=True)
    g.reset()
    dom_name = max(("layer_decode", "ffn_decode"), key=lambda n: prof[n][2])
    dom = prof[dom_name]
    dom_ms = dom[2] / max(1, dom[1])
    mean_distinct = distinct / NL
    roof = _roofline(dom_name, dom_ms, w, mean_distinct, args.fmt, clk, peaks)
    weight_bytes = distinct * bytes_per_expert(w.H, w.I, args.fmt)
    cpu = None
    if want_cpu and rank == 0 and world == 1:
        cpu = cpu_baseline(layers[0], w, w.T, 1, args.fmt, budget_s=2.0)
        if cpu:   # one layer's token rate -> tokens through all 48 layers
            cpu = dict(cpu, value=round(cpu["value"] / NL, 4), unit="tokens/s through 48 layers",
                       sample=cpu["sample"] + f"; rate divided by {NL} layers")
    out = {
        "value": round(world * 1e3 / median_ms, 2), "unit": "tokens/s through 48 layers",
        "ms_per_token_48_layers": round(median_ms, 5), "median_of": n,
        "block_ms_per_token_48_layers": round(block_ms, 5),
        "ms_per_layer": round(median_ms / NL, 5),
        "eager_ms_per_token_48_layers": round(eager_ms, 5),
        "config": dict(run_config(args, {"workload": "wide_decode_T1 x 48 layers", "T": 1, "E": w.E, "k": w.k,
                                         "H": w.H, "I": w.I, "route": "topk_softmax", "layers": NL,
                                         "parallelism": f"dp{world} (independent batches)",
                                         "l2": "48 resident layers in one graph; one token reads each "
                                               "layer's selected experts once (~2.7 GB)"})),
        "layer": {"distinct_experts_per_layer": round(mean_distinct, 2),
                  "weight_GBps": round(weight_bytes / (median_ms * 1e-3) / 1e9, 1),
                  "hbm_frac_of_measured": round(weight_bytes / (median_ms * 1e-3) / 1e9 / peaks[0], 4)},
        "roofline": roof,
        "gpu_launches_per_token": sum(v[0] for v in prof.values()) // 3,
        "kernels": {k: {"launches": v[0], "avg_ms": round(v[2] / v[1], 5) if v[1] else None}
                    for k, v in prof.items() if v[0]},
        "clocks": clk,
        "cpu_baseline": cpu,
    }
    del layers, pool, g
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    peaks = measured_peaks()
    want_cpu = not args.no_cpu_baseline
    head = measure_workload(args, args.workload, rank, world, local, dev, peaks, headline=True, want_cpu=want_cpu)
    others = {}
    if not args.only:
        for name in ALL_WORKLOADS:
            if name == args.workload:
                continue
            others[name] = measure_workload(args, name, rank, world, local, dev, peaks, headline=False,
                                            want_cpu=want_cpu)
        others["wide_decode_T1_48_layers"] = measure_sweep(args, rank, world, local, dev, peaks, want_cpu)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": f"{args.fmt} weights, f16 MMA operands, fp32 accumulate",
        "data": "synthetic (seeded N(0,1) activations, N(0,sigma) logits, N(0,0.02) weights packed to "
                f"{args.fmt.upper()})",
        "config": head["config"],
        "median_ms_per_step": head["median_ms_per_step"], "median_of": head["median_of"],
        "layer": head["layer"], "roofline": head["roofline"], "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"], "eager_ms_per_step": head["eager_ms_per_step"],
        "kernels": head["kernels"], "clocks": head["clocks"], "cpu_baseline": head["cpu_baseline"],
    }
    if others:
        line["workloads"] = {args.workload: {k: v for k, v in head.items() if k != "config"}, **others}
    print(json.dumps(line))


def oracle_threads() -> int:
    """Host threads the C++ oracle runs on (its OpenMP default)."""
    v = os.environ.get("OMP_NUM_THREADS", "")
    return int(v) if v.isdigit() and int(v) > 0 else (os.cpu_count() or 1)


def cpu_baseline(L, w, T, n_tokens, fmt="nvfp4", budget_s=10.0):
    """The C++ oracle (as it stands) on a bounded sample of the same layer:
    the first n tokens, repeated until about budget_s of host time."""
    from oracle import cpp

    li = L["li"]
    pool = L["pool"]
    st = L["st_host"]
    n = min(T, n_tokens)
    ids, _ = cpp.route(li.logits[:n], w.k)
    need = sorted(set(int(v) for v in ids.reshape(-1)))
    Lo = pool.rows_layout                                     # slots read back row-major
    nb = int(Lo.slot_bytes)
    buf = np.zeros(len(need) * nb, np.uint8)                  # the selected experts' slots, on the host
    table = np.full(w.E, -1, np.int32)
    for i, e in enumerate(need):
        buf[i * nb:(i + 1) * nb] = pool.export_slot(int(st[e]))
        table[e] = i
    reps, dt = 0, 0.0
    while dt < budget_s and reps < 50:
        t0 = time.perf_counter()
        cpp.moe_layer(li.x_bits, li.logits, w.k, table, buf, nb, list(Lo.codes_off),
                      list(Lo.scales_off), list(Lo.global_off), list(Lo.ld_scale), w.H, w.I, tokens=np.arange(n),
                      fmt=int(Lo.scale_format))
        dt += time.perf_counter() - t0
        reps += 1
    return {"value": round(n * reps / dt, 3), "unit": "tokens/s", "cores": oracle_threads(), "kind": "oracle",
            "sample": f"{n} tokens of one {w.name} layer x {reps} (C++ oracle: route, {fmt.upper()} decode from the "
                      f"bytes of the {len(need)} experts they select, fp64 SwiGLU FFN, combine); {dt:.2f} s",
            "host_cpus": os.cpu_count()}


# ------------------------------------------------------ reference arm ---

REFERENCE_BUDGET_S = 120.0


def reference_layout(H: int, I: int) -> dict:
    """The slot layout of the library's C header (ft_nvfp4_slot_layout) from its
    documented definition, for the reference arm, which loads no library."""
    a256 = lambda v: (v + 255) // 256 * 256
    L = {"codes_off": [], "scales_off": [], "ld_scale": []}
    off = 0
    for N, K in ((I, H), (I, H), (H, I)):
        ld = (K // 16 + 15) // 16 * 16
        L["ld_scale"].append(ld)
        L["codes_off"].append(off)
        off = a256(off + N * K // 2)
        L["scales_off"].append(off)
        off = a256(off + N * ld)
    L["global_off"] = [off + 4 * m for m in range(3)]
    L["slot_bytes"] = a256(off + 12)
    return L


def run_reference(args):
    """The C++ oracle timed on the host cores, on this workload's metric."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from oracle import cpp

    w = inputs.WORKLOADS[args.workload]
    R = rotation_layers(w, args.layers)
    li = inputs.make_layer_inputs(w, 0)
    s = inputs.layer_seed(w.seed, 0)
    Lo = reference_layout(w.H, w.I)
    slots = {}

    def slot_bytes_of(e):
        """Expert e packed by the oracle into one slot of the layout (untimed)."""
        if e not in slots:
            b = np.zeros(Lo["slot_bytes"], np.uint8)
            for mat, (N, K) in enumerate(((w.I, w.H), (w.I, w.H), (w.H, w.I))):
                wt = inputs.make_weight_fp32_host(N, K, s, e, mat)
                if args.fmt == "mxfp4":   # E8M0 bytes at both of their 16-K positions; no global
                    c, sc32 = cpp.pack_mxfp4(wt)
                    sc = np.zeros((N, Lo["ld_scale"][mat]), np.uint8)
                    sc[:, 0:K // 16:2] = sc32
                    sc[:, 1:K // 16:2] = sc32
                    g = np.float32(1.0)
                else:
                    c, sc, g = cpp.pack(wt, Lo["ld_scale"][mat])
                b[Lo["codes_off"][mat]:Lo["codes_off"][mat] + c.size] = c.reshape(-1)
                b[Lo["scales_off"][mat]:Lo["scales_off"][mat] + sc.size] = sc.reshape(-1)
                b[Lo["global_off"][mat]:Lo["global_off"][mat] + 4] = np.frombuffer(np.float32(g).tobytes(), np.uint8)
            slots[e] = b
        return slots[e]

    def step(i, n):
        tok = (np.arange(n) + i * n) % w.T
        ids, _ = cpp.route(li.logits[tok], w.k)
        need = sorted(set(int(v) for v in ids.reshape(-1)))
        buf = np.concatenate([slot_bytes_of(e) for e in need])
        table = np.full(w.E, -1, np.int32)
        table[need] = np.arange(len(need), dtype=np.int32)
        t0 = time.perf_counter()
        cpp.moe_layer(li.x_bits, li.logits, w.k, table, buf, Lo["slot_bytes"], Lo["codes_off"], Lo["scales_off"],
                      Lo["global_off"], Lo["ld_scale"], w.H, w.I, tokens=tok, fmt=1 if args.fmt == "mxfp4" else 0)
        return time.perf_counter() - t0

    # size each step's sample so that warm-up and timed steps together take
    # about REFERENCE_BUDGET_S of host time
    n0 = min(w.T, 2)
    per_token = step(0, n0) / n0
    n = int(max(1, min(w.T, args.cpu_sample_tokens,
                       REFERENCE_BUDGET_S / max(1, args.steps + args.warmup) / max(per_token, 1e-9))))
    for i in range(args.warmup):
        step(i, n)
    times = [step(args.warmup + i, n) for i in range(args.steps)]
    total = sum(times)
    value = n * args.steps / total
    threads = oracle_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": run_config(args, workload_config(w, R, max(w.slots, R * w.E), world)),
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"{n} tokens of one {w.name} layer per step"},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


CHURN_CONFIG = dict(T=8, E=128, k=8, H=2048, I=768, layers=8, domains=4, hot=16, capacity=192)


def run_slot_churn(args):
    """Expert-cache churn (one GPU): decode steps of 8 layers (E128 k8 H2048
    I768, T=8) whose experts live in pinned host banks; the device pool holds
    192 slots, 1.5 domains' worth.  The domain switches every
    `steps_per_domain` steps, so the first step of a domain misses on every
    layer.  Both work orders (demand, prefetch) are timed with CUDA events."""
    import torch
    from moe_expert_layer_renorm_b200 import churn

    if args.slot_churn == "prefill_stream":
        run_prefill_stream()
        return
    cfg = churn.ChurnConfig(**CHURN_CONFIG)
    hs = churn.hot_sets(cfg)
    banks = churn.ExpertBanks(cfg, hs)
    out = {"metric": "expert-cache churn: decode step time with misses (switch) and without (steady)",
           "unit": "ms/step", "n_gpus": 1, "data": "synthetic (domain-rotation routing)",
           "config": dict(CHURN_CONFIG, steps_per_domain=8, rounds=2, slot_mb=round(banks.slot_bytes / 1e6, 3))}
    for mode in ("demand", "prefetch"):
        r = churn.run_churn(cfg, mode, steps_per_domain=8, rounds=2, banks=banks)
        sw, st = statistics.median(r["switch_ms"]), statistics.median(r["steady_ms"])
        miss = statistics.median(r["misses_per_switch"])
        bytes_sw = statistics.median(r["h2d_bytes_per_switch"])
        out[mode] = {"switch_ms": round(sw, 4), "steady_ms": round(st, 4), "misses_per_switch": miss,
                     "h2d_MB_per_switch": round(bytes_sw / 1e6, 1),
                     "miss_cost_ms": round(sw - st, 4),
                     "h2d_GBps_effective": round(bytes_sw / max(sw - st, 1e-6) / 1e6, 1),
                     "stats": r["stats"]}
        torch.cuda.synchronize()
    print(json.dumps(out))


STREAM_CONFIG = dict(T=4096, E=128, k=8, H=2048, I=768, layers=4, domains=1, hot=128, capacity=256)


def run_prefill_stream():
    """Double-buffered prefill expert streaming (one GPU): 4 prefill layers
    (T=4096, E128 k8 H2048 I768, uniform routing) whose 128 experts each come
    from pinned host banks into a 256-slot pool (two layers' worth): layer
    l + 1's experts are filled while layer l runs.  Reports the streamed step,
    the same step with every expert resident, and a plain copy of the same
    bytes."""
    import torch
    from moe_expert_layer_renorm_b200 import churn

    cfg = churn.ChurnConfig(**STREAM_CONFIG)
    banks = churn.ExpertBanks(cfg, churn.hot_sets(cfg), keep_device=True)
    r = churn.run_stream(cfg, steps=4, banks=banks)
    sm, rm = statistics.median(r["stream_ms"]), statistics.median(r["resident_ms"])
    b = statistics.median(r["h2d_bytes_per_step"])
    copy_ms = b / (r["copy_only_GBps"] * 1e6)
    print(json.dumps({
        "metric": "prefill expert streaming: step time of 4 layers with every expert filled from the host",
        "unit": "ms/step", "n_gpus": 1, "data": "synthetic (uniform routing)",
        "config": dict(STREAM_CONFIG, steps=4, slot_mb=round(banks.slot_bytes / 1e6, 3)),
        "stream_ms": round(sm, 3), "resident_ms": round(rm, 3), "h2d_MB_per_step": round(b / 1e6, 1),
        "copy_only_GBps": round(r["copy_only_GBps"], 1), "copy_only_ms_for_step_bytes": round(copy_ms, 3),
        "overlap": round((rm + copy_ms - sm) / min(rm, copy_ms), 3),
        "stats": r["stats"]}))


def run_ep(args):
    """The layer with its experts split over the ranks (ExpertParallelMoE over
    NCCL; a one-rank group when run without torchrun).  Every rank routes its
    own batch; the step is eager (the exchange plan needs the routed counts on
    the host), timed with CUDA events, max over ranks."""
    import datetime
    import socket

    import torch
    import torch.distributed as dist

    from moe_expert_layer_renorm_b200.ep import ExpertParallelMoE, owned_experts
    from moe_expert_layer_renorm_b200.layer import ExpertPool

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    else:
        with socket.socket() as so:
            so.bind(("127.0.0.1", 0))
            port = so.getsockname()[1]
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                                timeout=datetime.timedelta(seconds=120), device_id=dev)
    w = inputs.WORKLOADS[args.workload]
    mine = owned_experts(w.E, world, rank)
    from moe_expert_layer_renorm_b200 import _lib
    pool = ExpertPool(w.H, w.I, len(mine), device=dev, tiled=args.layout == "tiled",
                      fmt=_lib.FT_SCALE_MXFP4 if args.fmt == "mxfp4" else _lib.FT_SCALE_NVFP4)
    for j, e in enumerate(mine):                     # the same experts as one GPU would hold, split by owner
        for mat in range(3):
            N, K = pool.shape(mat)
            pool.pack_into(j, mat, inputs.make_weight_fp32_torch(N, K, w.seed, e, mat, dev))
    table = torch.arange(len(mine), dtype=torch.int32, device=dev)
    li = inputs.make_layer_inputs(inputs.custom_workload(w, seed=rank_layer_seed(w, rank, 0)), 0)
    x = torch.from_numpy(li.x_bits.view(np.int16)).view(torch.bfloat16).to(dev)
    lg = torch.from_numpy(li.logits).to(dev)
    ep = ExpertParallelMoE(w.T, w.E, w.k, w.H, w.I, mode=w.route_mode, device=dev)
    for _ in range(max(3, args.warmup)):
        ep.forward(x, lg, table, pool)
    dist.barrier()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    recv = 0
    for _ in range(args.steps):
        ep.forward(x, lg, table, pool)
        recv += ep.plan.n_recv
    b.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), dev)
    line = {"metric": "MoE-layer tokens/s, experts split over the ranks", "value": round(world * w.T * args.steps /
                                                                                        (ms * 1e-3), 1),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms / args.steps, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": f"{args.fmt} weights, f16 MMA operands, fp32 accumulate",
            "data": "synthetic (seeded; each rank its own batch, the experts of one layer split by owner)",
            "config": dict(run_config(args, {"workload": w.name, "T_per_rank": w.T, "E": w.E, "k": w.k, "H": w.H,
                                             "I": w.I}),
                           parallelism=f"ep{world}", experts_per_rank=len(mine),
                           rows_received_per_step_rank0=round(recv / args.steps, 1),
                           timing="eager steps (one host synchronisation per step for the exchange plan)")}
    dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    elif args.slot_churn:
        run_slot_churn(args)
    elif args.ep:
        run_ep(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
