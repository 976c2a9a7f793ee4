"""Benchmark of the Spark2_5 hybrid GQA attention core on B200.

Headline workload (one step): prefill of B=4 sequences of T=8192 tokens
through one sliding-window layer and one full layer, q/k/v bf16 ~N(0,1) with
k scaled 0.5, gate logits ~N(0, 2^2), positions 0..8191, seed 1.  A step runs
the whole hot path: RoPE on q and k, the attention prefill, and the KV-cache
append, for both layer kinds.  Secondary workload: one decode step of the
36-layer stack for B=64 sequences with 32768 cached tokens (27 sliding layers
with 512-slot rings, 9 full layers with linear caches), captured in one CUDA
graph.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun each rank runs its own replica (independent sequences, no
collective on the data path); timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
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

SLIDING, FULL = 0, 1
HQ, HKV, D, WINDOW = 16, 4, 256, 512
PREFILL_B, PREFILL_T, PREFILL_SEED = 4, 8192, 1
DECODE_B, DECODE_CTX, DECODE_SEED = 64, 32768, 3
N_LAYERS = 36


# ----------------------------------------------------------- work models ----

def visible_pairs(T: int, pos0: int, kind: int, with_history: bool = True) -> int:
    """Exact number of visible (query, key) pairs of a chunk of T queries at pos0."""
    first = pos0 if not with_history else 0
    if kind == FULL:
        # query at pos0+t sees keys first..pos0+t
        return T * (pos0 - first + 1) + T * (T - 1) // 2
    total = 0
    for t in range(T):
        qp = pos0 + t
        total += qp - max(first, qp - WINDOW + 1) + 1
    return total


def prefill_flops(B: int, T: int, pos0: int, kind: int, with_history: bool = True) -> int:
    """Algorithmic FLOPs: 2*256 for QK^T plus 2*256 for PV per visible pair and query head."""
    return B * visible_pairs(T, pos0, kind, with_history) * HQ * 4 * D


def prefill_tile_flops(B: int, T: int, kind: int) -> int:
    """FLOPs the prefill kernels execute for a chunk without history: every 128-query tile against
    every 128-key tile it touches (diagonal and window-edge tiles in full, masked or not)."""
    n_qt = (T + 127) // 128
    tiles = 0
    for qt in range(n_qt):
        first = max(0, qt * 128 - (WINDOW - 1)) // 128 if kind == SLIDING else 0
        tiles += qt - first + 1
    return B * HQ * tiles * 128 * 128 * 4 * D


def decode_kv_bytes(B: int, p: int, kind: int) -> int:
    """Algorithmic KV bytes a decode step reads: visible keys x 4 heads x (K+V) x 256 x 2 B."""
    keys = p + 1 if kind == FULL else min(p + 1, WINDOW)
    return B * keys * HKV * 2 * D * 2


def decode_q8_kv_bytes(B: int, p: int, kind: int) -> int:
    """The same for the 8-bit cache: per key and KV head, K and V codes (256 B each) and scales (16 B each)."""
    keys = p + 1 if kind == FULL else min(p + 1, WINDOW)
    return B * keys * HKV * 2 * (D + 2 * (D // 32))


# ------------------------------------------------------------- plumbing -----

def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def hbm_roofline(kernel: str, achieved_gbs: float, peaks, traffic=None):
    """Roofline entry of a kernel that only reads HBM (the decode kernels read the KV cache and write
    a few KB): held to the measured read-only ceiling; the copy figure of MEASURED_PEAKS.json (read +
    write bytes of a device copy) is kept beside it for reference."""
    read = peaks.get("hbm_read_gbs")
    peak, src = (read, "read-only stream over 8 GiB, measured in this run") if read else \
        (peaks["hbm_gbs"], f"hbm_gbs copy, {peaks['source']} (no read probe in this run)")
    return {"bound": "hbm", "kernel": kernel, "achieved": achieved_gbs, "peak": peak, "unit": "GB/s",
            "frac": achieved_gbs / peak, "peak_source": src, "copy_peak_gbs": peaks["hbm_gbs"],
            "frac_of_copy": achieved_gbs / peaks["hbm_gbs"], "traffic": traffic}


def kernel_source_sha():
    """Hash of the CUDA sources' code (comments and blank space removed), which keys the ncu traffic
    figures in profiles/traffic.json: they hold until the code changes."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "full_gqa_attention_spark2_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(f.encode())
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it matches the current kernels."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    e = t.get(kernel)
    if not e or e.get("source_sha") != kernel_source_sha():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling every 10 ms; the summary covers the samples taken
    between begin() and end() (the timed region), so idle samples around it do not hide a clock that
    dropped under load."""
    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.t_begin = self.t_end = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "10"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.15)

    def begin(self):
        self.t_begin = datetime.datetime.now()

    def end(self):
        self.t_end = datetime.datetime.now()

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.03)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 10:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None

        def when(r):
            try:
                return datetime.datetime.strptime(r[0], "%Y/%m/%d %H:%M:%S.%f")
            except ValueError:
                return None
        inside = [r for r in rows if self.t_begin is not None and self.t_end is not None and when(r) is not None
                  and self.t_begin <= when(r) <= self.t_end]
        use = inside or rows
        sm = [float(r[2]) for r in use if r[2].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in use:
            for name, val in zip(names, r[6:10]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_min_mhz": min(sm) if sm else None,
                "sm_max_mhz": float(rows[0][3]) if rows[0][3].replace(".", "").isdigit() else None,
                "reasons": sorted(reasons), "samples": len(use), "in_timed_region": bool(inside),
                "interval_ms": 10}


# ------------------------------------------------------------ our arm -------

def prefill_workload(torch, sa, synth, dev, B=PREFILL_B, T=PREFILL_T, seed=PREFILL_SEED, k_sigma=0.5,
                     g_sigma=2.0):
    """Device buffers of a prefill workload for both layer kinds (default: the headline workload)."""
    W = {}
    for kind, layer in ((SLIDING, 0), (FULL, 3)):
        cfg = sa.spark_layer_cfg_for_kind(kind)
        q = torch.empty(B, T, HQ, D, dtype=torch.bfloat16, device=dev)
        k = torch.empty(B, T, HKV, D, dtype=torch.bfloat16, device=dev)
        v = torch.empty_like(k)
        g = torch.empty(B, T, HQ, dtype=torch.bfloat16, device=dev)
        synth.fill_tokens(q, seed, synth.tensor_id(layer, synth.ROLE_Q), 0)
        synth.fill_tokens(k, seed, synth.tensor_id(layer, synth.ROLE_K), 0, sigma=k_sigma)
        synth.fill_tokens(v, seed, synth.tensor_id(layer, synth.ROLE_V), 0)
        synth.fill_tokens(g, seed, synth.tensor_id(layer, synth.ROLE_GATE), 0, sigma=g_sigma)
        cap = WINDOW if kind == SLIDING else T
        kc = torch.empty(B, HKV, cap, D, dtype=torch.bfloat16, device=dev)
        vc = torch.empty_like(kc)
        W[kind] = dict(cfg=cfg, q=q, k=k, v=v, g=g, out=torch.empty_like(q), kc=kc, vc=vc)
    pos0 = torch.zeros(B, dtype=torch.int32, device=dev)
    return W, pos0


def prefill_step(sa, W, pos0, events=None):
    """One pass of the hot path over the batch, for both layer kinds: RoPE on k, the prefill
    (which rotates its raw q at load), the KV append.  events: {kind: (start, end)} recorded
    around each kind's prefill launch."""
    for kind in (SLIDING, FULL):
        w = W[kind]
        sa.spark_rope_apply(w["k"], pos0, w["cfg"])
        if events is not None:
            events[kind][0].record()
        sa.spark_attn_prefill(w["out"], w["q"], w["k"], w["v"], w["g"], None, None, pos0, w["cfg"],
                              flags=sa.SPARK_ROPE_FUSED)
        if events is not None:
            events[kind][1].record()
        sa.spark_kv_append(w["kc"], w["vc"], w["k"], w["v"], pos0, w["cfg"])


def max_over_ranks(torch, dist, ms: float, device: str = "cuda") -> float:
    """The slowest rank's time: every rank reports its own device-timed milliseconds."""
    if dist is None:
        return ms
    x = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(x, op=dist.ReduceOp.MAX)
    return float(x.item())


def weak_scaling_rate(units_per_rank: float, world: int, ms: float) -> float:
    """Whole-job throughput: every rank processed its own units in at most `ms`."""
    return units_per_rank * world / (ms * 1e-3)


def timed_region(torch, dist, fn, steps, clocks=None):
    """Time `steps` calls of fn on the device, bracketed by a barrier and a synchronize; max over ranks.
    clocks: a running ClockSampler, told where the region begins and ends."""
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    if clocks is not None:
        clocks.begin()
    t0.record()
    for i in range(steps):
        fn(i)
    t1.record()
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.end()
    if dist is not None:
        dist.barrier()
    return max_over_ranks(torch, dist, t0.elapsed_time(t1))


def run_prefill(torch, sa, synth, dist, args, peaks, world):
    dev = torch.device("cuda")
    W, pos0 = prefill_workload(torch, sa, synth, dev)
    for _ in range(args.warmup):
        prefill_step(sa, W, pos0)
    sa.spark_check()
    # per-launch duration of the full-layer prefill kernel, on its stream
    pairs = [{kind: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for kind in (SLIDING, FULL)} for _ in range(args.steps)]
    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    clocks.start()
    ms = timed_region(torch, dist, lambda i: prefill_step(sa, W, pos0, pairs[i]), args.steps, clocks)
    clk = clocks.stop()
    sa.spark_check()
    full_each = [ev[FULL][0].elapsed_time(ev[FULL][1]) for ev in pairs]
    kern_ms = statistics.mean(full_each)
    slide_ms = statistics.mean(ev[SLIDING][0].elapsed_time(ev[SLIDING][1]) for ev in pairs)
    B, T = PREFILL_B, PREFILL_T
    f_full = prefill_flops(B, T, 0, FULL, False)
    f_slide = prefill_flops(B, T, 0, SLIDING, False)
    ms_eager = ms / args.steps
    clk_eager = clk
    # the headline: the same step replayed from one CUDA graph (its six launches with no host work
    # between them), after a pause that lets the power draw settle back
    time.sleep(1.5)
    graph = graph_of(torch, lambda: prefill_step(sa, W, pos0))
    for _ in range(3):
        graph.replay()
    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    clocks.start()
    ms = timed_region(torch, dist, lambda i: graph.replay(), args.steps, clocks)
    clk = clocks.stop()
    sa.spark_check()
    del graph
    ms_step = ms / args.steps
    tokens = B * T * world
    achieved = f_full / (kern_ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]

    # end to end: pinned host inputs -> device, the path, outputs -> pinned host, every step.
    # Pipelined across steps with two sets of device buffers: the copy-in of step i+1 and the
    # copy-out of step i-1 run on their own streams while step i computes (PCIe is full duplex).
    host_in = {kind: {n: torch.empty(W[kind][n].shape, dtype=torch.bfloat16, pin_memory=True)
                      for n in ("q", "k", "v", "g")} for kind in W}
    host_out = {kind: torch.empty(W[kind]["out"].shape, dtype=torch.bfloat16, pin_memory=True) for kind in W}
    for kind in W:
        for n in ("q", "k", "v", "g"):
            host_in[kind][n].copy_(W[kind][n])
    h2d = sum(t.numel() * 2 for kind in W for t in host_in[kind].values())
    d2h = sum(t.numel() * 2 for t in host_out.values())
    W2 = {kind: dict(W[kind], **{n: torch.empty_like(W[kind][n]) for n in ("q", "k", "v", "g", "out", "kc", "vc")})
          for kind in W}
    bufs = (W, W2)
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_pipeline(steps):
        ev_in = [torch.cuda.Event() for _ in range(steps)]
        ev_cmp = [torch.cuda.Event() for _ in range(steps)]
        ev_out = [torch.cuda.Event() for _ in range(steps)]

        def step(i):
            cur = torch.cuda.current_stream()
            if i == 0:
                for st in (s_in, s_cmp, s_out):
                    st.wait_stream(cur)
            Wi = bufs[i % 2]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_cmp[i - 2])          # step i-2 has read these inputs
                for kind in Wi:
                    for n in ("q", "k", "v", "g"):
                        Wi[kind][n].copy_(host_in[kind][n], non_blocking=True)
                ev_in[i].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ev_in[i])
                if i >= 2:
                    s_cmp.wait_event(ev_out[i - 2])         # step i-2's output has been copied out
                prefill_step(sa, Wi, pos0)
                ev_cmp[i].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[i])
                for kind in Wi:
                    host_out[kind].copy_(Wi[kind]["out"], non_blocking=True)
                ev_out[i].record(s_out)
            if i == steps - 1:
                cur.wait_event(ev_out[i])
        return step

    warm = e2e_pipeline(2)
    warm(0)
    warm(1)
    torch.cuda.synchronize()
    e2e_steps = max(3, min(args.steps, 30))              # the pipeline's fill and drain amortised
    ms_e2e = timed_region(torch, dist, e2e_pipeline(e2e_steps), e2e_steps)
    del W2, bufs
    sa.spark_check()
    del W
    torch.cuda.empty_cache()
    return {
        "metric": "prefill attn tok/s & TFLOP/s; decode KV-read GB/s (36-layer stack); % roofline",
        "value": weak_scaling_rate(B * T, world, ms_step),
        "unit": "tok/s",
        "ms_per_step": ms_step,
        "tflops": (f_full + f_slide) * world / (ms_step * 1e-3) / 1e12,
        "eager": {"ms_per_step": ms_eager, "value": weak_scaling_rate(B * T, world, ms_eager), "clocks": clk_eager,
                  "note": "the same step with eager launches; the kernel times below come from its events"},
        "prefill_full_kernel": {"ms": kern_ms, "tflops": achieved, "flops": f_full,
                                # the mean over the first and the last ten timed steps: under the power
                                # cap, which a continuous run reaches after ~40 ms, the clocks drop
                                "ms_first_10_steps": statistics.mean(full_each[:10]),
                                "ms_last_10_steps": statistics.mean(full_each[-10:])},
        "per_layer_kind": {
            name: {"kernel_us": ms * 1e3, "tok_s": B * T / (ms * 1e-3),
                   "tflops": f / (ms * 1e-3) / 1e12, "algorithmic_flops": f,
                   "tile_flops": prefill_tile_flops(B, T, kind),
                   "roofline": {"bound": "tensor", "kernel": f"prefill3_kernel ({name} layer)",
                                "achieved": f / (ms * 1e-3) / 1e12, "peak": peak, "unit": "TFLOP/s",
                                "frac": f / (ms * 1e-3) / 1e12 / peak,
                                "peak_source": f"bf16_tflops burst, {peaks['source']}",
                                "traffic": ncu_traffic(f"prefill3_kernel_{name}")}}
            for name, kind, ms, f in (("sliding", SLIDING, slide_ms, f_slide), ("full", FULL, kern_ms, f_full))},
        "stack36_derived": {"ms": 27 * slide_ms + 9 * kern_ms,
                            "tok_s": B * T / ((27 * slide_ms + 9 * kern_ms) * 1e-3),
                            "note": "derived, not measured: 27 sliding + 9 full layer kernels of this step"},
        "roofline": {"bound": "tensor", "kernel": "prefill3_kernel (full layer, persistent SM pairs)", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": f"bf16_tflops burst, {peaks['source']}",
                     "frac_of_sustained": (achieved / peaks["bf16_tflops_sustained"]
                                           if peaks.get("bf16_tflops_sustained") else None),
                     "traffic": ncu_traffic("prefill3_kernel_full")},
        "e2e": {"value": tokens / (ms_e2e / e2e_steps * 1e-3), "unit": "tok/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "clocks": clk,
        "gpu_launches": 6 * args.steps,
    }


TINY_B, TINY_T, TINY_SEED = 1, 1024, 0


def run_prefill_stack36(torch, sa, synth, dist, args, peaks, world):
    """The headline prefill step through all 36 layers (27 sliding, 9 full, in the pages' order), each
    layer with its own q, k, v, gate, output and cache (B=4, T=8192: about 25 GB in all)."""
    dev = torch.device("cuda")
    B, T = PREFILL_B, PREFILL_T
    layers = []
    for layer in range(N_LAYERS):
        cfg = sa.spark_layer_cfg_for_layer(layer)
        q = torch.empty(B, T, HQ, D, dtype=torch.bfloat16, device=dev)
        k = torch.empty(B, T, HKV, D, dtype=torch.bfloat16, device=dev)
        v = torch.empty_like(k)
        g = torch.empty(B, T, HQ, dtype=torch.bfloat16, device=dev)
        synth.fill_tokens(q, PREFILL_SEED, synth.tensor_id(layer, synth.ROLE_Q), 0)
        synth.fill_tokens(k, PREFILL_SEED, synth.tensor_id(layer, synth.ROLE_K), 0, sigma=0.5)
        synth.fill_tokens(v, PREFILL_SEED, synth.tensor_id(layer, synth.ROLE_V), 0)
        synth.fill_tokens(g, PREFILL_SEED, synth.tensor_id(layer, synth.ROLE_GATE), 0, sigma=2.0)
        cap = WINDOW if cfg.kind == SLIDING else T
        kc = torch.empty(B, HKV, cap, D, dtype=torch.bfloat16, device=dev)
        layers.append(dict(cfg=cfg, q=q, k=k, v=v, g=g, out=torch.empty_like(q), kc=kc, vc=torch.empty_like(kc)))
    pos0 = torch.zeros(B, dtype=torch.int32, device=dev)

    def step(i=0):
        for w in layers:
            sa.spark_rope_apply(w["k"], pos0, w["cfg"])
            sa.spark_attn_prefill(w["out"], w["q"], w["k"], w["v"], w["g"], None, None, pos0, w["cfg"],
                                  flags=sa.SPARK_ROPE_FUSED)
            sa.spark_kv_append(w["kc"], w["vc"], w["k"], w["v"], pos0, w["cfg"])

    for _ in range(max(1, min(args.warmup, 3))):
        step()
    sa.spark_check()
    steps = max(5, min(args.steps, 10))
    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    clocks.start()
    ms = timed_region(torch, dist, step, steps, clocks) / steps
    clk = clocks.stop()
    sa.spark_check()
    flops = sum(prefill_flops(B, T, 0, w["cfg"].kind, False) for w in layers)
    del layers
    torch.cuda.empty_cache()
    tflops = flops / (ms * 1e-3) / 1e12
    sustained = peaks.get("bf16_tflops_sustained")
    return {"workload": f"prefill_b{B}_t{T}_36layers", "value": B * T * world / (ms * 1e-3), "unit": "tok/s",
            "ms_per_step": ms, "tflops": tflops * world, "gpu_launches_per_step": 3 * N_LAYERS,
            "frac_of_sustained_bf16": tflops / sustained if sustained else None, "clocks": clk,
            "note": "measured: per layer RoPE on k, the prefill (q rotated at load), the append; eager launches; "
                    "a step of ~30 ms at full tensor load runs under the power cap (clocks sampled here)"}


def run_prefill_tiny(torch, sa, synth, dist, args, peaks, world):
    """The small prefill workload: B=1, T=1024, seed 0, q/k/v/gate ~N(0,1), one sliding and one full
    layer, the same step as the headline (RoPE on k, prefill with q rotated at load, the append)."""
    dev = torch.device("cuda")
    B, T = TINY_B, TINY_T
    W, pos0 = prefill_workload(torch, sa, synth, dev, B, T, TINY_SEED, 1.0, 1.0)
    for _ in range(max(3, args.warmup)):
        prefill_step(sa, W, pos0)
    sa.spark_check()
    steps = max(20, min(args.steps, 200))
    pairs = [{kind: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for kind in (SLIDING, FULL)} for _ in range(steps)]
    ms = timed_region(torch, dist, lambda i: prefill_step(sa, W, pos0, pairs[i]), steps) / steps
    sa.spark_check()
    per = {}
    for name, kind in (("sliding", SLIDING), ("full", FULL)):
        k_ms = statistics.mean(ev[kind][0].elapsed_time(ev[kind][1]) for ev in pairs)
        f = prefill_flops(B, T, 0, kind, False)
        per[name] = {"kernel_us": k_ms * 1e3, "tok_s": B * T / (k_ms * 1e-3), "tflops": f / (k_ms * 1e-3) / 1e12,
                     "algorithmic_flops": f, "tile_flops": prefill_tile_flops(B, T, kind)}
    f_all = prefill_flops(B, T, 0, SLIDING, False) + prefill_flops(B, T, 0, FULL, False)
    # the same step's six launches replayed from one CUDA graph (no host work between them)
    graph = graph_of(torch, lambda: prefill_step(sa, W, pos0))
    for _ in range(3):
        graph.replay()
    ms_g = timed_region(torch, dist, lambda i: graph.replay(), steps) / steps
    sa.spark_check()
    del graph, W
    return {"workload": f"prefill_tiny_b{B}_t{T}_sliding+full", "value": B * T * world / (ms_g * 1e-3),
            "unit": "tok/s", "ms_per_step": ms_g, "tflops": f_all * world / (ms_g * 1e-3) / 1e12,
            "eager": {"ms_per_step": ms, "value": B * T * world / (ms * 1e-3)},
            "per_layer_kind": per, "gpu_launches_per_step": 6,
            "note": "one CUDA graph per step (eager launches beside it); 8 query tiles x 4 KV heads x 2 head "
                    "pairs = 64 units on 74 SM pairs: launch- and latency-bound, not a roofline case"}


def decode_layers(torch, sa, synth, dev, B: int, p: int, layer_ids=range(N_LAYERS), seed: int = DECODE_SEED):
    """Caches holding positions 0..p-1 and the new token's q/k/v/gate at p, per layer."""
    layers = []
    for l in layer_ids:
        kind = FULL if l % 4 == 3 else SLIDING
        cfg = sa.spark_layer_cfg_for_kind(kind)
        cap = WINDOW if kind == SLIDING else p + 1
        kc = torch.empty(B, HKV, cap, D, dtype=torch.bfloat16, device=dev)
        vc = torch.empty_like(kc)
        synth.fill_cache(kc, seed, synth.tensor_id(l, synth.ROLE_K), p, kind == SLIDING)
        synth.fill_cache(vc, seed, synth.tensor_id(l, synth.ROLE_V), p, kind == SLIDING)
        q = torch.empty(B, 1, HQ, D, dtype=torch.bfloat16, device=dev)
        kn = torch.empty(B, 1, HKV, D, dtype=torch.bfloat16, device=dev)
        vn = torch.empty_like(kn)
        g = torch.empty(B, 1, HQ, dtype=torch.bfloat16, device=dev)
        synth.fill_tokens(q, seed, synth.tensor_id(l, synth.ROLE_Q), p)
        synth.fill_tokens(kn, seed, synth.tensor_id(l, synth.ROLE_K), p)
        synth.fill_tokens(vn, seed, synth.tensor_id(l, synth.ROLE_V), p)
        synth.fill_tokens(g, seed, synth.tensor_id(l, synth.ROLE_GATE), p)
        layers.append(dict(layer=l, kind=kind, cfg=cfg, cap=cap, kc=kc, vc=vc, q=q.view(B, HQ, D), kn=kn, vn=vn,
                           g=g.view(B, HQ), out=torch.empty(B, HQ, D, dtype=torch.bfloat16, device=dev)))
    return layers


def decode_launches(sa, B: int, layers, q8: bool = False) -> int:
    """Kernels one decode step launches: per layer the append and the split kernel, plus the
    combine kernel where the split plan has more than one split (read back from the workspace size,
    B * 16 * splits * 258 fp32)."""
    n = 0
    for L in layers:
        fn = sa.spark_decode_q8_workspace_bytes if q8 else sa.spark_decode_workspace_bytes
        splits = fn(B, L["cap"], L["cfg"]) // (B * HQ * (D + 2) * 4)
        n += 2 + (1 if splits > 1 else 0)
    return n


def decode_step(sa, layers, pos, ws):
    """One decode step in two calls per layer: append the new token (RoPE fused on k), then attend
    (RoPE fused on q)."""
    for L in layers:
        sa.spark_kv_append(L["kc"], L["vc"], L["kn"], L["vn"], pos, L["cfg"], flags=sa.SPARK_ROPE_FUSED)
        sa.spark_attn_decode(L["out"], L["q"], L["g"], L["kc"], L["vc"], pos, L["cfg"], ws,
                             flags=sa.SPARK_ROPE_FUSED)


def decode_fused_step(sa, layers, pos, wsf):
    """One decode step in one launch per layer: append, attention and combine fused (RoPE on q and k)."""
    for L in layers:
        sa.spark_attn_decode_fused(L["out"], L["q"], L["kn"], L["vn"], L["g"], L["kc"], L["vc"], pos, L["cfg"], wsf,
                                   flags=sa.SPARK_ROPE_FUSED)


def graph_of(torch, fn):
    """fn() captured in a CUDA graph (after one eager run on a side stream)."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def event_ms(torch, fn, reps: int = 10) -> float:
    """Mean device time of fn() over reps back-to-back calls captured in one CUDA graph (CUDA events
    around its replay): the calls' own host-side cost does not leave the device idle between them."""
    g = graph_of(torch, lambda: [fn() for _ in range(reps)])
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) / reps


def run_decode(torch, sa, synth, dist, args, peaks, world):
    """One decode step of the 36-layer stack, B=64, 32768 cached tokens, in one CUDA graph: one
    fused launch per layer (the headline decode figure), and the two-call path on the same caches."""
    dev = torch.device("cuda")
    B, p = DECODE_B, DECODE_CTX
    layers = decode_layers(torch, sa, synth, dev, B, p)
    pos = torch.full((B,), p, dtype=torch.int32, device=dev)
    ws = torch.empty(max(sa.spark_decode_workspace_bytes(B, L["cap"], L["cfg"]) for L in layers),
                     dtype=torch.uint8, device=dev)
    wsf = torch.zeros(max(sa.spark_decode_fused_workspace_bytes(B, L["cap"], L["cfg"]) for L in layers),
                      dtype=torch.uint8, device=dev)
    dsteps = max(5, min(args.steps, 30))
    res = {}
    for name, step in (("two_call", lambda: decode_step(sa, layers, pos, ws)),
                       ("fused", lambda: decode_fused_step(sa, layers, pos, wsf))):
        graph = graph_of(torch, step)
        sa.spark_check()
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize()
        res[name] = timed_region(torch, dist, lambda i: graph.replay(), dsteps) / dsteps
        sa.spark_check()
        del graph
    ms_step = res["fused"]
    # one layer of each kind alone (ten calls in one CUDA graph) for the rooflines
    per_kind = {}
    for name, L in (("sliding", layers[0]), ("full", layers[3])):
        k_ms = event_ms(torch, lambda: sa.spark_attn_decode_fused(
            L["out"], L["q"], L["kn"], L["vn"], L["g"], L["kc"], L["vc"], pos, L["cfg"], wsf,
            flags=sa.SPARK_ROPE_FUSED))
        nbytes = decode_kv_bytes(B, p, L["kind"])
        per_kind[name] = {"kernel_us": k_ms * 1e3, "kv_bytes": nbytes,
                          "roofline": hbm_roofline(f"decode_fused_kernel ({name} layer)", nbytes / (k_ms * 1e-3) / 1e9,
                                                   peaks, ncu_traffic(f"decode_fused_kernel_{name}"))}
    sa.spark_check()
    total_bytes = sum(decode_kv_bytes(B, p, L["kind"]) for L in layers)
    launches = decode_launches(sa, B, layers)
    del layers, ws, wsf
    torch.cuda.empty_cache()
    return {
        "value": total_bytes * world / (ms_step * 1e-3) / 1e9, "unit": "GB/s",
        "ms_per_step": ms_step, "steps_per_s": 1e3 / ms_step, "kv_bytes_per_step": total_bytes,
        "workload": f"decode_b{B}_ctx{p}_36layers", "gpu_launches_per_step": N_LAYERS,
        "two_call": {"ms_per_step": res["two_call"], "gpu_launches_per_step": launches,
                     "value": total_bytes * world / (res["two_call"] * 1e-3) / 1e9},
        "per_layer_kind": per_kind,
        "roofline": per_kind["full"]["roofline"],
    }


def decode_append_layers(torch, sa, synth, dev, B: int, p: int, layer_ids=range(N_LAYERS),
                         seed: int = DECODE_SEED, q8: bool = False, page: int = 0, chunk: int = 2048):
    """Caches holding positions 0..p-1 written through the library's own append (the generator's
    tokens, keys taken as rotated) and the new token's q/k/v/gate at p, per layer.  q8: 8-bit
    caches; page > 0: paged pools of `page`-row pages, each sequence's pages in shuffled order."""
    import numpy as np
    layers = []
    rng = np.random.default_rng(11)
    for l in layer_ids:
        kind = FULL if l % 4 == 3 else SLIDING
        cfg = sa.spark_layer_cfg_for_kind(kind)
        cap = WINDOW if kind == SLIDING else p + 1
        dt = torch.uint8 if q8 else torch.bfloat16
        L = dict(layer=l, kind=kind, cfg=cfg, cap=cap, q8=q8, page=page)
        if page:
            max_pages = -(-cap // page)
            n_pages = B * max_pages
            L["table"] = torch.from_numpy(rng.permutation(n_pages).reshape(B, max_pages).astype(np.int32)).to(dev)
            shape, sshape = (n_pages, HKV, page, D), (n_pages, HKV, page, D // 32)
        else:
            shape, sshape = (B, HKV, cap, D), (B, HKV, cap, D // 32)
        L["kc"] = torch.empty(shape, dtype=dt, device=dev)
        L["vc"] = torch.empty_like(L["kc"])
        if q8:
            L["ks"] = torch.empty(sshape, dtype=torch.float16, device=dev)
            L["vs"] = torch.empty_like(L["ks"])
        if page:
            L["kv"] = sa.paged_kv(L["kc"], L["vc"], L["table"], L.get("ks"), L.get("vs"))
        first = 0 if kind == FULL else max(0, p - WINDOW)
        for c0 in range(first, p, chunk):
            n = min(chunk, p - c0)
            kt = torch.empty(B, n, HKV, D, dtype=torch.bfloat16, device=dev)
            vt = torch.empty_like(kt)
            synth.fill_tokens(kt, seed, synth.tensor_id(l, synth.ROLE_K), c0)
            synth.fill_tokens(vt, seed, synth.tensor_id(l, synth.ROLE_V), c0)
            append_layer(sa, L, kt, vt, torch.full((B,), c0, dtype=torch.int32, device=dev), 0)
            del kt, vt
        q = torch.empty(B, 1, HQ, D, dtype=torch.bfloat16, device=dev)
        kn = torch.empty(B, 1, HKV, D, dtype=torch.bfloat16, device=dev)
        vn = torch.empty_like(kn)
        g = torch.empty(B, 1, HQ, dtype=torch.bfloat16, device=dev)
        synth.fill_tokens(q, seed, synth.tensor_id(l, synth.ROLE_Q), p)
        synth.fill_tokens(kn, seed, synth.tensor_id(l, synth.ROLE_K), p)
        synth.fill_tokens(vn, seed, synth.tensor_id(l, synth.ROLE_V), p)
        synth.fill_tokens(g, seed, synth.tensor_id(l, synth.ROLE_GATE), p)
        L.update(q=q.view(B, HQ, D), kn=kn, vn=vn, g=g.view(B, HQ),
                 out=torch.empty(B, HQ, D, dtype=torch.bfloat16, device=dev))
        layers.append(L)
    sa.spark_check()
    return layers


def decode_q8_layers(torch, sa, synth, dev, B: int, p: int, layer_ids=range(N_LAYERS), seed: int = DECODE_SEED):
    """8-bit dense caches for the decode step (see decode_append_layers)."""
    return decode_append_layers(torch, sa, synth, dev, B, p, layer_ids, seed, q8=True)


def append_layer(sa, L, k, v, pos, flags):
    if L["page"]:
        sa.spark_kv_append_paged(L["kv"], k, v, pos, L["cfg"], flags=flags)
    elif L["q8"]:
        sa.spark_kv_append_q8(L["kc"], L["ks"], L["vc"], L["vs"], k, v, pos, L["cfg"], flags=flags)
    else:
        sa.spark_kv_append(L["kc"], L["vc"], k, v, pos, L["cfg"], flags=flags)


def attend_layer(sa, L, pos, ws):
    f = sa.SPARK_ROPE_FUSED
    if L["page"]:
        sa.spark_attn_decode_paged(L["out"], L["q"], L["g"], L["kv"], pos, L["cfg"], ws, flags=f)
    elif L["q8"]:
        sa.spark_attn_decode_q8(L["out"], L["q"], L["g"], L["kc"], L["ks"], L["vc"], L["vs"], pos, L["cfg"], ws,
                                flags=f)
    else:
        sa.spark_attn_decode(L["out"], L["q"], L["g"], L["kc"], L["vc"], pos, L["cfg"], ws, flags=f)


def layer_ws_bytes(sa, B, L):
    if L["page"]:
        return sa.spark_decode_paged_workspace_bytes(B, L["kv"], L["cfg"])
    if L["q8"]:
        return sa.spark_decode_q8_workspace_bytes(B, L["cap"], L["cfg"])
    return sa.spark_decode_workspace_bytes(B, L["cap"], L["cfg"])


def decode_q8_step(sa, layers, pos, ws):
    """One decode step over caches built by decode_append_layers: per layer, append the new token
    (RoPE fused on k, quantised if the cache is 8-bit), then attend (RoPE fused on q)."""
    for L in layers:
        append_layer(sa, L, L["kn"], L["vn"], pos, sa.SPARK_ROPE_FUSED)
        attend_layer(sa, L, pos, ws)


def run_decode_variant(torch, sa, synth, dist, args, peaks, world, q8: bool, page: int):
    """The decode step of run_decode (36 layers, B=64, 32768 cached tokens, one CUDA graph) over
    an 8-bit cache (q8) and/or paged pools (page > 0)."""
    dev = torch.device("cuda")
    B, p = DECODE_B, DECODE_CTX
    layers = decode_append_layers(torch, sa, synth, dev, B, p, q8=q8, page=page)
    pos = torch.full((B,), p, dtype=torch.int32, device=dev)
    ws = torch.empty(max(layer_ws_bytes(sa, B, L) for L in layers), dtype=torch.uint8, device=dev)
    decode_q8_step(sa, layers, pos, ws)
    torch.cuda.synchronize()
    sa.spark_check()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        decode_q8_step(sa, layers, pos, ws)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    dsteps = max(5, min(args.steps, 30))
    ms_step = timed_region(torch, dist, lambda i: graph.replay(), dsteps) / dsteps
    sa.spark_check()
    full = layers[3]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 10
    e0.record()
    for _ in range(reps):
        attend_layer(sa, full, pos, ws)
    e1.record()
    torch.cuda.synchronize()
    k_ms = e0.elapsed_time(e1) / reps
    per_key = decode_q8_kv_bytes if q8 else decode_kv_bytes
    total_bytes = sum(per_key(B, p, L["kind"]) for L in layers)
    full_bytes = per_key(B, p, FULL)
    launches = sum(2 + (1 if layer_ws_bytes(sa, B, L) // (B * HQ * (D + 2) * 4) > 1 else 0) for L in layers)
    del graph, layers, ws
    torch.cuda.empty_cache()
    name = ("decode_q8" if q8 else "decode") + (f"_paged{page}" if page else "")
    kern = ("decode_q8_partial_kernel" if q8 else "decode_partial_kernel") + ("<paged>" if page else "")
    return {
        "value": total_bytes * world / (ms_step * 1e-3) / 1e9, "unit": "GB/s",
        "ms_per_step": ms_step, "steps_per_s": 1e3 / ms_step, "kv_bytes_per_step": total_bytes,
        "workload": f"{name}_b{B}_ctx{p}_36layers", "gpu_launches_per_step": launches,
        "roofline": hbm_roofline(f"{kern}+combine (full layer)", full_bytes / (k_ms * 1e-3) / 1e9, peaks,
                                 None if page else ncu_traffic("decode_q8_partial_kernel_full" if q8 else
                                                               "decode_partial_kernel_full")),
    }


def run_decode_q8(torch, sa, synth, dist, args, peaks, world):
    return run_decode_variant(torch, sa, synth, dist, args, peaks, world, q8=True, page=0)


RAGGED_B, RAGGED_SEED, RAGGED_PAGE = 16, 6, 256


def ragged_workload():
    """The serving mix: 16 sequences with seeded chunk lengths in [256, 4096] and history lengths in
    [0, 16384] (positions before the chunk, already in a paged pool of 256-row pages)."""
    import numpy as np
    rng = np.random.default_rng(RAGGED_SEED)
    lens = rng.integers(256, 4097, RAGGED_B).tolist()
    hist = rng.integers(0, 16385, RAGGED_B).tolist()
    return lens, hist


def run_prefill_ragged(torch, sa, synth, dist, args, peaks, world):
    """One sliding and one full layer over the ragged batch: RoPE on the packed k, the prefill with
    paged history (RoPE on q fused at load), the append of the chunk into the pages."""
    import numpy as np
    dev = torch.device("cuda")
    lens, hist = ragged_workload()
    B, P = RAGGED_B, RAGGED_PAGE
    total = sum(lens)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=dev)
    hcu = torch.tensor(np.concatenate([[0], np.cumsum(hist)]), dtype=torch.int32, device=dev)
    pos0 = torch.tensor(hist, dtype=torch.int32, device=dev)
    zeros = torch.zeros(B, dtype=torch.int32, device=dev)
    max_len = max(lens)
    L = {}
    rng = np.random.default_rng(RAGGED_SEED + 1)
    for kind, layer in ((SLIDING, 0), (FULL, 3)):
        cfg = sa.spark_layer_cfg_for_kind(kind)
        max_pages = WINDOW // P if kind == SLIDING else -(-max(h + n for h, n in zip(hist, lens)) // P)
        n_pages = B * max_pages
        table = torch.from_numpy(rng.permutation(n_pages).reshape(B, max_pages).astype(np.int32)).to(dev)
        kp = torch.zeros(n_pages, HKV, P, D, dtype=torch.bfloat16, device=dev)
        vp = torch.zeros_like(kp)
        kv = sa.paged_kv(kp, vp, table)
        # history: each sequence's positions 0..hist-1, generated per sequence and appended raw (RoPE fused)
        hk = torch.empty(sum(hist), HKV, D, dtype=torch.bfloat16, device=dev)
        hv = torch.empty_like(hk)
        for b in range(B):
            if hist[b]:
                sl = slice(int(hcu[b]), int(hcu[b + 1]))
                synth.fill_tokens(hk[sl].view(1, hist[b], HKV, D), RAGGED_SEED, synth.tensor_id(layer, synth.ROLE_K) + 16 * b, 0)
                synth.fill_tokens(hv[sl].view(1, hist[b], HKV, D), RAGGED_SEED, synth.tensor_id(layer, synth.ROLE_V) + 16 * b, 0)
        sa.spark_kv_append_varlen(kv, hk, hv, hcu, max(hist), zeros, cfg, flags=sa.SPARK_ROPE_FUSED)
        del hk, hv
        q = torch.empty(total, HQ, D, dtype=torch.bfloat16, device=dev)
        k = torch.empty(total, HKV, D, dtype=torch.bfloat16, device=dev)
        v = torch.empty_like(k)
        g = torch.empty(total, HQ, dtype=torch.bfloat16, device=dev)
        for b in range(B):
            sl = slice(int(cu[b]), int(cu[b + 1]))
            for t_, role, H in ((q, synth.ROLE_Q, HQ), (k, synth.ROLE_K, HKV), (v, synth.ROLE_V, HKV)):
                synth.fill_tokens(t_[sl].view(1, lens[b], H, D), RAGGED_SEED, synth.tensor_id(layer, role) + 16 * b,
                                  hist[b])
            synth.fill_tokens(g[sl].view(1, lens[b], HQ), RAGGED_SEED, synth.tensor_id(layer, synth.ROLE_GATE) + 16 * b,
                              hist[b])
        L[kind] = dict(cfg=cfg, kv=kv, q=q, k=k, v=v, g=g, out=torch.empty_like(q), keep=(kp, vp, table))
    sa.spark_check()

    def step(i=0):
        for kind in (SLIDING, FULL):
            w = L[kind]
            sa.spark_rope_apply_varlen(w["k"], cu, max_len, pos0, w["cfg"])
            sa.spark_attn_prefill_varlen(w["out"], w["q"], w["k"], w["v"], w["g"], cu, max_len, pos0, w["kv"],
                                         w["cfg"], flags=sa.SPARK_ROPE_FUSED)
            sa.spark_kv_append_varlen(w["kv"], w["k"], w["v"], cu, max_len, pos0, w["cfg"])

    for _ in range(max(3, min(args.warmup, 5))):
        step()
    sa.spark_check()
    steps = max(3, min(args.steps, 20))
    ms = timed_region(torch, dist, step, steps) / steps
    sa.spark_check()
    flops = sum(prefill_flops(1, n, h, kind, True) for kind in (SLIDING, FULL) for n, h in zip(lens, hist))
    f_full = sum(prefill_flops(1, n, h, FULL, True) for n, h in zip(lens, hist))
    # the full layer's prefill alone, for its roofline
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w = L[FULL]
    e0.record()
    for _ in range(5):
        sa.spark_attn_prefill_varlen(w["out"], w["q"], w["k"], w["v"], w["g"], cu, max_len, pos0, w["kv"], w["cfg"],
                                     flags=sa.SPARK_ROPE_FUSED)
    e1.record()
    torch.cuda.synchronize()
    k_ms = e0.elapsed_time(e1) / 5
    del L
    torch.cuda.empty_cache()
    return {"workload": f"prefill_ragged_b{B}_len256-4096_hist0-16384_page{P}_sliding+full",
            "lens": lens, "history": hist, "value": total * world / (ms * 1e-3), "unit": "tok/s",
            "ms_per_step": ms, "tflops": flops * world / (ms * 1e-3) / 1e12, "gpu_launches_per_step": 6,
            "full_layer_kernel": {"ms": k_ms, "tflops": f_full / (k_ms * 1e-3) / 1e12,
                                  "frac": f_full / (k_ms * 1e-3) / 1e12 / peaks["bf16_tflops"]}}


def run_long_prefill(torch, sa, synth, dist, args, peaks, world):
    """B=1, T=131072 in 16 chunks of 8192 over the growing cache, one full and one sliding layer."""
    dev = torch.device("cuda")
    T, C, seed = 131072, 8192, 4
    L = {}
    for kind, layer in ((SLIDING, 0), (FULL, 3)):
        cfg = sa.spark_layer_cfg_for_kind(kind)
        q = torch.empty(1, T, HQ, D, dtype=torch.bfloat16, device=dev)
        k = torch.empty(1, T, HKV, D, dtype=torch.bfloat16, device=dev)
        v = torch.empty_like(k)
        g = torch.empty(1, T, HQ, dtype=torch.bfloat16, device=dev)
        synth.fill_tokens(q, seed, synth.tensor_id(layer, synth.ROLE_Q), 0)
        synth.fill_tokens(k, seed, synth.tensor_id(layer, synth.ROLE_K), 0)
        synth.fill_tokens(v, seed, synth.tensor_id(layer, synth.ROLE_V), 0)
        synth.fill_tokens(g, seed, synth.tensor_id(layer, synth.ROLE_GATE), 0)
        cap = WINDOW if kind == SLIDING else T
        kc = torch.empty(1, HKV, cap, D, dtype=torch.bfloat16, device=dev)
        L[kind] = dict(cfg=cfg, q=q, k=k, v=v, g=g, out=torch.empty_like(q), kc=kc, vc=torch.empty_like(kc))
    pos = [torch.full((1,), c * C, dtype=torch.int32, device=dev) for c in range(T // C)]

    def step(i=0):
        for kind in (SLIDING, FULL):
            w = L[kind]
            for c in range(T // C):
                sl = slice(c * C, (c + 1) * C)
                q, k = w["q"][:, sl], w["k"][:, sl]
                sa.spark_rope_apply(k, pos[c], w["cfg"])
                sa.spark_attn_prefill(w["out"][:, sl], q, k, w["v"][:, sl], w["g"][:, sl],
                                      w["kc"] if c else None, w["vc"] if c else None, pos[c], w["cfg"],
                                      flags=sa.SPARK_ROPE_FUSED)
                sa.spark_kv_append(w["kc"], w["vc"], k, w["v"][:, sl], pos[c], w["cfg"])

    # the same chunks over 8-bit caches: a chunk with history reads it through spark_attn_prefill_q8
    # (the history dequantised into a workspace, then the bf16 prefill) and appends itself quantised
    for kind in (SLIDING, FULL):
        w = L[kind]
        cap = w["kc"].shape[2]
        w["kq"] = torch.empty(1, HKV, cap, D, dtype=torch.uint8, device=dev)
        w["vq"] = torch.empty_like(w["kq"])
        w["ks"] = torch.empty(1, HKV, cap, D // 32, dtype=torch.float16, device=dev)
        w["vs"] = torch.empty_like(w["ks"])
        w["ws"] = torch.empty(sa.spark_prefill_q8_workspace_bytes(1, cap, w["cfg"]), dtype=torch.uint8, device=dev)

    def step_q8(i=0):
        for kind in (SLIDING, FULL):
            w = L[kind]
            for c in range(T // C):
                sl = slice(c * C, (c + 1) * C)
                q, k, v, g = w["q"][:, sl], w["k"][:, sl], w["v"][:, sl], w["g"][:, sl]
                sa.spark_rope_apply(k, pos[c], w["cfg"])
                if c == 0:
                    sa.spark_attn_prefill(w["out"][:, sl], q, k, v, g, None, None, pos[c], w["cfg"],
                                          flags=sa.SPARK_ROPE_FUSED)
                    sa.spark_kv_append_q8(w["kq"], w["ks"], w["vq"], w["vs"], k, v, pos[c], w["cfg"])
                else:
                    sa.spark_attn_prefill_q8(w["out"][:, sl], q, k, v, g, w["kq"], w["ks"], w["vq"], w["vs"], pos[c],
                                             w["cfg"], w["ws"], flags=sa.SPARK_ROPE_FUSED | sa.SPARK_APPEND_FUSED)

    for _ in range(max(1, min(args.warmup, 3))):
        step()
    sa.spark_check()
    steps = max(2, min(args.steps, 5))
    ms = timed_region(torch, dist, step, steps) / steps
    sa.spark_check()
    for _ in range(max(1, min(args.warmup, 3))):
        step_q8()
    sa.spark_check()
    ms_q8 = timed_region(torch, dist, step_q8, steps) / steps
    sa.spark_check()
    f_full = sum(prefill_flops(1, C, c * C, FULL, True) for c in range(T // C))
    f_slide = sum(prefill_flops(1, C, c * C, SLIDING, True) for c in range(T // C))
    del L
    torch.cuda.empty_cache()
    n_ch = T // C
    return {"workload": "long_prefill_b1_t131072_chunks8192_sliding+full", "value": T * world / (ms * 1e-3),
            "unit": "tok/s", "ms_per_step": ms, "tflops": (f_full + f_slide) * world / (ms * 1e-3) / 1e12,
            "gpu_launches_per_step": 2 * n_ch * 3,
            "q8_cache": {"value": T * world / (ms_q8 * 1e-3), "unit": "tok/s", "ms_per_step": ms_q8,
                         "gpu_launches_per_step": 2 * (3 + (n_ch - 1) * 4),
                         "note": "history in 8-bit q8_0 caches, dequantised per chunk into a bf16 workspace"}}


def run_long_decode(torch, sa, synth, dist, args, peaks, world):
    """One 36-layer decode step at long context: B=1 at 2^20 and B=16 at 131072 (positions at the end)."""
    dev = torch.device("cuda")
    out = {}
    for B, ctx in ((1, 1 << 20), (16, 131072)):
        p = ctx - 1
        layers = decode_layers(torch, sa, synth, dev, B, p, seed=5)
        pos = torch.full((B,), p, dtype=torch.int32, device=dev)
        ws = torch.empty(max(sa.spark_decode_workspace_bytes(B, L["cap"], L["cfg"]) for L in layers),
                         dtype=torch.uint8, device=dev)
        wsf = torch.zeros(max(sa.spark_decode_fused_workspace_bytes(B, L["cap"], L["cfg"]) for L in layers),
                          dtype=torch.uint8, device=dev)
        steps = max(5, min(args.steps, 20))
        ms = {}
        for name, step in (("two_call", lambda: decode_step(sa, layers, pos, ws)),
                           ("fused", lambda: decode_fused_step(sa, layers, pos, wsf))):
            graph = graph_of(torch, step)
            for _ in range(3):
                graph.replay()
            ms[name] = timed_region(torch, dist, lambda i: graph.replay(), steps) / steps
            sa.spark_check()
            del graph
        total = sum(decode_kv_bytes(B, p, L["kind"]) for L in layers)
        m = ms["fused"]
        out[f"b{B}_ctx{ctx}"] = {"value": total * world / (m * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": m,
                                 "steps_per_s": 1e3 / m, "kv_bytes_per_step": total,
                                 "frac_of_hbm": total / (m * 1e-3) / 1e9 / (peaks.get("hbm_read_gbs") or
                                                                            peaks["hbm_gbs"]),
                                 "two_call_ms_per_step": ms["two_call"], "gpu_launches_per_step": N_LAYERS}
        del layers, ws, wsf
        torch.cuda.empty_cache()
    return out


def run_cp_decode(torch, sa, synth, dist, args, peaks, world):
    """Context-parallel decode, B=1 at 2^20: each full layer's cache split by position over the
    ranks (append to the owning shard, each rank's record, one all-gather, the merge); the sliding
    layers replicated on every rank.  The same sequence for every N (strong scaling).  Eager
    launches: between ranks the exchange is an NCCL all-gather."""
    from full_gqa_attention_spark2_b200.context_parallel import FullLayerShard
    dev = torch.device("cuda")
    B, ctx = 1, 1 << 20
    p = ctx - 1
    seed = 5
    layers = []
    for l in range(N_LAYERS):
        kind = FULL if l % 4 == 3 else SLIDING
        cfg = sa.spark_layer_cfg_for_kind(kind)
        toks = {}
        for name, role, H in (("q", synth.ROLE_Q, HQ), ("kn", synth.ROLE_K, HKV), ("vn", synth.ROLE_V, HKV),
                              ("g", synth.ROLE_GATE, HQ)):
            t = torch.empty(B, 1, H, *(() if name == "g" else (D,)), dtype=torch.bfloat16, device=dev)
            synth.fill_tokens(t, seed, synth.tensor_id(l, role), p)
            toks[name] = t
        L = dict(kind=kind, cfg=cfg, q=toks["q"].view(B, HQ, D), kn=toks["kn"], vn=toks["vn"],
                 g=toks["g"].view(B, HQ), out=torch.empty(B, HQ, D, dtype=torch.bfloat16, device=dev))
        if kind == FULL:
            L["shard"] = FullLayerShard(B, ctx, cfg, device=dev)
        else:
            kc = torch.empty(B, HKV, WINDOW, D, dtype=torch.bfloat16, device=dev)
            vc = torch.empty_like(kc)
            synth.fill_cache(kc, seed, synth.tensor_id(l, synth.ROLE_K), p, True)
            synth.fill_cache(vc, seed, synth.tensor_id(l, synth.ROLE_V), p, True)
            L.update(kc=kc, vc=vc)
        layers.append(L)
    pos = torch.full((B,), p, dtype=torch.int32, device=dev)
    cfg_s = sa.spark_layer_cfg_for_kind(SLIDING)
    ws = torch.empty(sa.spark_decode_workspace_bytes(B, WINDOW, cfg_s), dtype=torch.uint8, device=dev)
    fused = sa.SPARK_ROPE_FUSED

    def step(i=0):
        for L in layers:
            if L["kind"] == FULL:
                L["shard"].append(L["kn"].view(B, HKV, D), L["vn"].view(B, HKV, D), pos, flags=fused)
                L["shard"].attend(L["out"], L["q"], L["g"], pos, flags=fused)
            else:
                sa.spark_kv_append(L["kc"], L["vc"], L["kn"], L["vn"], pos, L["cfg"], flags=fused)
                sa.spark_attn_decode(L["out"], L["q"], L["g"], L["kc"], L["vc"], pos, L["cfg"], ws, flags=fused)

    for _ in range(3):
        step()
    sa.spark_check()
    steps = max(5, min(args.steps, 20))
    ms = timed_region(torch, dist, step, steps) / steps
    sa.spark_check()
    total = sum(decode_kv_bytes(B, p, L["kind"]) for L in layers)
    res = {"b1_ctx1048576": {"value": total / (ms * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": ms,
                             "steps_per_s": 1e3 / ms, "kv_bytes_per_step": total, "ranks": world,
                             "scaling": "strong", "record_bytes_per_rank": sa.spark_decode_cp_record_bytes(B),
                             "frac_of_hbm_x_ranks": total / (ms * 1e-3) / 1e9 / ((peaks.get("hbm_read_gbs") or
                                                                                     peaks["hbm_gbs"]) * world)}}
    del layers, ws
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------- oracle timing -------

class OracleSampler:
    """The fp64 oracle on the headline workload, one bounded sample at a time: `rows` random query
    rows of sequence 0 (all 16 heads) through both layers, against all of that sequence's keys."""

    def __init__(self, rows_per_sample: int = 4, seed: int = 0):
        import synth
        from oracle import spark_oracle as O
        self.O, self.synth = O, synth
        self.R = rows_per_sample
        self.pos = np.arange(PREFILL_T)
        self.layer_of = {SLIDING: 0, FULL: 3}
        self.kv = {kind: (self._get(kind, synth.ROLE_K, HKV, D, self.pos, 0.5),
                          self._get(kind, synth.ROLE_V, HKV, D, self.pos)) for kind in self.layer_of}
        self.rng = np.random.default_rng(seed)

    def _get(self, kind, role, H, Dd, p, sig=1.0):
        s = self.synth
        return s.bf16_bits_to_f64(s.token_tensor(PREFILL_SEED, s.tensor_id(self.layer_of[kind], role), 1, H, Dd, p,
                                                 sig)[0])

    def sample(self) -> float:
        """Runs one sample; returns the seconds the oracle took (input regeneration excluded)."""
        rows = np.sort(self.rng.integers(0, PREFILL_T, size=self.R))
        t_used = 0.0
        for kind in (SLIDING, FULL):
            q_rows = self._get(kind, self.synth.ROLE_Q, HQ, D, rows)
            g_rows = self._get(kind, self.synth.ROLE_GATE, HQ, 1, rows, 2.0)
            t0 = time.perf_counter()
            self.O.layer_prefill_rows(q_rows, self.kv[kind][0], self.kv[kind][1], g_rows, self.pos, kind, rows)
            t_used += time.perf_counter() - t0
        return t_used


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        return os.cpu_count()


def oracle_prefill_rate(budget_s: float = 15.0):
    """The oracle's rate (query rows per second through both layers) over samples run until about
    budget_s seconds of oracle time; returns (tok/s, threads, description)."""
    sampler = OracleSampler()
    done, t_used = 0, 0.0
    while t_used < budget_s or done < 2 * sampler.R:
        t_used += sampler.sample()
        done += sampler.R
    return done / t_used, oracle_threads(), \
        f"{done} random query rows of sequence 0 through both layers (all 16 heads, all 8192 keys), {t_used:.1f} s"


def main_config(world: int) -> dict:
    """The headline line's config (both arms)."""
    return {"workload": "prefill_b4_t8192_sliding+full", "B": PREFILL_B, "T": PREFILL_T,
            "layers": ["sliding (window 512, rope theta 1e4, 256 dims)", "full (rope theta 5e6, first 64 dims)"],
            "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (q alone is 268 MB per layer); no flush",
            "regime": "burst: K steps replayed from a CUDA graph, ahead of the power cap; an eager pass of K "
                      "steps before it gives the kernel times (the full-layer kernel's first and last ten steps "
                      "are reported); the 36-layer leg runs under the cap"}


def run_reference(args, rank):
    """The oracle arm: W untimed and K timed steps, each step one bounded sample of the headline
    workload (4 random query rows of sequence 0 through both layers, fp64, all host threads).  The
    line reports what was measured: rows per second and the measured seconds per sampled step."""
    if rank != 0:
        return
    sampler = OracleSampler(rows_per_sample=4)
    for _ in range(args.warmup):
        sampler.sample()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        sampler.sample()
    wall = time.perf_counter() - t0
    rows = args.steps * sampler.R
    rate = rows / wall
    threads = oracle_threads()
    sample = (f"{args.steps} timed steps of {sampler.R} random query rows of sequence 0 through both layers "
              f"(all 16 heads, all 8192 keys), {wall:.1f} s measured; {args.warmup} untimed steps before")
    line = {
        "impl": "reference", "metric": "prefill attn tok/s & TFLOP/s; decode KV-read GB/s (36-layer stack); % roofline",
        "value": rate, "unit": "tok/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": wall / args.steps * 1e3, "tokens_per_step": sampler.R, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded counter generator)",
        "config": main_config(args.gpus),
        "cpu_baseline": {"value": rate, "unit": "tok/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": rate, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- main -----

def run_profile_case(torch, sa, synth, which: str):
    """A small case for ncu: one warm-up and two launches of one kernel, nothing timed.

    prefill_full / prefill_sliding: B=4, T=8192 (q alone 268 MB > L2);
    decode_full: B=16, 32768 cached tokens, one full layer (2.1 GB of KV)."""
    dev = torch.device("cuda")
    if which in ("prefill_full", "prefill_sliding"):
        kind = FULL if which == "prefill_full" else SLIDING
        W, pos0 = prefill_workload(torch, sa, synth, dev)
        w = W[kind]
        sa.spark_rope_apply(w["k"], pos0, w["cfg"])
        for _ in range(3):            # as in prefill_step: q raw, rotated at load
            sa.spark_attn_prefill(w["out"], w["q"], w["k"], w["v"], w["g"], None, None, pos0, w["cfg"],
                                  flags=sa.SPARK_ROPE_FUSED)
    elif which == "decode_full":
        B, p = 16, DECODE_CTX
        cfg = sa.spark_layer_cfg_for_kind(FULL)
        kc = torch.empty(B, HKV, p + 1, D, dtype=torch.bfloat16, device=dev)
        vc = torch.empty_like(kc)
        synth.fill_cache(kc, DECODE_SEED, synth.tensor_id(3, synth.ROLE_K), p + 1, False)
        synth.fill_cache(vc, DECODE_SEED, synth.tensor_id(3, synth.ROLE_V), p + 1, False)
        q = torch.empty(B, 1, HQ, D, dtype=torch.bfloat16, device=dev)
        g = torch.empty(B, 1, HQ, dtype=torch.bfloat16, device=dev)
        synth.fill_tokens(q, DECODE_SEED, synth.tensor_id(3, synth.ROLE_Q), p)
        synth.fill_tokens(g, DECODE_SEED, synth.tensor_id(3, synth.ROLE_GATE), p)
        out = torch.empty(B, HQ, D, dtype=torch.bfloat16, device=dev)
        pos = torch.full((B,), p, dtype=torch.int32, device=dev)
        ws = torch.empty(sa.spark_decode_workspace_bytes(B, p + 1, cfg), dtype=torch.uint8, device=dev)
        for _ in range(3):
            sa.spark_attn_decode(out, q.view(B, HQ, D), g.view(B, HQ), kc, vc, pos, cfg, ws, flags=sa.SPARK_ROPE_FUSED)
    elif which in ("decode_fused_full", "decode_fused_sliding"):
        # one layer of the fused decode: full, B=16 at 32768 (2.1 GB of KV); sliding, B=128 (268 MB > L2)
        full = which == "decode_fused_full"
        B, p = (16, DECODE_CTX) if full else (128, DECODE_CTX)
        L = decode_layers(torch, sa, synth, dev, B, p, (3,) if full else (0,))[0]
        pos = torch.full((B,), p, dtype=torch.int32, device=dev)
        wsf = torch.zeros(sa.spark_decode_fused_workspace_bytes(B, L["cap"], L["cfg"]), dtype=torch.uint8, device=dev)
        for _ in range(3):
            sa.spark_attn_decode_fused(L["out"], L["q"], L["kn"], L["vn"], L["g"], L["kc"], L["vc"], pos, L["cfg"], wsf,
                                       flags=sa.SPARK_ROPE_FUSED)
    elif which == "prefill_ragged_full":
        # run_prefill_ragged at its smallest: the second prefill2_kernel launch is the full layer's
        import types
        run_prefill_ragged(torch, sa, synth, None, types.SimpleNamespace(steps=1, warmup=0), load_peaks(), 1)
    elif which == "decode_q8_full":
        B, p = 16, DECODE_CTX
        L = decode_q8_layers(torch, sa, synth, dev, B, p, layer_ids=(3,))[0]
        pos = torch.full((B,), p, dtype=torch.int32, device=dev)
        ws = torch.empty(sa.spark_decode_q8_workspace_bytes(B, L["cap"], L["cfg"]), dtype=torch.uint8, device=dev)
        for _ in range(3):
            sa.spark_attn_decode_q8(L["out"], L["q"], L["g"], L["kc"], L["ks"], L["vc"], L["vs"], pos, L["cfg"], ws,
                                    flags=sa.SPARK_ROPE_FUSED)
    else:
        raise SystemExit(f"unknown profile case {which}")
    sa.spark_check()
    print(json.dumps({"profile_case": which, "ok": True}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    # 20 steps: the headline's timed region (~41 ms) stays ahead of the power cap, which a continuous
    # tensor-core load reaches after ~40 ms (the denominator is the burst bf16 figure); the 36-layer
    # prefill leg reports the capped regime
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-long", action="store_true", help="skip the long-context prefill and decode workloads")
    ap.add_argument("--cp-decode", action="store_true",
                    help="also run context-parallel decode (B=1 at 2^20, full-layer caches split over the ranks)")
    ap.add_argument("--profile", choices=["prefill_full", "prefill_sliding", "decode_full", "decode_q8_full",
                                          "prefill_ragged_full", "decode_fused_full", "decode_fused_sliding"],
                    default=None,
                    help="run a small case of one kernel for ncu and exit")
    args = ap.parse_args()
    rank, world, local = dist_env()
    if args.impl == "reference":
        run_reference(args, rank)
        return

    import torch
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        torch.cuda.set_device(local)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    else:
        torch.cuda.set_device(0)
    import full_gqa_attention_spark2_b200 as sa
    import synth
    sa._lib()
    synth.load_lib()
    peaks = load_peaks()
    if args.profile:
        run_profile_case(torch, sa, synth, args.profile)
        return

    res = run_prefill(torch, sa, synth, dist, args, peaks, world)
    tiny = run_prefill_tiny(torch, sa, synth, dist, args, peaks, world)
    stack36 = run_prefill_stack36(torch, sa, synth, dist, args, peaks, world)
    if not args.no_decode:
        peaks["hbm_read_gbs"] = synth.read_probe_gbs()
    dec = None if args.no_decode else run_decode(torch, sa, synth, dist, args, peaks, world)
    dec_q8 = None if args.no_decode else run_decode_q8(torch, sa, synth, dist, args, peaks, world)
    dec_paged = None if args.no_decode else run_decode_variant(torch, sa, synth, dist, args, peaks, world,
                                                               q8=False, page=256)
    ragged = run_prefill_ragged(torch, sa, synth, dist, args, peaks, world)
    long_pf = None if args.no_long else run_long_prefill(torch, sa, synth, dist, args, peaks, world)
    long_dec = None if (args.no_long or args.no_decode) else run_long_decode(torch, sa, synth, dist, args, peaks, world)
    cp_dec = run_cp_decode(torch, sa, synth, dist, args, peaks, world) if args.cp_decode else None
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, threads, sample = oracle_prefill_rate()
        cpu = {"value": rate, "unit": "tok/s", "cores": threads, "kind": "oracle", "sample": sample}
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": res["metric"], "value": res["value"], "unit": res["unit"], "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded counter generator, shapes of the pages' workloads)",
        "config": main_config(world),
        "tflops": res["tflops"], "eager": res["eager"], "prefill_full_kernel": res["prefill_full_kernel"],
        "per_layer_kind": res["per_layer_kind"], "stack36_derived": res["stack36_derived"],
        "prefill_stack36": stack36,
        "roofline": res["roofline"], "e2e": res["e2e"], "clocks": res["clocks"],
        "gpu_launches": res["gpu_launches"] + (0 if dec is None else 0),
        "cpu_baseline": cpu, "prefill_tiny": tiny, "hbm_read_gbs": peaks.get("hbm_read_gbs"),
        "prefill_ragged": ragged, "decode": dec, "decode_q8": dec_q8,
        "decode_paged256": dec_paged,
        "long_prefill": long_pf, "long_decode": long_dec,
        "long_decode_cp": cp_dec,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
