#!/usr/bin/env python
"""Throughput of the QE linear layer on B200: one JSON line on stdout.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the hot path over one batch: every projection of the
workload's layer set goes through the QE forward, in three stages: the
tensor-core down-projection with the router logits; routing, the bucket
sort and quantization with the expert-masked adapter rows (one cooperative
launch); and the int8 tcgen05 product with its adapter epilogue. The default
workload is the largest layer set that fits one GPU: the Qwen2VL-72B-shaped
projections at T = 8192. The step is captured once as a CUDA graph of the
public forward calls with a timing event at each end, and replayed. Inputs
are synthetic and seeded, with the shapes of the named model (qe_inputs),
and resident in HBM when the timed region starts. L2 is flushed between
steps, outside the timed intervals. A second graph with events between the
stages, replayed after the timed region, gives the per-stage breakdown
(per_projection) and the product kernels' time for the roofline. With the
default workload, the line also carries `decode`: the 72B decode-shaped
gate/up/down layers (W4A8 and W3A16, T = 16 and T = 1), each timed the same
way against the HBM roofline. Under torchrun each rank runs an independent
replica on its own token batch (weak scaling, no data-path collective), and
the time is the max over ranks; `--gpus N` without torchrun launches the N
ranks itself. e2e times the plain public call with pinned host buffers and
the copies inside the timed region.

`--impl reference` times the CPU oracle (a deliberately slow, plain program)
on a bounded token sample of the same workload, on the host's cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import qe_inputs as qi  # noqa: E402

WORKLOADS = {
    # name: (config, T override, description)
    "qwen2vl2b": ("qwen2vl2b", None, "Qwen2VL-2B-shaped layer set (q,o 1536x1536; gate,up 1536->8960; down 8960->1536), "
                                     "T=2048, W4A6 g128, r_s=32, N_r=8, r_r=4"),
    "internvl2_8b": ("internvl2_8b", None, "InternVL2-8B-shaped layer set, T=4096, W4A8 g128"),
    "qwen2vl72b": ("qwen2vl72b", None, "Qwen2VL-72B-shaped layer set, T=8192, W4A6 g128"),
    "qwen2vl2b_sparse": ("qwen2vl2b", None, "Qwen2VL-2B-shaped layer set, T=2048, W4A6 g128, r_s=32, N_r=8, "
                                            "r_r=4, cluster-sparse routed experts on 32 channels each", 32),
    "qwen2vl2b_w4a16": ("qwen2vl2b_w4a16", None, "Qwen2VL-2B-shaped layer set, T=2048, W4A16 g128 (weight-only "
                                                 "prefill), r_s=32, N_r=8, r_r=4"),
    "qwen2vl2b_w3a16": ("qwen2vl2b_w3a16", None, "Qwen2VL-2B-shaped layer set, T=2048, W3A16 g128 (weight-only "
                                                 "prefill), r_s=32, N_r=8, r_r=4"),
    "decode72b_w4a8": ("decode72b_w4a8", 16, "72B decode gate/up/down, T=16, W4A8 g128"),
    "decode72b_w4a8_t1": ("decode72b_w4a8", 1, "72B decode gate/up/down, T=1, W4A8 g128"),
    "decode72b_w3a16": ("decode72b_w3a16", 16, "72B decode gate/up/down, T=16, W3A16 g128"),
    "decode72b_w3a16_t1": ("decode72b_w3a16", 1, "72B decode gate/up/down, T=1, W3A16 g128"),
    "decode72b_w4a8_t4": ("decode72b_w4a8", 4, "72B decode gate/up/down, T=4, W4A8 g128"),
    "decode72b_w3a16_t4": ("decode72b_w3a16", 4, "72B decode gate/up/down, T=4, W3A16 g128"),
    "qwen2vl2b_w4a8_s16": ("qwen2vl2b_w4a8_s16", None, "Qwen2VL-2B-shaped layer set, T=2048, W4A8 g128 with fp16 "
                                                       "group scales, r_s=32, N_r=8, r_r=4"),
    "decode72b_w4a8_s16": ("decode72b_w4a8_s16", 16, "72B decode gate/up/down, T=16, W4A8 g128, fp16 group scales"),
    "qwen2vl72b_rr32": ("qwen2vl72b_rr32", None, "Qwen2VL-72B-shaped layer set, T=8192, W4A6 g128, routed rank 32 "
                                                 "(ablation)"),
    "qwen2vl72b_rr32_sparse": ("qwen2vl72b_rr32", None, "Qwen2VL-72B-shaped layer set, T=8192, W4A6 g128, routed rank "
                                                        "32 (ablation), cluster-sparse routed experts on 32 channels",
                               32),
}
METRIC = "QE linear tokens/s and effective TOPS; % of int8-TC / HBM roofline, 1 B200"
# The largest layer set that fits one GPU: the Qwen2VL-72B-shaped projections at T = 8192.
DEFAULT_WORKLOAD = "qwen2vl72b"

# The calibration statistics: per-token Top-k importance with its histogram, the channel split,
# the co-occurrence counts of the token-dependent channels and their NPMI.
CALIB_WORKLOADS = {
    # name: (T, d, k, N_r, description)
    "calib72b": (8192, 29568, 32, 8, "Qwen2VL-72B-shaped calibration statistic: T=8192 tokens of the 29568-wide down "
                                     "projection input, Top-k k=32, N_r=8 (C=256 token-dependent channels), NPMI "
                                     "threshold 0.2"),
}
CALIB_METRIC = "QE calibration statistic tokens/s (Top-k, split, co-occurrence, NPMI); % of HBM roofline, 1 B200"


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + sorted(CALIB_WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-decode", action="store_true",
                    help="leave out the decode-shaped 72B layers measured beside the default workload")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-mode", choices=["serial", "overlap"], default="overlap",
                    help="serial: each layer's copy in, forward and copy out on one stream; overlap: copies "
                         "on their own streams, so layer i+1's input and layer i-1's output cross PCIe while "
                         "layer i computes")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="oracle time the cpu_baseline sample is sized for (the reference arm: per step, "
                         "capped so that all steps take about two minutes)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="token count per GPU instead of the workload's own (smaller cases for ncu captures)")
    return ap.parse_args(argv)


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d.get("hbm_gbs", 6650.0), "bf16_tflops": d.get("bf16_tflops", 1590.0),
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", 1400.0), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def git_src_hash(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def read_traffic(kernel_file: str, name: str):
    """Per-launch DRAM bytes from a committed ncu summary (profiles/<name>.md), or None when
    absent or when the kernel source changed since the capture."""
    p = os.path.join(ROOT, "profiles", name + ".md")
    if not os.path.exists(p):
        return None
    vals = {}
    with open(p) as f:
        lines = f.read().splitlines()
    for line in lines:
        if ":" in line and line.strip().startswith("- "):
            k, v = line.strip()[2:].split(":", 1)
            v = v.strip()
            if v.startswith("`") and "`" in v[1:]:
                v = v[1:v.index("`", 1)]  # the value is the first backticked word
            vals[k.strip()] = v
    try:
        if vals.get("source_hash") != git_src_hash([kernel_file]):
            return None
        return float(vals["dram_bytes_per_launch_full_workload"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.thread = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            if self.thread:
                self.thread.join(timeout=2)

    def summary(self):
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower() in ("active", "1", "yes"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- reference arm (CPU oracle)

ORACLE_PREP_TOKENS = 2048  # token rows prepared for the oracle's timed sample


def oracle_layer_set(cfg, n_tokens, seed_shift=0):
    """The oracle's inputs for every projection (weights quantized once, outside any timing) and a
    function that times its forward over the first n of `n_tokens` tokens. Returns (run, n_tokens)."""
    import oracle
    prep = []
    for pi, proj in enumerate(cfg.projections):
        inp = qi.layer_inputs(cfg, proj, T=n_tokens, proj_index=pi + seed_shift)
        codes, scales, _, _ = oracle.quantize_weights(inp["W"], inp["s"], cfg.group, cfg.w_bits,
                                                      scale_fp16=cfg.scale_fp16)
        del inp["W"]
        prep.append((inp, codes, scales))

    def run(n):
        t0 = time.perf_counter()
        for inp, codes, scales in prep:
            oracle.qe_forward(inp["X"][:n], codes, scales, oracle.smoothing_inverse(inp["s"]), inp["A_s"], inp["B_s"], inp["A_r"],
                              inp["B_r"], inp["G"], cfg.group, cfg.a_bits)
        return time.perf_counter() - t0
    return run, n_tokens


def sized_oracle_sample(run, n_avail, target_s, probe=16, max_passes=10):
    """Times `run(n)` (the oracle over the first n tokens, in seconds) on a sample sized for about
    target_s seconds: a probe of a few tokens gives the rate, then n = min(n_avail, rate * target_s)
    tokens, passed again over the same tokens while the total is short of the target (tokens are
    independent, so a pass costs the same each time). Returns (tokens processed, seconds, n)."""
    p = max(1, min(probe, n_avail))
    sp = run(p)
    n = int(min(n_avail, max(p, p * target_s / max(sp, 1e-9))))
    tok, secs = 0, 0.0
    for _ in range(max_passes):
        secs += run(n)
        tok += n
        if secs >= 0.8 * target_s:
            break
    return tok, secs, n


def reference_step_seconds(args):
    """Oracle time per reference-arm step: the cpu_baseline target, capped so that all steps take
    about two minutes."""
    return max(0.5, min(args.cpu_seconds, 120.0 / max(1, args.steps)))


def run_reference(args, workload):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    cfg_name, t_over, desc = WORKLOADS[workload][:3]
    cfg = qi.CONFIGS[cfg_name]
    T = args.tokens or t_over or cfg.T
    cores = os.cpu_count() or 1
    os.environ.setdefault("OMP_NUM_THREADS", str(cores))
    run, n_avail = oracle_layer_set(cfg, min(T, ORACLE_PREP_TOKENS))
    for _ in range(args.warmup):
        run(min(n_avail, 4))
    target = reference_step_seconds(args)
    tok, tot, sample = 0, 0.0, 0
    for _ in range(args.steps):
        t_, s_, sample = sized_oracle_sample(run, n_avail, target)
        tok += t_
        tot += s_
    value = tok / tot
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64/f64", "data": "synthetic",
        "config": {"workload": workload, "description": desc, "T": T, "sample_tokens_per_step": tok // args.steps},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{tok // args.steps} token passes of every projection per step, about "
                                   f"{target:.0f} s each (passes over the first {sample} tokens; tokens are "
                                   f"independent)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- our arm

def replica_x_seed(rank: int, proj_index: int) -> int:
    """Seed of replica `rank`'s token batch for one projection (rank 0 uses the config's own seed)."""
    return 1000 + 7919 * rank + proj_index


def max_over_ranks(value: float, pg, device=None) -> float:
    """The slowest rank's time: every rank contributes its own, all receive the max."""
    if pg is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def build_layers(cfg, T, rank, dev, routed_channels=0):
    import torch
    import quantized_gemm_moe_b200 as qe
    layers = []
    for pi, proj in enumerate(cfg.projections):
        inp = qi.layer_inputs(cfg, proj, T=T, proj_index=pi)
        if rank:
            # each replica gets its own token batch (same weights)
            spec = cfg.outlier_spec(proj.d_in)
            x = qi.outlier_activations(T, proj.d_in, replica_x_seed(rank, pi), spec)
            inp["X"] = qi.to_bf16(x) if cfg.x_dtype == "bf16" else x
        desc = qe.make_desc(proj.d_in, proj.d_out, cfg.group, cfg.w_bits, cfg.a_bits, cfg.rank_shared, cfg.n_routed,
                            cfg.rank_routed, routed_channels, cfg.scale_fp16)

        def c(a):
            t = torch.from_numpy(np.ascontiguousarray(a)) if isinstance(a, np.ndarray) else a
            return t.contiguous().to(dev)

        channels = None
        if routed_channels:
            # cluster-sparse routed experts: seeded disjoint channel clusters with their own A_r
            channels, inp["A_r"] = qi.sparse_routed(proj.d_in, cfg.n_routed, routed_channels, cfg.rank_routed,
                                                    6000 + pi)
            channels = c(channels)
        layer = qe.QELayer.from_float(desc, c(inp["W"]), c(inp["s"]), c(inp["A_s"]), c(inp["B_s"]), c(inp["A_r"]),
                                      c(inp["B_r"]), c(inp["G"]), channels=channels)
        X = c(inp["X"])
        Y = torch.empty((T, proj.d_out), dtype=torch.bfloat16, device=dev)
        ws = layer.workspace(T)
        layers.append(dict(proj=proj, desc=desc, layer=layer, X=X, Y=Y, ws=ws, x_host=inp["X"]))
        del inp
    torch.cuda.synchronize()
    return layers


def e2e_overlapped_step(qe, layers, xh, yh, stream, s_in, s_out):
    """One end-to-end step with the copies on their own streams: layer i's input crosses PCIe on
    s_in while earlier layers compute on `stream`, and its output returns on s_out while later
    layers compute. Ordering: each copy in waits for the step's start (the previous step ended
    with a full synchronize), each forward for its own input, each copy out for its forward; the
    step ends when `stream` has waited for the last copy out."""
    import torch
    start = torch.cuda.Event()
    start.record(stream)
    s_in.wait_event(start)
    s_out.wait_event(start)
    x_ready = []
    for L, x in zip(layers, xh):
        with torch.cuda.stream(s_in):
            L["X"].copy_(x, non_blocking=True)
        ev = torch.cuda.Event()
        ev.record(s_in)
        x_ready.append(ev)
    for L, y, ev in zip(layers, yh, x_ready):
        stream.wait_event(ev)
        qe.linear_forward(L["desc"], L["layer"].weights, L["X"], L["Y"], L["ws"], stream=stream)
        done = torch.cuda.Event()
        done.record(stream)
        s_out.wait_event(done)
        with torch.cuda.stream(s_out):
            y.copy_(L["Y"], non_blocking=True)
    out_done = torch.cuda.Event()
    out_done.record(s_out)
    stream.wait_event(out_done)


def time_layer_set(qe, layers, T, args, flush, pg, stages, clocks=True):
    """Times one step (every projection through the public forward call, T tokens each) as a CUDA
    graph replay with an event at each end, L2 flushed before each replay. A second graph splits
    each forward into its stages with events between them; its replays after the timed region give
    the per-stage breakdown. Returns (step_ms [steps], stage_ms [n_diag, proj, stage], clocks)."""
    import torch
    ins = [(L["desc"], L["layer"].weights, L["X"][:T], L["Y"][:T], L["layer"].workspace(T)) for L in layers]

    def step_plain():
        for d, w, X, Y, ws in ins:
            qe.linear_forward(d, w, X, Y, ws)

    for _ in range(max(args.warmup, 0)):
        flush.zero_()
        step_plain()
    torch.cuda.synchronize()
    assert qe.device_error() == 0, "a device wait ran out during warm-up"
    cap = torch.cuda.Stream()
    ev0 = torch.cuda.Event(enable_timing=True, external=True)
    ev1 = torch.cuda.Event(enable_timing=True, external=True)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cap):
        ev0.record()
        step_plain()
        ev1.record()
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(stages) + 1)] for _ in ins]
    sgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(sgraph, stream=cap):
        for (d, w, X, Y, ws), e in zip(ins, evs):
            e[0].record()
            for i, sm in enumerate(stages):
                qe.linear_forward_stages(d, w, X, Y, ws, sm)
                e[i + 1].record()
    for _ in range(2):
        graph.replay()
        sgraph.replay()
    torch.cuda.synchronize()
    step_ms = np.zeros(args.steps)
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    clk = ClockSampler(torch.cuda.current_device()) if clocks else None
    if clk:
        clk.__enter__()
    try:
        for s_i in range(args.steps):
            flush.zero_()
            graph.replay()
            torch.cuda.synchronize()
            step_ms[s_i] = ev0.elapsed_time(ev1)
    finally:
        if clk:
            clk.__exit__(None, None, None)
    if pg:
        pg.barrier()
    n_diag = max(3, min(args.steps, 10))
    stage_ms = np.zeros((n_diag, len(ins), len(stages)))
    for s_i in range(n_diag):
        flush.zero_()
        sgraph.replay()
        torch.cuda.synchronize()
        for p_i, e in enumerate(evs):
            for k in range(len(stages)):
                stage_ms[s_i, p_i, k] = e[k].elapsed_time(e[k + 1])
    err = qe.device_error()
    assert err == 0, f"device wait ran out (code {err:#x})"
    del graph, sgraph
    return step_ms, stage_ms, (clk.summary() if clk else None)


def measure_int8_peak(dev):
    """Dense int8 tensor-core throughput of the library GEMM on this GPU: torch._int_mm (cuBLASLt)
    of 8192^3, best of 10 CUDA-event timings after warm-up. None if the call is unavailable."""
    import torch
    n = 8192
    try:
        a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev)
        b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev).t()
        for _ in range(3):
            torch._int_mm(a, b)
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._int_mm(a, b)
            e1.record()
            e1.synchronize()
            best = min(best, e0.elapsed_time(e1))
        del a, b
        torch.cuda.empty_cache()
        return 2.0 * n ** 3 / (best / 1e3) / 1e12
    except Exception:  # pragma: no cover - reported as unavailable
        return None


def product_roofline(cfg, layers, T, prod_ms, peaks, int8, traffic):
    """Roofline of the dominant kernel (the main product) for one timed layer set."""
    from quantized_gemm_moe_b200 import roofline
    wonly = cfg.a_bits == 16
    kernel = "qdec" if T <= 16 else ("wgemm" if wonly else "qgemm")
    if T <= 16:
        # decode: HBM bound; the product streams the packed codes, the scales and the adapters
        by = sum(roofline.layer_bytes(T, L["proj"].d_in, L["proj"].d_out, cfg.group, cfg.w_bits, cfg.rank_shared,
                                      cfg.n_routed, cfg.rank_routed, 1 if not wonly else 2, 2,
                                      2 if cfg.scale_fp16 else 4) for L in layers)
        ach = by / (prod_ms / 1e3) / 1e9
        return {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"], "traffic": traffic, "kernel": kernel,
                "peak_source": peaks["source"] + " hbm copy (of measured)"}
    if wonly:
        wfl = sum(2 * T * L["proj"].d_in * L["proj"].d_out for L in layers)
        ach = wfl / (prod_ms / 1e3) / 1e12
        return {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": ach / peaks["bf16_tflops"], "traffic": traffic, "kernel": kernel,
                "peak_source": f"{peaks['source']} bf16 burst (of measured)"}
    ints = sum(roofline.int_ops(T, L["proj"].d_in, L["proj"].d_out) for L in layers)
    ach = ints / (prod_ms / 1e3) / 1e12
    return {"bound": "tensor", "achieved": ach, "peak": int8["peak"], "unit": "TOP/s", "frac": ach / int8["peak"],
            "traffic": traffic, "kernel": kernel, "peak_source": int8["source"]}


def per_projection(cfg, layers, T, stage_ms):
    from quantized_gemm_moe_b200 import roofline
    wonly = cfg.a_bits == 16
    out = []
    for p_i, L in enumerate(layers):
        ms = stage_ms[:, p_i, :].mean(axis=0)
        K, N = L["proj"].d_in, L["proj"].d_out
        tot = ms.sum()
        out.append({
            "proj": L["proj"].name, "K": K, "N": N, "ms": float(tot),
            "stage_ms": {"project": float(ms[0]), "route_quant": float(ms[1]), "product": float(ms[2])},
            "product_tops": (roofline.int_ops(T, K, N) / (ms[2] / 1e3) / 1e12) if not wonly else None,
            "product_gbs": roofline.layer_bytes(T, K, N, cfg.group, cfg.w_bits, cfg.rank_shared, cfg.n_routed,
                                                cfg.rank_routed, 1 if not wonly else 2, 2,
                                                2 if cfg.scale_fp16 else 4) / (ms[2] / 1e3) / 1e9,
            "layer_tokens_per_s": T / (tot / 1e3),
        })
    return out


def oracle_baseline(cfg, T, seconds):
    """The oracle timed on the host cores on a bounded token sample of the workload."""
    cores = os.cpu_count() or 1
    os.environ.setdefault("OMP_NUM_THREADS", str(cores))
    run, n_avail = oracle_layer_set(cfg, min(T, ORACLE_PREP_TOKENS))
    tok, secs, sample = sized_oracle_sample(run, n_avail, seconds)
    return {"value": tok / secs, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{tok} token passes through every projection of the layer set in {secs:.1f} s "
                      f"(the first {sample} tokens of the workload; tokens are independent)"}


# Decode-shaped 72B layers (gate/up/down at T <= 16), measured beside the headline workload:
# each variant's layers are built once and timed at every T of the list.
DECODE_SETS = (("decode72b_w4a8", (16, 1)), ("decode72b_w3a16", (16, 1)), ("decode72b_w4a8_s16", (16, 1)))


def run_ours(args, workload):
    import torch
    import quantized_gemm_moe_b200 as qe
    from quantized_gemm_moe_b200 import roofline

    rank, local_rank, world = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the product path has no CPU fallback)")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    qe.load()
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist
    cfg_name, t_over, desc_txt = WORKLOADS[workload][:3]
    routed_channels = WORKLOADS[workload][3] if len(WORKLOADS[workload]) > 3 else 0
    cfg = qi.CONFIGS[cfg_name]
    T = args.tokens or t_over or cfg.T
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    wonly = cfg.a_bits == 16
    stages = (qe.QE_STAGE_PROJECT, qe.QE_STAGE_ROUTE | qe.QE_STAGE_QUANT, qe.QE_STAGE_PRODUCT)
    peaks = load_peaks()

    # int8 denominator: the library GEMM measured here, or 2x the bf16 burst (the nominal
    # int8:bf16 ratio), whichever is larger (the smaller fraction)
    int8_meas = measure_int8_peak(dev) if not wonly else None
    twice_bf16 = 2.0 * peaks["bf16_tflops"]
    if int8_meas is not None and int8_meas >= twice_bf16:
        int8 = {"peak": int8_meas, "source": f"measured torch._int_mm 8192^3 on this GPU: {int8_meas:.0f} TOP/s "
                                             f"(2x the bf16 burst: {twice_bf16:.0f})"}
    else:
        meas = "unavailable" if int8_meas is None else f"{int8_meas:.0f} TOP/s"
        int8 = {"peak": twice_bf16, "source": f"{peaks['source']} bf16 burst {peaks['bf16_tflops']} TF/s x 2 "
                                              f"(int8:bf16 nominal ratio); torch._int_mm 8192^3 measured {meas}"}

    layers = build_layers(cfg, T, rank, dev, routed_channels)
    step_ms, stage_ms, clocks = time_layer_set(qe, layers, T, args, flush, pg, stages)
    total_ms = max_over_ranks(float(step_ms.sum()), pg, dev)
    ms_per_step = total_ms / args.steps
    value = world * T * args.steps / (total_ms / 1e3)

    # algorithmic work per step
    ints = sum(roofline.int_ops(T, L["proj"].d_in, L["proj"].d_out) for L in layers) if not wonly else 0
    fl = sum(roofline.adapter_flops(T, L["proj"].d_in, L["proj"].d_out, cfg.rank_shared, cfg.n_routed,
                                    cfg.rank_routed) for L in layers)
    if wonly:
        fl += sum(2 * T * L["proj"].d_in * L["proj"].d_out for L in layers)
    xb = 2 if cfg.x_dtype == "bf16" else 4
    nbytes = sum(roofline.layer_bytes(T, L["proj"].d_in, L["proj"].d_out, cfg.group, cfg.w_bits, cfg.rank_shared,
                                      cfg.n_routed, cfg.rank_routed, xb, 2, 2 if cfg.scale_fp16 else 4)
                 for L in layers)
    prod_ms = stage_ms[:, :, 2].sum(axis=1).mean()  # the product kernels of one step
    if T <= 16:
        kernel_file, kname = "quantized_gemm_moe_b200/csrc/k_decode.cu", "qdec_"
    elif wonly:
        kernel_file, kname = "quantized_gemm_moe_b200/csrc/k_wgemm.cu", "wgemm_"
    else:
        kernel_file, kname = "quantized_gemm_moe_b200/csrc/k_gemm.cu", "qgemm_"
    traffic = read_traffic(kernel_file, kname + workload) if not args.tokens else None
    roof = product_roofline(cfg, layers, T, prod_ms, peaks, int8, traffic)
    per_proj = per_projection(cfg, layers, T, stage_ms)

    # end to end through the public call with host buffers (pinned), copies inside the timed region
    e2e = None
    if not args.no_e2e:
        xh = [torch.from_numpy(np.ascontiguousarray(L["x_host"])) if isinstance(L["x_host"], np.ndarray)
              else L["x_host"] for L in layers]
        xh = [x.contiguous().pin_memory() for x in xh]
        yh = [torch.empty(L["Y"].shape, dtype=L["Y"].dtype).pin_memory() for L in layers]
        h2d = sum(x.numel() * x.element_size() for x in xh)
        d2h = sum(y.numel() * y.element_size() for y in yh)
        e_ms = 0.0
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        for it in range(args.warmup + args.steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            if args.e2e_mode == "serial":
                for L, x, y in zip(layers, xh, yh):
                    L["X"].copy_(x, non_blocking=True)
                    qe.linear_forward(L["desc"], L["layer"].weights, L["X"], L["Y"], L["ws"])
                    y.copy_(L["Y"], non_blocking=True)
            else:
                e2e_overlapped_step(qe, layers, xh, yh, stream, s_in, s_out)
            e1.record(stream)
            e1.synchronize()
            if it >= args.warmup:
                e_ms += e0.elapsed_time(e1)
        e_ms = max_over_ranks(e_ms, pg, dev)
        e2e = {"value": world * T * args.steps / (e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "mode": args.e2e_mode}
        del xh, yh

    launches = sum(qe.linear_kernel_launches(L["desc"], T, qe.QE_BF16 if cfg.x_dtype == "bf16" else qe.QE_F32)
                   for L in layers) * args.steps
    for L in layers:
        L.clear()
    del layers
    torch.cuda.empty_cache()

    # decode-shaped layers (HBM bound), each at its own roofline
    decode = None
    if not args.no_decode and args.tokens == 0 and workload == DEFAULT_WORKLOAD:
        decode = []
        for dname, Ts in DECODE_SETS:
            dcfg = qi.CONFIGS[dname]
            dl = build_layers(dcfg, max(Ts), rank, dev)
            dcpu = None
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                dcpu = oracle_baseline(dcfg, max(Ts), args.cpu_seconds / 2)
            for dT in Ts:
                s_ms, st_ms, dclk = time_layer_set(qe, dl, dT, args, flush, pg, stages)
                tot = max_over_ranks(float(s_ms.sum()), pg, dev)
                pm = st_ms[:, :, 2].sum(axis=1).mean()
                dtraffic = read_traffic("quantized_gemm_moe_b200/csrc/k_decode.cu", f"qdec_{dname}_t{dT}")
                decode.append({
                    "workload": dname, "T": dT,
                    "description": f"72B decode gate/up/down, T={dT}, {'W3A16' if dcfg.w_bits == 3 else 'W4A8'} g128"
                                   + (", fp16 group scales" if dcfg.scale_fp16 else ""),
                    "value": world * dT * args.steps / (tot / 1e3), "unit": "tokens/s",
                    "ms_per_step": tot / args.steps,
                    "roofline": product_roofline(dcfg, dl, dT, pm, peaks, int8, dtraffic),
                    "per_projection": per_projection(dcfg, dl, dT, st_ms),
                    "cpu_baseline": dcpu, "clocks": dclk,
                })
            for L in dl:
                L.clear()
            del dl
            torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_baseline(cfg, T, args.cpu_seconds)

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if wonly else "int8", "data": "synthetic",
        "config": {"workload": workload, "description": desc_txt, "T_per_gpu": T,
                   "projections": [[p.name, p.d_in, p.d_out] for p in cfg.projections],
                   "l2": "flushed between steps (256 MB write outside the per-step events)",
                   "parallelism": f"replicas x{world}"},
        "effective_tops": (ints + fl) / (ms_per_step / 1e3) / 1e12 * world,
        "hbm_gbs_algorithmic": nbytes / (ms_per_step / 1e3) / 1e9,
        "roofline": roof,
        "int8_peak": {"torch_int_mm_tops": int8_meas, "twice_bf16_burst_tops": twice_bf16, "used": int8["peak"]},
        "per_projection": per_proj,
        "decode": decode,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "clocks": clocks,
        "gpu_launches": launches,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    return 0

# ---------------------------------------------------------------- calibration statistic

def calib_inputs(T, d, seed=0):
    """Activations with the 72B outlier structure and the weight column means w_mean."""
    cfg = qi.CONFIGS["qwen2vl72b"]
    X = qi.to_bf16(qi.outlier_activations(T, d, 4242 + seed, cfg.outlier_spec(d)))
    w_mean = np.abs(qi.gaussian(d, 0.02, 4243)).astype(np.float32)
    return X, w_mean


def calib_oracle_run(X, w_mean, k, C):
    """The oracle's calibration chain on a token sample. Returns seconds."""
    import oracle
    t0 = time.perf_counter()
    idx, hist = oracle.topk(X, w_mean, k)
    pos = oracle.split_channels(hist, k, C)
    O = oracle.cooccurrence(idx, pos, C)
    oracle.npmi(O, X.shape[0], 0.2)
    return time.perf_counter() - t0


def run_calib(args, workload):
    T, d, k, n_routed, desc_txt = CALIB_WORKLOADS[workload]
    T = args.tokens or T
    C = n_routed * k
    rank, local_rank, world = dist_env()
    if args.impl == "reference":
        if rank != 0:
            return 0
        cores = 1   # the oracle's Top-k, counts and NPMI run on one thread
        X, w_mean = calib_inputs(min(T, ORACLE_PREP_TOKENS), d)
        for _ in range(args.warmup):
            calib_oracle_run(X[:4], w_mean, k, C)
        target = reference_step_seconds(args)
        tok, tot, sample = 0, 0.0, 0
        for _ in range(args.steps):
            t_, s_, sample = sized_oracle_sample(lambda n: calib_oracle_run(X[:n], w_mean, k, C), len(X), target)
            tok += t_
            tot += s_
        value = tok / tot
        print(json.dumps({
            "impl": "reference", "metric": CALIB_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32/int64/f64",
            "data": "synthetic", "config": {"workload": workload, "description": desc_txt, "T": T,
                                            "sample_tokens_per_step": tok // args.steps},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"{tok // args.steps} tokens through Top-k, split, co-occurrence and NPMI "
                                       f"per step, about {target:.0f} s each (samples of the first {sample} tokens)"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }), flush=True)
        return 0

    import torch
    import quantized_gemm_moe_b200 as qe
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the product path has no CPU fallback)")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    qe.load()
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist
    X_h, w_mean_h = calib_inputs(T, d, seed=rank)
    X = X_h.to(dev)
    w_mean = torch.from_numpy(w_mean_h).to(dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    hist = torch.empty(d, dtype=torch.int32, device=dev)
    pos = torch.empty(d, dtype=torch.int32, device=dev)
    O = torch.empty((C, C), dtype=torch.int32, device=dev)
    S = torch.empty((C, C), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]

    def step(record=False):
        if record:
            ev[0].record(stream)
        qe.topk_importance(X, w_mean, k, idx, hist)
        if record:
            ev[1].record(stream)
        qe.split_channels(hist, k, C, pos)
        if record:
            ev[2].record(stream)
        qe.cooccurrence_npmi(idx, pos, C, O, S, 0.2)
        if record:
            ev[3].record(stream)

    for _ in range(max(args.warmup, 0)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    step_ms = np.zeros(args.steps)
    part_ms = np.zeros((args.steps, 3))
    with ClockSampler(torch.cuda.current_device()) as clk:
        for s_i in range(args.steps):
            flush.zero_()
            step(record=True)
            torch.cuda.synchronize()
            step_ms[s_i] = ev[0].elapsed_time(ev[3])
            part_ms[s_i] = [ev[i].elapsed_time(ev[i + 1]) for i in range(3)]
    if pg:
        pg.barrier()
    total_ms = max_over_ranks(float(step_ms.sum()), pg, dev)
    ms_per_step = total_ms / args.steps
    value = world * T * args.steps / (total_ms / 1e3)
    parts = part_ms.mean(axis=0)

    peaks = load_peaks()
    # the committed capture is per full-size launch; DRAM traffic grows with the tokens
    scaled_traffic = read_traffic("quantized_gemm_moe_b200/csrc/k_misc.cu", "topk_" + workload)
    if scaled_traffic is not None:
        scaled_traffic *= T / CALIB_WORKLOADS[workload][0]
    # Top-k reads X (bf16) and w_mean once and writes idx and hist
    topk_bytes = T * d * 2 + d * 4 + T * k * 4 + d * 4
    ach = topk_bytes / (parts[0] / 1e3) / 1e9
    roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": ach / peaks["hbm_gbs"],
            "traffic": scaled_traffic, "kernel": "topk",
            "peak_source": peaks["source"] + " hbm copy"}

    e2e = None
    if not args.no_e2e:
        xh = X_h.contiguous().pin_memory()
        Oh = torch.empty((C, C), dtype=torch.int32).pin_memory()
        Sh = torch.empty((C, C), dtype=torch.float32).pin_memory()
        e_ms = 0.0
        for it in range(args.warmup + args.steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            X.copy_(xh, non_blocking=True)
            step()
            Oh.copy_(O, non_blocking=True)
            Sh.copy_(S, non_blocking=True)
            e1.record(stream)
            e1.synchronize()
            if it >= args.warmup:
                e_ms += e0.elapsed_time(e1)
        e_ms = max_over_ranks(e_ms, pg, dev)
        e2e = {"value": world * T * args.steps / (e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": xh.numel() * xh.element_size(), "d2h_bytes_per_step": 2 * C * C * 4}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n_avail = min(T, ORACLE_PREP_TOKENS)
        tok, secs, sample = sized_oracle_sample(lambda n: calib_oracle_run(X_h[:n], w_mean_h, k, C), n_avail,
                                                args.cpu_seconds)
        cpu = {"value": tok / secs, "unit": "tokens/s", "cores": 1, "kind": "oracle",
               "sample": f"{tok} tokens through Top-k, split, co-occurrence and NPMI in {secs:.1f} s "
                         f"(samples of the first {sample} tokens)"}
    line = {
        "metric": CALIB_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32/int32", "data": "synthetic",
        "config": {"workload": workload, "description": desc_txt, "T_per_gpu": T, "d": d, "k": k, "C": C,
                   "l2": "inputs larger than L2 (X is 484 MB) and a 256 MB flush between steps",
                   "parallelism": f"replicas x{world}"},
        "stage_ms": {"topk": float(parts[0]), "split": float(parts[1]), "cooc_npmi": float(parts[2])},
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "clocks": clk.summary(),
        "gpu_launches": 4 * args.steps,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    return 0


def free_port() -> int:
    import socket
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


def spawn_ranks(args, argv) -> int:
    """--gpus N > 1 outside torchrun: run this script again under torch.distributed.run with N
    ranks on this node (rendezvous on 127.0.0.1). Returns the launcher's exit status."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()), os.path.abspath(__file__)] + list(argv)
    return subprocess.call(cmd)


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    args = parse_args(argv)
    if args.gpus < 1:
        raise SystemExit("--gpus must be >= 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        return spawn_ranks(args, argv)
    if "WORLD_SIZE" in os.environ and int(os.environ["WORLD_SIZE"]) != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but the launcher started {os.environ['WORLD_SIZE']} ranks")
    if args.workload in CALIB_WORKLOADS:
        return run_calib(args, args.workload)
    if args.impl == "reference":
        return run_reference(args, args.workload)
    return run_ours(args, args.workload)


if __name__ == "__main__":
    sys.exit(main())
