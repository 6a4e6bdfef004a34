#!/usr/bin/env python
"""Benchmark of the routed MoE expert-FFN layer (moe_forward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config prompt] [--impl own|reference]

One step = one moe_forward over one batch: route → permute → expert FFN →
combine, every kernel of the library, inputs resident in HBM. W warm-up steps,
then K timed steps, each bracketed by CUDA events on the launching stream, with
L2 flushed between steps outside the events (a 256 MiB write, then a 256 MiB read
so the dirty lines are written back before the next step). For N > 1 each
rank (one per GPU, launched by torch.distributed.run) runs its own replica of
the workload — the layer shards by tokens with no exchange — and the time is
the max over ranks (NCCL all-reduce of the measured times only).

One JSON line on rank 0: value = tokens/s of the whole job; plus TFLOP/s (or
GB/s for the decode configs), the roofline of the dominant kernel measured live
(per-kernel CUDA events inside the library, moe_profile_*), the end-to-end
number through the host-buffer entry points (copies of every step's inputs in
and output back inside the timed region; a pipelined loop over three streams
with moe_forward_host_async, and one synchronous moe_forward_host per step),
SM clocks sampled through NVML during the timed region, and the fp64 CPU
oracle's throughput on this host as a baseline. At N = 1 the line also carries
`per_config`: the other stated workloads (capped, decode T=1/8/32, quantised)
measured the same way in the same run, each with its dominant kernel's roofline
and its own clock samples.

--impl reference times that oracle alone (on the host cores, rank 0 only) on
this arm's config, a bounded sample of the workload per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time
import types

ROOT = os.path.dirname(os.path.abspath(__file__))
TILE_ARG = {"auto": 0, "one": 1, "pair": 2}  # moe_params.tile_ctas (MOE_TILE_*)
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "MoE layer tokens/sec and TFLOP/s (% BF16 tensor peak); decode GB/s (% HBM)"
FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="prompt", choices=sorted(synth.CONFIGS))
    ap.add_argument("--impl", default="own", choices=["own", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the other stated workloads (capped, decode1/8/32, quant) in the JSON line")
    ap.add_argument("--tokens", type=int, default=0, help="override T of the workload (profiling small cases)")
    ap.add_argument("--experts", type=int, default=0,
                    help="override E of the workload (profiling: a decode layer with fewer untouched experts "
                         "runs the same kernels on the same touched weights, with less memory held)")
    ap.add_argument("--profile-calls", type=int, default=0,
                    help="only run this many moe_forward calls and exit (for ncu: no timing, no other kernels)")
    ap.add_argument("--profile-op", default="forward", choices=["forward", "backward", "route_stats"],
                    help="entry point the --profile-calls calls make")
    ap.add_argument("--tile", default="auto", choices=["auto", "one", "pair"],
                    help="SMs per tcgen05 tile (moe_params.tile_ctas); auto = the library's choice")
    ap.add_argument("--sweep-threshold", action="store_true",
                    help="time moe_forward for each stream_max_rows and print one JSON line")
    ap.add_argument("--variant-table", action="store_true",
                    help="time tiles against streaming on layers of exact rows per expert; one JSON line")
    return ap.parse_args()


# --------------------------------------------------------------------------- workload numbers

class L2Flush:
    """Between timed steps: write a 256 MiB buffer (every L2 line is evicted), then read another
    256 MiB buffer, so that the lines the write left dirty are written back before the next timed
    step starts. The step then begins with a cold L2 holding only clean lines of the second buffer,
    and does not pay for the flush's write-back traffic."""

    def __init__(self, torch):
        self.w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        self.r = torch.zeros(FLUSH_BYTES // 4, dtype=torch.int32, device="cuda")

    def __call__(self):
        self.w.zero_()
        self.r.max()  # a reduction reading the whole buffer; the result stays on the device


def workload_numbers(cfg, P, touched):
    """Algorithmic FLOPs and bytes of one layer call (no padding, no intermediates)."""
    T, d, f = cfg.T, cfg.d, cfg.f
    fl_gateup = 2.0 * P * 2 * d * f
    fl_down = 2.0 * P * f * d
    wbytes = 2.0 if cfg.weight_format == "bf16" else 0.5 + 2.0 / 32  # q4g32: nibble + fp16 scale / 32
    n_exp = touched + (1 if cfg.has_shared else 0)
    if cfg.has_shared:
        fl_gateup += 2.0 * T * 2 * d * cfg.f_shared
        fl_down += 2.0 * T * cfg.f_shared * d
    w_gateup = n_exp * 2 * d * f * wbytes
    w_down = n_exp * f * d * wbytes
    io = T * d * 2 + T * d * 4 + T * cfg.E * 4  # x bf16 in, out fp32, logits
    return {"flops": fl_gateup + fl_down, "flops_gateup": fl_gateup, "flops_down": fl_down,
            "bytes": w_gateup + w_down + io, "bytes_gateup": w_gateup + T * d * 2,
            "bytes_down": w_down + T * d * 2}


def workload_name(cfg):
    s = f"{cfg.name}: T={cfg.T} d_model={cfg.d} d_ff={cfg.f} E={cfg.E} top-{cfg.k}"
    if cfg.capacity_factor:
        s += f" cf={cfg.capacity_factor}"
    if cfg.has_shared:
        s += f" +shared(d_ff={cfg.f_shared})"
    if cfg.bias != "none":
        s += f" bias={cfg.bias}"
    return s + f" weights={cfg.weight_format}"


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            return json.load(fh), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(files):
    """SHA-256 (first 16 hex digits) of the kernel sources with their // comments and blank lines
    removed, so that a comment edit does not invalidate counters taken on the same code."""
    h = hashlib.sha256()
    for fn in files:
        with open(os.path.join(ROOT, "mixture_experts_routed_04_b200", "csrc", fn)) as fh:
            for line in fh:
                code = line.split("//", 1)[0].rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def committed_traffic(kernel, files, cfg_name):
    """DRAM bytes per launch (read + write) from the committed ncu summary table, if its row was
    taken on the current kernel source; None otherwise."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.md")
    if not os.path.exists(path):
        return None
    want = kernel_source_hash(files)
    with open(path) as fh:
        for line in fh:
            cells = [c.strip().strip("`") for c in line.strip().strip("|").split("|")]
            if len(cells) >= 5 and cells[0] == kernel and cells[1] == cfg_name and cells[2] == want:
                return int(cells[3]) + int(cells[4])
    return None


def max_over_ranks(value, dist=None, device="cpu"):
    """The largest of every rank's value (all ranks call it in the same order); the value itself
    without a process group. Multi-GPU runs are replicas, so this timing reduction is the only
    collective on the path."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tokens_per_s(tokens_per_rank, world, max_ms_per_step):
    """Whole-job throughput: every rank processes tokens_per_rank per step; the step takes the
    slowest rank's time."""
    return tokens_per_rank * world / (max_ms_per_step / 1e3)


# --------------------------------------------------------------------------- roofline of the dominant kernel

ONE_SM_SRC = ["gemm_tc.cu", "gemm_tc.cuh", "common.cuh"]
TWO_SM_SRC = ["gemm_pair.cu", "gemm_tc.cuh", "common.cuh"]
STREAM_SRC = ["stream.cu", "common.cuh"]


def dominant_roofline(prof, wl, K, ms, pk, pk_src, pair, down_f16, cfg_name):
    """Roofline object of the expert GEMM with the largest measured share of the step.

    achieved = the kernel's algorithmic work per launch (FLOPs when the workload's intensity is
    at or above the measured ridge, else bytes: touched weights + x) / its mean launch time
    (library CUDA events); traffic = DRAM bytes per launch from the committed ncu table while
    the kernel source is unchanged; traffic_over_algorithmic = traffic / those algorithmic bytes
    (weights + x, the scope table's count: the gathered rows, h and y_rows are not in it)."""
    ridge = pk["bf16_tflops"] * 1e12 / (pk["hbm_gbs"] * 1e9)
    tensor_bound = wl["flops"] / wl["bytes"] >= ridge
    names = {"tc_gateup": ("grouped_gemm_pair_kernel<0> (tcgen05 SM pairs, gate/up + clamped SwiGLU)", "gateup",
                           TWO_SM_SRC) if pair else
             ("grouped_gemm_kernel<0> (tcgen05 gate/up + clamped SwiGLU)", "gateup", ONE_SM_SRC),
             "tc_down": ("grouped_gemm_pair_kernel<1> (tcgen05 SM pairs, down + gate scale)", "down", TWO_SM_SRC)
             if pair and down_f16 else ("grouped_gemm_kernel<1> (tcgen05 down + gate scale)", "down", ONE_SM_SRC),
             "stream_gateup": ("stream_kernel<0> (few-rows gate/up)", "gateup", STREAM_SRC),
             "stream_down": ("stream_kernel<1> (few-rows down)", "down", STREAM_SRC)}
    kern = max(names, key=lambda k: prof.get(k, (0.0, 0))[0])
    kms, kn = prof.get(kern, (0.0, 0))
    k_avg = kms / kn if kn else float("nan")
    label, part, src = names[kern]
    alg_bytes = wl["bytes_" + part]
    if tensor_bound:
        work = wl["flops_" + part]
        achieved = work / (k_avg / 1e3) / 1e12
        peak = pk["bf16_tflops"]
        roof = {"kernel": label, "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "peak_source": f"{pk_src} bf16_tflops (burst)"}
    else:
        work = alg_bytes
        achieved = work / (k_avg / 1e3) / 1e9
        peak = pk["hbm_gbs"]
        roof = {"kernel": label, "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_source": f"{pk_src} hbm_gbs"}
    traffic = committed_traffic(kern, src, cfg_name)
    roof.update({"avg_launch_ms": k_avg, "algorithmic_per_launch": work, "share_of_step": kms / K / ms,
                 "algorithmic_bytes_per_launch": alg_bytes, "traffic": traffic,
                 "traffic_over_algorithmic": traffic / alg_bytes if traffic else None})
    return roof


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """Polls SM clock and throttle reasons through NVML in a thread (read only)."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # NVML missing: report no samples
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.001)

    def __enter__(self):
        if self._nv:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._nv:
            self._t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------------------- CPU oracle

def cpu_oracle_runner(cfg):
    """Prepare the oracle's inputs (fp64 weights of every expert) once; return run(tokens)->seconds."""
    import oracle
    from synth.device import expert_f64, shared_f64
    x = synth.bf16_bits_to_f32(synth.x_bits(cfg)).astype(np.float64)
    lg = synth.logits(cfg)
    if cfg.weight_format == "q4g32":
        def load(e):
            return tuple(oracle.dequant_q4g32(*synth.expert_q4_weights(cfg, e, w)) for w in ("gate", "up", "down"))
    else:
        def load(e):
            return expert_f64(cfg, e)
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(8) as ex:
        Ws = dict(zip(range(cfg.E), ex.map(load, range(cfg.E))))
    sh = shared_f64(cfg) if cfg.has_shared else None

    def run(tokens):
        xs, ls = x[tokens], lg[tokens]
        t0 = time.perf_counter()
        oracle.forward(xs, ls, cfg.k, Ws.__getitem__, cfg.swiglu_limit, cfg.capacity_factor, shared=sh)
        return time.perf_counter() - t0

    return run


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(cfg, budget_s=15.0):
    """The oracle timed on the host cores on whole-layer calls of the workload, until ~budget_s."""
    run = cpu_oracle_runner(cfg)
    toks = np.arange(cfg.T)
    run(toks[: min(cfg.T, 64)])  # warm BLAS
    times = []
    t_end = time.perf_counter() + budget_s
    while not times or (time.perf_counter() < t_end and len(times) < 50):
        times.append(run(toks))
    tps = cfg.T * len(times) / sum(times)
    return {"value": tps, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{len(times)} whole-layer call(s) of the {cfg.name} workload (T={cfg.T}), fp64 NumPy, "
                      f"weights pre-converted to fp64 outside the timing"}


# --------------------------------------------------------------------------- reference arm

def reference_arm(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    run = cpu_oracle_runner(cfg)
    est = run(np.arange(min(cfg.T, 256)))  # seconds for 256 tokens
    per_tok = est / min(cfg.T, 256)
    budget = 120.0  # seconds of timed CPU work in total
    n = int(max(1, min(cfg.T, budget / max(args.steps, 1) / max(per_tok, 1e-9))))
    rng = np.random.default_rng(0)
    for _ in range(args.warmup):
        run(np.sort(rng.choice(cfg.T, n, replace=False)))
    times = [run(np.sort(rng.choice(cfg.T, n, replace=False))) for _ in range(args.steps)]
    sec = sum(times)
    tps = n * args.steps / sec
    line = {"metric": METRIC, "value": tps, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * sec / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": workload_name(cfg), "tokens_per_step": n, "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": tps, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": f"{n} random tokens of the {cfg.name} workload per step (all experts' "
                                       f"weights resident as fp64)"},
            "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- the other stated workloads

PER_CONFIG = ("capped", "decode1", "decode8", "decode32", "quant")


def upload_routed(cfg, b, torch):
    """Device inputs with every routed expert's weights (others NaN, never read): the routing
    is the library's own (moe_route on the device), so only the experts it picks are drawn."""
    from synth.device import upload
    lg = torch.from_numpy(synth.logits(cfg)).cuda()
    p = b.params_for(cfg)
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device="cuda")
    w = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device="cuda")
    b.route(p, lg, idx, w, b.workspace(p, b.WS_ROUTE))
    routed = sorted(set(idx.cpu().numpy().reshape(-1).tolist()))
    del lg, idx, w
    return upload(cfg, "cuda", experts=routed if len(routed) < cfg.E else None)


def measure_workload(cfg, args, b, torch, flush, pk, pk_src, steps):
    """One stated workload on this GPU: moe_forward as a CUDA-graph replay with L2 flushed
    between steps (CUDA events on the launching stream), the library's per-kernel events over
    the same number of steps, the dominant kernel's roofline and the SM clocks sampled while
    the timed steps ran."""
    local = int(os.environ.get("LOCAL_RANK", "0"))
    d = upload_routed(cfg, b, torch)
    f16 = cfg.weight_format == "bf16"
    wd = b.prepare_down_f16(d["w_down"]) if f16 else d["w_down"]
    sh = None
    if cfg.has_shared:
        sh = (d["shared_gate"], d["shared_up"], b.prepare_down_f16(d["shared_down"]))
    p = b.params_for(cfg, down_dtype=b.DOWN_F16 if f16 else b.DOWN_BF16, tile_ctas=TILE_ARG[args.tile])
    W = b.weights(d["w_gate"], d["w_up"], wd, d.get("s_gate"), d.get("s_up"), d.get("s_down"), shared=sh)
    ws = b.workspace(p, b.WS_FORWARD)
    out = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device="cuda")
    counts = torch.empty(cfg.E + int(cfg.has_shared), dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        b.forward(p, d["x"], d["logits"], W, out, ws)

    b.forward(p, d["x"], d["logits"], W, out, ws, counts_out=counts)
    cap = b.capacity(p)
    kept = counts[: cfg.E].cpu().numpy()
    kept = np.minimum(kept, cap) if cap is not None else kept
    P, touched = int(kept.sum()), int((kept > 0).sum())
    wl = workload_numbers(cfg, P, touched)
    for _ in range(3):
        flush()
        step()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(3):
        flush()
        graph.replay()
    torch.cuda.synchronize()
    s_ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    e_ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    with ClockSampler(local) as clocks:
        for i in range(steps):
            flush()
            s_ev[i].record(stream)
            graph.replay()
            e_ev[i].record(stream)
        torch.cuda.synchronize()
    ms = sum(a.elapsed_time(z) for a, z in zip(s_ev, e_ev)) / steps
    b.profile_collect()
    b.profile_enable(True)
    for _ in range(steps):
        flush()
        step()
    torch.cuda.synchronize()
    prof = b.profile_collect()
    b.profile_enable(False)
    if b.get_error(ws):
        raise RuntimeError(f"device error word set ({cfg.name})")
    roof = dominant_roofline(prof, wl, steps, ms, pk, pk_src, b.tile_ctas(p) == b.TILE_PAIR, f16, cfg.name)
    tflops = wl["flops"] / (ms / 1e3) / 1e12
    gbs = wl["bytes"] / (ms / 1e3) / 1e9
    entry = {"workload": workload_name(cfg), "ms_per_step": ms, "tokens_per_s": cfg.T / (ms / 1e3),
             "routed_rows": P, "touched_experts": touched,
             "tflops": tflops, "tensor_frac_of_peak": tflops / pk["bf16_tflops"],
             "gbs": gbs, "hbm_frac_of_peak": gbs / pk["hbm_gbs"], "bound": roof["bound"],
             "layer_frac": gbs / pk["hbm_gbs"] if roof["bound"] == "hbm" else tflops / pk["bf16_tflops"],
             "roofline": roof, "kernels_ms_per_step": {k: v[0] / steps for k, v in prof.items() if v[1]},
             "steps": steps, "step_launch": "CUDA graph replay of one moe_forward call, L2 flushed between steps",
             "clocks": clocks.summary()}
    del graph, d, W, ws, out, wd, sh
    torch.cuda.empty_cache()
    return entry


def extra_ops(cfg, b, torch):
    """Closures running one moe_expert_ffn_backward and one moe_route_stats call on the workload
    (routing and permutation done once beforehand), and the workspaces whose error words they set."""
    from synth.device import upload
    d = upload(cfg, "cuda")
    p = b.params_for(cfg, down_dtype=b.DOWN_F16)
    T, E, k, dm, f = cfg.T, cfg.E, cfg.k, cfg.d, cfg.f
    Et = E + int(cfg.has_shared)
    rows = b.max_rows(p)
    i32 = dict(dtype=torch.int32, device="cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    idx, w = torch.empty(T, k, **i32), torch.empty(T, k, **f32)
    counts, kept, offsets = torch.empty(Et, **i32), torch.empty(Et, **i32), torch.empty(Et + 1, **i32)
    st, sp, pr = torch.empty(rows, **i32), torch.empty(rows, **i32), torch.empty(T * k, **i32)
    b.route(p, d["logits"], idx, w, b.workspace(p, b.WS_ROUTE))
    b.permute(p, idx, counts, kept, offsets, st, sp, pr, b.workspace(p, b.WS_PERMUTE))
    sh = (d["shared_gate"], d["shared_up"], b.prepare_down_f16(d["shared_down"])) if cfg.has_shared else None
    W = b.weights(d["w_gate"], d["w_up"], b.prepare_down_f16(d["w_down"]), shared=sh)
    dout = torch.from_numpy(synth.dout(cfg)).cuda()
    g = dict(dx=torch.empty(T, dm, **f32), dwg=torch.empty(E, dm, f, **f32), dwu=torch.empty(E, dm, f, **f32),
             dwd=torch.empty(E, f, dm, **f32), dtw=torch.empty(T, k, **f32), dl=torch.empty(T, E, **f32))
    shg = tuple(torch.empty(s_, **f32) for s_ in ((dm, f), (dm, f), (f, dm))) if cfg.has_shared else None
    G = b.grads(g["dx"], g["dwg"], g["dwu"], g["dwd"], g["dtw"], g["dl"], shared=shg)
    wsb = b.workspace(p, b.WS_BACKWARD)
    stats = torch.empty(5, **f32)
    wss = b.workspace(p, b.WS_ROUTE_STATS)
    idx2, w2 = torch.empty(T, k, **i32), torch.empty(T, k, **f32)

    def bwd():
        b.expert_ffn_backward(p, d["x"], idx, w, offsets, st, sp, pr, W, dout, G, wsb)

    def rstats():
        b.route_stats(p, d["logits"], idx2, w2, stats, wss)

    return types.SimpleNamespace(bwd=bwd, rstats=rstats, ws=(wsb, wss), offsets=offsets, tensors=(d, W, G, g))


def measure_extra_rows(cfg, b, torch, flush, pk, pk_src, steps):
    """The layer's backward (moe_expert_ffn_backward) and the router with its telemetry
    (moe_route_stats) on the workload, each timed with CUDA events around a graph replay of one
    call, L2 flushed between calls. Backward work: 16 d f FLOPs per routed row (recomputed gate/up
    4df, dh 2df, dx 4df, weight gradients 6df) plus the shared expert's rows; telemetry: the
    logits read once (4 E bytes per token)."""
    T, E, dm, f = cfg.T, cfg.E, cfg.d, cfg.f
    ops = extra_ops(cfg, b, torch)
    bwd, rstats, (wsb, wss) = ops.bwd, ops.rstats, ops.ws
    out = {}
    for name, fn in (("backward", bwd), ("route_stats", rstats)):
        for _ in range(3):
            fn()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            fn()
        tot = 0.0
        for i in range(steps + 3):
            flush()
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record()
            graph.replay()
            s1.record()
            s1.synchronize()
            if i >= 3:
                tot += s0.elapsed_time(s1)
        out[name] = tot / steps
        del graph
    if b.get_error(wsb) or b.get_error(wss):
        raise RuntimeError("device error word set (backward / route_stats)")
    P = int(ops.offsets[E].item())
    counts = ops.offsets[1:E + 1] - ops.offsets[:E]
    touched = int((counts > 0).sum().item())
    fl = 16.0 * P * dm * f + (16.0 * T * dm * f if cfg.has_shared else 0.0)
    tfl = fl / (out["backward"] / 1e3) / 1e12
    # algorithmic bytes: each touched expert's weights read once (bf16 gate/up, fp16 W_down), every
    # expert's three fp32 weight gradients written (zeros for the untouched), x and dout read, dx
    # written, the routing weights and logits' gradients (small)
    nsh = 1 if cfg.has_shared else 0
    bb = ((touched + nsh) * 3.0 * dm * f * 2 + (E + nsh) * 3.0 * dm * f * 4 + T * dm * (2 + 4 + 4)
          + T * cfg.k * 4 * 3 + T * E * 4 * 2)
    bgbs = bb / (out["backward"] / 1e3) / 1e9
    t_tensor = fl / (pk["bf16_tflops"] * 1e12)
    t_hbm = bb / (pk["hbm_gbs"] * 1e9)
    gbs = T * E * 4 / (out["route_stats"] / 1e3) / 1e9
    res = {"backward": {"call": "moe_expert_ffn_backward", "ms": out["backward"], "flops": fl, "tflops": tfl,
                        "frac_of_peak": tfl / pk["bf16_tflops"], "peak_source": f"{pk_src} bf16_tflops (burst)",
                        "bytes": bb, "gbs": bgbs, "hbm_frac_of_peak": bgbs / pk["hbm_gbs"],
                        "bound": "hbm" if t_hbm > t_tensor else "tensor",
                        "frac_of_bound": max(t_hbm, t_tensor) / (out["backward"] / 1e3),
                        "work": "16 d f FLOPs per routed row: recomputed gate/up, dh, dx, three weight gradients; "
                                "bytes: touched weights read once, all fp32 weight gradients written, x, dout, dx"},
           "route_stats": {"call": "moe_route_stats", "ms": out["route_stats"], "gbs": gbs,
                           "frac_of_peak": gbs / pk["hbm_gbs"], "peak_source": f"{pk_src} hbm_gbs",
                           "work": "the logits read once (4 E bytes per token); latency-bound at this size"},
           "workload": workload_name(cfg), "steps": steps,
           "step_launch": "CUDA graph replay of one call, L2 flushed between calls"}
    del ops, bwd, rstats, wsb, wss
    torch.cuda.empty_cache()
    return res


# --------------------------------------------------------------------------- own arm

def own_arm(args, cfg):
    import torch
    from mixture_experts_routed_04_b200 import binding as b
    from synth.device import upload

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    d = upload(cfg, "cuda")
    # load-time preparation (outside every step): an fp16 copy of W_down, so the
    # down GEMM reads fp16 directly (the layer keeps h in fp16)
    prep_ms = None
    down_f16 = cfg.weight_format == "bf16"
    if down_f16:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        d["w_down_f16"] = b.prepare_down_f16(d["w_down"])
        if cfg.has_shared:
            d["shared_down_f16"] = b.prepare_down_f16(d["shared_down"])
        e1.record()
        e1.synchronize()
        prep_ms = e0.elapsed_time(e1)
    tile = TILE_ARG[args.tile]
    p = b.params_for(cfg, down_dtype=b.DOWN_F16 if down_f16 else b.DOWN_BF16, tile_ctas=tile)
    pair = b.tile_ctas(p) == b.TILE_PAIR
    sh = None
    if cfg.has_shared:
        sh = (d["shared_gate"], d["shared_up"], d["shared_down_f16" if down_f16 else "shared_down"])
    W = b.weights(d["w_gate"], d["w_up"], d["w_down_f16" if down_f16 else "w_down"], d.get("s_gate"),
                  d.get("s_up"), d.get("s_down"), shared=sh)
    ws = b.workspace(p, b.WS_FORWARD)
    out = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device="cuda")
    flush = L2Flush(torch)
    stream = torch.cuda.current_stream()

    def step():
        b.forward(p, d["x"], d["logits"], W, out, ws)

    # routed rows P and touched experts, from the layer's own per-expert counts
    counts = torch.empty(cfg.E + int(cfg.has_shared), dtype=torch.int32, device="cuda")
    b.forward(p, d["x"], d["logits"], W, out, ws, counts_out=counts)
    cap = b.capacity(p)
    kept = counts[: cfg.E].cpu().numpy()
    kept = np.minimum(kept, cap) if cap is not None else kept
    P, touched = int(kept.sum()), int((kept > 0).sum())
    wl = workload_numbers(cfg, P, touched)

    for _ in range(max(args.warmup, 3)):
        flush()
        step()
    torch.cuda.synchronize()
    if b.get_error(ws):
        raise RuntimeError("device error word set during warm-up")

    # The layer makes no host synchronisation, so one call captures into a CUDA
    # graph; every timed step replays it (all kernels run, on the real buffers).
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    torch.cuda.synchronize()

    def timed_steps(fn, n):
        s_ev = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        e_ev = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for i in range(n):
            flush()
            s_ev[i].record(stream)
            fn()
            e_ev[i].record(stream)
        torch.cuda.synchronize()
        return sum(a.elapsed_time(z) for a, z in zip(s_ev, e_ev))

    K = args.steps
    for _ in range(3):
        flush()
        graph.replay()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        total_ms = timed_steps(graph.replay, K)
    if dist:
        dist.barrier()
    total_ms = max_over_ranks(total_ms, dist, "cuda")
    eager_ms = max_over_ranks(timed_steps(step, max(3, min(K, 50))) / max(3, min(K, 50)), dist, "cuda")
    if b.get_error(ws):
        raise RuntimeError("device error word set during the timed steps")
    ms = total_ms / K

    # per-kernel times, CUDA events inside the library around each launch (same steps, same flushes)
    b.profile_collect()
    b.profile_enable(True)
    for i in range(K):
        flush()
        step()
    torch.cuda.synchronize()
    prof = b.profile_collect()
    b.profile_enable(False)

    # the same steps with W_down given as bf16 (converted to fp16 per tile inside the down GEMM)
    ms_down_bf16 = None
    if down_f16:
        p_bf = b.params_for(cfg, down_dtype=b.DOWN_BF16, tile_ctas=tile)
        W_bf = b.weights(d["w_gate"], d["w_up"], d["w_down"],
                         shared=(d["shared_gate"], d["shared_up"], d["shared_down"]) if cfg.has_shared else None)
        kb = max(3, min(K, 50))
        tot = 0.0
        for i in range(kb + 3):
            flush()
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            b.forward(p_bf, d["x"], d["logits"], W_bf, out, ws)
            s1.record(stream)
            s1.synchronize()
            if i >= 3:
                tot += s0.elapsed_time(s1)
        ms_down_bf16 = tot / kb

    # End to end through the host-buffer entry points: every step copies its x and logits in
    # from pinned host memory and its output back. "value": a pipelined loop over three streams
    # (moe_forward_host_async, separate workspaces and host buffers per stream), so one step's
    # copies overlap other steps' kernels and copies, as a serving loop runs; "sync": one
    # moe_forward_host call per step (copies, layer and copy back in sequence, then a host
    # synchronisation).
    e2e = None
    if not args.no_e2e:
        h2d = cfg.T * cfg.d * 2 + cfg.T * cfg.E * 4
        d2h = cfg.T * cfg.d * 4
        ek = max(3, min(K, 50))
        slots = [dict(stream=torch.cuda.Stream(), ws=b.workspace(p, b.WS_FORWARD_HOST),
                      x=d["x"].cpu().pin_memory(), l=d["logits"].cpu().pin_memory(),
                      o=torch.empty(cfg.T, cfg.d, dtype=torch.float32).pin_memory()) for _ in range(3)]

        def step_async(i):
            sl = slots[i % len(slots)]
            b.forward_host_async(p, sl["x"], sl["l"], W, sl["o"], sl["ws"], stream=sl["stream"])

        for i in range(2 * len(slots)):
            step_async(i)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for sl in slots:
            sl["stream"].wait_event(t0)
        for i in range(ek):
            step_async(i)
        for sl in slots:
            ev = torch.cuda.Event()
            ev.record(sl["stream"])
            stream.wait_event(ev)
        t1.record(stream)
        t1.synchronize()
        for sl in slots:
            if b.get_error(sl["ws"]):
                raise RuntimeError("device error word set (pipelined end-to-end loop)")
        pipe_ms = max_over_ranks(t0.elapsed_time(t1) / ek, dist, "cuda")

        pe = slots[0]["ws"]
        x_h, l_h, o_h = slots[0]["x"], slots[0]["l"], slots[0]["o"]
        for _ in range(3):
            b.forward_host(p, x_h, l_h, W, o_h, pe)
        e_ms = 0.0
        for _ in range(ek):
            flush()
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            b.forward_host(p, x_h, l_h, W, o_h, pe)
            s1.record(stream)
            s1.synchronize()
            e_ms += s0.elapsed_time(s1)
        e_ms = max_over_ranks(e_ms, dist, "cuda")
        e2e = {"value": aggregate_tokens_per_s(cfg.T, world, pipe_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": pipe_ms,
               "mode": "pipelined: moe_forward_host_async on 3 streams, pinned host buffers; no L2 flush "
                       "(the touched weights exceed L2)",
               "sync": {"value": aggregate_tokens_per_s(cfg.T, world, e_ms / ek), "ms_per_step": e_ms / ek,
                        "mode": "one moe_forward_host call per step (L2 flushed between steps)"}}

    pk, pk_src = peaks()
    roof = dominant_roofline(prof, wl, K, ms, pk, pk_src, pair, down_f16, cfg.name)

    line = None
    if rank == 0:
        tflops = wl["flops"] / (ms / 1e3) / 1e12
        gbs = wl["bytes"] / (ms / 1e3) / 1e9
        line = {"metric": METRIC, "value": aggregate_tokens_per_s(cfg.T, world, ms), "unit": "tokens/s",
                "n_gpus": world,
                "steps": K, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": workload_name(cfg), "tokens_per_gpu": cfg.T, "routed_rows": P,
                           "touched_experts": touched, "parallelism": f"replicas x{world} (no exchange)",
                           "l2": "flushed between steps (256 MiB write + 256 MiB read), touched weights also larger than L2"},
                "tflops": tflops, "tensor_frac_of_peak": tflops / pk["bf16_tflops"],
                "gbs": gbs, "hbm_frac_of_peak": gbs / pk["hbm_gbs"], "peaks": pk_src,
                "roofline": roof,
                "kernels_ms_per_step": {k: v[0] / K for k, v in prof.items() if v[1]},
                "gpu_launches": b.launch_count(p, b.WS_FORWARD) * K,
                "step_launch": "CUDA graph replay of one moe_forward call",
                "ms_per_step_eager": eager_ms,
                "w_down": "fp16 copy prepared once at load time" if down_f16 else "n/a",
                "tile_ctas": b.tile_ctas(p),
                "w_down_prep_ms": prep_ms, "ms_per_step_w_down_bf16": ms_down_bf16,
                "clocks": clocks.summary(), "e2e": e2e}
    if rank == 0 and world == 1 and not args.no_per_config:
        # the other stated workloads, measured in the same run (graph replay, L2 flushed);
        # one GPU only, so that no rank waits at a barrier meanwhile
        del graph
        torch.cuda.empty_cache()
        pc = {}
        for name in PER_CONFIG:
            if name != cfg.name:
                pc[name] = measure_workload(synth.CONFIGS[name], args, b, torch, flush, pk, pk_src,
                                            max(3, min(args.steps, 20)))
        line["per_config"] = pc
        # the scope table's next rows on this workload: the backward and the router telemetry
        line["next_rows"] = measure_extra_rows(cfg, b, torch, flush, pk, pk_src, max(3, min(args.steps, 20)))
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(cfg)
        print(json.dumps(line), flush=True)
    return 0


def prepared_layer(cfg, b, torch, stream_max_rows=-1, tile_ctas=0):
    """Device inputs, load-time fp16 W_down, params, weights struct, workspace, output."""
    from synth.device import upload
    d = upload(cfg, "cuda")
    f16 = cfg.weight_format == "bf16"
    wd = b.prepare_down_f16(d["w_down"]) if f16 else d["w_down"]
    sh = None
    if cfg.has_shared:
        sh = (d["shared_gate"], d["shared_up"], b.prepare_down_f16(d["shared_down"]))
    p = b.params_for(cfg, down_dtype=b.DOWN_F16 if f16 else b.DOWN_BF16, stream_max_rows=stream_max_rows,
                     tile_ctas=tile_ctas)
    W = b.weights(d["w_gate"], d["w_up"], wd, d.get("s_gate"), d.get("s_up"), d.get("s_down"), shared=sh)
    out = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device="cuda")
    return d, p, W, out


def profile_calls(args, cfg):
    """Only `n` calls of one entry point (the first one warms up): a short, fixed launch sequence
    for ncu. --profile-op: moe_forward (default), moe_expert_ffn_backward or moe_route_stats."""
    import torch
    from mixture_experts_routed_04_b200 import binding as b
    if args.profile_op == "forward":
        d, p, W, out = prepared_layer(cfg, b, torch, tile_ctas=TILE_ARG[args.tile])
        ws = b.workspace(p, b.WS_FORWARD)
        wss = (ws,)

        def fn():
            b.forward(p, d["x"], d["logits"], W, out, ws)
    else:
        ops = extra_ops(cfg, b, torch)
        wss = ops.ws
        fn = ops.bwd if args.profile_op == "backward" else ops.rstats
    torch.cuda.synchronize()
    for _ in range(args.profile_calls):
        fn()
    torch.cuda.synchronize()
    if any(b.get_error(w) for w in wss):
        raise RuntimeError("device error word set")
    print(json.dumps({"profile_calls": args.profile_calls, "op": args.profile_op, "workload": workload_name(cfg)}))
    return 0


def sweep_threshold(args, cfg):
    """moe_forward time (graph replay, L2 flushed) for each streaming threshold."""
    import torch
    from mixture_experts_routed_04_b200 import binding as b
    d, _, W, out = prepared_layer(cfg, b, torch)
    flush = L2Flush(torch)
    res = {}
    for smax in (0, 4, 8, 16, 24, 32, 48, 64, 96, 128):
        p = b.params_for(cfg, down_dtype=b.DOWN_F16 if cfg.weight_format == "bf16" else b.DOWN_BF16,
                         stream_max_rows=smax)
        ws = b.workspace(p, b.WS_FORWARD)
        for _ in range(3):
            b.forward(p, d["x"], d["logits"], W, out, ws)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            b.forward(p, d["x"], d["logits"], W, out, ws)
        tot, n = 0.0, max(args.steps, 5)
        for i in range(n + 3):
            flush()
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record()
            g.replay()
            s1.record()
            s1.synchronize()
            if i >= 3:
                tot += s0.elapsed_time(s1)
        if b.get_error(ws):
            raise RuntimeError("device error word set")
        res[smax] = tot / n
        del g, ws
    print(json.dumps({"sweep_stream_max_rows_ms": res, "workload": workload_name(cfg), "steps": max(args.steps, 5)}))
    return 0


def variant_table_sweep(args):
    """The measured table behind the library's variant choice: moe_forward time (graph replay,
    L2 flushed) with every expert on the tcgen05 tiles against every routed expert on the
    weight-streaming kernels, on decode-shaped layers (d=4096, f=1536, E=256, top-8, shared
    expert) whose routing gives `touched` experts exactly `rows` rows each. One JSON line."""
    import torch
    from mixture_experts_routed_04_b200 import binding as b
    from synth.device import upload
    touched_list = (8, 12, 16, 20, 24, 32, 48)
    rows_list = (1, 2, 4, 8, 16)
    base = synth.LayerConfig("vt", T=48, d=4096, f=1536, E=256, k=8, bias="balanced", touched=48,
                             has_shared=True, f_shared=1536)
    d = upload(base, "cuda", experts=range(max(touched_list)))
    wd = b.prepare_down_f16(d["w_down"])
    sh = (d["shared_gate"], d["shared_up"], b.prepare_down_f16(d["shared_down"]))
    W = b.weights(d["w_gate"], d["w_up"], wd, shared=sh)
    flush = L2Flush(torch)
    res = []
    for n in touched_list:
        for r in rows_list:
            if (r * n) % base.k:
                continue
            cfg = base.replace(T=r * n // base.k, touched=n)
            x = torch.from_numpy(synth.x_bits(cfg).view(np.int16)).cuda().view(torch.bfloat16)
            lg = torch.from_numpy(synth.logits(cfg)).cuda()
            out = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device="cuda")
            row = {"touched": n, "rows": r, "T": cfg.T, "gateup_tiles": (n + 1) * ((cfg.f + 127) // 128)}
            for name, v in (("tiles", b.VARIANT_TENSOR), ("stream", b.VARIANT_STREAM)):
                p = b.params_for(cfg, variant=v, down_dtype=b.DOWN_F16)
                ws = b.workspace(p, b.WS_FORWARD)
                for _ in range(3):
                    b.forward(p, x, lg, W, out, ws)
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    b.forward(p, x, lg, W, out, ws)
                tot, k = 0.0, max(args.steps, 5)
                for i in range(k + 3):
                    flush()
                    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    s0.record()
                    g.replay()
                    s1.record()
                    s1.synchronize()
                    if i >= 3:
                        tot += s0.elapsed_time(s1)
                if b.get_error(ws):
                    raise RuntimeError("device error word set")
                row[name + "_us"] = 1e3 * tot / k
                del g, ws
            res.append(row)
    print(json.dumps({"variant_table": res, "sms": torch.cuda.get_device_properties(0).multi_processor_count,
                      "steps": max(args.steps, 5)}))
    return 0


def main():
    args = parse()
    cfg = synth.CONFIGS[args.config]
    if args.tokens:
        cfg = cfg.replace(T=args.tokens)
    if args.experts:
        cfg = cfg.replace(E=args.experts)
    if args.impl == "reference":
        return reference_arm(args, cfg)
    if args.profile_calls:
        return profile_calls(args, cfg)
    if args.sweep_threshold:
        return sweep_threshold(args, cfg)
    if args.variant_table:
        return variant_table_sweep(args)
    return own_arm(args, cfg)


if __name__ == "__main__":
    sys.exit(main())
