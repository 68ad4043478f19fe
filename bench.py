#!/usr/bin/env python
"""Multi-Router Latent MoE layer forward: tokens/s on B200, and its roofline.

One step = one forward of the whole layer (down-projection, routers + top-k,
dispatch, gate/up + SiLU-GLU, expert down-projection, combine + RMSNorm,
up-projection) over one batch of T synthetic tokens already in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config c2_prefill]
    python bench.py --impl reference ...     # the CPU oracle on a bounded sample

For N > 1 launch with torchrun; every rank runs its own batch on its own GPU
(weak scaling, no data-path collective) and rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import glob
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer fwd tokens/s on 1 B200 (T=8192, full width); % of roofline"
UNIT = "tokens/s"
KERNELS_PER_STEP = 11          # launches of this library's kernels per forward (+1 router merge)


def kernels_per_step(s, sms: int) -> int:
    """Kernel launches of one forward: 11, plus the router's merge kernel when
    the library splits the expert chunks of a token tile over several CTAs
    (same rule as router_parts in the library), or plus two (the score pass
    and the top-k) when it splits the router's K range instead (small T; same
    rule as router_ksplit)."""
    ec = 16
    for c in (256, 128, 64, 32, 16):
        if c * s.n_routers <= 256 and s.n_experts % c == 0:
            ec = c
            break
    m_tiles = (s.T + 127) // 128
    chunks = s.n_experts // ec
    # FP8 variant: the x and n quantisers replace nothing and the z quantiser
    # replaces the gather; h is quantised in the gate/up GEMM's epilogue,
    # except with FP4 expert weights and a d_lat that does not split into
    # 256-wide slices, where a quantiser pass over h follows the GEMM
    extra = (3 if s.fp4 and s.d_lat % 256 else 2) if s.fp8 else 0
    if 2 * m_tiles * chunks <= 148 and s.d_lat // 64 % 2 == 0:
        return KERNELS_PER_STEP + 2 + extra
    parts = 1
    while parts * 2 <= chunks and chunks % (parts * 2) == 0 and m_tiles * parts * 2 <= sms:
        parts *= 2
    return KERNELS_PER_STEP + (1 if parts > 1 else 0) + extra
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="c2_prefill")
    ap.add_argument("--tokens", type=int, default=None, help="override T (small profiling runs)")
    ap.add_argument("--experts", type=int, default=None,
                    help="override the routed expert count (small profiling runs only)")
    ap.add_argument("--cpu-sample", type=int, default=256,
                    help="tokens of the workload the CPU oracle baseline runs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--aggregation", choices=["mean", "sum", "max"], default=None,
                    help="router score aggregation (default: the config's, the mean)")
    ap.add_argument("--routers", type=int, default=None, help="override the number of routers R")
    ap.add_argument("--no-train-summary", action="store_true",
                    help="leave the training-step summary out of the forward's line")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="leave the c1_decode / c3_skew / c4_fp8 / c1_fp4 summaries out of the headline's line")
    ap.add_argument("--train", action="store_true",
                    help="time a training step (forward that keeps its activations + backward) instead")
    ap.add_argument("--route-only", action="store_true",
                    help="time routing from x alone (down-projection, routers, top-k, dispatch: "
                         "mrlmoe_route) and print its own JSON line; bf16 configs")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def csrc_hash() -> str:
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "sparse_moe_layer_mean_b200", "csrc", "*"))):
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", f"{kernel}__{workload}.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("csrc_hash") != csrc_hash():
        return None
    return d.get("dram_bytes_per_launch_full")


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during a region
    (every 20 ms, so a short timed region still gets several samples)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.samples = []
        self.window = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20", "-i", gpu_id], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.th = threading.Thread(target=self._read, daemon=True)
        self.th.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def begin(self):
        self.window = [time.time(), None]

    def end(self):
        if self.window:
            self.window[1] = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        t0, t1 = self.window
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, mx, reasons, power = [], None, set(), []
        for ts, line in self.samples:
            if not (t0 - 0.05 <= ts <= t1 + 0.15):
                continue
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_median": statistics.median(power) if power else None}


def max_over_ranks(values, device):
    """Element-wise max of a list of floats over all ranks of the default group."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(world: int, tokens_per_rank: int, steps: int, max_ms: float) -> float:
    """Whole-job tokens/s: every rank processes its own batch each step."""
    return world * tokens_per_rank * steps / (max_ms * 1e-3)


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def shape_from_args(args):
    import dataclasses
    import workloads as W
    s = W.CONFIGS[args.config]
    if args.tokens:
        s = s.with_T(args.tokens)
    if args.experts:
        s = dataclasses.replace(s, n_experts=args.experts, name=f"{s.name}_E{args.experts}")
    if args.routers:
        s = dataclasses.replace(s, n_routers=args.routers, name=f"{s.name}_R{args.routers}")
    if args.aggregation and args.aggregation != s.aggregation:
        s = dataclasses.replace(s, aggregation=args.aggregation, name=f"{s.name}_{args.aggregation}")
    return s


def layer_bytes_flops(s, counts):
    """Algorithmic bytes and FLOPs of one forward (weights of touched experts,
    the dense weights, x read and y written)."""
    import workloads as W
    touched = int((counts > 0).sum())
    D, L, E, F, R, T = s.d_model, s.d_lat, s.n_experts, s.d_ff, s.n_routers, s.T
    wb = 1 if s.fp8 else 2                       # bytes per projection weight
    we = 0.5 if s.fp4 else wb                    # bytes per expert weight (e2m1: half a byte)
    expert = int(3 * F * L * we)
    byts = (touched + 1) * expert + (L * D + D * L) * wb + R * E * L * 2 + L * 4 + 2 * T * D * 2
    return byts, W.flops_per_token(s) * T, touched


def glu_kernel_bytes(s, touched):
    """Algorithmic bytes of one gate/up + SiLU-GLU launch, counted as the
    layer's byte count counts them: the gate and up weights of the touched
    experts and of the shared expert (one 128-wide d_ff slice of both per
    unit, 2 * 128 * d_lat * 2 bytes in bf16).  The dispatched latent rows it
    reads and the h it writes are intermediates and are not counted; the
    profiled DRAM traffic shows them."""
    we = 0.5 if s.fp4 else (1 if s.fp8 else 2)
    return int((touched + 1) * 2 * s.d_ff * s.d_lat * we)


def glu_kernel_flops(s):
    """FLOPs of one gate/up launch: 2 * rows * d_lat * 2 d_ff."""
    return 2 * (s.T * s.top_k + s.T) * s.d_lat * 2 * s.d_ff


def fp8_peak_probe(dev, n=8192, seconds=1.0):
    """Sustained e4m3 GEMM throughput of the vendor library on this GPU
    (torch._scaled_mm, n x n x n, per-tensor scales), for context next to the
    assumed e4m3 peak (2 x the measured sustained bf16 peak)."""
    import torch
    try:
        a = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn).t()
        one = torch.ones((), device=dev)
        for _ in range(3):
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        e1.record()
        torch.cuda.synchronize()
        reps = max(10, int(seconds * 1e3 / max(e0.elapsed_time(e1), 1e-3)))
        e0.record()
        for _ in range(reps):
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        e1.record()
        torch.cuda.synchronize()
        tflops = 2.0 * n ** 3 * reps / (e0.elapsed_time(e1) * 1e-3) / 1e12
        return {"tflops": round(tflops, 1), "gemm": f"{n}x{n}x{n} e4m3 -> bf16, torch._scaled_mm",
                "reps": reps}
    except (RuntimeError, AttributeError) as e:   # not available in this torch build
        return {"unavailable": str(e).splitlines()[0][:200]}


_E4M3_PROBE = {}


def e4m3_peak(dev, peaks, peak_kind):
    """The tensor peak an e4m3 kernel is measured against: the vendor
    library's sustained e4m3 GEMM rate on this GPU (fp8_peak_probe, taken once
    per process), or 2 x the sustained bf16 peak where the probe cannot run."""
    if dev not in _E4M3_PROBE:
        _E4M3_PROBE[dev] = fp8_peak_probe(dev)
    probe = _E4M3_PROBE[dev]
    if "tflops" in probe:
        return probe["tflops"], "measured (vendor e4m3 GEMM probe on this GPU: " + probe["gemm"] + ")", probe
    return peaks["bf16_tflops_sustained"] * 2, f"of {peak_kind} (sustained bf16 x 2 for e4m3, assumed)", probe


def glu_roofline(s, glu_ms, touched, peaks, peak_kind, dev):
    """The gate/up kernel against its bound, the larger of its two floors:
    the touched experts' gate and up weight bytes at the measured HBM copy
    rate, or its FLOPs at the tensor peak of its operand type (e4m3 / e2m1:
    the vendor e4m3 GEMM probe; bf16: the measured sustained bf16 peak)."""
    if s.fp8:
        tpeak, tkind, _ = e4m3_peak(dev, peaks, peak_kind)
    else:
        tpeak, tkind = peaks["bf16_tflops_sustained"], f"of {peak_kind} (sustained bf16)"
    byts, flops = glu_kernel_bytes(s, touched), glu_kernel_flops(s)
    if flops / (tpeak * 1e12) > byts / (peaks["hbm_gbs"] * 1e9):
        achieved = flops / (glu_ms * 1e-3) / 1e12
        return {"bound": "tensor", "achieved": achieved, "peak": tpeak, "unit": "TFLOP/s",
                "frac": achieved / tpeak, "peak_kind": tkind}
    achieved = byts / (glu_ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "peak_kind": f"of {peak_kind}"}


OTHER_CONFIGS = ("c1_decode", "c3_skew", "c4_fp8", "c1_fp4")


def config_summary(name, dev, bf16_weights, steps=20, warmup=3, shape=None):
    """One more workload, timed on its own after the headline's timed region:
    ms per forward (CUDA events on the launching stream), tokens/s, the
    layer's roofline fraction and the stage times; the skewed workload also
    times its balancing-bias update.  The bf16 workloads reuse the headline's
    weights (same layer shape); the e4m3 one draws its own.  ``shape``
    replaces the named config's (e.g. another router aggregation)."""
    import torch
    import sparse_moe_layer_mean_b200 as M
    import workloads as W
    try:
        s = shape if shape is not None else W.CONFIGS[name]
        weights = W.make_layer_weights(s, dev) if s.fp8 else bf16_weights
        x = W.make_x(s, dev)
        bias = W.make_bias(s, dev)
        layer = M.MRLMoELayer(s, weights, device=dev)
        y = torch.empty(s.T, s.d_model, dtype=torch.bfloat16, device=dev)
        routing = layer.routing_buffers()
        for _ in range(max(3, warmup)):
            layer(x, bias, y=y, routing=routing)
        torch.cuda.synchronize()
        if layer.device_status() != 0:
            raise RuntimeError("device status non-zero after warm-up")
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(M._native.NUM_STAGE_EVENTS)]
               for _ in range(steps)]
        for row in evs:          # torch creates the event handles on their first record
            for e in row:
                e.record()
        torch.cuda.synchronize()
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record()
        for i in range(steps):
            M.mrlmoe_forward_timed(layer.cfg, layer.cw, bias, x, y, None, layer.workspace, layer.ws_bytes, evs[i])
        stop.record()
        torch.cuda.synchronize()
        if layer.device_status() != 0:
            raise RuntimeError("device status non-zero after the timed region")
        ms = start.elapsed_time(stop) / steps
        stage = [sum(r[j].elapsed_time(r[j + 1]) for r in evs) / steps for j in range(M._native.NUM_STAGE_EVENTS - 1)]
        counts = routing["counts"].cpu()
        byts, flops, touched = layer_bytes_flops(s, counts)
        peaks, peak_kind = load_peaks()
        if s.fp8:
            tpeak, tkind, _ = e4m3_peak(dev, peaks, peak_kind)
        else:
            tpeak, tkind = peaks["bf16_tflops_sustained"], f"{peak_kind}"
        t_bytes, t_flops = byts / (peaks["hbm_gbs"] * 1e9), flops / (tpeak * 1e12)
        out = {"T": s.T, "dtype": "e4m3" if s.fp8 else "bf16", "ms_per_step": round(ms, 4),
               "tokens_per_s": s.T / (ms * 1e-3), "steps": steps, "warmup": max(3, warmup),
               "touched_experts": touched,
               "layer_roofline": {"bound": "hbm" if t_bytes >= t_flops else "tensor",
                                  "t_bytes_ms": round(t_bytes * 1e3, 4), "t_flops_ms": round(t_flops * 1e3, 4),
                                  "frac": max(t_bytes, t_flops) / (ms * 1e-3),
                                  "peaks": f"{peak_kind}" + (f"; e4m3 peak {tpeak} TFLOP/s {tkind}" if s.fp8 else "")},
               "stage_ms": dict(zip(M._native.STAGES, [round(v, 4) for v in stage])),
               "gate_up_roofline": glu_roofline(s, stage[M._native.STAGES.index("gate_up_glu")], touched, peaks,
                                                peak_kind, dev),
               "gpu_launches": kernels_per_step(s, torch.cuda.get_device_properties(dev).multi_processor_count) * steps}
        if s.bias_kind == "zipf":
            c = counts.double()
            out["max_over_mean_load"] = round(float(c.max() / c.mean()), 2)
            b2 = bias.clone()
            for _ in range(3):
                M.mrlmoe_bias_update(layer.cfg, routing["counts"], b2, 1e-3)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(steps):
                M.mrlmoe_bias_update(layer.cfg, routing["counts"], b2, 1e-3)
            b.record()
            torch.cuda.synchronize()
            out["bias_update_ms"] = round(a.elapsed_time(b) / steps, 5)
        del layer, routing, y, x
        if s.fp8:
            del weights
        torch.cuda.empty_cache()
        return out
    except Exception as e:  # the headline line is printed either way
        return {"error": str(e).splitlines()[0][:200] if str(e) else type(e).__name__}


def ep_summary(n, dev, bf16_weights, T=4096, iters=5, steps=20):
    """The expert-parallel form emulated on one GPU: n ranks in one process,
    the headline's full-width weights, T tokens per rank.  Rank d routes its
    own tokens, runs experts [d E/n, (d+1) E/n) on every rank's rows for them
    and combines its tokens (sparse_moe_layer_mean_b200.ep.emulate_forward).
    Each phase's device time per rank comes from CUDA events (median of
    ``iters`` runs), next to the single-GPU forward of one rank's T tokens.
    The exchanges are device copies of the slices here; on n GPUs they cross
    NVLink, so the line gives the bytes each rank sends and receives, not a
    transfer time (the exchange over NVLink is unmeasured: every GPU call on
    this pool has one GPU)."""
    import torch
    import sparse_moe_layer_mean_b200 as M
    import workloads as W
    from sparse_moe_layer_mean_b200 import ep as EP
    try:
        s = W.CONFIGS["c2_prefill"].with_T(T)
        ranks = [EP.ExpertParallelRank(s, bf16_weights, r, n, device=dev) for r in range(n)]
        xs = [W.make_x(s, dev, seed=100 + r) for r in range(n)]
        bias = W.make_bias(s, dev)
        EP.emulate_forward(ranks, xs, bias)                      # warm-up
        torch.cuda.synchronize()
        runs, splits = [], None
        for _ in range(iters):
            ev = {}
            EP.emulate_forward(ranks, xs, bias, events=ev)
            torch.cuda.synchronize()
            splits = ev.pop("splits")
            runs.append({k: [a.elapsed_time(b) for a, b in v] for k, v in ev.items()})
        if any(rk.status() != 0 for rk in ranks):
            raise RuntimeError("device status non-zero after the expert-parallel runs")

        def med(vals):
            return sorted(vals)[len(vals) // 2]
        phase = {ph: [round(med([r[ph][i] for r in runs]), 4) for i in range(n)]
                 for ph in ("dispatch", "experts", "combine")}
        per_rank = [phase["dispatch"][i] + phase["experts"][i] + phase["combine"][i] for i in range(n)]
        del ranks
        torch.cuda.empty_cache()
        # the single-GPU forward of one rank's tokens, same weights
        layer = M.MRLMoELayer(s, bf16_weights, device=dev)
        y = torch.empty(T, s.d_model, dtype=torch.bfloat16, device=dev)
        for _ in range(3):
            layer(xs[0], bias, y=y)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            layer(xs[0], bias, y=y)
        b.record()
        torch.cuda.synchronize()
        if layer.device_status() != 0:
            raise RuntimeError("device status non-zero after the single-GPU forward")
        fwd = a.elapsed_time(b) / steps
        L = s.d_lat
        out_rows = [sum(splits[r][d] for d in range(n) if d != r) for r in range(n)]
        in_rows = [sum(splits[q][r] for q in range(n) if q != r) for r in range(n)]
        return {"n_ranks": n, "tokens_per_rank": T, "experts_per_rank": s.n_experts // n,
                "phase_ms": phase, "compute_ms_per_rank_max": round(max(per_rank), 4),
                "single_gpu_forward_ms": round(fwd, 4),
                "emulated_exchange_copies_ms": {ph: round(med([r[ph][0] for r in runs]), 4) for ph in ("rows", "back")},
                "bytes_per_rank_max": {"rows_out_bf16": max(out_rows) * L * 2, "rows_in_bf16": max(in_rows) * L * 2,
                                       "outputs_back_fp32": max(in_rows) * L * 4},
                "exchange": "unmeasured (one GPU): device copies stand in for the NVLink all-to-alls"}
    except Exception as e:  # the headline line is printed either way
        return {"error": str(e).splitlines()[0][:200] if str(e) else type(e).__name__}


def cpu_baseline(s, weights_dev, x_dev, bias_dev, ntok):
    """The CPU oracle, as it stands, on the first ntok tokens of the batch."""
    import torch
    import oracle as O
    wh = {k: v.cpu() for k, v in weights_dev.items()}
    xs = x_dev[:ntok].cpu()
    b = bias_dev.cpu()
    t0 = time.perf_counter()
    O.forward(xs, wh, b, s.top_k, s.rms_eps, fp8=s.fp8, fp4=s.fp4)
    dt = time.perf_counter() - t0
    return {"value": ntok / dt, "unit": UNIT, "cores": torch.get_num_threads(), "kind": "oracle",
            "sample": f"first {ntok} tokens of the {s.name} batch (fp64 oracle, {dt:.1f} s)"}


def run_reference(args):
    """--impl reference: the CPU oracle timed on the host cores, one bounded
    sample of the workload per step."""
    world, rank, local = dist_setup()
    if rank != 0:
        return
    import torch
    import oracle as O
    import workloads as W
    s = shape_from_args(args)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    w = {k: v.cpu() for k, v in W.make_layer_weights(s, dev).items()}
    per_step = 1
    n = args.warmup + args.steps
    x = W.make_x(s, dev, T=min(s.T, n * per_step)).cpu()
    b = W.make_bias(s, "cpu")
    for i in range(args.warmup):
        O.forward(x[i:i + 1], w, b, s.top_k, s.rms_eps, fp8=s.fp8, fp4=s.fp4)
    t0 = time.perf_counter()
    for i in range(args.steps):
        j = (args.warmup + i) % x.shape[0]
        O.forward(x[j:j + per_step], w, b, s.top_k, s.rms_eps, fp8=s.fp8, fp4=s.fp4)
    dt = time.perf_counter() - t0
    v = args.steps * per_step / dt
    line = {"metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": s.name, "T": s.T, "sample_tokens_per_step": per_step},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": torch.get_num_threads(),
                             "kind": "oracle",
                             "sample": f"{per_step} token of the {s.name} batch per step"},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_route_only(args):
    """Routing from x (S1-S6 through mrlmoe_route) on one GPU: only the
    down-projection and router weights are built.  Each call is timed alone
    with CUDA events, an L2 flush (a 256 MB write) between calls."""
    import torch
    import sparse_moe_layer_mean_b200 as M
    import workloads as W
    s = shape_from_args(args)
    if s.fp8:
        raise SystemExit("--route-only runs the bf16 configs")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    weights = W.make_routing_weights(s, dev)
    x = W.make_x(s, dev)
    bias = W.make_bias(s, dev)
    layer = M.MRLMoELayer(s, weights, device=dev)
    routing = layer.routing_buffers()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(max(3, args.warmup)):
        layer.route(bias, x=x, routing=routing)
    torch.cuda.synchronize()
    times = []
    for _ in range(args.steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        layer.route(bias, x=x, routing=routing)
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    st = layer.device_status()
    if st != 0:
        raise SystemExit(f"device status {M.status_string(st)}")
    ms = sum(times) / len(times)
    print(json.dumps({"metric": "routing from x, tokens/s (down-projection, routers, top-k, dispatch)",
                      "value": s.T / (ms * 1e-3), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
                      "warmup": max(3, args.warmup), "ms_per_step": ms, "higher_is_better": True,
                      "dtype": "bf16", "data": "synthetic",
                      "config": {"workload": f"{s.name} routing: T={s.T} tokens, d_model {s.d_model} -> "
                                             f"d_lat {s.d_lat}, {s.n_experts} experts top-{s.top_k}, "
                                             f"R={s.n_routers} routers, bf16",
                                 "T": s.T, "l2": "flushed between calls"}}),
          flush=True)


TRAIN_METRIC = "MoE-layer training step (fwd + bwd) tokens/s on 1 B200 (full width); % of roofline"
BACKWARD_KERNELS = 12          # launches of this library's kernels per backward


def wgrad_kernel_bytes(s):
    """Algorithmic bytes of the expert weight-gradient launch: the fp32
    gradients of gate, up and down for every routed expert and the shared
    one written once, and its operands (dg, du, z, do, h rows) read once."""
    rows = s.T * s.top_k + s.T
    return 3 * (s.n_experts + 1) * s.d_ff * s.d_lat * 4 + rows * (3 * s.d_ff + 2 * s.d_lat) * 2


def train_flops(s):
    """FLOPs of one training step: the forward plus twice its GEMM FLOPs
    (dgrad and wgrad of every GEMM)."""
    import workloads as W
    return 3 * W.flops_per_token(s) * s.T


def _time_training(layer, x, bias, dy, cg, steps, warmup, clocks=None):
    """Warm-up, then `steps` training steps (forward_train + backward) between
    CUDA events on the current stream; returns (total ms, mean forward_train
    ms, mean ms of each backward stage)."""
    import torch
    import sparse_moe_layer_mean_b200 as M
    y = torch.empty(layer.cfg.T, layer.cfg.d_model, dtype=torch.bfloat16, device=x.device)
    for _ in range(max(3, warmup)):
        layer.forward_train(x, bias, y=y)
        M.mrlmoe_backward(layer.cfg, layer.cw, x, dy, cg, layer.workspace, layer.ws_bytes)
    torch.cuda.synchronize()
    if layer.device_status() != 0:
        raise RuntimeError("device status non-zero after warm-up")
    NB = M._native.NUM_BACKWARD_EVENTS
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(NB + 1)] for _ in range(steps)]
    for row in evs:
        for e in row:
            e.record()
    torch.cuda.synchronize()
    if clocks is not None:
        time.sleep(0.6)
        clocks.begin()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(steps):
        evs[i][0].record()
        layer.forward_train(x, bias, y=y)
        M.mrlmoe_backward_timed(layer.cfg, layer.cw, x, dy, cg, layer.workspace, layer.ws_bytes, evs[i][1:])
    stop.record()
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.end()
    if layer.device_status() != 0:
        raise RuntimeError("device status non-zero after the timed region")
    ms = start.elapsed_time(stop)
    fwd_ms = sum(r[0].elapsed_time(r[1]) for r in evs) / steps
    stage = [sum(r[j + 1].elapsed_time(r[j + 2]) for r in evs) / steps for j in range(NB - 1)]
    return ms, fwd_ms, stage


def train_summary(s, dev, weights, x, bias, steps=10, warmup=3):
    """The training step (forward_train + backward) on the same workload,
    timed on its own after the forward's timed region: a summary object for
    the forward's JSON line."""
    import torch
    import sparse_moe_layer_mean_b200 as M
    import workloads as W
    try:
        w = dict(weights)
        w["rms_gain"] = W.make_train_gain(s, dev)
        dy = W.make_dy(s, dev)
        layer = M.MRLMoELayer(s, w, device=dev, train=True)
        grads = M.grad_buffers(layer.cfg, dev)
        ms, fwd_ms, stage = _time_training(layer, x, bias, dy, M.make_grads(grads), steps, warmup)
        peaks, peak_kind = load_peaks()
        wg_ms = stage[M._native.BACKWARD_STAGES.index("expert_wgrad")]
        wg_bytes = wgrad_kernel_bytes(s)
        out = {"metric": "training step (forward_train + backward) tokens/s", "value": s.T * steps / (ms * 1e-3),
               "unit": UNIT, "ms_per_step": ms / steps, "steps": steps, "warmup": max(3, warmup),
               "forward_train_ms": round(fwd_ms, 4), "backward_ms": round(sum(stage), 4),
               "backward_stage_ms": dict(zip(M._native.BACKWARD_STAGES, [round(v, 4) for v in stage])),
               "roofline": {"kernel": "expert_wgrad", "bound": "hbm",
                            "achieved": wg_bytes / (wg_ms * 1e-3) / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                            "frac": wg_bytes / (wg_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                            "traffic": profiled_traffic("expert_wgrad", s.name), "peak_kind": f"of {peak_kind}"},
               "gpu_launches": BACKWARD_KERNELS * steps,
               "note": "python bench.py --train gives the full line (e2e, clocks, CPU baseline)"}
        del layer, grads
        torch.cuda.empty_cache()
        return out
    except Exception as e:  # the forward's line is printed either way
        return {"error": str(e).splitlines()[0][:200] if str(e) else type(e).__name__}


def run_train(args):
    """--train: one step = mrlmoe_forward_train + mrlmoe_backward over one batch
    (fp32 weight gradients of every expert, bf16 dx)."""
    import torch
    import sparse_moe_layer_mean_b200 as M
    import workloads as W
    world, rank, local = dist_setup()
    if world > 1:
        raise SystemExit("--train runs on one GPU")
    s = shape_from_args(args)
    if s.fp8:
        raise SystemExit("--train runs the bf16 configs")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    weights = W.make_layer_weights(s, dev)
    weights["rms_gain"] = W.make_train_gain(s, dev)
    x = W.make_x(s, dev)
    bias = W.make_bias(s, dev)
    dy = W.make_dy(s, dev)
    layer = M.MRLMoELayer(s, weights, device=dev, train=True)
    y = torch.empty(s.T, s.d_model, dtype=torch.bfloat16, device=dev)
    grads = M.grad_buffers(layer.cfg, dev)
    cg = M.make_grads(grads)
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    clocks = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    ms, fwd_ms, stage = _time_training(layer, x, bias, dy, cg, args.steps, args.warmup, clocks)
    clk = clocks.stop()
    bwd_ms = sum(stage)

    # e2e: x and dy from pinned host memory, the step, dx back to pinned host memory, every step
    e2e = None
    if not args.no_e2e:
        xh, dyh = x.cpu().pin_memory(), dy.cpu().pin_memory()
        dxh = torch.empty_like(grads["dx"], device="cpu").pin_memory()
        xd, dyd = torch.empty_like(x), torch.empty_like(dy)

        def e2e_run(n):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(n):
                xd.copy_(xh, non_blocking=True)
                dyd.copy_(dyh, non_blocking=True)
                layer.forward_train(xd, bias, y=y)
                M.mrlmoe_backward(layer.cfg, layer.cw, xd, dyd, cg, layer.workspace, layer.ws_bytes)
                dxh.copy_(grads["dx"], non_blocking=True)
            b.record()
            torch.cuda.synchronize()
            return a.elapsed_time(b)

        e2e_run(2)
        e2e_ms = e2e_run(args.steps)
        e2e = {"value": s.T * args.steps / (e2e_ms * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": 2 * x.numel() * x.element_size(),
               "d2h_bytes_per_step": grads["dx"].numel() * grads["dx"].element_size()}

    peaks, peak_kind = load_peaks()
    wg_ms = stage[M._native.BACKWARD_STAGES.index("expert_wgrad")]
    wg_bytes = wgrad_kernel_bytes(s)
    flops = train_flops(s)
    line = {
        "metric": TRAIN_METRIC, "value": s.T * args.steps / (ms * 1e-3), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"{s.name} training step: T={s.T} tokens, d_model {s.d_model} -> d_lat {s.d_lat}, "
                               f"{s.n_experts} experts top-{s.top_k} + 1 shared, d_ff {s.d_ff}, "
                               f"R={s.n_routers} routers, bf16 operands, fp32 weight gradients",
                   "T": s.T, "l2": "inputs larger than L2 (expert weights and gradients streamed every step)",
                   "forward_train_ms": round(fwd_ms, 4), "backward_ms": round(bwd_ms, 4),
                   "backward_stage_ms": dict(zip(M._native.BACKWARD_STAGES, [round(v, 4) for v in stage])),
                   "step_tensor_frac_of_bf16_peak": flops / (ms / args.steps * 1e-3) / (peaks["bf16_tflops"] * 1e12)},
        "roofline": {"kernel": "expert_wgrad (grouped tcgen05 GEMM over ragged token K, fp32 gradients)",
                     "bound": "hbm", "achieved": wg_bytes / (wg_ms * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": wg_bytes / (wg_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                     "traffic": profiled_traffic("expert_wgrad", s.name), "algorithmic_bytes": wg_bytes,
                     "peak_kind": f"of {peak_kind}"},
        "clocks": clk,
        "gpu_launches": (kernels_per_step(s, torch.cuda.get_device_properties(dev).multi_processor_count)
                         + BACKWARD_KERNELS) * args.steps,
    }
    if e2e:
        line["e2e"] = e2e
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_train(s, weights, x, bias, dy, min(args.cpu_sample, 4))
    print(json.dumps(line), flush=True)


def cpu_baseline_train(s, weights_dev, x_dev, bias_dev, dy_dev, ntok):
    """The oracle's forward + backward, as they stand, on the first ntok
    tokens (the routed experts' weight gradients for the experts those
    tokens select; the others are zero)."""
    import torch
    from oracle import mrlmoe_backward as OB
    wh = {k: v.cpu() for k, v in weights_dev.items()}
    t0 = time.perf_counter()
    fc = OB.forward_for_grad(x_dev[:ntok].cpu(), wh, bias_dev.cpu(), s.top_k, rms_eps=s.rms_eps,
                             aggregation=s.aggregation)
    used = torch.unique(fc.idx).tolist()
    OB.backward(fc, wh, dy_dev[:ntok].cpu(), s.top_k, aggregation=s.aggregation, experts=used)
    dt = time.perf_counter() - t0
    return {"value": ntok / dt, "unit": UNIT, "cores": torch.get_num_threads(), "kind": "oracle",
            "sample": f"first {ntok} tokens of the {s.name} batch, forward + backward (fp64 oracle, {dt:.1f} s)"}


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.route_only:
        return run_route_only(args)
    if args.train:
        return run_train(args)
    world, rank, local = dist_setup()
    import torch
    import torch.distributed as dist

    import sparse_moe_layer_mean_b200 as M
    import workloads as W

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    s = shape_from_args(args)
    weights = W.make_layer_weights(s, dev)
    x = W.make_x(s, dev, seed=s.seed + rank)
    bias = W.make_bias(s, dev)
    layer = M.MRLMoELayer(s, weights, device=dev)
    y = torch.empty(s.T, s.d_model, dtype=torch.bfloat16, device=dev)
    routing = layer.routing_buffers()

    # warm-up (also yields this batch's routing for the byte counts)
    for _ in range(max(1, args.warmup)):
        layer(x, bias, y=y, routing=routing)
    torch.cuda.synchronize()
    st = layer.device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")
    counts = routing["counts"].cpu()
    byts, flops, touched = layer_bytes_flops(s, counts)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(M._native.NUM_STAGE_EVENTS)]
           for _ in range(args.steps)]
    for row in evs:          # materialise the event handles
        for e in row:
            e.record()
    torch.cuda.synchronize()

    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    clocks = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    time.sleep(0.6)
    if world > 1:
        dist.barrier(device_ids=[local])
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks.begin()
    start.record()
    for i in range(args.steps):
        M.mrlmoe_forward_timed(layer.cfg, layer.cw, bias, x, y, None, layer.workspace, layer.ws_bytes,
                               evs[i])
    stop.record()
    torch.cuda.synchronize()
    clocks.end()
    if world > 1:
        dist.barrier(device_ids=[local])
    clk = clocks.stop()
    ms = start.elapsed_time(stop)
    stage_ms = [0.0] * (M._native.NUM_STAGE_EVENTS - 1)
    for row in evs:
        for j in range(len(stage_ms)):
            stage_ms[j] += row[j].elapsed_time(row[j + 1])
    stage_ms = [v / args.steps for v in stage_ms]
    if layer.device_status() != 0:
        raise RuntimeError("device status non-zero after the timed region")

    # e2e: pinned host x -> device, forward, y -> pinned host, every step.  The
    # copies run on the copy engines, pipelined as a server would run them:
    # step i+1's x goes up (H2D stream) while step i computes, step i-1's y
    # comes back (D2H stream); device x / y are double-buffered.  Every step's
    # copies lie inside the timed region.
    e2e = None
    if not args.no_e2e:
        xh = x.cpu().pin_memory()
        yh = [torch.empty_like(y, device="cpu").pin_memory() for _ in range(2)]
        xd = [torch.empty_like(x) for _ in range(2)]
        yd = [torch.empty_like(y) for _ in range(2)]
        comp = torch.cuda.current_stream()
        h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()

        def pipelined(n):
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(comp)
            h2d.wait_event(t0)
            fwd_done, y_read = [None, None], [None, None]
            for i in range(n):
                j = i % 2
                if fwd_done[j] is not None:          # step i-2 has read xd[j]
                    h2d.wait_event(fwd_done[j])
                with torch.cuda.stream(h2d):
                    xd[j].copy_(xh, non_blocking=True)
                up = torch.cuda.Event()
                up.record(h2d)
                comp.wait_event(up)
                if y_read[j] is not None:            # step i-2's y has left yd[j]
                    comp.wait_event(y_read[j])
                layer(xd[j], bias, y=yd[j], stream=comp)
                fwd_done[j] = torch.cuda.Event()
                fwd_done[j].record(comp)
                d2h.wait_event(fwd_done[j])
                with torch.cuda.stream(d2h):
                    yh[j].copy_(yd[j], non_blocking=True)
                y_read[j] = torch.cuda.Event()
                y_read[j].record(d2h)
            for ev in y_read:
                if ev is not None:
                    comp.wait_event(ev)
            t1.record(comp)
            torch.cuda.synchronize()
            return t0.elapsed_time(t1)

        pipelined(3)
        if world > 1:
            dist.barrier(device_ids=[local])
        e2e_ms = pipelined(args.steps)
        # the layer is bitwise reproducible: the last step read back equals the device-only result
        if not torch.equal(yh[(args.steps - 1) % 2], y.cpu()):
            raise RuntimeError("pipelined end-to-end result differs from the device-only forward")
        e2e = [e2e_ms, x.numel() * x.element_size(), y.numel() * y.element_size()]

    # the balancing-bias update (the skewed workload's step after the forward), timed alone
    bias_ms = None
    if s.bias_kind == "zipf":
        b2 = bias.clone()
        for _ in range(3):
            M.mrlmoe_bias_update(layer.cfg, routing["counts"], b2, 1e-3)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.steps):
            M.mrlmoe_bias_update(layer.cfg, routing["counts"], b2, 1e-3)
        b.record()
        torch.cuda.synchronize()
        bias_ms = a.elapsed_time(b) / args.steps

    # max over ranks
    if world > 1:
        red = max_over_ranks([ms, e2e[0] if e2e else 0.0] + stage_ms, dev)
        ms = red[0]
        if e2e:
            e2e[0] = red[1]
        stage_ms = red[2:]

    if rank == 0:
        peaks, peak_kind = load_peaks()
        glu_ms = stage_ms[M._native.STAGES.index("gate_up_glu")]
        glu_bytes = glu_kernel_bytes(s, touched)
        glu_flops = glu_kernel_flops(s)
        # the gate/up kernel's bound: HBM bytes or tensor FLOPs (e4m3: the probe's peak)
        if s.fp8:
            tensor_peak, tensor_kind, probe = e4m3_peak(dev, peaks, peak_kind)
        else:
            tensor_peak, tensor_kind = peaks["bf16_tflops_sustained"], f"of {peak_kind} (sustained bf16)"
        glu_tensor_bound = glu_flops / (tensor_peak * 1e12) > glu_bytes / (peaks["hbm_gbs"] * 1e9)
        achieved = glu_bytes / (glu_ms * 1e-3) / 1e9
        step_s = ms / args.steps * 1e-3
        t_bytes = byts / (peaks["hbm_gbs"] * 1e9)
        t_flops = flops / (tensor_peak * 1e12)
        workload = s.name
        line = {
            "metric": METRIC, "value": job_throughput(world, s.T, args.steps, ms), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3" if s.fp8 else "bf16", "data": "synthetic",
            "config": {
                "workload": f"{workload}: T={s.T} tokens, d_model {s.d_model} -> d_lat {s.d_lat}, "
                            f"{s.n_experts} experts top-{s.top_k} + 1 shared, d_ff {s.d_ff}, "
                            f"R={s.n_routers} routers, "
                            + ("e2m1 experts, e4m3 projections (128x128 block scales), e4m3 activations, bf16 routers"
                               if s.fp4 else
                               "e4m3 experts and projections (128x128 block scales), bf16 routers" if s.fp8 else "bf16"),
                "T": s.T, "parallelism": f"replicas x{world} (expert weights replicated, own batch per GPU)",
                "l2": "inputs larger than L2 (expert weights streamed every step)",
                "touched_experts": touched,
                "layer_roofline": {"bytes": byts, "flops": flops,
                                   "t_bytes_ms": t_bytes * 1e3, "t_flops_ms": t_flops * 1e3,
                                   "frac": max(t_bytes, t_flops) / step_s,
                                   "tensor_frac_of_bf16_peak": flops / step_s / (peaks["bf16_tflops"] * 1e12),
                                   "peaks": peak_kind + (f"; e4m3 peak {tensor_peak} TFLOP/s {tensor_kind}"
                                                         if s.fp8 else ""),
                                   # the same against the nominal datasheet figures (HBM 8 TB/s,
                                   # dense bf16 2.25 PFLOP/s, dense e4m3 4.5 PFLOP/s)
                                   "frac_nominal": max(byts / 8.0e12,
                                                       flops / ((4.5e15 if s.fp8 else 2.25e15))) / step_s},
                "stage_ms": dict(zip(M._native.STAGES, [round(v, 4) for v in stage_ms])),
            },
            "roofline": ({"kernel": "gate_up_glu (grouped tcgen05 GEMM, SiLU-GLU epilogue)",
                          "bound": "tensor", "achieved": glu_flops / (glu_ms * 1e-3) / 1e12,
                          "peak": tensor_peak, "unit": "TFLOP/s",
                          "frac": glu_flops / (glu_ms * 1e-3) / 1e12 / tensor_peak,
                          "traffic": profiled_traffic("gate_up_glu", workload),
                          "algorithmic_flops": glu_flops,
                          "peak_kind": tensor_kind}
                         if glu_tensor_bound else
                         {"kernel": "gate_up_glu (grouped tcgen05 GEMM, SiLU-GLU epilogue)",
                          "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                          "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                          "traffic": profiled_traffic("gate_up_glu", workload),
                          "algorithmic_bytes": glu_bytes, "peak_kind": f"of {peak_kind}"}),
            "clocks": clk,
            "gpu_launches": kernels_per_step(s, torch.cuda.get_device_properties(dev).multi_processor_count)
            * args.steps,
        }
        if e2e:
            line["e2e"] = {"value": job_throughput(world, s.T, args.steps, e2e[0]), "unit": UNIT,
                           "h2d_bytes_per_step": e2e[1], "d2h_bytes_per_step": e2e[2]}
        if bias_ms is not None:
            line["config"]["bias_update_ms"] = bias_ms
        if s.fp8:
            line["config"]["e4m3_peak_probe"] = probe
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(s, weights, x, bias, min(args.cpu_sample, s.T))
        if world == 1 and not s.fp8 and not args.no_train_summary:
            line["train_step"] = train_summary(s, dev, weights, x, bias)
        if world == 1 and s.name == "c2_prefill" and not args.no_other_configs:
            line["other_configs"] = {n: config_summary(n, dev, weights) for n in OTHER_CONFIGS}
            # the router aggregation variants (sum, max) of the headline workload
            line["aggregation_variants"] = {
                agg: config_summary("c2_prefill", dev, weights,
                                    shape=dataclasses.replace(s, aggregation=agg, name=f"c2_prefill_{agg}"))
                for agg in ("sum", "max")}
            line["ep_emulated"] = ep_summary(8, dev, weights)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
