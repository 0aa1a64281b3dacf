#!/usr/bin/env python3
"""Benchmark of the MoE layer forward on B200: tokens/s, TFLOP/s and roofline fractions.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload mixtral] [--impl ours|reference]

A step is one full layer forward (route -> dispatch -> layer0 grouped GEMM + SwiGLU ->
layer1 grouped GEMM + gate scale -> top-k combine) through the C ABI on one batch of
synthetic, seeded inputs already resident in HBM. With N > 1 (torchrun, one rank per GPU)
every rank runs its own batch of the same workload with the same weights (data-parallel
replicas, weak scaling); there is no collective on the data path, and the reported time is
the max over ranks. Rank 0 prints one JSON line.

The per-step working set (Mixtral-shaped layer: 2.8 GB of expert weights plus 0.8 GB of
intermediates) is far larger than the 126 MB L2, so every step streams its inputs from HBM;
no separate L2 flush is inserted.

--impl reference times the CPU oracle (oracle/, plain C + OpenMP) on a bounded token sample
of the same workload on the host cores; rank 0 only.
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
from pathlib import Path

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# layer0 grouped GEMM + SwiGLU, by GEMM mode (the single-CTA launch is the select kernel,
# which runs the 128-row body, or the operand-swapped one when every expert is single-tile)
DOMINANT_KERNEL = {"auto": "moe_grouped_gemm_select_kernel<0>",
                   "single": "moe_grouped_gemm_select_kernel<0>",
                   "pair": "moe_grouped_gemm_pair_kernel<0>",
                   "fused": "moe_fused_layer_kernel<0>"}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mixtral")
    ap.add_argument("--T", type=int, default=None)
    ap.add_argument("--E", type=int, default=None)
    ap.add_argument("--k", type=int, default=None)
    ap.add_argument("--H", type=int, default=None)
    ap.add_argument("--F", type=int, default=None)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--gemm-mode", choices=["auto", "single", "pair", "fused"], default="auto",
                    help="grouped-GEMM variant (moe_set_gemm_mode)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="measure only the named workload (default: the Mixtral-shaped run also "
                         "reports the other four bench workloads under 'workloads')")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU seconds of the oracle sample")
    ap.add_argument("--fp8", action="store_true",
                    help="e4m3 experts (moe_forward_fp8; weights quantised once before timing)")
    ap.add_argument("--backward", action="store_true",
                    help="time moe_backward (the layer's gradients) instead of the forward")
    ap.add_argument("--trace", default=None, metavar="FILE",
                    help="after timing, run one forward with the persistent launch's schedule "
                         "trace on; write the raw records to FILE (.npy) and a summary into the "
                         "JSON line")
    ap.add_argument("--router-mode", choices=["auto", "sequential", "filter"], default="auto",
                    help="router variant (moe_set_router_mode)")
    ap.add_argument("--ep-local", type=int, default=0, metavar="N",
                    help="the expert-parallel layer (moe_ep_layer_forward) with the workload's "
                         "tokens split over N ranks carried by one launch on this GPU (each rank "
                         "1/N of the SMs, every exchange buffer local): the EP machinery's cost "
                         "against the single-GPU layer, not NVLink")
    ap.add_argument("--router-only", action="store_true",
                    help="time moe_route alone (router logits + top-k); no expert weights allocated")
    return ap.parse_args()


def workload(args):
    from mixture_experts_layer_forward_b200 import synth
    from dataclasses import replace

    cfg = synth.CONFIGS[args.workload]
    over = {k: getattr(args, k) for k in ("T", "E", "k", "H", "F") if getattr(args, k) is not None}
    if over:
        cfg = replace(cfg, name=cfg.name + "_" + "_".join(f"{k}{v}" for k, v in over.items()), **over)
    return cfg


WORKLOAD_NAMES = {
    "tiny": "tiny MoE layer",
    "mixtral": "Mixtral-8x7B-shaped MoE layer",
    "phi35": "Phi-3.5-MoE-shaped MoE layer",
    "qwen2": "Qwen2-57B-A14B-shaped MoE layer",
    "skew": "skewed fine-grained MoE layer (Zipf 1.2 expert prior)",
    "skew_decode": "skewed fine-grained MoE layer, decode batch",
}


def config_dict(cfg, args, n):
    return {
        "workload": WORKLOAD_NAMES.get(args.workload, args.workload) + f" ({cfg.name})",
        "T_per_gpu": cfg.T, "H": cfg.H, "F": cfg.F, "E": cfg.E, "top_k": cfg.k,
        "act": ["swiglu", "gelu_tanh", "relu", "identity"][cfg.act],
        "gate": ["softmax_topk", "softmax_all", "select_bias"][cfg.gate],
        "global_tokens": cfg.T * n, "parallelism": f"dp{n} replicas (no collective)",
        "l2": "inputs larger than L2 (per-step working set >> 126 MB); no flush",
        "seed": args.seed,
        "gemm_mode": getattr(args, "gemm_mode", "auto"),
        "experts": "e4m3 codes, fp32 row/column scales" if getattr(args, "fp8", False) else "bf16",
    }


def load_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def tensor_peak(peaks, clocks, fp8=False):
    """Tensor-core peak for the clock regime of a timed region, read from the median sampled
    SM clock: the measured burst figure when the median is within 10% of the maximum clock,
    the measured sustained (power-capped) figure otherwise. e4m3: the bf16 figure times the
    nominal e4m3/bf16 ratio of 2. Returns (peak, burst_peak, regime, clock_frac)."""
    mult = 2.0 if fp8 else 1.0
    burst = peaks["bf16_tflops"] * mult
    sust = (peaks.get("bf16_tflops_sustained") or peaks["bf16_tflops"]) * mult
    cf = None
    if clocks and clocks.get("sm_max_mhz"):
        cf = clocks["sm_mhz"] / clocks["sm_max_mhz"]
    regime = "sustained" if (cf is not None and cf < 0.9) else "burst"
    return (sust if regime == "sustained" else burst), burst, regime, cf


def tensor_fracs(achieved, peaks, clocks, fp8=False):
    """frac against the regime's peak, against the burst peak, and against the burst peak
    scaled by the sampled clock (median SM MHz / max MHz), with the figures used."""
    peak, burst, regime, cf = tensor_peak(peaks, clocks, fp8)
    d = {"peak": peak, "frac": achieved / peak, "regime": regime, "peak_burst": burst,
         "frac_burst": achieved / burst}
    if cf is not None:
        d["clock_frac"] = cf
        d["frac_clock_scaled"] = achieved / (burst * cf)
    return d


def launches_in_mode(moe, p, mode):
    prev = moe.moe_set_gemm_mode(mode)
    try:
        return moe.moe_forward_launches(p)
    finally:
        moe.moe_set_gemm_mode(prev)


def layer0_roofline(cfg, g0_ms, active_experts, peaks, peak_src, clocks, fp8, kernel, fused=False,
                    whole=False):
    """Roofline of the dominant kernel. Separate launches: the layer0 grouped GEMM, with its
    useful FLOPs (padding rows not counted) and algorithmic bytes (each active expert's W1
    once, x once, h of the routed rows written once). One persistent launch (`fused`):
    layer0 + layer1 + combine, with both GEMMs' useful FLOPs and the bytes that must cross
    HBM (the active experts' W1 and W2, the sorted x rows, the output); the whole layer in
    that launch (`whole`) adds the router's FLOPs and its reads of x and W_g. The bound is
    whichever takes longer at the measured peaks."""
    w1_cols = 2 * cfg.F if cfg.act == 0 else cfg.F
    wb = 1 if fp8 else 2   # e4m3 experts: 1-byte weights and x codes; h is still bf16
    if fused:
        flops = 2 * cfg.T * cfg.k * cfg.H * (w1_cols + cfg.F)
        nbytes = (wb * (active_experts * cfg.H * (w1_cols + cfg.F) + cfg.T * cfg.k * cfg.H) +
                  2 * cfg.T * cfg.H)
        if whole:
            flops += 2 * cfg.T * cfg.H * cfg.E
            nbytes += 2 * cfg.T * cfg.H + 2 * cfg.H * cfg.E
    else:
        flops = 2 * cfg.T * cfg.k * cfg.H * w1_cols
        nbytes = wb * (active_experts * cfg.H * w1_cols + cfg.T * cfg.H) + 2 * cfg.T * cfg.k * cfg.F
    g0_s = g0_ms / 1e3
    tpk, _, _, _ = tensor_peak(peaks, clocks, fp8)
    hbm_bound = nbytes / (peaks["hbm_gbs"] * 1e9) > flops / (tpk * 1e12)
    r = {"bound": "hbm" if hbm_bound else "tensor", "kernel": kernel}
    if hbm_bound:
        achieved = nbytes / g0_s / 1e9
        r.update({"achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                  "frac": achieved / peaks["hbm_gbs"],
                  "peak_source": f"{peak_src} HBM copy bandwidth"})
    else:
        achieved = flops / g0_s / 1e12
        r.update({"achieved": achieved, "unit": "TFLOP/s"})
        r.update(tensor_fracs(achieved, peaks, clocks, fp8))
        r["peak_source"] = (f"{peak_src} bf16 {r['regime']}" + (" x 2 (nominal e4m3/bf16 ratio)" if fp8 else "") +
                            "; regime from the median sampled SM clock (>= 0.9 of max: burst)")
    r.update({"traffic": traffic_for(kernel, cfg.name), "algorithmic_flops_per_launch": flops,
              "algorithmic_bytes_per_launch": nbytes, "active_experts": active_experts,
              "ms_per_launch": g0_ms})
    return r


STAGE_NAMES = ["route", "dispatch", "layer0_gemm_swiglu", "layer1_gemm_scale", "combine"]


def schedule_trace(torch, moe, fwd, dev, out_file, cap=1 << 18):
    """One forward with the persistent launch's schedule trace on. Summary: the span of each
    kind of work item (layer0 and layer1 tile epilogues, combine items), the gap between
    the last layer0 and the first layer1 tile, and how much of the combine work ended
    inside the layer1 window (the in-device analogue of hidden communication)."""
    import numpy as np

    rec = torch.zeros(4 + 4 * cap, dtype=torch.int64, device=dev)
    moe.moe_set_schedule_trace(rec, cap)
    try:
        fwd()
        torch.cuda.synchronize(dev)
    finally:
        moe.moe_set_schedule_trace(None, 0)
    n = min(int(rec[0].item()), cap)
    r = rec[4:4 + 4 * n].view(n, 4).cpu().numpy().astype(np.int64)
    if out_file:
        np.save(out_file, r)
    if n == 0:
        return {"records": 0}
    kind = r[:, 0] >> 32
    t0 = r[:, 2] - r[:, 2].min()
    t1 = r[:, 3] - r[:, 2].min()
    summ = {"records": n, "span_us": float(t1.max()) / 1e3}
    names = {0: "layer0", 1: "layer1", 2: "combine", 3: "front", 4: "scatter"}
    for k, nm in names.items():
        m = kind == k
        if m.any():
            summ[nm] = {"items": int(m.sum()), "first_begin_us": float(t0[m].min()) / 1e3,
                        "last_end_us": float(t1[m].max()) / 1e3,
                        "busy_us_sum": float((t1[m] - t0[m]).sum()) / 1e3,
                        "sms": int(len(np.unique(r[m, 1])))}
    if (kind == 0).any() and (kind == 1).any():
        summ["layer0_to_layer1_gap_us"] = float(t0[kind == 1].min() - t1[kind == 0].max()) / 1e3
    if (kind == 2).any() and (kind == 1).any():
        end1 = t1[kind == 1].max()
        c = kind == 2
        dur = (t1[c] - t0[c]).astype(np.float64)
        inside = np.clip(np.minimum(t1[c], end1) - t0[c], 0, None).astype(np.float64)
        summ["combine_hidden_frac"] = float(inside.sum() / max(dur.sum(), 1.0))
        summ["combine_after_layer1_us"] = float(max(0, t1[c].max() - end1)) / 1e3
    return summ


def new_sampler(torch, dev, enabled):
    if not enabled:
        return None
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    smp = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
    smp.start()
    return smp


def timed_staged(torch, fwd_staged, K, stream, dev, sampler, barrier=None):
    """K back-to-back staged forwards between two events on the launch stream; returns
    (total ms, per-stage mean ms, clock summary of the timed region)."""
    import mixture_experts_layer_forward_b200 as moe

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(moe.MOE_NUM_STAGE_EVENTS)]
           for _ in range(K)]
    for row in evs:          # create the CUDA events now, outside the timed region
        for e in row:
            e.record(stream)
    torch.cuda.synchronize(dev)
    if barrier is not None:
        barrier()
    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_begin = time.time()
    start.record(stream)
    for i in range(K):
        fwd_staged(evs[i])
    end.record(stream)
    torch.cuda.synchronize(dev)
    t_end = time.time()
    if barrier is not None:
        barrier()
    clocks = sampler.stop(t_begin, t_end) if sampler is not None else None
    stage_ms = {nm: sum(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(K)) / K
                for j, nm in enumerate(STAGE_NAMES)}
    return start.elapsed_time(end), stage_ms, clocks


def measure_workload(torch, name, dev, K, W, seed, clocks_on, peaks, peak_src):
    """One workload (its own inputs and weights) on this GPU: K staged layer forwards after W
    warm-up ones; step time, stage times, clocks and the layer0 roofline."""
    import mixture_experts_layer_forward_b200 as moe
    from mixture_experts_layer_forward_b200 import synth

    cfg = synth.CONFIGS[name]
    stream = torch.cuda.current_stream(dev)
    inp = synth.make_inputs(cfg, seed=seed, device=dev)
    p = moe.Problem.from_config(cfg)
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(moe.moe_workspace_size(p), dtype=torch.uint8, device=dev)
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=dev)
    a = (p, inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W2"], out, ws)
    for _ in range(W):
        moe.moe_forward(*a, idx)
    torch.cuda.synchronize(dev)
    assert moe.moe_get_device_status(ws) == 0, f"{name}: device status after warm-up"
    active = int(torch.unique(idx).numel())
    sampler = new_sampler(torch, dev, clocks_on)
    ms, stage_ms, clocks = timed_staged(torch, lambda ev: moe.moe_forward_staged(*a, ev), K,
                                        stream, dev, sampler)
    assert moe.moe_get_device_status(ws) == 0, f"{name}: device status"
    ms_step = ms / K
    tflops = cfg.useful_flops / (ms_step / 1e3) / 1e12
    layer = {"bound": "tensor", "achieved": tflops, "unit": "TFLOP/s"}
    layer.update(tensor_fracs(tflops, peaks, clocks))
    fused = moe.moe_forward_launches(p) < launches_in_mode(moe, p, moe.GEMM_SINGLE_CTA)
    lay = ("layer0_gemm_swiglu", "layer1_gemm_scale", "combine")
    g_ms = sum(stage_ms[k] for k in lay) if fused else stage_ms["layer0_gemm_swiglu"]
    kernel = "moe_fused_layer_kernel<0>" if fused else DOMINANT_KERNEL["auto"]
    res = {"workload": WORKLOAD_NAMES.get(name, name), "T": cfg.T, "H": cfg.H, "F": cfg.F,
           "E": cfg.E, "top_k": cfg.k, "steps": K, "warmup": W, "ms_per_step": ms_step,
           "tokens_per_s": cfg.T / (ms_step / 1e3), "tflops": tflops, "layer_roofline": layer,
           "stage_ms": stage_ms, "launch": "persistent" if fused else "separate",
           "roofline": layer0_roofline(cfg, g_ms, active, peaks, peak_src, clocks, False, kernel,
                                       fused),
           "clocks": clocks, "active_experts": active}
    if fused:
        prev = moe.moe_set_gemm_mode(moe.GEMM_SINGLE_CTA)
        try:
            for _ in range(W):
                moe.moe_forward(*a, idx)
            ms_s, stage_s, _ = timed_staged(torch, lambda ev: moe.moe_forward_staged(*a, ev), K,
                                            stream, dev, None)
        finally:
            moe.moe_set_gemm_mode(prev)
        sep = sum(stage_s[k] for k in lay)
        res["overlap"] = {"separate_ms_per_step": ms_s / K, "separate_stage_ms": stage_s,
                          "separate_layers_ms": sep, "fused_layers_ms": g_ms,
                          "hidden_frac": 1.0 - g_ms / sep}
    del inp, out, ws, idx, a
    torch.cuda.empty_cache()
    return res


def source_hash(files):
    h = hashlib.sha256()
    for f in files:
        h.update((ROOT / "mixture_experts_layer_forward_b200" / "csrc" / f).read_bytes())
    return h.hexdigest()[:16]


def traffic_for(kernel, cfg_name):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if the kernel's
    sources are unchanged since the counters were taken; else None."""
    p = ROOT / "profiles" / "traffic.json"
    if not p.exists():
        return None
    d = json.loads(p.read_text())
    ent = d.get(kernel, {}).get(cfg_name)
    if not ent:
        return None
    try:
        if source_hash(ent["source_files"]) != ent.get("source_hash"):
            return None
    except (OSError, KeyError):
        return None
    return ent.get("bytes_per_launch")


class ClockSampler:
    """Samples the SM clock, power and clock-event (throttle) reasons of one GPU through NVML
    every ~20 ms on a background thread (read-only queries; no setting is changed).
    Falls back to `nvidia-smi -lms 200` when NVML is unavailable."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, uuid, period_s=0.02):
        self.uuid = uuid
        self.period = period_s
        self.samples = []  # (host time, sm MHz, max sm MHz, power W, reason bitmask)
        self._stop = threading.Event()
        self.t = None
        self.source = None

    def start(self):
        try:
            import pynvml

            pynvml.nvmlInit()
            self.h = pynvml.nvmlDeviceGetHandleByUUID(self.uuid)
            self.pynvml = pynvml
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
            self.source = "nvml"
        except Exception:  # noqa: BLE001 - no NVML: the clock record is simply absent
            return
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()

    def _run(self):
        nv = self.pynvml
        while not self._stop.is_set():
            try:
                clk = float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                pw = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                rs = int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
                self.samples.append((time.time(), clk, self.max_mhz, pw, rs))
            except Exception:  # noqa: BLE001
                pass
            self._stop.wait(self.period)

    def stop(self, t_begin, t_end):
        """Summary of the samples taken inside the timed region [t_begin, t_end]."""
        if self.t is None:
            return None
        self._stop.set()
        self.t.join(timeout=5)
        win = [x for x in self.samples if t_begin <= x[0] <= t_end]
        if not win:  # a region shorter than one period: take the nearest sample
            win = sorted(self.samples, key=lambda x: abs(x[0] - 0.5 * (t_begin + t_end)))[:1]
        if not win:
            return None
        sm = sorted(x[1] for x in win)
        seen = 0
        for x in win:
            seen |= x[4]
        reasons = sorted(n for n, bit in self.REASONS.items() if seen & bit)
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": win[0][2], "reasons": reasons,
                "samples": len(win), "power_w_max": max(x[3] for x in win), "source": self.source}


def cpu_oracle_sample(cfg, inputs_host, seconds, tokens_hint=None):
    """Time the oracle's per-token layer on a token sample sized to ~`seconds` of CPU work.
    Returns (tokens_per_s, n_tokens, elapsed_s, threads)."""
    try:
        threads = len(os.sched_getaffinity(0))
    except AttributeError:
        threads = os.cpu_count() or 1
    os.environ.setdefault("OMP_NUM_THREADS", str(threads))
    threads = int(os.environ["OMP_NUM_THREADS"])
    import numpy as np

    import oracle

    lib = oracle.load()
    x, Wg, W1, W2, b = inputs_host
    rng = np.random.default_rng(1234)

    def run(n):
        toks = rng.choice(cfg.T, size=min(n, cfg.T), replace=False).astype(np.int32)
        t0 = time.perf_counter()
        oracle.moe_tokens(x, Wg, b, W1, W2, cfg.k, toks, act=cfg.act, gate=cfg.gate, lib=lib)
        return len(toks), time.perf_counter() - t0

    n0, t0 = run(max(threads, 4))              # calibration
    per_tok = t0 / n0
    n = tokens_hint or int(max(threads, min(cfg.T, seconds / max(per_tok, 1e-9))))
    n = max(threads, (n // threads) * threads) if n >= threads else n
    n = min(n, cfg.T)
    n1, t1 = run(n)
    return n1 / t1, n1, t1, threads


def host_inputs(inp):
    from mixture_experts_layer_forward_b200 import synth

    b = None if inp["bias"] is None else inp["bias"].cpu().numpy()
    return (synth.bf16_bits(inp["x"]), synth.bf16_bits(inp["Wg"]), synth.bf16_bits(inp["W1"]),
            synth.bf16_bits(inp["W2"]), b)


def set_router_mode(moe, args):
    moe.moe_set_router_mode({"auto": moe.ROUTER_AUTO, "sequential": moe.ROUTER_SEQUENTIAL,
                             "filter": moe.ROUTER_FILTER}[args.router_mode])


def emit(obj):
    print(json.dumps(obj), flush=True)


# ---------------------------------------------------------------------------------------
# reference arm: the CPU oracle
# ---------------------------------------------------------------------------------------

def run_reference(args):
    from mixture_experts_layer_forward_b200 import dp, synth

    rank, _, world = dp.env_rank()
    if rank != 0:
        return 0
    cfg = workload(args)
    inp = synth.make_inputs(cfg, seed=args.seed, device="cpu")
    hin = host_inputs(inp)
    K, W = max(1, args.steps), max(0, args.warmup)
    # each step is a bounded token sample; the whole run stays within a few minutes
    per_step_s = max(1.0, min(args.cpu_seconds, 150.0 / (K + W)))
    _, n_tok, _, threads = cpu_oracle_sample(cfg, hin, per_step_s)
    for _ in range(W):
        cpu_oracle_sample(cfg, hin, per_step_s, tokens_hint=n_tok)
    tot_t, tot_n = 0.0, 0
    for _ in range(K):
        _, n, t, _ = cpu_oracle_sample(cfg, hin, per_step_s, tokens_hint=n_tok)
        tot_t += t
        tot_n += n
    value = tot_n / tot_t
    flops_per_tok = cfg.useful_flops / cfg.T
    emit({
        "impl": "reference", "metric": "MoE-layer forward tokens/s", "value": value,
        "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": 1000.0 * tot_t / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64 (router logits f32)", "data": "synthetic",
        "config": config_dict(cfg, args, 1),
        "tflops": value * flops_per_tok / 1e12,
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"{n_tok} random tokens of the {cfg.T}-token batch per step "
                                   f"(per-token definition path, fp64)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    })
    return 0


# ---------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------

def run_ours(args):
    import torch
    import torch.distributed as dist

    import mixture_experts_layer_forward_b200 as moe
    from mixture_experts_layer_forward_b200 import dp, synth

    rank, local_rank, world = dp.env_rank()
    if world != args.gpus:
        print(f"warning: WORLD_SIZE={world} but --gpus={args.gpus}", file=sys.stderr)
    n = world
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    cfg = workload(args)
    K, W = args.steps, max(3, args.warmup)
    moe.moe_set_gemm_mode({"auto": moe.GEMM_AUTO, "single": moe.GEMM_SINGLE_CTA,
                           "pair": moe.GEMM_CTA_PAIR, "fused": moe.GEMM_FUSED}[args.gemm_mode])
    set_router_mode(moe, args)

    inp = synth.make_inputs(cfg, seed=args.seed, device=dev,
                            x_seed=dp.replica_x_seed(args.seed, rank) if world > 1 else None)
    p = moe.Problem.from_config(cfg)
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    if args.fp8:
        # one-off weight preparation, outside the timed region
        w1c = 2 * cfg.F if cfg.act == 0 else cfg.F
        q = (torch.empty(cfg.E, w1c, cfg.H, dtype=torch.uint8, device=dev),
             torch.empty(cfg.E, w1c, dtype=torch.float32, device=dev),
             torch.empty(cfg.E, cfg.H, cfg.F, dtype=torch.uint8, device=dev),
             torch.empty(cfg.E, cfg.H, dtype=torch.float32, device=dev))
        moe.moe_quantize_experts_fp8(p, inp["W1"], inp["W2"], *q)
        del inp["W1"], inp["W2"]
        torch.cuda.empty_cache()
        ws = torch.empty(moe.moe_workspace_size_fp8(p), dtype=torch.uint8, device=dev)
        args_fwd = (p, inp["x"], inp["Wg"], inp["bias"], *q, out, ws)
        fwd = lambda idx=None: moe.moe_forward_fp8(*args_fwd, topk_idx_out=idx)
        fwd_staged = lambda ev: moe.moe_forward_fp8_staged(*args_fwd, ev)
    else:
        ws = torch.empty(moe.moe_workspace_size(p), dtype=torch.uint8, device=dev)
        args_fwd = (p, inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W2"], out, ws)
        fwd = lambda idx=None: moe.moe_forward(*args_fwd, idx)
        fwd_staged = lambda ev: moe.moe_forward_staged(*args_fwd, ev)

    idx_buf = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=dev)
    for _ in range(W):
        fwd(idx_buf)
    torch.cuda.synchronize(dev)
    assert moe.moe_get_device_status(ws) == 0, "device status after warm-up"
    active_experts = int(torch.unique(idx_buf).numel())  # for the layer0 byte count below
    counts = torch.bincount(idx_buf.flatten().long(), minlength=cfg.E).cpu()
    nz = counts[counts > 0]
    routing = {"active_experts": active_experts,
               "rows_max": int(counts.max()), "rows_min_active": int(nz.min()) if nz.numel() else 0,
               "single_tile_experts": int(((counts > 0) & (counts <= 128)).sum()),
               "padded_rows": int(((counts + 127) // 128 * 128).sum()), "routed_rows": cfg.T * cfg.k}
    if cfg.E <= 64:
        routing["expert_histogram"] = [int(c) for c in counts]

    # K staged steps: stage events recorded on the launch stream by the library
    sampler = new_sampler(torch, dev, not args.no_clocks)
    ms_local, stage_ms, clocks = timed_staged(torch, fwd_staged, K, stream, dev, sampler,
                                              barrier=lambda: dp.barrier(dev))
    status = moe.moe_get_device_status(ws)
    assert status == 0, f"device status {status}"
    ms = dp.max_over_ranks(ms_local, device=dev)
    ms_per_step = ms / K

    # the same layer with a cold L2: a 256 MiB buffer written before each step (outside each
    # step's events); a reported figure beside the warm, back-to-back value above
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    n_cold = min(K, 20)
    cold_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n_cold)]
    for a, b in cold_ev:
        flush.zero_()
        a.record(stream)
        fwd()
        b.record(stream)
    torch.cuda.synchronize(dev)
    cold_ms = dp.max_over_ranks(sum(a.elapsed_time(b) for a, b in cold_ev) / n_cold, device=dev)
    del flush


    # end to end through the public API with host buffers: every step copies its x in and
    # its out back (pinned host memory); moe_forward_host_batches overlaps step i's compute
    # with step i+1's copy in and step i-1's copy out
    e2e = None
    if not args.no_e2e and not args.fp8:
        x_h = inp["x"].cpu().pin_memory()
        out_h = [torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        outs = [out_h[i & 1] for i in range(K)]
        moe.moe_forward_host_batches(p, [x_h, x_h], inp["Wg"], inp["bias"], inp["W1"], inp["W2"],
                                     out_h, ws)
        dp.barrier(dev)
        torch.cuda.synchronize(dev)
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        moe.moe_forward_host_batches(p, [x_h] * K, inp["Wg"], inp["bias"], inp["W1"], inp["W2"],
                                     outs, ws)
        e2.record(stream)
        torch.cuda.synchronize(dev)
        dp.barrier(dev)
        e2e_ms = dp.max_over_ranks(s2.elapsed_time(e2), device=dev) / K
        e2e = {"value": n * cfg.T / (e2e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": cfg.T * cfg.H * 2, "d2h_bytes_per_step": cfg.T * cfg.H * 2,
               "ms_per_step": e2e_ms, "api": "moe_forward_host_batches (copies overlapped across steps)"}

    peaks, peak_src = load_peaks()
    layer_tflops = cfg.useful_flops / (ms_per_step / 1e3) / 1e12
    # the persistent launch replaces layer0, layer1 and the combine (stage events 3..5 all
    # mark its end)
    fused = (not args.fp8 and
             moe.moe_forward_launches(p) < launches_in_mode(moe, p, moe.GEMM_SINGLE_CTA))
    # the whole layer in one launch: that kernel is the step (the timed region holds it and one
    # 32-byte memset per step), so its duration is the step's
    whole = not args.fp8 and moe.moe_forward_launches(p) == 1
    if whole:
        kernel = f"moe_fused_layer_kernel<{cfg.act if cfg.act == 0 else 1}, true>"
        g_ms = ms_per_step
    elif fused:
        kernel = "moe_fused_layer_kernel<0>" if cfg.act == 0 else "moe_fused_layer_kernel<1>"
        g_ms = sum(stage_ms[k] for k in ("layer0_gemm_swiglu", "layer1_gemm_scale", "combine"))
    else:
        kernel = ("moe_grouped_gemm_select_f8_kernel<0>" if args.fp8
                  else DOMINANT_KERNEL[args.gemm_mode])
        g_ms = stage_ms["layer0_gemm_swiglu"]
    roofline = layer0_roofline(cfg, g_ms, active_experts, peaks, peak_src, clocks, args.fp8, kernel,
                               fused or whole, whole)
    layer_roof = {"bound": "tensor", "achieved": layer_tflops, "unit": "TFLOP/s per GPU"}
    layer_roof.update(tensor_fracs(layer_tflops, peaks, clocks, args.fp8))
    layer_roof["peak_source"] = f"{peak_src} bf16 {layer_roof['regime']}" + (" x 2" if args.fp8 else "")

    line = {
        "metric": "MoE-layer forward tokens/s", "value": n * cfg.T / (ms_per_step / 1e3),
        "unit": "tokens/s", "n_gpus": n, "steps": K, "warmup": W, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3 experts (bf16 router, fp32 accumulation)" if args.fp8 else "bf16",
        "data": "synthetic (seeded random inputs and random-init weights of the layer's shape)",
        "config": config_dict(cfg, args, n),
        "tflops": layer_tflops * n,
        "layer_roofline": layer_roof,
        "roofline": roofline,
        "stage_ms": stage_ms,
        # FP8: the bf16 path's launches (router, dispatch, [the gather into sorted rows],
        # layer0, layer1, combine) plus the x and h quantisers
        "gpu_launches": (moe.moe_forward_launches(p) + (2 if args.fp8 else 0)) * K,
        "clocks": clocks,
        "e2e": e2e,
        "cold_l2": {"ms_per_step": cold_ms, "steps": n_cold,
                    "how": "256 MiB buffer written before each step, outside its events"},
        "routing": routing,
    }

    # the three-launch form of the same layer, staged: the sum of its stage times against
    # the default launch (hidden-overlap ratio: the share of the separate stages' time that
    # the default form does not spend, the in-device analogue of hidden communication)
    if not args.fp8 and fused:
        prev = moe.moe_set_gemm_mode(moe.GEMM_SINGLE_CTA)
        try:
            for _ in range(W):
                fwd()
            Ks = max(1, min(K, 20))
            ms_s, stage_s, _ = timed_staged(torch, fwd_staged, Ks, stream, dev, None)
        finally:
            moe.moe_set_gemm_mode(prev)
        sep = {k: v for k, v in stage_s.items()}
        sum_layers = sep["layer0_gemm_swiglu"] + sep["layer1_gemm_scale"] + sep["combine"]
        fused_ms = stage_ms["layer0_gemm_swiglu"] + stage_ms["layer1_gemm_scale"] + stage_ms["combine"]
        line["overlap"] = {
            "separate_stage_ms": sep, "separate_ms_per_step": ms_s / Ks,
            "fused_layers_ms": fused_ms, "separate_layers_ms": sum_layers,
            "hidden_frac": 1.0 - fused_ms / sum_layers,
            "combine_ms": sep["combine"],
            "how": "layer0 + layer1 + combine as three launches (staged, same run) against the "
                   "one persistent launch",
            # the layer0 grouped GEMM of the separate launches, for comparison with runs
            # whose dominant kernel is that launch
            "separate_layer0_roofline": layer0_roofline(
                cfg, sep["layer0_gemm_swiglu"], active_experts, peaks, peak_src, clocks, False,
                DOMINANT_KERNEL["single"])}
    if args.trace is not None and not args.fp8:
        line["schedule_trace"] = schedule_trace(torch, moe, fwd, dev, args.trace or None)

    # the other bench workloads, measured in the same run (one GPU only): step time, stage
    # times, layer0 roofline and clocks of each, beside the headline Mixtral-shaped layer
    if world == 1 and not args.fp8 and not args.no_workloads and args.workload == "mixtral" and \
            not any(getattr(args, k) is not None for k in ("T", "E", "k", "H", "F")):
        hin = host_inputs(inp) if (rank == 0 and not args.no_cpu_baseline) else None
        del inp, out, ws, args_fwd, fwd, fwd_staged
        torch.cuda.empty_cache()
        Kw = max(1, min(K, 20))
        line["workloads"] = {
            nm: measure_workload(torch, nm, dev, Kw, W, args.seed, not args.no_clocks, peaks, peak_src)
            for nm in ("phi35", "qwen2", "skew", "skew_decode")}
    else:
        hin = None

    # the CPU oracle baseline: rank 0 of a one-GPU run only
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.fp8:
        if hin is None:
            hin = host_inputs(inp)
        v, n_tok, t, threads = cpu_oracle_sample(cfg, hin, args.cpu_seconds)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                "sample": f"{n_tok} random tokens of the {cfg.T}-token batch, "
                                          f"{t:.1f} s (per-token definition path, fp64)"}
    if rank == 0:
        emit(line)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_router(args):
    """Router alone on one GPU: K timed moe_route calls on the workload's x and W_g."""
    import torch

    import mixture_experts_layer_forward_b200 as moe
    from mixture_experts_layer_forward_b200 import synth

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    cfg = workload(args)
    K, W = args.steps, max(3, args.warmup)
    set_router_mode(moe, args)
    inp = synth.make_inputs(cfg, seed=args.seed, device=dev, experts=False)
    p = moe.Problem.from_config(cfg)
    ws = torch.empty(moe.moe_workspace_size(p), dtype=torch.uint8, device=dev)
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=dev)
    w = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device=dev)
    call = lambda: moe.moe_route(p, inp["x"], inp["Wg"], inp["bias"], idx, w, ws)
    for _ in range(W):
        call()
    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(K):
        call()
    end.record()
    torch.cuda.synchronize(dev)
    assert moe.moe_get_device_status(ws) == 0
    ms = start.elapsed_time(end) / K
    cfgd = config_dict(cfg, args, 1)
    cfgd["l2"] = "no flush between calls (x and W_g may stay in L2)"
    emit({"metric": "MoE router tokens/s", "value": cfg.T / (ms / 1e3), "unit": "tokens/s",
          "n_gpus": 1, "steps": K, "warmup": W, "ms_per_step": ms, "higher_is_better": True,
          "dtype": "f32 logits from bf16 inputs", "data": "synthetic", "config": cfgd,
          "router": "filter" if moe.moe_route_uses_filter(p) else "sequential"})
    return 0


def run_ep_local(args):
    """The expert-parallel layer for N ranks in one launch on one GPU: rank r routes tokens
    [r T/N, (r+1) T/N) of the workload and holds experts [r E/N, (r+1) E/N); K timed calls
    (the same total work as the single-GPU layer; its exchange stores stay on this GPU)."""
    import torch

    import mixture_experts_layer_forward_b200 as moe
    from mixture_experts_layer_forward_b200 import ep, synth

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    cfg = workload(args)
    N = args.ep_local
    K, W = args.steps, max(3, args.warmup)
    if cfg.T % N or cfg.E % N:
        raise SystemExit(f"--ep-local {N} must divide T = {cfg.T} and E = {cfg.E}")
    inp = synth.make_inputs(cfg, seed=args.seed, device=dev)
    T, el = cfg.T // N, cfg.E // N
    xs = [inp["x"][r * T:(r + 1) * T].contiguous() for r in range(N)]
    W1s = [inp["W1"][r * el:(r + 1) * el].contiguous() for r in range(N)]
    W2s = [inp["W2"][r * el:(r + 1) * el].contiguous() for r in range(N)]
    p = moe.Problem.make(T, cfg.H, cfg.F, cfg.E, cfg.k, cfg.act, cfg.gate)
    bufs = [ep.ep_layer_buffers(p, N, dev) for _ in range(N)]
    wss = [torch.empty(moe.moe_ep_workspace_size(p, N), dtype=torch.uint8, device=dev)
           for _ in range(N)]
    outs = [torch.empty(T, cfg.H, dtype=torch.bfloat16, device=dev) for _ in range(N)]
    epoch = [0]

    def call():
        epoch[0] += 1
        ep.ep_layer_forward_local(p, xs, inp["Wg"], inp["bias"], W1s, W2s, outs, bufs, wss,
                                  epoch[0])

    for _ in range(W):
        call()
    torch.cuda.synchronize(dev)
    sampler = new_sampler(torch, dev, not args.no_clocks)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.time()
    start.record()
    for _ in range(K):
        call()
    end.record()
    torch.cuda.synchronize(dev)
    t1 = time.time()
    clocks = sampler.stop(t0, t1) if sampler else None
    for w in wss:
        assert moe.moe_get_device_status(w) == 0
    ms = start.elapsed_time(end) / K
    cfgd = config_dict(cfg, args, 1)
    cfgd["parallelism"] = f"ep{N} emulated: {N} ranks in one launch on one GPU"
    line = {"metric": "MoE-layer forward tokens/s", "value": cfg.T / (ms / 1e3), "unit": "tokens/s",
            "n_gpus": 1, "steps": K, "warmup": W, "ms_per_step": ms, "higher_is_better": True,
            "dtype": "bf16", "data": "synthetic", "config": cfgd, "impl": "ep_local",
            "gpu_launches": K, "clocks": clocks}
    if args.trace is not None:
        # rank 0's CTAs record their work items (front, scatter, GEMM tiles, combine items)
        line["schedule_trace"] = schedule_trace(torch, moe, call, dev, args.trace or None)
    emit(line)
    return 0


def run_backward(args):
    """The layer's backward on one GPU: K timed moe_backward calls (each recomputes the
    routing, the dispatch and z = x W1) on a seeded dL/dout."""
    import torch

    import mixture_experts_layer_forward_b200 as moe
    from mixture_experts_layer_forward_b200 import synth

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    cfg = workload(args)
    K, W = args.steps, max(3, args.warmup)
    inp = synth.make_inputs(cfg, seed=args.seed, device=dev)
    p = moe.Problem.from_config(cfg)
    g = torch.Generator(device=dev).manual_seed(args.seed + 1)
    dy = torch.randn(cfg.T, cfg.H, generator=g, device=dev).to(torch.bfloat16)
    w1c = 2 * cfg.F if cfg.act == 0 else cfg.F
    dx = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=dev)
    dWg = torch.empty(cfg.H, cfg.E, dtype=torch.float32, device=dev)
    dbias = torch.empty(cfg.E, dtype=torch.float32, device=dev)
    dW1 = torch.empty(cfg.E, cfg.H, w1c, dtype=torch.bfloat16, device=dev)
    dW2 = torch.empty(cfg.E, cfg.F, cfg.H, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(moe.moe_backward_workspace_size(p), dtype=torch.uint8, device=dev)
    call = lambda: moe.moe_backward(p, inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W2"], dy,
                                    dx, dWg, dbias, dW1, dW2, ws)
    for _ in range(W):
        call()
    torch.cuda.synchronize(dev)
    assert moe.moe_get_device_status(ws) == 0
    sampler = None
    if not args.no_clocks:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
        sampler.start()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_begin = time.time()
    start.record()
    for _ in range(K):
        call()
    end.record()
    torch.cuda.synchronize(dev)
    clocks = sampler.stop(t_begin, time.time()) if sampler is not None else None
    assert moe.moe_get_device_status(ws) == 0
    ms = start.elapsed_time(end) / K
    # GEMM FLOPs: z = x W1 recomputed (2 T k H w1c), u = dy W2^T (2 T k H F), dW2 (2 T k F H),
    # dW1 (2 T k H w1c), dx rows (2 T k w1c H); "useful" leaves out the recomputation
    tk = cfg.T * cfg.k
    flops = 2 * tk * cfg.H * (3 * w1c + 2 * cfg.F)
    useful = flops - 2 * tk * cfg.H * w1c
    peaks, peak_src = load_peaks()
    tf = flops / (ms / 1e3) / 1e12
    rf = {"bound": "tensor", "achieved": tf, "unit": "TFLOP/s"}
    rf.update(tensor_fracs(tf, peaks, clocks))
    rf["peak_source"] = f"{peak_src} bf16 {rf['regime']}; regime from the median sampled SM clock"
    emit({"metric": "MoE-layer backward tokens/s", "value": cfg.T / (ms / 1e3), "unit": "tokens/s",
          "n_gpus": 1, "steps": K, "warmup": W, "ms_per_step": ms, "higher_is_better": True,
          "dtype": "bf16 (fp32 accumulation)", "data": "synthetic", "config": config_dict(cfg, args, 1),
          "gemm_tflops": tf, "useful_tflops": useful / (ms / 1e3) / 1e12,
          "roofline": rf,
          "clocks": clocks})
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.router_only:
        return run_router(args)
    if args.ep_local:
        return run_ep_local(args)
    if args.backward:
        return run_backward(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
