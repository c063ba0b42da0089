#!/usr/bin/env python
"""Benchmark of the GLM-5.2 MoE feed-forward layer forward pass on B200.

One step = one moe_forward call over one batch (router logits, routing,
grouping, row gather, gate/up GEMM with the SiLU gate, down GEMM, merge) on
inputs already resident in HBM; the L2 cache is flushed (256 MiB memset)
before every timed step, outside the step's events.  Prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config decode]
  python bench.py --impl reference ...   # the CPU oracle on the host cores

Multi-GPU (torchrun, one process per GPU): every rank runs an independent
replica on its own batch (the layer shards over tokens with no exchange), so
scaling is weak; the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time
from datetime import timedelta

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import moe_inputs as mi  # noqa: E402

METRIC = "MoE-layer tokens/sec on 1 B200 and % of roofline (HBM or bf16 tensor peak)"
FLUSH_BYTES = 256 << 20
L2_BYTES = 126 * 10**6        # B200 L2 capacity
STAGES = ["router_logits", "route", "permute", "gather", "expert_ffn", "combine"]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------
# ranks: one process per GPU, one independent replica per rank
# ---------------------------------------------------------------------------
def rank_env():
    """(rank, world, local_rank) from the torchrun environment (1 process if unset)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def replica_seed(rank: int) -> int:
    """Seed of a rank's token batch: rank 0 runs the seed-0 workload the tests check."""
    return rank


def max_over_ranks(values, world: int, device="cpu"):
    """Element-wise max of per-rank floats over all ranks (the slowest rank sets
    the step time)."""
    if world <= 1:
        return list(values)
    t = torch.tensor(list(values), device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def aggregate_tokens_per_s(tokens_per_rank: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's step time."""
    return world * tokens_per_rank / (max_ms / 1e3)


# ---------------------------------------------------------------------------
# accounting
# ---------------------------------------------------------------------------
def expert_weight_bytes(rows: int, K: int, weights: str) -> int:
    """Bytes of one expert matrix [rows, K]: bf16, or FP8 codes plus one int8
    exponent per 128 x 128 block."""
    if weights == "fp8":
        return rows * K + -(-rows // 128) * -(-K // 128)
    return rows * K * 2


def layer_bytes_flops(cfg, U: int, weights: str = "bf16"):
    """Algorithmic bytes and flops of one layer pass (touched experts only):
    expert weights of the touched routed experts and of the shared experts, the
    router weight and bias, the bf16 input, the fp32 output, the routing."""
    T, D, E, F, k, S, Fs = cfg.T, cfg.D, cfg.E, cfg.F, cfg.k, cfg.S, cfg.Fs
    wb = 3 * (U * expert_weight_bytes(F, D, weights) + S * expert_weight_bytes(Fs, D, weights))
    B = wb + E * D * 4 + E * 4 + T * D * 2 + T * D * 4 + T * k * 8
    FL = 2 * T * D * E + 6 * D * F * T * k + 6 * D * Fs * T * S
    return B, FL


def ffn_bytes(cfg, U: int, weights: str = "bf16", shared: bool = True):
    """Algorithmic bytes of one expert-FFN launch (gate/up and down GEMMs in one
    kernel): W1, W3 and W2 of the touched routed experts and (with `shared`) of
    the shared experts, the gathered bf16 input rows, and the fp32 expert
    outputs written.  The gated activations stay inside the kernel's working
    set and are not counted."""
    T, D, F, k, Fs = cfg.T, cfg.D, cfg.F, cfg.k, cfg.Fs
    S = cfg.S if shared else 0
    wb = 3 * (U * expert_weight_bytes(F, D, weights) + S * expert_weight_bytes(Fs, D, weights))
    return wb + (T * k + S * T) * D * 2 + (T * k + S * T) * D * 4


def ffn_flops(cfg, shared: bool = True):
    S = cfg.S if shared else 0
    return 6 * cfg.D * (cfg.F * cfg.T * cfg.k + cfg.Fs * cfg.T * S)


def workload_name(cfg) -> str:
    """The workload a bench line measures, named the same way by both arms."""
    family = {"glm45air": "GLM-4.5-Air-shaped ", "glm52": "GLM-5.2-shaped "}.get(cfg.weight_family,
                                                                               "small ")
    return (f"{cfg.name}: {family}MoE layer T={cfg.T} D={cfg.D} E={cfg.E} k={cfg.k} "
            f"F={cfg.F} S={cfg.S} Fs={cfg.Fs} scale={cfg.scale}")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_digest(paths) -> str:
    """First 16 hex digits of the SHA-256 of the given source files, concatenated."""
    import hashlib
    h = hashlib.sha256()
    for rel in paths:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def stored_traffic(kernel_key: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel_key)
    if not rec:
        return None
    srcs = rec["sources"]
    if not all(os.path.exists(os.path.join(ROOT, s)) for s in srcs):
        return None
    if source_digest(srcs) != rec["sources_sha256_16"]:
        return None
    return rec["dram_bytes_per_launch"]


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            gid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gid, f"--query-gpu={self.FIELDS}", "--format=csv,noheader",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        mhz, maxs, reasons = [], [], set()
        capped = 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz.append(float(parts[1].split()[0]))
                maxs.append(float(parts[2].split()[0]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
            capped += parts[8].lower() == "active"
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": max(maxs),
                "reasons": sorted(reasons), "samples": len(mhz),
                "power_cap_fraction": capped / len(mhz)}


# ---------------------------------------------------------------------------
# CPU oracle timing (test infrastructure; the product path never imports it)
# ---------------------------------------------------------------------------
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads") for p in threadpool_info() if p.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_sample_runner(cfg, h_rows: np.ndarray, Wr: np.ndarray, bias: np.ndarray, expert_fn,
                         shared):
    from oracle import moe_oracle as orc

    def run():
        return orc.moe_layer_tokens(h_rows, Wr, bias, cfg.k, cfg.scale, expert_fn, shared)
    return run


def time_oracle(run, n_tokens: int, min_s: float, max_s: float):
    run()  # untimed: fills the host copies of the touched experts
    t0 = time.perf_counter()
    reps = 0
    while True:
        run()
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_s or el >= max_s:
            break
    return n_tokens * reps / el, reps, el


def cpu_baseline_from_device(cfg, inp, n_tokens: int, fp8=None):
    """The oracle on the first tokens of the batch; with `fp8` (codes and
    exponents) the experts are the oracle's decoding of the FP8 weights."""
    from oracle import moe_oracle as orc

    h = inp["h"][:n_tokens].float().cpu().numpy()
    Wr = inp["Wr"].cpu().numpy()
    bias = inp["bias"].cpu().numpy()
    cache = {}

    def matrices(names, g):
        if fp8 is None:
            return tuple(inp[n][g].cpu().double().numpy() for n in names)
        return tuple(orc.dequantize_fp8_blocks(fp8[n + "q"][g].cpu().numpy(),
                                               fp8[n + "e"][g].cpu().numpy()) for n in names)

    def expert(e):
        if e not in cache:
            cache[e] = matrices(("W1", "W3", "W2"), e)
        return cache[e]
    shared = [matrices(("Ws1", "Ws3", "Ws2"), s) for s in range(cfg.S)]
    run = oracle_sample_runner(cfg, h, Wr, bias, expert, shared)
    tps, reps, el = time_oracle(run, n_tokens, 10.0, 30.0)
    return {"value": tps, "unit": "tokens/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"first {n_tokens} tokens of the {cfg.name} batch, whole layer in numpy "
                      f"(fp32 routing, fp64 experts), {reps} passes in {el:.1f} s; touched "
                      f"expert weights pre-copied to the host"}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args, rank, world, local_rank):
    import sparse_moe_layer_04_b200 as moe

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = mi.CONFIGS[args.config]
    if args.experts or args.tokens:
        cfg = mi.custom_config(args.config, E=args.experts or cfg.E, T=args.tokens or cfg.T)
    inp = mi.layer_weights(cfg, 0, device=dev)
    inp["h"] = mi.hidden(cfg, seed=replica_seed(rank), device=dev)
    fp8 = None
    if args.weights == "fp8":
        # the FP8 layer stores only codes and block exponents
        fp8 = mi.fp8_layer_weights(inp)
        for n in ("W1", "W3", "W2", "Ws1", "Ws3", "Ws2"):
            del inp[n]
        torch.cuda.empty_cache()
        w8 = moe.fp8_weights(*(fp8[n + "q"] for n in ("W1", "W3", "W2", "Ws1", "Ws3", "Ws2")),
                             *(fp8[n + "e"] for n in ("W1", "W3", "W2", "Ws1", "Ws3", "Ws2")))
    d = moe.dims_of(cfg)
    ws = moe.alloc_workspace(d, dev)
    out = torch.empty((cfg.T, cfg.D), dtype=torch.float32, device=dev)
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=dev)
    wgt = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def forward(h, o, i=None, w=None):
        if fp8 is not None:
            moe.moe_forward_fp8(h, inp["Wr"], inp["bias"], w8, d, o, ws, i, w)
        else:
            moe.moe_forward(h, inp["Wr"], inp["bias"], inp["W1"], inp["W3"], inp["W2"],
                            inp["Ws1"], inp["Ws3"], inp["Ws2"], d, o, ws, i, w)

    def step():
        forward(inp["h"], out, idx, wgt)

    sampler = ClockSampler(local_rank)
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if moe.moe_get_device_status(ws) != 0:
        raise RuntimeError("device status error during warm-up: " + moe.moe_last_error())
    launches_per_step = moe.moe_last_launch_count()

    K = args.steps
    # headline loop: one event pair around each step (nothing recorded between
    # the step's kernels, so their programmatic launch overlap is intact)
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    for e in ev0 + ev1:  # create the CUDA events before the timed region
        e.record()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    for i in range(K):
        flush.zero_()
        ev0[i].record()
        step()
        ev1[i].record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    step_ms = [ev0[i].elapsed_time(ev1[i]) for i in range(K)]

    # profiled loop: events at every stage boundary (stage times and the
    # dominant kernel's duration, measured on the launching stream)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(moe.MOE_PROFILE_EVENTS)]
          for _ in range(K)]
    for evs in ev:
        for e in evs:
            e.record()
    torch.cuda.synchronize()
    for i in range(K):
        flush.zero_()
        moe.moe_set_profile_events(ev[i])
        step()
    moe.moe_set_profile_events(None)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if moe.moe_get_device_status(ws) != 0:
        raise RuntimeError("device status error in the timed region: " + moe.moe_last_error())

    stage_ms = {name: statistics.mean(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(K))
                for j, name in enumerate(STAGES)}
    profiled_ms = statistics.mean(ev[i][0].elapsed_time(ev[i][len(STAGES)]) for i in range(K))
    ms, ffn_ms = max_over_ranks([statistics.mean(step_ms), stage_ms["expert_ffn"]], world, dev)

    counts = torch.bincount(idx.flatten().long(), minlength=cfg.E)
    U = int((counts > 0).sum().item())

    # end to end, serial: pinned host input -> device -> layer -> pinned host
    # output, each step waited for (context for the pipelined figure below)
    h_pin = inp["h"].cpu().pin_memory()
    out_pin = torch.empty((cfg.T, cfg.D), dtype=torch.float32).pin_memory()
    h_dev = torch.empty_like(inp["h"])
    e2e_steps = min(K, 200)
    e2e_ms = []
    for i in range(e2e_steps + 3):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        h_dev.copy_(h_pin, non_blocking=True)
        forward(h_dev, out)
        out_pin.copy_(out, non_blocking=True)
        b.record()
        b.synchronize()
        if i >= 3:
            e2e_ms.append(a.elapsed_time(b))
    e2e_serial = max_over_ranks([statistics.mean(e2e_ms)], world, dev)[0]

    # end to end through the library's host-buffer pipeline (the C ABI call a
    # caller with host-resident activations makes): every step copies its
    # input from pinned host memory and its output back to pinned host memory;
    # the copies of steps n+1 and n-1 run on their own streams while step n's
    # layer runs.  Timed over all steps, from an idle device to the last
    # output in host memory.
    if fp8 is not None:
        pipe = moe.moe_pipeline_create(d, inp["Wr"], inp["bias"], w8=w8, keep=(fp8,))
    else:
        pipe = moe.moe_pipeline_create(d, inp["Wr"], inp["bias"], inp["W1"], inp["W3"], inp["W2"],
                                       inp["Ws1"], inp["Ws3"], inp["Ws2"])
    outs_pin = [out_pin, torch.empty_like(out_pin).pin_memory()]
    for i in range(3):
        moe.moe_pipeline_submit(pipe, h_pin, outs_pin[i % 2])
    moe.moe_pipeline_wait(pipe)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    # a step that streams less than twice the L2 gets the flush between steps,
    # on the compute stream and inside the timed region
    flush_e2e = ffn_bytes(cfg, U, args.weights) < 2 * L2_BYTES
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(e2e_steps):
        if flush_e2e:
            flush.zero_()
        moe.moe_pipeline_submit(pipe, h_pin, outs_pin[i % 2])
    moe.moe_pipeline_wait(pipe)   # every output is in host memory
    b.record()
    b.synchronize()
    moe.moe_pipeline_destroy(pipe)
    e2e = max_over_ranks([a.elapsed_time(b) / e2e_steps], world, dev)[0]

    if rank != 0:
        return None

    peaks, peak_src = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    bf16_burst = float(peaks["bf16_tflops"])
    bf16_sust = float(peaks.get("bf16_tflops_sustained", bf16_burst))
    # The tensor denominator: the burst figure for a step the power cap left
    # alone, the sustained one when the clock record of the run shows the power
    # cap active in at least a quarter of the samples (long tensor-heavy steps
    # run at the capped clock).  Both fractions are reported.
    capped = bool(clocks) and clocks.get("power_cap_fraction", 0.0) >= 0.25
    bf16 = bf16_sust if capped else bf16_burst
    tc_peak_choice = ("sustained (sw_power_cap active in >= 25% of the clock samples)" if capped
                      else "burst (power cap active in < 25% of the clock samples)")
    B, FL = layer_bytes_flops(cfg, U, args.weights)
    t_s = ms / 1e3
    t_roof_hbm = B / (hbm * 1e9)
    t_roof_tc = FL / (bf16 * 1e12)
    # With the shared experts beside the routing on their own stream, the FFN
    # launch timed here carries the routed experts only.
    overlap = moe.moe_forward_shared_overlap(d, fp8 is not None)
    f_bytes = ffn_bytes(cfg, U, args.weights, shared=not overlap)
    f_flops = ffn_flops(cfg, shared=not overlap)
    f_gbs = f_bytes / (ffn_ms / 1e3) / 1e9
    f_tfs = f_flops / (ffn_ms / 1e3) / 1e12
    f_bound = "hbm" if f_bytes / (hbm * 1e9) >= f_flops / (bf16 * 1e12) else "tensor"
    if f_bound == "hbm":
        roof = {"bound": "hbm", "achieved": f_gbs, "peak": hbm, "unit": "GB/s",
                "frac": f_gbs / hbm}
    else:
        roof = {"bound": "tensor", "achieved": f_tfs, "peak": bf16, "unit": "TFLOP/s",
                "frac": f_tfs / bf16}
    traffic_key = (("expert_ffn_fp8" if fp8 is not None else "expert_ffn")
                   + ("_routed/" if overlap else "/") + cfg.name)
    kernel = ("ffn_fp8_kernel (fused gate/up + down expert FFN, FP8 weights decoded into TMEM)"
              if fp8 is not None else "grouped_gemm_kernel (fused gate/up + down expert FFN)")
    if overlap:
        kernel += ("; routed experts (the shared expert's FFN runs beside the routing on an "
                   "internal stream)")
    roof.update({"traffic": stored_traffic(traffic_key), "kernel": kernel, "ms": ffn_ms,
                 "algorithmic_bytes": f_bytes, "algorithmic_flops": f_flops,
                 "tensor_peak": tc_peak_choice,
                 "tensor_frac_burst": f_tfs / bf16_burst, "tensor_frac_sustained": f_tfs / bf16_sust,
                 "peak_source": f"{peak_src} (MEASURED_PEAKS.json)" if peak_src == "measured"
                 else "fallback (profiling recipe)"})

    res = {
        "metric": METRIC,
        "value": aggregate_tokens_per_s(cfg.T, world, ms),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded counter-based generator; random-init weights of the layer's shapes)",
        "config": {"workload": workload_name(cfg),
                   "T": cfg.T, "touched_experts": U, "global_batch": world * cfg.T,
                   "weights": ("fp8 e4m3 codes + power-of-two 128x128 block exponents, decoded "
                               "exactly to bf16 in the kernel" if fp8 is not None else "bf16"),
                   "parallelism": f"replicas x{world} (token-parallel, no exchange)",
                   "l2": "flushed: 256 MiB memset before every timed step, outside its events",
                   "ms_p10_p90": [float(np.percentile(step_ms, 10)), float(np.percentile(step_ms, 90))],
                   "stage_ms": stage_ms, "profiled_step_ms": profiled_ms},
        "roofline": roof,
        "layer_roofline": {
            "bytes": B, "flops": FL, "t_roof_ms": max(t_roof_hbm, t_roof_tc) * 1e3,
            "binding": "hbm" if t_roof_hbm >= t_roof_tc else "tensor",
            "frac": max(t_roof_hbm, t_roof_tc) / t_s,
            "hbm_frac": t_roof_hbm / t_s, "tensor_frac": t_roof_tc / t_s,
            "tensor_frac_burst": FL / (bf16_burst * 1e12) / t_s,
            "tensor_frac_sustained": FL / (bf16_sust * 1e12) / t_s,
            "peaks": {"hbm_gbs": hbm, "bf16_tflops": bf16, "bf16_tflops_burst": bf16_burst,
                      "bf16_tflops_sustained": bf16_sust, "tensor_peak": tc_peak_choice,
                      "source": peak_src}},
        "e2e": {"value": aggregate_tokens_per_s(cfg.T, world, e2e), "unit": "tokens/s",
                "h2d_bytes_per_step": cfg.T * cfg.D * 2, "d2h_bytes_per_step": cfg.T * cfg.D * 4,
                "ms_per_step": e2e, "steps": e2e_steps,
                "api": "moe_pipeline_submit / moe_pipeline_wait (pinned host buffers)",
                "mode": "pipelined: input copy of step n+1 and output copy of step n-1 overlap "
                        "the layer of step n; " + (
                            "L2 flushed between steps inside the timed region" if flush_e2e else
                            "L2 not flushed (each step streams the touched experts' weights, "
                            "more than twice the 126 MB L2)"),
                "serial": {"value": aggregate_tokens_per_s(cfg.T, world, e2e_serial),
                           "ms_per_step": e2e_serial,
                           "mode": "copy in, layer, copy out, then wait, per step; L2 flushed "
                                   "before every step outside its events"}},
        "gpu_launches": launches_per_step * K,
        "gpu_launches_note": "kernels of the headline timed loop (the profiled loop runs as many again)",
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline_from_device(cfg, inp, min(cfg.T, args.cpu_tokens), fp8)
    return res


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle, as it stands, on the host cores
# ---------------------------------------------------------------------------
def run_reference(args):
    from oracle import moe_oracle as orc

    cfg = mi.CONFIGS[args.config]
    n = min(cfg.T, args.cpu_tokens)
    h = mi.hidden(cfg, 0).float().numpy()[:n]
    Wr = mi.router_weight(cfg, 0).numpy()
    bias = mi.correction_bias(cfg, 0).numpy()
    cache = {}

    def matrices(ws):
        if args.weights == "fp8":   # the weights the FP8 codes stand for
            return tuple(orc.dequantize_fp8_blocks(*(t.numpy() for t in mi.quantize_fp8_blocks(x)))
                         for x in ws)
        return tuple(x.double().numpy() for x in ws)

    def expert(e):
        if e not in cache:
            cache[e] = matrices(mi.expert_weights(cfg, e, 0))
        return cache[e]
    shared = [matrices(mi.expert_weights(cfg, s, 0, shared=True)) for s in range(cfg.S)]

    def step():
        return orc.moe_layer_tokens(h, Wr, bias, cfg.k, cfg.scale, expert, shared)

    step()  # untimed: generates the touched experts' weights
    for _ in range(args.warmup):
        step()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        step()
        times.append(time.perf_counter() - t0)
    ms = statistics.mean(times) * 1e3
    value = n / (ms / 1e3)
    cores = _blas_threads()
    sample = (f"first {n} tokens of the {cfg.name} batch per step, whole layer in numpy "
              f"(fp32 routing, fp64 experts); touched experts generated before timing")
    return {
        "metric": METRIC, "value": value, "unit": "tokens/s", "impl": "reference",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded counter-based generator)",
        "config": {"workload": workload_name(cfg), "T": cfg.T,
                   "sample_tokens": n, "weights": args.weights},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="decode", choices=sorted(mi.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-tokens", type=int, default=128,
                    help="tokens of the batch the CPU oracle processes per pass")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--weights", default="bf16", choices=["bf16", "fp8"],
                    help="expert weight storage: bf16 (the headline layer) or FP8 E4M3 with "
                         "128x128 block scales")
    ap.add_argument("--experts", type=int, default=None,
                    help="override E (small cases for profiler captures; not a bench line)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override T (small cases for profiler captures; not a bench line)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    rank, world, local_rank = rank_env()

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args)), flush=True)
        return 0

    if world > 1:
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        res = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    if res is not None:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
