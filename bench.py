#!/usr/bin/env python
"""Benchmark of the GLM-5.2 MoE feed-forward layer forward pass on B200.

One step = one moe_forward call over one batch (router logits, routing,
grouping, row gather, gate/up GEMM with the SiLU gate, down GEMM, merge) on
inputs already resident in HBM; the L2 cache is flushed (256 MiB memset)
before every timed step, outside the step's events.  Prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config decode]
  python bench.py --impl reference ...   # the CPU oracle on the host cores

The headline is the --config workload (decode by default).  The same run then
times the other workloads in `--per-config` (prefill, skew, GLM-4.5-Air and
the N(0, 1)-hidden decode batch by default) with the same steps, warm-up and
L2 flush, each with its own roofline and clock record, under
"per_config" in the JSON line.

Multi-GPU: one process per GPU.  Under torchrun (RANK/WORLD_SIZE set) every
rank runs an independent replica on its own batch (the layer shards over
tokens with no exchange), so scaling is weak and the step time is the max
over ranks.  Without torchrun, `--gpus N` (N > 1) starts the N ranks itself
through torch.distributed.run.
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
    """Algorithmic bytes of one expert-FFN launch: W1, W3 and W2 of the touched
    routed experts and (with `shared`) of the shared experts, plus each token's
    bf16 hidden row read once.  The gathered rows, the gated activations and
    the fp32 expert outputs are the kernel's own intermediates and are not
    counted."""
    T, D, F, Fs = cfg.T, cfg.D, cfg.F, cfg.Fs
    S = cfg.S if shared else 0
    wb = 3 * (U * expert_weight_bytes(F, D, weights) + S * expert_weight_bytes(Fs, D, weights))
    return wb + T * D * 2


def ffn_kernel_bytes(cfg, U: int, weights: str = "bf16", shared: bool = True):
    """The FFN launch's bytes with its row traffic: the weights, the gathered
    bf16 input rows read and the fp32 expert outputs written (a secondary
    figure; the roofline uses ffn_bytes)."""
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


def workload_config(cfg, n_gpus: int, fp8: bool) -> dict:
    """The workload a line measures, the same in both arms' lines (the
    measurement's own details go under "run")."""
    return {"workload": workload_name(cfg), "T": cfg.T, "global_batch": n_gpus * cfg.T,
            "weights": ("fp8 e4m3 codes + power-of-two 128x128 block exponents, decoded "
                        "exactly to bf16" if fp8 else "bf16")}


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
_REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}


def summarize_clocks(samples):
    """Clock record of a run from (sm_mhz, sm_max_mhz, reason_bits) samples:
    median SM clock, the maximum, the throttle reasons seen, and the share of
    samples with the power cap active."""
    if not samples:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                "power_cap_fraction": 0.0}
    reasons = sorted({n for _, _, bits in samples for n, b in _REASON_BITS.items() if bits & b})
    capped = sum(1 for _, _, bits in samples if bits & _REASON_BITS["sw_power_cap"])
    return {"sm_mhz": statistics.median(m for m, _, _ in samples),
            "sm_max_mhz": max(x for _, x, _ in samples), "reasons": reasons,
            "samples": len(samples), "power_cap_fraction": capped / len(samples)}


class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons of one GPU
    every `period_s` in a background thread (NVML) between start() and stop(),
    i.e. during the timed loops."""

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.period_s = period_s
        self.samples = []
        self.handle = None
        self.thread = None
        self.running = False
        try:
            import pynvml
            self.nvml = pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            gid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(gid.encode())
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
            self.reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception:
            self.handle = None

    def _run(self):
        nv = self.nvml
        while self.running:
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                bits = self.reasons_fn(self.handle)
                self.samples.append((float(mhz), float(self.max_mhz), int(bits)))
            except Exception:
                pass
            time.sleep(self.period_s)

    def start(self):
        import threading
        self.samples = []
        if self.handle is None:
            return self
        self.running = True
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()
        return self

    def stop(self):
        if self.thread is not None:
            self.running = False
            self.thread.join()
            self.thread = None
        rec = summarize_clocks(self.samples)
        rec["source"] = "NVML, sampled every %.0f ms during the timed loops" % (self.period_s * 1e3) \
            if self.handle is not None else "unavailable"
        return rec


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
FP8_NAMES = ("W1", "W3", "W2", "Ws1", "Ws3", "Ws2")


def pick_tensor_peak(clocks, bf16_burst: float, bf16_sust: float):
    """The tensor denominator: the burst figure for a step the power cap left
    alone, the sustained one when the clock record shows the power cap active
    in at least a quarter of the samples (long tensor-heavy steps run at the
    capped clock).  Both fractions are reported either way."""
    capped = bool(clocks) and clocks.get("power_cap_fraction", 0.0) >= 0.25
    if capped:
        return bf16_sust, "sustained (sw_power_cap active in >= 25% of the clock samples)"
    return bf16_burst, "burst (power cap active in < 25% of the clock samples)"


def roofline_report(cfg, U: int, weights: str, overlap: bool, ms: float, ffn_ms: float, clocks,
                    peaks, peak_src: str, fp8: bool):
    """The dominant kernel's roofline (the expert FFN launch) and the whole
    layer's, for one measured configuration."""
    hbm = float(peaks["hbm_gbs"])
    bf16_burst = float(peaks["bf16_tflops"])
    bf16_sust = float(peaks.get("bf16_tflops_sustained", bf16_burst))
    bf16, tc_peak_choice = pick_tensor_peak(clocks, bf16_burst, bf16_sust)
    B, FL = layer_bytes_flops(cfg, U, weights)
    t_s = ms / 1e3
    t_roof_hbm = B / (hbm * 1e9)
    t_roof_tc = FL / (bf16 * 1e12)
    # With the shared experts beside the routing on their own stream, the FFN
    # launch timed here carries the routed experts only.
    f_bytes = ffn_bytes(cfg, U, weights, shared=not overlap)
    f_kbytes = ffn_kernel_bytes(cfg, U, weights, shared=not overlap)
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
    traffic_key = (("expert_ffn_fp8" if fp8 else "expert_ffn")
                   + ("_routed/" if overlap else "/") + cfg.name)
    kernel = ("ffn_fp8_kernel (fused gate/up + down expert FFN, FP8 weights decoded into TMEM)"
              if fp8 else "grouped_gemm_kernel (fused gate/up + down expert FFN)")
    if overlap:
        kernel += ("; routed experts (the shared expert's FFN runs beside the routing on an "
                   "internal stream)")
    roof.update({
        "traffic": stored_traffic(traffic_key), "kernel": kernel, "ms": ffn_ms,
        "algorithmic_bytes": f_bytes,
        "algorithmic_bytes_def": "touched expert weights + each token's hidden row read once",
        "algorithmic_flops": f_flops,
        "hbm_frac": f_gbs / hbm,
        "hbm_frac_with_row_traffic": f_kbytes / (ffn_ms / 1e3) / 1e9 / hbm,
        "tensor_peak": tc_peak_choice,
        "tensor_frac_burst": f_tfs / bf16_burst, "tensor_frac_sustained": f_tfs / bf16_sust,
        "peak_source": f"{peak_src} (MEASURED_PEAKS.json)" if peak_src == "measured"
        else "fallback (profiling recipe)"})
    layer = {
        "bytes": B, "flops": FL, "t_roof_ms": max(t_roof_hbm, t_roof_tc) * 1e3,
        "binding": "hbm" if t_roof_hbm >= t_roof_tc else "tensor",
        "frac": max(t_roof_hbm, t_roof_tc) / t_s,
        "hbm_frac": t_roof_hbm / t_s, "tensor_frac": t_roof_tc / t_s,
        "tensor_frac_burst": FL / (bf16_burst * 1e12) / t_s,
        "tensor_frac_sustained": FL / (bf16_sust * 1e12) / t_s,
        "peaks": {"hbm_gbs": hbm, "bf16_tflops": bf16, "bf16_tflops_burst": bf16_burst,
                  "bf16_tflops_sustained": bf16_sust, "tensor_peak": tc_peak_choice,
                  "source": peak_src}}
    return roof, layer


class Layer:
    """One workload's inputs on the device and the layer call on them."""

    def __init__(self, moe, cfg, inp, w8, dev):
        self.moe, self.cfg, self.inp, self.w8 = moe, cfg, inp, w8
        self.d = moe.dims_of(cfg)
        self.ws = moe.alloc_workspace(self.d, dev)
        self.out = torch.empty((cfg.T, cfg.D), dtype=torch.float32, device=dev)
        self.idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=dev)
        self.wgt = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device=dev)

    def forward(self, h, o, i=None, w=None):
        moe, inp = self.moe, self.inp
        if self.w8 is not None:
            moe.moe_forward_fp8(h, inp["Wr"], inp["bias"], self.w8, self.d, o, self.ws, i, w)
        else:
            moe.moe_forward(h, inp["Wr"], inp["bias"], inp["W1"], inp["W3"], inp["W2"],
                            inp["Ws1"], inp["Ws3"], inp["Ws2"], self.d, o, self.ws, i, w)

    def step(self):
        self.forward(self.inp["h"], self.out, self.idx, self.wgt)

    def status_check(self, where: str):
        if self.moe.moe_get_device_status(self.ws) != 0:
            raise RuntimeError(f"device status error {where} ({self.cfg.name}): "
                               + self.moe.moe_last_error())

    def touched(self) -> int:
        counts = torch.bincount(self.idx.flatten().long(), minlength=self.cfg.E)
        return int((counts > 0).sum().item())


def time_layer(L: Layer, K: int, warmup: int, flush, world: int, dev, sampler: ClockSampler):
    """W untimed steps, then K timed steps (one event pair per step, nothing
    recorded between the step's kernels), then K profiled steps (events at the
    stage boundaries: stage times and the FFN launch's duration).  L2 flushed
    before every step.  Returns the per-rank timings and the clock record of
    the timed loops."""
    moe = L.moe
    for _ in range(warmup):
        flush.zero_()
        L.step()
    torch.cuda.synchronize()
    L.status_check("during warm-up")
    launches = moe.moe_last_launch_count()
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    for e in ev0 + ev1:  # create the CUDA events before the timed region
        e.record()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(moe.MOE_PROFILE_EVENTS)]
          for _ in range(K)]
    for evs in ev:
        for e in evs:
            e.record()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler.start()
    for i in range(K):
        flush.zero_()
        ev0[i].record()
        L.step()
        ev1[i].record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    step_ms = [ev0[i].elapsed_time(ev1[i]) for i in range(K)]
    for i in range(K):
        flush.zero_()
        moe.moe_set_profile_events(ev[i])
        L.step()
    moe.moe_set_profile_events(None)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    L.status_check("in the timed region")
    stage_ms = {name: statistics.mean(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(K))
                for j, name in enumerate(STAGES)}
    profiled_ms = statistics.mean(ev[i][0].elapsed_time(ev[i][len(STAGES)]) for i in range(K))
    ms, ffn_ms = max_over_ranks([statistics.mean(step_ms), stage_ms["expert_ffn"]], world, dev)
    return {"ms": ms, "ffn_ms": ffn_ms, "step_ms": step_ms, "stage_ms": stage_ms,
            "profiled_ms": profiled_ms, "launches": launches, "clocks": clocks}


def config_inputs(moe, cfg, rank: int, dev, cache: dict, fp8_mode: bool):
    """Device inputs of a workload: the weights of its family (generated once
    per family and shared, with their FP8 codes in FP8 mode), its bias and its
    hidden states (seeded by rank)."""
    # weights are shared by the workloads of one family and one shape only (a
    # run with --experts / --tokens has its own)
    fam = (cfg.weight_family, cfg.E, cfg.D, cfg.F, cfg.S, cfg.Fs)
    if fam not in cache:
        w = mi.layer_weights(cfg, 0, device=dev)
        w8 = None
        if fp8_mode:
            # the FP8 layer stores only codes and block exponents
            q = mi.fp8_layer_weights(w)
            for n in FP8_NAMES:
                del w[n]
            torch.cuda.empty_cache()
            w8 = moe.fp8_weights(*(q[n + "q"] for n in FP8_NAMES), *(q[n + "e"] for n in FP8_NAMES))
            w["_fp8"] = q
        cache[fam] = (w, w8)
    w, w8 = cache[fam]
    inp = dict(w)
    inp["bias"] = mi.correction_bias(cfg, 0, device=dev)
    inp["h"] = mi.hidden(cfg, seed=replica_seed(rank), device=dev)
    return inp, w8


def run_ours(args, rank, world, local_rank):
    import sparse_moe_layer_04_b200 as moe

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = mi.CONFIGS[args.config]
    if args.experts or args.tokens:
        cfg = mi.custom_config(args.config, E=args.experts or cfg.E, T=args.tokens or cfg.T)
    fp8_mode = args.weights == "fp8"
    cache = {}
    inp, w8 = config_inputs(moe, cfg, rank, dev, cache, fp8_mode)
    L = Layer(moe, cfg, inp, w8, dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    sampler = ClockSampler(local_rank)
    peaks, peak_src = load_peaks()

    K = args.steps
    t = time_layer(L, K, args.warmup, flush, world, dev, sampler)
    ms, ffn_ms = t["ms"], t["ffn_ms"]
    U = L.touched()

    # end to end, serial: pinned host input -> device -> layer -> pinned host
    # output, each step waited for (context for the pipelined figure below)
    h_pin = inp["h"].cpu().pin_memory()
    out_pin = torch.empty((cfg.T, cfg.D), dtype=torch.float32).pin_memory()
    h_dev = torch.empty_like(inp["h"])
    e2e_steps = min(K, 200)
    e2e_ms = []
    sampler_e2e = ClockSampler(local_rank).start()
    for i in range(e2e_steps + 3):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        h_dev.copy_(h_pin, non_blocking=True)
        L.forward(h_dev, L.out)
        out_pin.copy_(L.out, non_blocking=True)
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
    if w8 is not None:
        pipe = moe.moe_pipeline_create(L.d, inp["Wr"], inp["bias"], w8=w8, keep=(inp["_fp8"],))
    else:
        pipe = moe.moe_pipeline_create(L.d, inp["Wr"], inp["bias"], inp["W1"], inp["W3"],
                                       inp["W2"], inp["Ws1"], inp["Ws3"], inp["Ws2"])
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
    clocks_e2e = sampler_e2e.stop()
    moe.moe_pipeline_destroy(pipe)
    e2e = max_over_ranks([a.elapsed_time(b) / e2e_steps], world, dev)[0]

    overlap = bool(moe.moe_forward_shared_overlap(L.d, w8 is not None))
    roof, layer = roofline_report(cfg, U, args.weights, overlap, ms, ffn_ms, t["clocks"], peaks,
                                  peak_src, w8 is not None)

    # the other workloads, same steps, warm-up and L2 flush
    per_config = {}
    names = [n for n in (args.per_config.split(",") if args.per_config else []) if n]
    for name in names:
        if name == cfg.name:
            continue
        c = mi.CONFIGS[name]
        cinp, cw8 = config_inputs(moe, c, rank, dev, cache, fp8_mode)
        CL = Layer(moe, c, cinp, cw8, dev)
        ct = time_layer(CL, K, args.warmup, flush, world, dev, sampler)
        cU = CL.touched()
        c_overlap = bool(moe.moe_forward_shared_overlap(CL.d, cw8 is not None))
        croof, clayer = roofline_report(c, cU, args.weights, c_overlap, ct["ms"], ct["ffn_ms"],
                                        ct["clocks"], peaks, peak_src, cw8 is not None)
        per_config[name] = {
            "workload": workload_name(c), "T": c.T, "touched_experts": cU,
            "value": aggregate_tokens_per_s(c.T, world, ct["ms"]), "unit": "tokens/s",
            "ms_per_step": ct["ms"],
            "ms_p10_p90": [float(np.percentile(ct["step_ms"], 10)),
                           float(np.percentile(ct["step_ms"], 90))],
            "stage_ms": ct["stage_ms"], "roofline": croof, "layer_roofline": clayer,
            "clocks": ct["clocks"], "gpu_launches": ct["launches"] * K}
        del CL, cinp
        torch.cuda.empty_cache()

    if rank != 0:
        return None

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
        "config": workload_config(cfg, world, w8 is not None),
        "run": {"touched_experts": U,
                "parallelism": f"replicas x{world} (token-parallel, no exchange)",
                "l2": "flushed: 256 MiB memset before every timed step, outside its events",
                "ms_p10_p90": [float(np.percentile(t["step_ms"], 10)),
                               float(np.percentile(t["step_ms"], 90))],
                "stage_ms": t["stage_ms"], "profiled_step_ms": t["profiled_ms"]},
        "roofline": roof,
        "layer_roofline": layer,
        "e2e": {"value": aggregate_tokens_per_s(cfg.T, world, e2e), "unit": "tokens/s",
                "h2d_bytes_per_step": cfg.T * cfg.D * 2, "d2h_bytes_per_step": cfg.T * cfg.D * 4,
                "ms_per_step": e2e, "steps": e2e_steps,
                "api": "moe_pipeline_submit / moe_pipeline_wait (pinned host buffers)",
                "mode": "pipelined: input copy of step n+1 and output copy of step n-1 overlap "
                        "the layer of step n; " + (
                            "L2 flushed between steps inside the timed region" if flush_e2e else
                            "L2 not flushed (each step streams the touched experts' weights, "
                            "more than twice the 126 MB L2)"),
                "clocks": clocks_e2e,
                "serial": {"value": aggregate_tokens_per_s(cfg.T, world, e2e_serial),
                           "ms_per_step": e2e_serial,
                           "mode": "copy in, layer, copy out, then wait, per step; L2 flushed "
                                   "before every step outside its events"}},
        "gpu_launches": t["launches"] * K,
        "gpu_launches_note": "kernels of the headline timed loop (the profiled loop runs as many again)",
        "clocks": t["clocks"],
        "per_config": per_config,
    }
    if world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline_from_device(
            cfg, inp, min(cfg.T, args.cpu_tokens), inp.get("_fp8"))
    return res


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle, as it stands, on the host cores
# ---------------------------------------------------------------------------
def host_memory_available() -> int:
    try:
        import psutil
        return int(psutil.virtual_memory().available)
    except Exception:
        return 0


def run_reference(args):
    from oracle import moe_oracle as orc

    cfg = mi.CONFIGS[args.config]
    n = min(cfg.T, args.cpu_tokens)
    # the seeded inputs are made on the GPU when there is one (the same values
    # as on the CPU, much faster) and copied to the host; the timed oracle
    # passes run on the host cores only
    gen = "cuda" if torch.cuda.is_available() else "cpu"
    h = mi.hidden(cfg, 0, device=gen).float().cpu().numpy()[:n]
    Wr = mi.router_weight(cfg, 0, device=gen).cpu().numpy()
    bias = mi.correction_bias(cfg, 0, device=gen).cpu().numpy()
    # The oracle takes each selected expert's weights as fp64 arrays.  They are
    # made once, before timing, and kept when they fit in half the free host
    # memory; otherwise each pass makes them again from bf16 host copies (and
    # that conversion is then inside the timed passes).
    touched = np.unique(orc.route(orc.router_logits(h, Wr), bias, cfg.k, cfg.scale)[0])
    per_expert = 3 * cfg.D * cfg.F * 8
    keep_fp64 = len(touched) * per_expert <= host_memory_available() // 2
    cache = {}
    bf16_copies = {}

    def matrices(ws):
        if args.weights == "fp8":   # the weights the FP8 codes stand for
            return tuple(orc.dequantize_fp8_blocks(*(t.numpy() for t in mi.quantize_fp8_blocks(x)))
                         for x in ws)
        return tuple(x.double().numpy() for x in ws)

    def host_weights(e, shared=False):
        return tuple(x.cpu() for x in mi.expert_weights(cfg, e, 0, device=gen, shared=shared))

    def expert(e):
        if keep_fp64:
            if e not in cache:
                cache[e] = matrices(host_weights(e))
            return cache[e]
        if e not in bf16_copies:
            bf16_copies[e] = host_weights(e)
        return matrices(bf16_copies[e])
    shared = [matrices(host_weights(s, shared=True)) for s in range(cfg.S)]

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
    sample = (f"first {n} of {cfg.T} tokens of the {cfg.name} batch per step, whole layer in "
              f"numpy (fp32 routing, fp64 experts); {len(touched)} touched experts' weights "
              + ("made before timing" if keep_fp64 else
                 "converted from bf16 host copies inside every pass (fp64 copies would not fit)"))
    res = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "impl": "reference",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded counter-based generator)",
        "config": workload_config(cfg, args.gpus, args.weights == "fp8"),
        "run": {"sample_tokens": n},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    if n < cfg.T:
        # linear extrapolation of the sample's rate to the whole batch (marked)
        res["run"]["full_batch_s_extrapolated"] = cfg.T / value
    return res


# ---------------------------------------------------------------------------
# launcher
# ---------------------------------------------------------------------------
def free_port() -> int:
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def spawn_ranks(n: int, argv) -> int:
    """Runs this script as n ranks (one process per GPU) under
    torch.distributed.run on this node; returns its exit code."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", f"--master-port={free_port()}",
           os.path.abspath(__file__), *argv]
    env = dict(os.environ)
    env.setdefault("NCCL_DEBUG", "INFO")   # the NCCL log shows the rank count
    env.setdefault("OMP_NUM_THREADS", "1")
    return subprocess.call(cmd, env=env)


def launcher_check(args, rank: int, world: int) -> int:
    """Checks the rank layout without any CUDA work: every rank joins the
    process group (gloo) and rank 0 prints the ranks it saw."""
    torch.distributed.init_process_group("gloo", timeout=timedelta(seconds=60))
    try:
        seen = [None] * world
        torch.distributed.all_gather_object(seen, {"rank": rank, "pid": os.getpid()})
        if rank == 0:
            print(json.dumps({"launcher_check": True, "n_gpus": world, "gpus_requested": args.gpus,
                              "ranks": sorted(r["rank"] for r in seen),
                              "pids": len({r["pid"] for r in seen})}), flush=True)
    finally:
        torch.distributed.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="decode", choices=sorted(mi.CONFIGS))
    ap.add_argument("--per-config", default="prefill,skew,air,decode_b",
                    help="comma-separated workloads timed after the headline (empty: none)")
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
    ap.add_argument("--launcher-check", action="store_true",
                    help="start the ranks and report them over gloo, without any CUDA work")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    for name in (args.per_config.split(",") if args.per_config else []):
        if name and name not in mi.CONFIGS:
            ap.error(f"--per-config: unknown workload {name}")

    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        return spawn_ranks(args.gpus, sys.argv[1:])
    rank, world, local_rank = rank_env()
    if world != args.gpus:
        raise SystemExit(f"bench.py: --gpus {args.gpus} but {world} ranks were started")

    if args.launcher_check:
        return launcher_check(args, rank, world)

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
