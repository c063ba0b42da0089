"""The benchmark's accounting on the CPU: algorithmic bytes and flops of the
layer and of the expert-FFN launch (the roofline numerators), FP8 weight
bytes, whole-job throughput, and the traffic record keyed by kernel sources."""
import json
import subprocess
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import moe_inputs as mi  # noqa: E402


def test_expert_weight_bytes():
    assert bench.expert_weight_bytes(2048, 6144, "bf16") == 2048 * 6144 * 2
    # codes + one exponent per 128 x 128 block (ragged blocks count whole)
    assert bench.expert_weight_bytes(2048, 6144, "fp8") == 2048 * 6144 + 16 * 48
    assert bench.expert_weight_bytes(200, 136, "fp8") == 200 * 136 + 2 * 2


def test_decode_ffn_bytes_and_flops():
    cfg = mi.CONFIGS["decode"]
    T, D, F, k = cfg.T, cfg.D, cfg.F, cfg.k
    rows = T * k + T                                   # routed rows + shared rows
    weights = 11 * 3 * F * D * 2                       # 10 touched + 1 shared expert
    # algorithmic: the touched weights and each token's hidden row read once
    assert bench.ffn_bytes(cfg, 10) == weights + T * D * 2 == 832045056
    # with the kernel's own row traffic (gathered rows in, fp32 rows out)
    assert bench.ffn_kernel_bytes(cfg, 10) == weights + rows * D * 2 + rows * D * 4 == 872939520
    assert bench.ffn_kernel_bytes(cfg, 10, "fp8") == 457728768
    assert bench.ffn_bytes(cfg, 10, "fp8") == 3 * 11 * (F * D + 16 * 48) + T * D * 2
    assert bench.ffn_flops(cfg) == 6 * D * F * (T * k + T)
    # the routed experts alone (shared expert on its own stream)
    assert bench.ffn_bytes(cfg, 10, shared=False) == 10 * 3 * F * D * 2 + T * D * 2
    assert bench.ffn_kernel_bytes(cfg, 10, shared=False) == 10 * 3 * F * D * 2 + T * k * D * 6
    assert bench.ffn_flops(cfg, shared=False) == 6 * D * F * T * k
    B, FL = bench.layer_bytes_flops(cfg, 10)
    assert B == weights + cfg.E * D * 4 + cfg.E * 4 + T * D * 2 + T * D * 4 + T * k * 8
    assert FL == 2 * T * D * cfg.E + bench.ffn_flops(cfg)


def test_roofline_frac_is_algorithmic_bytes_over_time_over_peak():
    cfg = mi.CONFIGS["decode"]
    peaks = {"hbm_gbs": 6541.1, "bf16_tflops": 1650.0, "bf16_tflops_sustained": 1382.0}
    clocks = bench.summarize_clocks([(1965.0, 1965.0, 0)] * 4)
    roof, layer = bench.roofline_report(cfg, 10, "bf16", True, 0.18677, 0.13878, clocks, peaks,
                                        "measured", False)
    assert roof["bound"] == "hbm"
    expect = bench.ffn_bytes(cfg, 10, shared=False) / 0.13878e-3 / 1e9 / 6541.1
    assert roof["frac"] == pytest.approx(expect) and roof["frac"] == pytest.approx(0.8334, abs=1e-3)
    assert roof["hbm_frac_with_row_traffic"] > roof["frac"]
    B, _ = bench.layer_bytes_flops(cfg, 10)
    assert layer["frac"] == pytest.approx(B / 6541.1e9 / 0.18677e-3)


def test_clock_record_and_tensor_peak_choice():
    assert bench.summarize_clocks([])["samples"] == 0
    s = [(1965.0, 1965.0, 0), (1300.0, 1965.0, 0x4), (1290.0, 1965.0, 0x4 | 0x1),
         (1310.0, 1965.0, 0x4)]
    rec = bench.summarize_clocks(s)
    assert rec["samples"] == 4 and rec["sm_mhz"] == pytest.approx(1305.0)
    assert rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["sw_power_cap"] and rec["power_cap_fraction"] == 0.75
    assert bench.pick_tensor_peak(rec, 1650.0, 1382.0)[0] == 1382.0
    quiet = bench.summarize_clocks([(1965.0, 1965.0, 0)] * 4 + [(1965.0, 1965.0, 0x4)])
    assert bench.pick_tensor_peak(quiet, 1650.0, 1382.0)[0] == 1650.0
    hot = bench.summarize_clocks([(1700.0, 1965.0, 0x40 | 0x8)])
    assert hot["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]


def test_throughput_counts_every_rank():
    assert bench.aggregate_tokens_per_s(128, 1, 0.2) == pytest.approx(128 / 2e-4)
    assert bench.aggregate_tokens_per_s(128, 8, 0.2) == pytest.approx(8 * 128 / 2e-4)
    assert bench.max_over_ranks([1.0, 2.0], 1) == [1.0, 2.0]


def test_traffic_record_follows_the_kernel_sources(tmp_path, monkeypatch):
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        recs = json.load(f)
    for key, rec in recs.items():
        for src in rec["sources"]:
            assert os.path.exists(os.path.join(ROOT, src)), src
        assert rec["dram_bytes_per_launch"] > 0
    assert bench.stored_traffic("no_such_kernel/decode") is None
    # a record taken on other sources is not reported
    fake = tmp_path / "profiles"
    fake.mkdir()
    rec = dict(recs["expert_ffn_routed/decode"], sources_sha256_16="0" * 16)
    (fake / "traffic.json").write_text(json.dumps({"expert_ffn_routed/decode": rec}))
    for src in rec["sources"]:
        dst = tmp_path / src
        dst.parent.mkdir(parents=True, exist_ok=True)
        dst.write_bytes(open(os.path.join(ROOT, src), "rb").read())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.stored_traffic("expert_ffn_routed/decode") is None
    rec["sources_sha256_16"] = bench.source_digest(rec["sources"])
    (fake / "traffic.json").write_text(json.dumps({"expert_ffn_routed/decode": rec}))
    assert bench.stored_traffic("expert_ffn_routed/decode") == rec["dram_bytes_per_launch"]


def test_both_arms_name_the_workload_alike():
    for name in ("decode", "air", "tiny"):
        w = bench.workload_name(mi.CONFIGS[name])
        assert w.startswith(name + ": ") and f"T={mi.CONFIGS[name].T} " in w
    assert "GLM-4.5-Air" in bench.workload_name(mi.CONFIGS["air"])


def test_both_arms_print_the_same_config():
    """The reference (oracle) arm, run as the driver runs it, prints the same
    `config` object as `workload_config` gives our arm for that workload."""
    cfg = mi.CONFIGS["tiny"]
    ours = bench.workload_config(cfg, 1, False)
    assert ours == {"workload": bench.workload_name(cfg), "T": cfg.T, "global_batch": cfg.T,
                    "weights": "bf16"}
    assert bench.workload_config(cfg, 4, False)["global_batch"] == 4 * cfg.T
    assert bench.workload_config(cfg, 1, True)["weights"].startswith("fp8")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--config", "tiny", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["config"] == ours
