"""The seeded input generator: determinism, moments, independence, stored bias."""
import numpy as np
import torch

import moe_inputs as mi


def test_counter_generator_is_deterministic_and_prefix_stable():
    a = mi.normal((1000,), 1.0, 0, "x")
    b = mi.normal((1000,), 1.0, 0, "x")
    c = mi.normal((2000,), 1.0, 0, "x")
    assert torch.equal(a, b)
    assert torch.equal(a, c[:1000])


def test_moments_and_stream_independence():
    a = mi.normal((400_000,), 0.02, 0, "a").double()
    b = mi.normal((400_000,), 0.02, 0, "b").double()
    assert abs(a.mean().item()) < 2e-4
    assert abs(a.std().item() / 0.02 - 1.0) < 5e-3
    corr = ((a - a.mean()) * (b - b.mean())).mean() / (a.std() * b.std())
    assert abs(corr.item()) < 1e-2
    # kurtosis of a normal is 3
    z = (a - a.mean()) / a.std()
    assert abs((z ** 4).mean().item() - 3.0) < 0.05


def test_mul32_matches_python_modular_product():
    x = torch.tensor([0, 1, 0xFFFFFFFF, 0x12345678, 0x80000000], dtype=torch.int64)
    for c in (0x85EBCA6B, 0xC2B2AE35, 0xFFFFFFFF):
        got = mi._mul32(x, c).tolist()
        assert got == [(int(v) * c) & 0xFFFFFFFF for v in x.tolist()]


def test_layer_shapes_and_dtypes():
    cfg = mi.CONFIGS["tiny"]
    w = mi.layer_weights(cfg)
    assert w["W1"].shape == (cfg.E, cfg.F, cfg.D) and w["W1"].dtype == torch.bfloat16
    assert w["W2"].shape == (cfg.E, cfg.D, cfg.F)
    assert w["Ws1"].shape == (cfg.S, cfg.Fs, cfg.D)
    assert w["Wr"].dtype == torch.float32 and w["bias"].shape == (cfg.E,)
    # bf16 tensors are the nearest-even rounding of the fp32 draw
    w32 = mi.layer_weights(cfg, fp32=True)
    assert torch.equal(w32["W1"].to(torch.bfloat16), w["W1"])


def test_skew_bias_file():
    cfg = mi.CONFIGS["skew"]
    b = mi.correction_bias(cfg).numpy()
    assert b.shape == (256,) and b.dtype == np.float32
    assert int((b == -2.0).sum()) == 16
    live = b[b != -2.0]
    assert live.min() > -1.0


def test_synthetic_topk_rows_are_distinct():
    idx = mi.synthetic_topk(100, 32, 8, 0, "t")
    for row in idx.tolist():
        assert len(set(row)) == 8 and all(0 <= e < 32 for e in row)
