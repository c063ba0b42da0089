"""Write the correction bias of the skewed-load workload (T=16384, E=256, k=8).

TEST INFRASTRUCTURE: this script computes an *input* (the bias vector is data
the layer is given), using only the oracle's routing and the seeded inputs.

The workload asks for a bias under which expert popularity follows Zipf(1.1):
a few experts receive more than ten times the mean load and some receive no
token at all.  The pages give no construction; this is the plain reading:

1. A seeded permutation assigns every expert a popularity rank r = 1..E.
2. The last 16 ranks get bias -2.  Every selection key of those experts is
   then below -1 while every other key is above -1 (scores lie in (0, 1) and
   the calibrated biases stay above -1), so they are never selected.
3. The other 240 experts get target loads proportional to r**-1.1, scaled to
   T*k assignments and capped at T (an expert can serve each token once);
   the excess of capped experts is spread over the rest in proportion.
4. Starting from zero, the biases move in log-load space towards their
   targets, using the oracle's sigmoid scores of the workload's own hidden
   states and router weights; the iterate with the smallest L1 load error is
   kept.

Run:  python -m oracle.make_skew_bias   (writes moe_inputs/skew_bias_T16384_seed0.txt)
"""
from __future__ import annotations

import os
import sys

import numpy as np

_ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if _ROOT not in sys.path:
    sys.path.insert(0, _ROOT)

import moe_inputs as mi  # noqa: E402
from oracle import moe_oracle as orc  # noqa: E402

ZIPF_S = 1.1
N_ZERO = 16
STEPS = 800


def zipf_targets(n: int, T: int, k: int) -> np.ndarray:
    p = np.arange(1, n + 1, dtype=np.float64) ** -ZIPF_S
    target = p / p.sum() * (T * k)
    capped = np.zeros(n, bool)
    for _ in range(n):
        over = (target > T) & ~capped
        if not over.any():
            break
        capped |= over
        excess = (target[capped] - T).sum()
        target[capped] = T
        free = ~capped
        target[free] += excess * target[free] / target[free].sum()
    return target


def loads_fast(scores: np.ndarray, bias: np.ndarray, k: int) -> np.ndarray:
    keys = (scores + bias[None, :].astype(np.float32)).astype(np.float32)
    top = np.argpartition(-keys, k - 1, axis=1)[:, :k]
    return np.bincount(top.reshape(-1), minlength=scores.shape[1])


def main() -> None:
    cfg = mi.CONFIGS["skew"]
    T, E, k = cfg.T, cfg.E, cfg.k
    h = mi.hidden(cfg, 0).float().numpy()
    Wr = mi.router_weight(cfg, 0).numpy()
    scores = orc.sigmoid_scores(orc.router_logits(h, Wr))

    rank_of = np.empty(E, np.int64)          # rank_of[e] in 0..E-1 (0 = most popular)
    order = np.argsort(mi.hash_u32(E, 0, "skew/rank").numpy(), kind="stable")
    rank_of[order] = np.arange(E)
    live = rank_of < E - N_ZERO
    target = np.zeros(E)
    target[live] = zipf_targets(E - N_ZERO, T, k)[rank_of[live]]

    bias = np.zeros(E)
    bias[~live] = -2.0
    best, best_err = bias.copy(), np.inf
    for step in range(STEPS):
        load = loads_fast(scores, bias, k)
        err = np.abs(load - target).sum() / (T * k)
        if err < best_err:
            best, best_err = bias.copy(), err
        eta = 0.02 if step < STEPS // 2 else 0.005
        bias[live] += eta * (np.log(target[live] + 1.0) - np.log(load[live] + 1.0))
        bias[live] = np.clip(bias[live], -0.9, 2.0)

    b32 = best.astype(np.float32)
    idx, _ = orc.route(orc.router_logits(h, Wr), b32, k, cfg.scale)
    load = np.bincount(idx.reshape(-1), minlength=E)
    mean = T * k / E
    r = rank_of[live] + 1
    slope = np.polyfit(np.log(r[load[live] > 0]), np.log(load[live][load[live] > 0]), 1)[0]
    out = os.path.join(_ROOT, "moe_inputs", cfg.skew_bias_file)
    with open(out, "w") as f:
        f.write("# fp32 correction bias of the skewed-load workload, one IEEE-754 bit pattern per line\n")
        f.write("# written by oracle/make_skew_bias.py (oracle routing on the seed-0 hidden states)\n")
        f.write(f"# realized loads: max/mean {load.max() / mean:.2f}, zero-load experts "
                f"{int((load == 0).sum())}, L1 error vs Zipf({ZIPF_S}) targets {best_err:.4f}, "
                f"fitted log-log slope {slope:.3f}\n")
        for v in b32:
            f.write(f"{int(v.view(np.uint32)):08x}\n")
    print(f"wrote {out}: max/mean {load.max() / mean:.2f} zero {int((load == 0).sum())} "
          f"L1 {best_err:.4f} slope {slope:.3f}")


if __name__ == "__main__":
    main()
