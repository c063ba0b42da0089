"""Shared helpers of the GPU parity tests: seeded inputs on the device, the
oracle on the same values on the host, and the comparison rules."""
from __future__ import annotations

import numpy as np
import torch

import moe_inputs as mi
from oracle import moe_oracle as orc

# Layer-output tolerance the benchmark spec states for the fp32 oracle comparison.
REL_L2_TOL = 1e-2
MAX_ABS_TOL = 2e-2
# Keys closer than this at the top-k boundary may legitimately flip between two
# fp32 routers that sum the hidden dimension in different orders.
NEAR_TIE = 1e-5


def layer_on_device(cfg, device="cuda", seed=0):
    """All inputs of one workload generated directly on the device."""
    w = mi.layer_weights(cfg, seed, device=device)
    w["h"] = mi.hidden(cfg, seed, device=device)
    return w


def host_f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


class HostExperts:
    """Routed experts copied to the host on demand (bf16 values widened exactly to fp64)."""

    def __init__(self, W1, W3, W2):
        self.W1, self.W3, self.W2 = W1, W3, W2
        self.cache = {}

    def __call__(self, e: int):
        if e not in self.cache:
            self.cache[e] = tuple(x[e].detach().cpu().double().numpy()
                                  for x in (self.W1, self.W3, self.W2))
        return self.cache[e]


def oracle_rows(inp, cfg, tokens: np.ndarray, gpu_idx: np.ndarray, experts: HostExperts):
    """Oracle outputs for the given tokens.

    For each token the oracle lists every routing that is correct up to fp32
    logit rounding (near ties at the k-th key); the GPU's selected expert set
    must be one of them, and the token is compared with the oracle output of
    that routing.  Returns (out [n, D] fp64, number of tokens whose GPU routing
    is a near-tie alternative rather than the oracle's strict choice, and the
    number of tokens whose GPU routing is not a correct routing at all).
    """
    h = host_f32(inp["h"][torch.as_tensor(tokens, device=inp["h"].device)])
    Wr = host_f32(inp["Wr"])
    bias = host_f32(inp["bias"])
    logits = orc.router_logits(h, Wr)
    shared = [tuple(x[s].detach().cpu().double().numpy() for x in (inp["Ws1"], inp["Ws3"], inp["Ws2"]))
              for s in range(cfg.S)]
    idx_rows, w_rows = [], []
    flips = wrong = 0
    for i in range(len(tokens)):
        cands = orc.routing_alternatives(logits[i], bias, cfg.k, cfg.scale, NEAR_TIE)
        gset = sorted(gpu_idx[i].tolist())
        match = [c for c in cands if sorted(c[0].tolist()) == gset]
        if not match:
            wrong += 1
            match = cands[:1]
        elif not np.array_equal(match[0][0], cands[0][0]):
            flips += 1
        idx_rows.append(match[0][0])
        w_rows.append(match[0][1])
    idx = np.stack(idx_rows)
    w = np.stack(w_rows)
    out = orc.routed_output_given_routing(h, idx, w, experts)
    if shared:
        out = out + orc.shared_output(h, shared)
    return out, flips, wrong


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))
