"""Seeded synthetic inputs for the GLM-5.2 MoE feed-forward layer.

This module is the one piece shared by the CUDA path's tests/bench and the CPU
oracle.  It draws random numbers and nothing else: it holds none of the
layer's arithmetic (no routing, no matmul, no activation).

Generator
---------
Every tensor element is a pure function of (seed, stream name, element index),
so the same values come out on the CPU and on any CUDA device, and one expert's
weights can be regenerated alone without materialising the others.

* counter -> 32-bit hash: two rounds of the MurmurHash3 32-bit finaliser
  ("fmix32", Austin Appleby's public-domain MurmurHash3), keyed by two 32-bit
  stream keys derived with BLAKE2b from the stream name.  All products are
  formed on 16-bit halves so int64 arithmetic never overflows, which keeps
  the CPU and CUDA results bit-identical.
* hash -> N(0, 1): the top 20 bits index a table of the 2**20 standard-normal
  quantiles at (q + 0.5) / 2**20 (computed once in fp64 with
  ``torch.special.ndtri`` and stored as fp32), then one fp32 multiply by the
  tensor's standard deviation.  bf16 tensors are rounded to nearest-even from
  that fp32 value.

Workloads (the layer shapes the GLM-5.2 and GLM-4.5-Air pages give)
--------------------------------------------------------------------
``CONFIGS`` lists the workloads: a tiny layer for exhaustive checks, the
GLM-5.2 layer at decode (T=128), prefill (T=4096) and skewed-load (T=16384)
batch sizes, the GLM-4.5-Air layer (T=8192), and a second decode batch
("decode_b") whose hidden states are N(0, 1) instead of N(0, 1/sqrt(D)).
Expert weights are N(0, 1/sqrt(fan_in)) (std = 1/sqrt(in-features)), the
router is fp32 N(0, 0.02), the correction bias fp32 N(0, 0.1).  The decode,
decode_b, prefill and skew workloads share one set of GLM-5.2 weights.  The
skew workload replaces the bias by a stored calibrated vector
(``skew_bias_T16384_seed0.txt``) that makes expert popularity follow Zipf(1.1)
with 16 experts that receive no tokens.
"""
from __future__ import annotations

import hashlib
import math
import os
from dataclasses import dataclass, replace
from typing import Dict, Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_MASK32 = 0xFFFFFFFF


@dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int          # tokens in the batch
    D: int          # hidden size
    E: int          # routed experts
    k: int          # experts selected per token
    F: int          # routed expert width
    S: int          # shared (always-on) experts
    Fs: int         # shared expert width
    scale: float    # routed scaling factor
    hidden_std: float
    weight_family: str          # configs that share one set of weights
    hidden_fp32: bool = False   # the tiny layer keeps fp32 originals too
    skew_bias_file: Optional[str] = None

    @property
    def dims(self) -> Dict[str, float]:
        return dict(T=self.T, D=self.D, E=self.E, F=self.F, k=self.k, S=self.S,
                    Fs=self.Fs, scale=self.scale)


CONFIGS: Dict[str, LayerConfig] = {
    "tiny": LayerConfig("tiny", T=64, D=128, E=8, k=2, F=64, S=1, Fs=64, scale=2.5,
                        hidden_std=1.0, weight_family="tiny", hidden_fp32=True),
    "decode": LayerConfig("decode", T=128, D=6144, E=256, k=8, F=2048, S=1, Fs=2048,
                          scale=2.5, hidden_std=1.0 / math.sqrt(6144),
                          weight_family="glm52"),
    # decode batch with N(0, 1) hidden states: the router logits then spread the
    # selection over about 108 experts instead of about 10 (reported, not a target)
    "decode_b": LayerConfig("decode_b", T=128, D=6144, E=256, k=8, F=2048, S=1, Fs=2048,
                            scale=2.5, hidden_std=1.0, weight_family="glm52"),
    "prefill": LayerConfig("prefill", T=4096, D=6144, E=256, k=8, F=2048, S=1, Fs=2048,
                           scale=2.5, hidden_std=1.0, weight_family="glm52"),
    "skew": LayerConfig("skew", T=16384, D=6144, E=256, k=8, F=2048, S=1, Fs=2048,
                        scale=2.5, hidden_std=1.0, weight_family="glm52",
                        skew_bias_file="skew_bias_T16384_seed0.txt"),
    "air": LayerConfig("air", T=8192, D=4096, E=128, k=8, F=1408, S=1, Fs=1408,
                       scale=1.0, hidden_std=1.0 / math.sqrt(4096),
                       weight_family="glm45air"),
}

ROUTER_STD = 0.02
BIAS_STD = 0.1


def custom_config(base: str, **overrides) -> LayerConfig:
    """A workload derived from ``base`` with some fields replaced (e.g. T)."""
    return replace(CONFIGS[base], **overrides)


# ----------------------------------------------------------------------------
# counter-based generator
# ----------------------------------------------------------------------------

def _stream_keys(seed: int, name: str):
    d = hashlib.blake2b(f"{seed}/{name}".encode(), digest_size=8).digest()
    return int.from_bytes(d[:4], "little"), int.from_bytes(d[4:], "little")


def _mul32(x: torch.Tensor, c: int) -> torch.Tensor:
    """(x * c) mod 2**32 for x in [0, 2**32), without int64 overflow."""
    lo, hi = c & 0xFFFF, c >> 16
    return (x * lo + (((x * hi) & 0xFFFF) << 16)) & _MASK32


def _fmix32(x: torch.Tensor) -> torch.Tensor:
    x = x ^ (x >> 16)
    x = _mul32(x, 0x85EBCA6B)
    x = x ^ (x >> 13)
    x = _mul32(x, 0xC2B2AE35)
    x = x ^ (x >> 16)
    return x


_QUANTILES: Dict[str, torch.Tensor] = {}
_QBITS = 20


def _quantile_table(device: torch.device) -> torch.Tensor:
    key = str(device)
    if key not in _QUANTILES:
        n = 1 << _QBITS
        p = (torch.arange(n, dtype=torch.float64) + 0.5) / n
        _QUANTILES[key] = torch.special.ndtri(p).to(torch.float32).to(device)
    return _QUANTILES[key]


def hash_u32(n: int, seed: int, name: str, device="cpu") -> torch.Tensor:
    """n 32-bit hashes (as int64 in [0, 2**32)) of the counters 0..n-1."""
    if n >= (1 << 32):
        raise ValueError("a stream holds fewer than 2**32 elements")
    k1, k2 = _stream_keys(seed, name)
    x = torch.arange(n, dtype=torch.int64, device=device)
    x = _fmix32(x ^ k1)
    return _fmix32(x ^ k2)


def normal(shape, std: float, seed: int, name: str, device="cpu") -> torch.Tensor:
    """fp32 tensor of N(0, std) samples, identical on every device."""
    n = 1
    for s in shape:
        n *= int(s)
    h = hash_u32(n, seed, name, device)
    table = _quantile_table(torch.device(device))
    z = table[(h >> (32 - _QBITS))]
    std_t = torch.tensor(std, dtype=torch.float32, device=device)
    return (z * std_t).reshape(shape)


def uniform_int(n: int, high: int, seed: int, name: str, device="cpu") -> torch.Tensor:
    """n integers in [0, high) (for synthetic routings and permutations)."""
    h = hash_u32(n, seed, name, device)
    return (h * high) >> 32


# ----------------------------------------------------------------------------
# layer tensors
# ----------------------------------------------------------------------------

def hidden(cfg: LayerConfig, seed: int = 0, device="cpu", fp32: bool = False) -> torch.Tensor:
    """Token hidden states [T, D]; bf16 unless fp32=True (the raw draw)."""
    x = normal((cfg.T, cfg.D), cfg.hidden_std, seed, f"{cfg.name}/hidden", device)
    return x if fp32 else x.to(torch.bfloat16)


def router_weight(cfg: LayerConfig, seed: int = 0, device="cpu") -> torch.Tensor:
    """fp32 router weight [E, D]."""
    return normal((cfg.E, cfg.D), ROUTER_STD, seed, f"{cfg.weight_family}/router", device)


def correction_bias(cfg: LayerConfig, seed: int = 0, device="cpu") -> torch.Tensor:
    """fp32 expert-score correction bias [E] (the stored Zipf vector for skew)."""
    if cfg.skew_bias_file is not None:
        return load_bias_file(os.path.join(_HERE, cfg.skew_bias_file), cfg.E).to(device)
    return normal((cfg.E,), BIAS_STD, seed, f"{cfg.weight_family}/bias", device)


def expert_weights(cfg: LayerConfig, e: int, seed: int = 0, device="cpu", fp32: bool = False,
                   shared: bool = False):
    """(w1 [F, D], w3 [F, D], w2 [D, F]) of routed expert e, or of shared expert e.

    nn.Linear layout (out-features, in-features); std = 1/sqrt(in-features).
    """
    F = cfg.Fs if shared else cfg.F
    tag = f"{cfg.weight_family}/{'shared' if shared else 'expert'}{e}"
    w1 = normal((F, cfg.D), 1.0 / math.sqrt(cfg.D), seed, tag + "/w1", device)
    w3 = normal((F, cfg.D), 1.0 / math.sqrt(cfg.D), seed, tag + "/w3", device)
    w2 = normal((cfg.D, F), 1.0 / math.sqrt(F), seed, tag + "/w2", device)
    if fp32:
        return w1, w3, w2
    return w1.to(torch.bfloat16), w3.to(torch.bfloat16), w2.to(torch.bfloat16)


def layer_weights(cfg: LayerConfig, seed: int = 0, device="cpu", fp32: bool = False):
    """All weights of one layer: dict with Wr, bias, W1, W3, W2, Ws1, Ws3, Ws2."""
    dt = torch.float32 if fp32 else torch.bfloat16
    W1 = torch.empty((cfg.E, cfg.F, cfg.D), dtype=dt, device=device)
    W3 = torch.empty_like(W1)
    W2 = torch.empty((cfg.E, cfg.D, cfg.F), dtype=dt, device=device)
    for e in range(cfg.E):
        W1[e], W3[e], W2[e] = expert_weights(cfg, e, seed, device, fp32)
    Ws1 = torch.empty((cfg.S, cfg.Fs, cfg.D), dtype=dt, device=device)
    Ws3 = torch.empty_like(Ws1)
    Ws2 = torch.empty((cfg.S, cfg.D, cfg.Fs), dtype=dt, device=device)
    for s in range(cfg.S):
        Ws1[s], Ws3[s], Ws2[s] = expert_weights(cfg, s, seed, device, fp32, shared=True)
    return dict(Wr=router_weight(cfg, seed, device), bias=correction_bias(cfg, seed, device),
                W1=W1, W3=W3, W2=W2, Ws1=Ws1, Ws3=Ws3, Ws2=Ws2)


def synthetic_logits(T: int, E: int, std: float, seed: int, name: str, device="cpu"):
    """fp32 router logits drawn directly (for routing checks fed identical logits)."""
    return normal((T, E), std, seed, f"logits/{name}", device)


def synthetic_topk(T: int, E: int, k: int, seed: int, name: str, device="cpu"):
    """int32 [T, k] rows of k distinct experts, uniformly random (for permute checks)."""
    keys = normal((T, E), 1.0, seed, f"topk/{name}", device)
    return torch.argsort(keys, dim=1, stable=True)[:, :k].to(torch.int32).contiguous()


# ----------------------------------------------------------------------------
# stored bias file
# ----------------------------------------------------------------------------

def load_bias_file(path: str, E: int) -> torch.Tensor:
    """Read an fp32 bias vector stored as one hex bit pattern per line ('#' comments)."""
    vals = []
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                vals.append(int(line, 16))
    if len(vals) != E:
        raise ValueError(f"{path}: expected {E} values, found {len(vals)}")
    signed = [v - (1 << 32) if v >= (1 << 31) else v for v in vals]
    return torch.tensor(signed, dtype=torch.int32).view(torch.float32)


def bias_file_path(cfg: LayerConfig) -> Optional[str]:
    return None if cfg.skew_bias_file is None else os.path.join(_HERE, cfg.skew_bias_file)


# ----------------------------------------------------------------------------
# FP8 weights (E4M3 codes, one power-of-two scale per 128 x 128 block)
# ----------------------------------------------------------------------------
FP8_BLOCK = 128
FP8_MAX = 448.0


def quantize_fp8_blocks(w: torch.Tensor):
    """E4M3 codes and block exponents of a weight matrix [..., rows, K].

    For each 128 x 128 block (ragged at the edges) the exponent e is the
    smallest integer with max|w| <= 448 * 2**e (0 for an all-zero block); the
    codes are torch's round-to-nearest-even float8_e4m3fn cast of w * 2**-e.
    The weight the codes stand for, code * 2**e, is exactly a bf16 value.
    Returns (codes uint8 [..., rows, K], exps int8 [..., ceil(rows/128), ceil(K/128)]).
    """
    *lead, R, K = w.shape
    RB, KB = -(-R // FP8_BLOCK), -(-K // FP8_BLOCK)
    wf = w.float()
    pad = torch.zeros(*lead, RB * FP8_BLOCK, KB * FP8_BLOCK, dtype=torch.float32, device=w.device)
    pad[..., :R, :K] = wf.abs()
    amax = pad.reshape(*lead, RB, FP8_BLOCK, KB, FP8_BLOCK).amax(dim=(-3, -1)).double()
    e = torch.ceil(torch.log2(torch.clamp(amax, min=1e-300) / FP8_MAX))
    lim = FP8_MAX * torch.pow(2.0, e)
    e = torch.where(amax > lim, e + 1, e)                       # exact corrections
    e = torch.where(amax <= FP8_MAX * torch.pow(2.0, e - 1), e - 1, e)
    e = torch.where(amax == 0, torch.zeros_like(e), e)
    exps = e.to(torch.int8)
    scale = torch.pow(2.0, -e).float()
    full = scale.repeat_interleave(FP8_BLOCK, dim=-2).repeat_interleave(FP8_BLOCK, dim=-1)
    codes = (wf * full[..., :R, :K]).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), exps.contiguous()


def fp8_layer_weights(weights: dict) -> dict:
    """FP8 copies of the expert weights of `layer_weights`: for each of W1,
    W3, W2, Ws1, Ws3, Ws2 the codes ("W1q" ...) and block exponents ("W1e" ...),
    on the weights' device.  Quantized one expert at a time, so the
    temporaries stay the size of one expert matrix."""
    out = {}
    for name in ("W1", "W3", "W2", "Ws1", "Ws3", "Ws2"):
        w = weights[name]
        parts = [quantize_fp8_blocks(w[g]) for g in range(w.shape[0])]
        R, K = w.shape[-2:]
        out[name + "q"] = (torch.stack([c for c, _ in parts]) if parts else
                           torch.empty((0, R, K), dtype=torch.uint8, device=w.device))
        out[name + "e"] = (torch.stack([e for _, e in parts]) if parts else
                           torch.empty((0, -(-R // FP8_BLOCK), -(-K // FP8_BLOCK)),
                                       dtype=torch.int8, device=w.device))
    return out
