"""GPU parity of the FP8-weight path (E4M3 codes with power-of-two 128 x 128
block scales, bf16 activations), called through the C ABI, against the CPU
oracle on the weights the codes stand for.

Bars: the decoding is bit-exact (every non-NaN code, the extreme exponents);
the expert MLPs and the whole layer meet the bf16 path's tolerances against
the oracle evaluated on the decoded weights; routing is the bf16 path's
(shared code) and is checked the same way.
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from oracle import moe_oracle as orc
from tests.gpu_helpers import (MAX_ABS_TOL, REL_L2_TOL, host_f32, layer_on_device, oracle_rows,
                               rel_l2)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import sparse_moe_layer_04_b200 as m
    return m


def _w8(moe, q):
    return moe.fp8_weights(q["W1q"], q["W3q"], q["W2q"], q.get("Ws1q"), q.get("Ws3q"),
                           q.get("Ws2q"), q["W1e"], q["W3e"], q["W2e"], q.get("Ws1e"),
                           q.get("Ws3e"), q.get("Ws2e"))


def _deq(q, name, g):
    """The oracle's decoding of matrix `name`, group g (fp64, host)."""
    return orc.dequantize_fp8_blocks(q[name + "q"][g].cpu().numpy(), q[name + "e"][g].cpu().numpy())


class HostFp8Experts:
    """Routed experts decoded by the oracle on demand."""

    def __init__(self, q):
        self.q = q
        self.cache = {}

    def __call__(self, e: int):
        if e not in self.cache:
            self.cache[e] = tuple(_deq(self.q, n, e) for n in ("W1", "W3", "W2"))
        return self.cache[e]


# ---------------------------------------------------------------------------
# decoding
# ---------------------------------------------------------------------------
def test_dequantize_every_code_bit_exact(moe):
    G, R, K = 3, 200, 272
    valid = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    pos = mi.uniform_int(G * R * K, len(valid), 0, "fp8/codes").numpy()
    codes = valid[pos].reshape(G, R, K)
    codes[0, 0, :len(valid)] = valid                 # every code at least once, exponent -117
    RB, KB = 2, 3
    exps = (mi.uniform_int(G * RB * KB, 125, 0, "fp8/exps").numpy() - 117).astype(np.int8)
    exps = exps.reshape(G, RB, KB)
    exps[0, 0, 0], exps[0, 0, 1], exps[1, 1, 2] = -117, 7, 0
    out = torch.empty((G, R, K), dtype=torch.bfloat16, device="cuda")
    d = moe.dims(T=1, D=128, E=8, F=64, k=2)
    ws = moe.alloc_workspace(d)
    moe.moe_fp8_dequantize(torch.from_numpy(codes).cuda(), torch.from_numpy(exps).cuda(), out, ws)
    assert moe.moe_get_device_status(ws) == 0
    ref = orc.dequantize_fp8_blocks(codes, exps)
    ref_bf16 = torch.from_numpy(ref).to(torch.bfloat16)
    assert torch.equal(ref_bf16.double(), torch.from_numpy(ref))        # exact in bf16
    assert torch.equal(out.cpu().view(torch.int16), ref_bf16.view(torch.int16))   # bit-exact, -0 too


def test_dequantize_flags_exponent_out_of_range(moe):
    codes = torch.full((1, 16, 32), 0x38, dtype=torch.uint8, device="cuda")
    out = torch.empty((1, 16, 32), dtype=torch.bfloat16, device="cuda")
    d = moe.dims(T=1, D=128, E=8, F=64, k=2)
    ws = moe.alloc_workspace(d)
    for e, ok in ((7, True), (-117, True), (8, False), (-118, False)):
        exps = torch.full((1, 1, 1), e, dtype=torch.int8, device="cuda")
        moe.moe_fp8_dequantize(codes, exps, out, ws)
        rc = moe.moe_get_device_status(ws)
        assert (rc == 0) == ok, e
        if not ok:
            assert rc == moe.MOE_ERR_BOUNDS


# ---------------------------------------------------------------------------
# expert MLPs
# ---------------------------------------------------------------------------
FFN_FP8_CASES = [
    (64, 128, 8, 64, 2, 1, 64),          # the tiny layer's shapes
    (128, 256, 16, 192, 8, 1, 320),      # F, Fs not multiples of the 64-feature tile
    (100, 144, 12, 80, 3, 2, 48),        # D not a multiple of 64, two shared experts
    (1, 128, 4, 64, 4, 1, 64),           # one token
    (120, 128, 64, 64, 1, 0, 0),         # no shared expert, many empty experts
    # more than 128 tokens: 256-token blocks, groups of several blocks
    (300, 256, 16, 192, 4, 1, 320),
    (700, 384, 8, 256, 2, 0, 0),
    (600, 512, 4, 128, 4, 2, 128),
]


@pytest.mark.parametrize("T,D,E,F,k,S,Fs", FFN_FP8_CASES)
def test_expert_ffn_fp8(moe, T, D, E, F, k, S, Fs):
    cfg = mi.LayerConfig("ffn8", T, D, E, k, F, S, max(Fs, 16), 2.5, 1.0, f"ffn8_{T}x{D}x{E}")
    inp = layer_on_device(cfg)
    q = mi.fp8_layer_weights(inp)
    idx = mi.synthetic_topk(T, E, k, 0, f"ffn8_{T}")
    _, offsets, perm, _ = orc.group_by_expert(idx.numpy(), E)
    d = moe.dims(T=T, D=D, E=E, F=F, k=k, S=S, Fs=max(Fs, 16))
    ws = moe.alloc_workspace(d)
    y = torch.full((T * k + S * T, D), float("nan"), device="cuda")
    if S == 0:
        for n in ("Ws1", "Ws3", "Ws2"):
            q[n + "q"] = q[n + "e"] = None
    w8 = _w8(moe, q)
    perm_d = torch.from_numpy(perm).cuda()
    offs_d = torch.from_numpy(offsets).cuda()
    moe.moe_expert_ffn_fp8(inp["h"], perm_d, offs_d, w8, d, y, ws)
    assert moe.moe_get_device_status(ws) == 0
    got = y.cpu().numpy().astype(np.float64)
    h = host_f32(inp["h"])
    ref = np.empty_like(got)
    ex = HostFp8Experts(q)
    for e in range(E):
        rows = slice(offsets[e], offsets[e + 1])
        if offsets[e + 1] > offsets[e]:
            ref[rows] = orc.swiglu_expert(h[perm[rows]], *ex(e))
    for s in range(S):
        ref[T * k + s * T: T * k + (s + 1) * T] = orc.swiglu_expert(
            h, _deq(q, "Ws1", s), _deq(q, "Ws3", s), _deq(q, "Ws2", s))
    assert np.all(np.isfinite(got))
    # as for bf16 weights: the gated activation is rounded to bf16 before the
    # w2 product (~1.1e-3 relative in L2 with independent signs)
    assert rel_l2(got, ref) < 4e-3
    row_err = np.linalg.norm(got - ref, axis=1) / np.maximum(np.linalg.norm(ref, axis=1), 1e-30)
    assert row_err.max() < 2e-2


def test_expert_ffn_fp8_flags_bad_exponent(moe):
    T, D, E, F, k = 16, 128, 4, 64, 2
    cfg = mi.LayerConfig("ffn8b", T, D, E, k, F, 1, 64, 2.5, 1.0, "ffn8b")
    inp = layer_on_device(cfg)
    q = mi.fp8_layer_weights(inp)
    q["W2e"] = q["W2e"].clone()
    q["W2e"][:] = 9
    idx = mi.synthetic_topk(T, E, k, 0, "ffn8b")
    _, offsets, perm, _ = orc.group_by_expert(idx.numpy(), E)
    d = moe.dims(T=T, D=D, E=E, F=F, k=k, S=1, Fs=64)
    ws = moe.alloc_workspace(d)
    y = torch.empty((T * k + T, D), device="cuda")
    moe.moe_expert_ffn_fp8(inp["h"], torch.from_numpy(perm).cuda(), torch.from_numpy(offsets).cuda(),
                           _w8(moe, q), d, y, ws)
    assert moe.moe_get_device_status(ws) == moe.MOE_ERR_BOUNDS


# ---------------------------------------------------------------------------
# the whole layer
# ---------------------------------------------------------------------------
def _forward_fp8(moe, cfg, inp, q):
    d = moe.dims_of(cfg)
    ws = moe.alloc_workspace(d)
    out = torch.empty((cfg.T, cfg.D), dtype=torch.float32, device="cuda")
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    w = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device="cuda")
    moe.moe_forward_fp8(inp["h"], inp["Wr"], inp["bias"], _w8(moe, q), d, out, ws, idx, w)
    assert moe.moe_get_device_status(ws) == 0
    return out, idx, w


def _check_layer_fp8(cfg, inp, q, out, idx, tokens, max_flip_frac=0.02):
    host = dict(h=inp["h"], Wr=inp["Wr"], bias=inp["bias"])
    for n in ("Ws1", "Ws3", "Ws2"):
        host[n] = torch.from_numpy(np.stack([_deq(q, n, s) for s in range(cfg.S)]))
    ref, flips, wrong = oracle_rows(host, cfg, tokens, idx.cpu().numpy()[tokens], HostFp8Experts(q))
    got = out.cpu().numpy()[tokens].astype(np.float64)
    assert wrong == 0, f"{wrong} tokens routed to a set that is not a correct top-k"
    assert flips <= max(1, max_flip_frac * len(tokens))
    assert rel_l2(got, ref) <= REL_L2_TOL
    assert np.max(np.abs(got - ref)) <= MAX_ABS_TOL


@pytest.mark.parametrize("T", [64, 1, 129, 300])
def test_forward_fp8_tiny(moe, T):
    cfg = mi.custom_config("tiny", T=T, name="tiny")
    inp = layer_on_device(cfg)
    q = mi.fp8_layer_weights(inp)
    out, idx, w = _forward_fp8(moe, cfg, inp, q)
    _check_layer_fp8(cfg, inp, q, out, idx, np.arange(T))
    # routing is the bf16 path's: identical indices and weights
    d = moe.dims_of(cfg)
    ws = moe.alloc_workspace(d)
    o2 = torch.empty_like(out)
    i2 = torch.empty_like(idx)
    w2 = torch.empty_like(w)
    moe.moe_forward(inp["h"], inp["Wr"], inp["bias"], inp["W1"], inp["W3"], inp["W2"], inp["Ws1"],
                    inp["Ws3"], inp["Ws2"], d, o2, ws, i2, w2)
    assert torch.equal(idx, i2) and torch.equal(w.view(torch.int32), w2.view(torch.int32))


def test_forward_fp8_deterministic(moe):
    cfg = mi.custom_config("tiny", T=300, name="tiny")
    inp = layer_on_device(cfg)
    q = mi.fp8_layer_weights(inp)
    a, ia, _ = _forward_fp8(moe, cfg, inp, q)
    b, ib, _ = _forward_fp8(moe, cfg, inp, q)
    assert torch.equal(a.view(torch.int32), b.view(torch.int32)) and torch.equal(ia, ib)


def test_forward_fp8_small_batch_many_tiles_per_cta(moe):
    """128 tokens over 64 experts of D=2048, F=512: ~1500 tiles, about ten per
    CTA, so every CTA cycles through both accumulator buffers of the 128-token
    path many times.  Every token against the oracle, and a second call gives
    the same bits."""
    cfg = mi.custom_config("decode", T=128, D=2048, E=64, k=8, F=512, S=1, Fs=512,
                           hidden_std=1.0, name="fp8_many_tiles")
    inp = layer_on_device(cfg)
    q = mi.fp8_layer_weights(inp)
    a, ia, wa = _forward_fp8(moe, cfg, inp, q)
    _check_layer_fp8(cfg, inp, q, a, ia, np.arange(cfg.T))
    b, ib, wb = _forward_fp8(moe, cfg, inp, q)
    assert torch.equal(ia, ib) and torch.equal(wa.view(torch.int32), wb.view(torch.int32))
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))


@pytest.fixture(scope="module")
def glm52_fp8():
    cfg = mi.CONFIGS["decode"]
    w = mi.layer_weights(cfg, 0, device="cuda")
    q = mi.fp8_layer_weights(w)
    for n in ("W1", "W3", "W2", "Ws1", "Ws3", "Ws2"):
        del w[n]
    torch.cuda.empty_cache()
    return w, q


@pytest.mark.parametrize("name,n", [("decode", 128), ("prefill", 24)])
def test_forward_fp8_glm52_full_size(moe, glm52_fp8, name, n):
    cfg = mi.CONFIGS[name]
    w, q = glm52_fp8
    inp = dict(w)
    inp["bias"] = mi.correction_bias(cfg, 0, device="cuda")
    inp["h"] = mi.hidden(cfg, 0, device="cuda")
    out, idx, _ = _forward_fp8(moe, cfg, inp, q)
    assert torch.isfinite(out).all()
    tokens = np.arange(cfg.T) if cfg.T <= n else np.unique(
        mi.uniform_int(n, cfg.T, 0, "sample/fp8" + name).numpy())
    _check_layer_fp8(cfg, inp, q, out, idx, tokens)
