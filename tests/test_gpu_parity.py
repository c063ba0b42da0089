"""GPU parity: every step of the CUDA path, called through the C ABI, against
the CPU oracle on the same seeded inputs.

Bars: integer results (expert indices, grouping) bit-exact; routing weights
bit-exact when both sides get identical fp32 logits (both take the decisions
in fp32 with the sigmoid in fp64); floating-point results within the
tolerances derived in each test; the layer output within relative L2 1e-2
and max-abs 2e-2 of the oracle.
"""
import math

import numpy as np
import pytest
import torch

import moe_inputs as mi
from oracle import moe_oracle as orc
from tests.gpu_helpers import (MAX_ABS_TOL, REL_L2_TOL, HostExperts, host_f32, layer_on_device,
                               oracle_rows, rel_l2)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import sparse_moe_layer_04_b200 as m
    return m


def _ws(moe, d):
    return moe.alloc_workspace(d)


# ---------------------------------------------------------------------------
# routing: identical logits -> identical indices and weights
# ---------------------------------------------------------------------------
ROUTE_CASES = [
    (1, 8, 2, "normal"), (37, 8, 3, "grid"), (128, 256, 8, "normal"), (1000, 256, 8, "grid"),
    (64, 1024, 32, "normal"), (513, 64, 1, "normal"), (16, 32, 32, "grid"), (200, 40, 6, "normal"),
    # more than 1024 tokens: the warp-per-token kernel
    (2000, 256, 8, "grid"), (1500, 64, 6, "normal"), (1100, 1024, 32, "normal"), (1025, 8, 2, "grid"),
]


@pytest.mark.parametrize("T,E,k,dist", ROUTE_CASES)
def test_route_bit_exact(moe, T, E, k, dist):
    name = f"route{T}x{E}x{k}"
    logits = mi.synthetic_logits(T, E, 1.5, 0, name)
    bias = mi.normal((E,), 0.1, 0, name + "/bias")
    if dist == "grid":  # many exact key ties
        logits = torch.round(logits * 4) / 4
        bias = torch.round(bias * 16) / 16
    d = moe.dims(T=T, D=64, E=E, F=64, k=k, scale=2.5)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    ws = _ws(moe, d)
    moe.moe_route(logits.cuda(), bias.cuda(), d, idx, w, ws)
    assert moe.moe_get_device_status(ws) == 0
    ridx, rw = orc.route(logits.numpy(), bias.numpy(), k, 2.5)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert np.array_equal(w.cpu().numpy().view(np.uint32), rw.view(np.uint32))


GROUPED_CASES = [
    (128, 256, 8, 8, 4, "normal"), (300, 256, 8, 8, 2, "grid"), (64, 64, 6, 4, 2, "normal"),
    (77, 160, 4, 32, 3, "grid"), (50, 1024, 32, 32, 16, "normal"), (40, 12, 3, 12, 3, "normal"),  # one-expert groups
]


@pytest.mark.parametrize("T,E,k,n_group,topk_group,dist", GROUPED_CASES)
def test_route_grouped_bit_exact(moe, T, E, k, n_group, topk_group, dist):
    name = f"groute{T}x{E}x{n_group}"
    logits = mi.synthetic_logits(T, E, 1.5, 0, name)
    bias = mi.normal((E,), 0.1, 0, name + "/bias")
    if dist == "grid":
        logits = torch.round(logits * 4) / 4
        bias = torch.round(bias * 16) / 16
    d = moe.dims(T=T, D=64, E=E, F=64, k=k, scale=2.5)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    ws = _ws(moe, d)
    moe.moe_route_grouped(logits.cuda(), bias.cuda(), d, n_group, topk_group, idx, w, ws)
    assert moe.moe_get_device_status(ws) == 0
    ridx, rw = orc.route_grouped(logits.numpy(), bias.numpy(), k, 2.5, n_group, topk_group)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert np.array_equal(w.cpu().numpy().view(np.uint32), rw.view(np.uint32))


def test_route_grouped_single_group_equals_route(moe):
    T, E, k = 200, 256, 8
    logits = mi.synthetic_logits(T, E, 1.5, 0, "g1").cuda()
    bias = mi.normal((E,), 0.1, 0, "g1/bias").cuda()
    d = moe.dims(T=T, D=64, E=E, F=64, k=k)
    outs = [(torch.empty((T, k), dtype=torch.int32, device="cuda"),
             torch.empty((T, k), device="cuda")) for _ in range(2)]
    moe.moe_route(logits, bias, d, *outs[0])
    moe.moe_route_grouped(logits, bias, d, 1, 1, *outs[1])
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def test_route_zero_router_tie(moe):
    T, E, k = 9, 64, 8
    d = moe.dims(T=T, D=64, E=E, F=64, k=k, scale=2.5)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    moe.moe_route(torch.zeros((T, E), device="cuda"), torch.zeros(E, device="cuda"), d, idx, w)
    assert np.array_equal(idx.cpu().numpy(), np.tile(np.arange(k, dtype=np.int32), (T, 1)))
    assert np.all(w.cpu().numpy() == np.float32(2.5 / 8))


# ---------------------------------------------------------------------------
# router logits: fp32 within the summation error bound, deterministic
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("T,D,E", [(64, 128, 8), (128, 6144, 256), (300, 1000, 64),
                                   (4096, 512, 256), (1, 64, 1024)])
def test_router_logits(moe, T, D, E):
    name = f"logit{T}x{D}x{E}"
    h = mi.normal((T, D), 1.0, 0, name + "/h").to(torch.bfloat16)
    Wr = mi.normal((E, D), 0.02, 0, name + "/w")
    d = moe.dims(T=T, D=D, E=E, F=64, k=1)
    ws = _ws(moe, d)
    out = torch.empty((T, E), dtype=torch.float32, device="cuda")
    moe.moe_router_logits(h.cuda(), Wr.cuda(), d, out, ws)
    out2 = torch.empty_like(out)
    moe.moe_router_logits(h.cuda(), Wr.cuda(), d, out2, ws)
    assert torch.equal(out, out2)
    hf, wf = h.float().numpy().astype(np.float64), Wr.numpy().astype(np.float64)
    ref = orc.router_logits(hf, wf).astype(np.float64)
    mag = np.abs(hf) @ np.abs(wf).T
    err = np.abs(out.cpu().numpy() - ref)
    if D % 64 == 0 and E % 8 == 0:
        # tensor path: 3D exact bf16 products (the split of Wr is within 2^-24)
        # summed in fp32 inside the tensor core; allow a full ulp per add
        bound = (3 * D + 64) * 2.0 ** -23 * mag + np.abs(ref) * 2.0 ** -24
    else:
        # fp32 FMA chain: (D + splits) * 2^-24 * sum_d |h w|
        bound = (D + 33) * 2.0 ** -24 * mag + np.abs(ref) * 2.0 ** -24
    assert np.all(err <= bound)
    # typical error stays at fp32 level (a dropped middle piece of the split
    # would leave ~2^-9 relative errors)
    assert np.sqrt(np.mean(err ** 2)) <= 1e-5 * np.sqrt(np.mean(ref ** 2)) + 1e-9


# ---------------------------------------------------------------------------
# grouping: bit-exact
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (100, 8, 8), (257, 256, 8), (4096, 256, 8),
                                   (1000, 1024, 32), (513, 64, 1), (3000, 16, 4)])
def test_permute_exact(moe, T, E, k):
    idx = mi.synthetic_topk(T, E, k, 0, f"perm{T}x{E}x{k}")
    if T == 3000:  # maximal skew: every token picks the same experts
        idx = torch.arange(k, dtype=torch.int32).repeat(T, 1)
    d = moe.dims(T=T, D=64, E=E, F=64, k=k)
    ws = _ws(moe, d)
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty((T, k), dtype=torch.int32, device="cuda")
    moe.moe_permute(idx.cuda(), d, counts, offsets, perm, inv, ws)
    assert moe.moe_get_device_status(ws) == 0
    rc, ro, rp, ri = orc.group_by_expert(idx.numpy(), E)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(perm.cpu().numpy(), rp)
    assert np.array_equal(inv.cpu().numpy(), ri)


# ---------------------------------------------------------------------------
# expert MLPs on grouped rows
# ---------------------------------------------------------------------------
FFN_CASES = [
    # T, D, E, F, k, S, Fs
    (64, 128, 8, 64, 2, 1, 64),        # the tiny layer
    (200, 256, 16, 192, 4, 1, 320),    # F, Fs not multiples of the 128-wide tile, Fs != F
    (300, 1024, 32, 512, 8, 2, 256),   # two shared experts
    (130, 512, 8, 128, 2, 0, 0),       # no shared expert, ragged T
    (1, 136, 4, 64, 4, 1, 64),         # one token, D not a multiple of 64
    # more than 512 tokens: the 256-wide tiles
    (700, 256, 16, 192, 4, 1, 320),
    (900, 384, 12, 320, 3, 2, 192),    # D not a multiple of the 256-wide tile
    (600, 512, 8, 128, 2, 0, 0),
]


@pytest.mark.parametrize("T,D,E,F,k,S,Fs", FFN_CASES)
def test_expert_ffn(moe, T, D, E, F, k, S, Fs):
    _check_expert_ffn(moe, T, D, E, F, k, S, Fs, mi.synthetic_topk(T, E, k, 0, f"ffn{T}"))


# Batches above 512 tokens (256-wide tiles): expert sizes around the 128-row
# tile (0, 1, 15-17, 127-129, 255-257, 513 rows), a K tail (D = 136), F and Fs
# not multiples of the 128-feature gate/up tile and D not a multiple of the
# 256-column down tile.
BLOCK_EDGE_COUNTS = [256, 257, 1, 0, 15, 16, 17, 138, 255, 513, 127, 128, 129]


@pytest.mark.parametrize("D,F,S,Fs", [(256, 256, 1, 128), (136, 192, 2, 64), (384, 64, 0, 0)])
def test_expert_ffn_block_edges(moe, D, F, S, Fs):
    E = len(BLOCK_EDGE_COUNTS)
    idx = np.repeat(np.arange(E, dtype=np.int32), BLOCK_EDGE_COUNTS)
    order = mi.uniform_int(len(idx), 1 << 30, 0, "pair_edges").numpy().argsort(kind="stable")
    idx = torch.from_numpy(idx[order].reshape(-1, 1).copy())   # k = 1, tokens shuffled
    _check_expert_ffn(moe, len(idx), D, E, F, 1, S, Fs, idx)


def _check_expert_ffn(moe, T, D, E, F, k, S, Fs, idx):
    cfg = mi.LayerConfig("ffn", T, D, E, k, F, S, max(Fs, 8), 2.5, 1.0, f"ffn{T}x{D}x{E}")
    inp = layer_on_device(cfg)
    _, offsets, perm, _ = orc.group_by_expert(idx.numpy(), E)
    d = moe.dims(T=T, D=D, E=E, F=F, k=k, S=S, Fs=max(Fs, 8))
    ws = _ws(moe, d)
    y = torch.full((T * k + S * T, D), float("nan"), device="cuda")
    sh = (inp["Ws1"], inp["Ws3"], inp["Ws2"]) if S > 0 else (None, None, None)
    moe.moe_expert_ffn(inp["h"], torch.from_numpy(perm).cuda(), torch.from_numpy(offsets).cuda(),
                       inp["W1"], inp["W3"], inp["W2"], *sh, d, y, ws)
    assert moe.moe_get_device_status(ws) == 0
    got = y.cpu().numpy().astype(np.float64)
    h = host_f32(inp["h"])
    ref = np.empty_like(got)
    ex = HostExperts(inp["W1"], inp["W3"], inp["W2"])
    for e in range(E):
        rows = slice(offsets[e], offsets[e + 1])
        if offsets[e + 1] > offsets[e]:
            ref[rows] = orc.swiglu_expert(h[perm[rows]], *ex(e))
    for s in range(S):
        ws_ = tuple(x[s].cpu().double().numpy() for x in (inp["Ws1"], inp["Ws3"], inp["Ws2"]))
        ref[T * k + s * T: T * k + (s + 1) * T] = orc.swiglu_expert(h, *ws_)
    assert np.all(np.isfinite(got))
    # the gated activation is rounded to bf16 (relative 2^-9 per element) before
    # the w2 product; with independent signs that is ~1.1e-3 relative in L2
    assert rel_l2(got, ref) < 4e-3
    row_err = np.linalg.norm(got - ref, axis=1) / np.maximum(np.linalg.norm(ref, axis=1), 1e-30)
    assert row_err.max() < 2e-2


# ---------------------------------------------------------------------------
# merge
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("T,D,k,S", [(50, 136, 4, 2), (128, 6144, 8, 1), (7, 64, 1, 0)])
def test_combine(moe, T, D, k, S):
    y = mi.normal((T * k + S * T, D), 1.0, 0, f"comb{T}/y")
    w = mi.normal((T, k), 0.5, 0, f"comb{T}/w")
    idx = mi.synthetic_topk(T, 32, k, 0, f"comb{T}")
    _, _, _, inv = orc.group_by_expert(idx.numpy(), 32)
    d = moe.dims(T=T, D=D, E=32, F=64, k=k, S=S, Fs=64)
    out = torch.empty((T, D), dtype=torch.float32, device="cuda")
    ws = _ws(moe, d)
    moe.moe_combine(y.cuda(), w.cuda(), torch.from_numpy(inv).cuda(), d, out, ws)
    assert moe.moe_get_device_status(ws) == 0
    yn = y.numpy()
    ref = orc.combine(yn[:T * k], w.numpy(), inv, yn[T * k:].reshape(S, T, D) if S else None)
    terms = np.abs(w.numpy().astype(np.float64))[:, :, None] * np.abs(yn[inv]).astype(np.float64)
    mag = terms.sum(axis=1) + (np.abs(yn[T * k:]).reshape(S, T, D).sum(axis=0) if S else 0)
    got = out.cpu().numpy().astype(np.float64)
    # fp32 sums of (k + S) terms: each add/fma rounds once (2^-24 relative of
    # the partial sum), so |error| <= (k + S + 1) 2^-24 sum|terms|
    assert np.all(np.abs(got - ref) <= (k + S + 1) * 2.0 ** -24 * mag + 1e-30)


# ---------------------------------------------------------------------------
# the whole layer
# ---------------------------------------------------------------------------
def _forward(moe, cfg, inp, T=None):
    d = moe.dims_of(cfg, T)
    Tn = d.T
    ws = _ws(moe, d)
    out = torch.empty((Tn, cfg.D), dtype=torch.float32, device="cuda")
    idx = torch.empty((Tn, cfg.k), dtype=torch.int32, device="cuda")
    w = torch.empty((Tn, cfg.k), dtype=torch.float32, device="cuda")
    h = inp["h"][:Tn].contiguous()
    moe.moe_forward(h, inp["Wr"], inp["bias"], inp["W1"], inp["W3"], inp["W2"], inp["Ws1"],
                    inp["Ws3"], inp["Ws2"], d, out, ws, idx, w)
    assert moe.moe_get_device_status(ws) == 0
    return out, idx, w, ws


def _check_layer(cfg, inp, out, idx, tokens, max_flip_frac=0.02):
    experts = HostExperts(inp["W1"], inp["W3"], inp["W2"])
    ref, flips, wrong = oracle_rows(inp, cfg, tokens, idx.cpu().numpy()[tokens], experts)
    got = out.float().cpu().numpy()[tokens].astype(np.float64)
    assert wrong == 0, f"{wrong} tokens routed to a set that is not a correct top-k"
    assert flips <= max(1, max_flip_frac * len(tokens))
    assert rel_l2(got, ref) <= REL_L2_TOL
    assert np.max(np.abs(got - ref)) <= MAX_ABS_TOL
    return rel_l2(got, ref), float(np.max(np.abs(got - ref))), flips


def test_forward_tiny_all_tokens(moe):
    cfg = mi.CONFIGS["tiny"]
    inp = layer_on_device(cfg)
    out, idx, w, _ = _forward(moe, cfg, inp)
    _check_layer(cfg, inp, out, idx, np.arange(cfg.T))
    # routing inside the layer equals the standalone entry points bit for bit
    d = moe.dims_of(cfg)
    ws = _ws(moe, d)
    logits = torch.empty((cfg.T, cfg.E), device="cuda")
    moe.moe_router_logits(inp["h"], inp["Wr"], d, logits, ws)
    i2 = torch.empty_like(idx)
    w2 = torch.empty_like(w)
    moe.moe_route(logits, inp["bias"], d, i2, w2, ws)
    assert torch.equal(idx, i2) and torch.equal(w.view(torch.int32), w2.view(torch.int32))


def test_forward_tiny_pure_fp32_oracle(moe):
    """The tiny layer against the oracle on the raw fp32 draws: the only
    difference left is the bf16 rounding of h and the expert weights."""
    cfg = mi.CONFIGS["tiny"]
    inp = layer_on_device(cfg)
    out, idx, _, _ = _forward(moe, cfg, inp)
    w32 = mi.layer_weights(cfg, fp32=True)
    h32 = mi.hidden(cfg, fp32=True).numpy()
    ref, ridx, _, _ = orc.moe_layer(h32, w32["Wr"].numpy(), w32["bias"].numpy(), w32["W1"].numpy(),
                                    w32["W3"].numpy(), w32["W2"].numpy(), w32["Ws1"].numpy(),
                                    w32["Ws3"].numpy(), w32["Ws2"].numpy(), cfg.k, cfg.scale)
    same = np.all(np.sort(idx.cpu().numpy(), 1) == np.sort(ridx, 1), axis=1)
    got = out.float().cpu().numpy()
    # bf16 inputs move logits by ~2^-9 relative, which may flip a few near ties
    assert same.mean() >= 0.9
    assert rel_l2(got[same], ref[same]) <= 2e-2


@pytest.mark.parametrize("T", [0, 1, 2, 127, 129, 256, 257, 300])
def test_forward_ragged_and_empty(moe, T):
    cfg = mi.custom_config("tiny", T=max(T, 1), name="tiny")
    inp = layer_on_device(cfg)
    if T == 0:
        d = moe.dims_of(cfg, 0)
        ws = _ws(moe, d)
        out = torch.empty((0, cfg.D), dtype=torch.float32, device="cuda")
        moe.moe_forward(inp["h"], inp["Wr"], inp["bias"], inp["W1"], inp["W3"], inp["W2"],
                        inp["Ws1"], inp["Ws3"], inp["Ws2"], d, out, ws)
        assert moe.moe_last_launch_count() == 0
        return
    out, idx, _, _ = _forward(moe, cfg, inp)
    _check_layer(cfg, inp, out, idx, np.arange(T))


@pytest.mark.parametrize("variant", ["k1", "no_shared", "E1024_k32", "two_shared", "zero_scale"])
def test_forward_variants(moe, variant):
    base = dict(T=100, D=256, E=16, k=4, F=128, S=1, Fs=128, scale=2.5)
    if variant == "k1":
        base.update(k=1)
    elif variant == "no_shared":
        base.update(S=0)
    elif variant == "E1024_k32":
        base.update(E=1024, k=32, F=64, Fs=64, D=128)
    elif variant == "two_shared":
        base.update(S=2, Fs=192)
    elif variant == "zero_scale":
        base.update(scale=0.0)
    cfg = mi.LayerConfig(f"v_{variant}", hidden_std=1.0, weight_family=f"v_{variant}", **base)
    inp = layer_on_device(cfg)
    if cfg.S == 0:
        inp["Ws1"] = inp["Ws3"] = inp["Ws2"] = None
    out, idx, _, _ = _forward(moe, cfg, inp)
    if cfg.S == 0:
        inp["Ws1"] = torch.empty((0, 8, cfg.D), dtype=torch.bfloat16, device="cuda")
        inp["Ws3"] = inp["Ws1"]
        inp["Ws2"] = torch.empty((0, cfg.D, 8), dtype=torch.bfloat16, device="cuda")
    _check_layer(cfg, inp, out, idx, np.arange(cfg.T))


def test_forward_deterministic(moe):
    cfg = mi.custom_config("tiny", T=300, name="tiny")
    inp = layer_on_device(cfg)
    a, ia, wa, _ = _forward(moe, cfg, inp)
    b, ib, wb, _ = _forward(moe, cfg, inp)
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    assert torch.equal(ia, ib) and torch.equal(wa, wb)


# ---------------------------------------------------------------------------
# full-size workloads, sampled tokens
# ---------------------------------------------------------------------------
@pytest.fixture(scope="module")
def glm52():
    cfg = mi.CONFIGS["skew"]  # largest T of the family; h rows are prefix-stable
    w = mi.layer_weights(cfg, 0, device="cuda")
    return w


def _sample(T, n, name):
    if T <= n:
        return np.arange(T)
    return np.unique(mi.uniform_int(n, T, 0, "sample/" + name).numpy())


@pytest.mark.parametrize("name,n", [("decode", 128), ("prefill", 24), ("skew", 16)])
def test_forward_glm52_full_size(moe, glm52, name, n):
    cfg = mi.CONFIGS[name]
    inp = dict(glm52)
    if name != "skew":
        inp["bias"] = mi.correction_bias(cfg, 0, device="cuda")
    inp["h"] = mi.hidden(cfg, 0, device="cuda")
    out, idx, _, ws = _forward(moe, cfg, inp)
    assert torch.isfinite(out.float()).all()
    _check_layer(cfg, inp, out, idx, _sample(cfg.T, n, name))
    # the routed load the workload describes: skew follows the stored Zipf bias;
    # the histogram kept in the workspace matches the returned indices
    counts = torch.bincount(idx.flatten().long(), minlength=cfg.E).cpu().numpy()
    d = moe.dims_of(cfg)
    assert np.array_equal(moe.moe_ws_expert_counts(ws, d).cpu().numpy(), counts)
    assert int(moe.moe_ws_touched_experts(ws, d).item()) == int((counts > 0).sum())
    if name == "skew":
        assert (counts == 0).sum() >= 16 and counts.max() > 10 * counts.mean()


def test_expert_ffn_full_size_heavy_experts(moe, glm52):
    """Every row of the three heaviest experts of the skewed workload (thousands
    of rows over many token blocks: the dynamic tile claims and the per-expert
    gate/up -> down hand-off at their busiest) and of one expert whose last
    token block is partial, at the GLM-5.2 sizes, against the oracle's expert
    MLP on the same grouped rows."""
    cfg = mi.CONFIGS["skew"]
    T, E, k, D = cfg.T, cfg.E, cfg.k, cfg.D
    inp = dict(glm52)
    inp["h"] = mi.hidden(cfg, 0, device="cuda")
    d = moe.dims_of(cfg)
    ws = _ws(moe, d)
    logits = torch.empty((T, E), device="cuda")
    moe.moe_router_logits(inp["h"], inp["Wr"], d, logits, ws)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), device="cuda")
    moe.moe_route(logits, inp["bias"], d, idx, w, ws)
    counts, offsets, perm, _ = orc.group_by_expert(idx.cpu().numpy(), E)
    y = torch.full((T * k + cfg.S * T, D), float("nan"), device="cuda")
    moe.moe_expert_ffn(inp["h"], torch.from_numpy(perm).cuda(), torch.from_numpy(offsets).cuda(),
                       inp["W1"], inp["W3"], inp["W2"], inp["Ws1"], inp["Ws3"], inp["Ws2"], d, y,
                       ws)
    assert moe.moe_get_device_status(ws) == 0
    by_load = np.argsort(-counts, kind="stable")
    heavy = [int(e) for e in by_load[:3]]
    partial = next(int(e) for e in by_load[3:] if counts[e] > 256 and counts[e] % 128)
    assert counts[heavy[-1]] > 1000
    h = host_f32(inp["h"])
    ex = HostExperts(inp["W1"], inp["W3"], inp["W2"])
    for e in heavy + [partial]:
        a, b = int(offsets[e]), int(offsets[e + 1])
        ref = orc.swiglu_expert(h[perm[a:b]], *ex(e))
        got = y[a:b].cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(got))
        assert rel_l2(got, ref) < 4e-3, e
        row_err = np.linalg.norm(got - ref, axis=1) / np.maximum(np.linalg.norm(ref, axis=1),
                                                                 1e-30)
        assert row_err.max() < 2e-2, e


def test_forward_air_full_size(moe):
    cfg = mi.CONFIGS["air"]
    inp = layer_on_device(cfg)
    out, idx, _, _ = _forward(moe, cfg, inp)
    _check_layer(cfg, inp, out, idx, _sample(cfg.T, 24, "air"))


# ---------------------------------------------------------------------------
# device-side error reporting (never a trap)
# ---------------------------------------------------------------------------
def test_status_nonfinite_logit(moe):
    d = moe.dims(T=4, D=64, E=8, F=64, k=2)
    ws = _ws(moe, d)
    logits = torch.zeros((4, 8), device="cuda")
    logits[2, 3] = float("nan")
    idx = torch.empty((4, 2), dtype=torch.int32, device="cuda")
    w = torch.empty((4, 2), device="cuda")
    moe.moe_route(logits, torch.zeros(8, device="cuda"), d, idx, w, ws)
    assert moe.moe_get_device_status(ws) == moe.MOE_ERR_NONFINITE
    assert moe.moe_get_device_status(ws) == 0  # cleared


def test_status_bad_indices(moe):
    d = moe.dims(T=4, D=64, E=8, F=64, k=2)
    ws = _ws(moe, d)
    outs = [torch.empty(8, dtype=torch.int32, device="cuda"),
            torch.empty(9, dtype=torch.int32, device="cuda"),
            torch.empty(8, dtype=torch.int32, device="cuda"),
            torch.empty((4, 2), dtype=torch.int32, device="cuda")]
    bad_range = torch.tensor([[0, 1], [2, 9], [3, 4], [5, 6]], dtype=torch.int32, device="cuda")
    moe.moe_permute(bad_range, d, *outs, ws)
    assert moe.moe_get_device_status(ws) == moe.MOE_ERR_BOUNDS
    dup = torch.tensor([[0, 1], [2, 2], [3, 4], [5, 6]], dtype=torch.int32, device="cuda")
    moe.moe_permute(dup, d, *outs, ws)
    assert moe.moe_get_device_status(ws) == moe.MOE_ERR_BOUNDS
    y = torch.zeros((4 * 2 + 4, 64), device="cuda")
    inv = torch.tensor([[0, 1], [2, 3], [4, 99], [6, 7]], dtype=torch.int32, device="cuda")
    out = torch.empty((4, 64), dtype=torch.float32, device="cuda")
    moe.moe_combine(y, torch.ones((4, 2), device="cuda"), inv, d, out, ws)
    assert moe.moe_get_device_status(ws) == moe.MOE_ERR_BOUNDS


def test_status_bad_offsets(moe):
    T, D, E, F, k = 8, 128, 4, 64, 2
    d = moe.dims(T=T, D=D, E=E, F=F, k=k, S=0)
    ws = _ws(moe, d)
    cfg = mi.LayerConfig("offs", T, D, E, k, F, 0, 8, 2.5, 1.0, "offs")
    inp = layer_on_device(cfg)
    perm = torch.zeros(T * k, dtype=torch.int32, device="cuda")
    offsets = torch.tensor([0, 4, 2, 10, 16], dtype=torch.int32, device="cuda")  # decreasing
    y = torch.zeros((T * k, D), device="cuda")
    moe.moe_expert_ffn(inp["h"], perm, offsets, inp["W1"], inp["W3"], inp["W2"], None, None, None,
                       d, y, ws)
    assert moe.moe_get_device_status(ws) == moe.MOE_ERR_BOUNDS


def test_bounded_wait_times_out_and_the_context_survives(moe):
    """A wait that can never end gives up after its clock budget and reports
    MOE_ERR_TIMEOUT; the next layer call on the same context still works."""
    d = moe.dims(T=4, D=64, E=8, F=64, k=2)
    ws = _ws(moe, d)
    moe.moe_selftest_bounded_wait(ws)
    assert moe.moe_get_device_status(ws) == moe.MOE_ERR_TIMEOUT
    cfg = mi.CONFIGS["tiny"]
    inp = layer_on_device(cfg)
    out, idx, _, _ = _forward(moe, cfg, inp)
    _check_layer(cfg, inp, out, idx, np.arange(8))
