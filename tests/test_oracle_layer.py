"""Pins of the oracle's expert MLP, grouping, merge and whole layer.

Checks against library routines (torch CPU linear/SiLU), closed forms
(identity experts), brute-force Python loops on tiny inputs, linearity in the
routed scale and metamorphic relations (token permutation, expert
relabelling).
"""
import numpy as np
import torch
import torch.nn.functional as Fn

import moe_inputs as mi
from oracle import moe_oracle as orc


def _tiny(seed=0, **over):
    cfg = mi.custom_config("tiny", **over) if over else mi.CONFIGS["tiny"]
    h = mi.hidden(cfg, seed).float().numpy()
    w = {k: v.float().numpy() for k, v in mi.layer_weights(cfg, seed).items()}
    return cfg, h, w


def _torch_swiglu(x, w1, w3, w2):
    x, w1, w3, w2 = (torch.from_numpy(np.asarray(a, np.float64)) for a in (x, w1, w3, w2))
    return Fn.linear(Fn.silu(Fn.linear(x, w1)) * Fn.linear(x, w3), w2).numpy()


def test_swiglu_matches_torch_linear_silu():
    cfg, h, w = _tiny()
    got = orc.swiglu_expert(h, w["W1"][3], w["W3"][3], w["W2"][3])
    assert np.allclose(got, _torch_swiglu(h, w["W1"][3], w["W3"][3], w["W2"][3]),
                       rtol=1e-12, atol=1e-12)


def test_zero_scale_leaves_the_shared_expert():
    cfg, h, w = _tiny()
    out, idx, rw, _ = orc.moe_layer(h, w["Wr"], w["bias"], w["W1"], w["W3"], w["W2"],
                                    w["Ws1"], w["Ws3"], w["Ws2"], cfg.k, 0.0)
    assert np.all(rw == 0)
    ref = _torch_swiglu(h, w["Ws1"][0], w["Ws3"][0], w["Ws2"][0])
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_identity_experts_give_silu_x_times_x():
    T, D = 9, 16
    rng = np.random.default_rng(2)
    x = rng.standard_normal((T, D))
    I = np.eye(D)
    y = orc.swiglu_expert(x, I, I, I)
    xt = torch.from_numpy(x)
    assert np.allclose(y, (Fn.silu(xt) * xt).numpy(), rtol=1e-14, atol=1e-14)


def test_layer_matches_bruteforce_loops_on_tiny():
    cfg, h, w = _tiny(T=6)
    out, idx, rw, logits = orc.moe_layer(h, w["Wr"], w["bias"], w["W1"], w["W3"], w["W2"],
                                         w["Ws1"], w["Ws3"], w["Ws2"], cfg.k, cfg.scale)
    for t in range(cfg.T):
        acc = _torch_swiglu(h[t:t + 1], w["Ws1"][0], w["Ws3"][0], w["Ws2"][0])[0]
        for j in range(cfg.k):
            e = idx[t, j]
            acc = acc + float(rw[t, j]) * _torch_swiglu(h[t:t + 1], w["W1"][e], w["W3"][e],
                                                        w["W2"][e])[0]
        assert np.allclose(out[t], acc, rtol=1e-12, atol=1e-12)


def test_linear_in_routed_scale():
    cfg, h, w = _tiny()
    args = (h, w["Wr"], w["bias"], w["W1"], w["W3"], w["W2"], w["Ws1"], w["Ws3"], w["Ws2"], cfg.k)
    shared = orc.moe_layer(*args, 0.0)[0]
    o1 = orc.moe_layer(*args, 1.0)[0] - shared
    o4 = orc.moe_layer(*args, 4.0)[0] - shared
    assert np.allclose(o4, 4.0 * o1, rtol=1e-10, atol=1e-12)


def test_token_permutation_permutes_outputs():
    cfg, h, w = _tiny()
    perm = np.random.default_rng(4).permutation(cfg.T)
    args = (w["Wr"], w["bias"], w["W1"], w["W3"], w["W2"], w["Ws1"], w["Ws3"], w["Ws2"],
            cfg.k, cfg.scale)
    out = orc.moe_layer(h, *args)[0]
    outp = orc.moe_layer(h[perm], *args)[0]
    assert np.allclose(outp, out[perm], rtol=1e-12, atol=1e-12)


def test_expert_relabelling_leaves_output_unchanged():
    cfg, h, w = _tiny()
    p = np.random.default_rng(6).permutation(cfg.E)
    out = orc.moe_layer(h, w["Wr"], w["bias"], w["W1"], w["W3"], w["W2"], w["Ws1"], w["Ws3"],
                        w["Ws2"], cfg.k, cfg.scale)[0]
    outp = orc.moe_layer(h, w["Wr"][p], w["bias"][p], w["W1"][p], w["W3"][p], w["W2"][p],
                         w["Ws1"], w["Ws3"], w["Ws2"], cfg.k, cfg.scale)[0]
    assert np.allclose(outp, out, rtol=1e-12, atol=1e-12)


def test_grouping_matches_bucket_loop():
    for seed in range(5):
        rng = np.random.default_rng(seed)
        T, E, k = 37, 11, 3
        idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
        counts, offsets, perm, inv = orc.group_by_expert(idx, E)
        rows = []
        inv_ref = np.full((T, k), -1)
        for e in range(E):
            for t in range(T):
                for j in range(k):
                    if idx[t, j] == e:
                        inv_ref[t, j] = len(rows)
                        rows.append(t)
        assert perm.tolist() == rows
        assert np.array_equal(inv, inv_ref)
        assert counts.tolist() == [int((idx == e).sum()) for e in range(E)]
        assert offsets[0] == 0 and offsets[-1] == T * k
        assert np.array_equal(np.diff(offsets), counts)


def test_combine_matches_loop():
    rng = np.random.default_rng(8)
    T, k, D, S = 7, 3, 5, 2
    y = rng.standard_normal((T * k, D))
    ys = rng.standard_normal((S, T, D))
    w = rng.standard_normal((T, k)).astype(np.float32)
    inv = rng.permutation(T * k).reshape(T, k).astype(np.int32)
    out = orc.combine(y, w, inv, ys)
    for t in range(T):
        ref = ys[0, t] + ys[1, t]
        for j in range(k):
            ref = ref + float(w[t, j]) * y[inv[t, j]]
        assert np.allclose(out[t], ref, rtol=1e-14, atol=1e-14)


def test_given_routing_equals_layer_on_its_own_routing():
    cfg, h, w = _tiny()
    out, idx, rw, _ = orc.moe_layer(h, w["Wr"], w["bias"], w["W1"], w["W3"], w["W2"],
                                    w["Ws1"], w["Ws3"], w["Ws2"], cfg.k, cfg.scale)
    routed = orc.routed_output_given_routing(h, idx, rw, lambda e: (w["W1"][e], w["W3"][e],
                                                                    w["W2"][e]))
    shared = _torch_swiglu(h, w["Ws1"][0], w["Ws3"][0], w["Ws2"][0])
    assert np.allclose(out, routed + shared, rtol=1e-12, atol=1e-12)
