"""Plain numpy oracle of the GLM-5.2 Mixture-of-Experts feed-forward layer.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never
imports this module.

What the layer computes, as the pages describe it:

* "Model anatomy -- GLM-5.2" (frontier-model-atlas), Decoder microscope,
  Feed-forward / Mixture of Experts panel: 256 routed experts, 8 active per
  token, 1 shared expert, expert width 2048, learned routing.  The router
  scores are sigmoids; an expert-score correction bias takes part in the
  top-k selection only; the selected scores *without* the bias are
  renormalised to sum to one and multiplied by 2.5; the weighted expert
  outputs are then merged with the output of the always-on shared expert.
  The same page's "Expert fan-out 8 + 1" counts the routed plus shared
  experts that every token uses.
* "GLM-5.2" (PocketLLM), Model specification table: hidden size 6144,
  256 routed experts, top-8, expert intermediate size 2048, 1 shared expert;
  Implemented execution path: the expert weights are named w1/w3 (the two
  input projections) and w2 (the output projection).
* "GLM-4.5 Full Forward", How it works: MoE layers use sigmoid routing, one
  shared expert and a routed scaling factor of 2.5 (1.0 for GLM-4.5-Air).

Readings where the pages are silent (each is listed in the design notes):
the expert MLP is SwiGLU, y = w2 (silu(w1 x) * (w3 x)), silu(z) = z/(1+e^-z);
weights use the (out-features, in-features) layout; ties between equal
selection keys go to the lower expert index and the slot order is the
selection order; the shared expert enters with weight 1 (it is not scaled);
routing is dropless (every token gets all k experts); no epsilon is added to
the renormalising sum.
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence, Tuple

import numpy as np

F32 = np.float32
F64 = np.float64


# ----------------------------------------------------------------------------
# router: logits, scores, selection, weights
# ----------------------------------------------------------------------------

def router_logits(h: np.ndarray, Wr: np.ndarray) -> np.ndarray:
    """Router logits l[t, e] = sum_d h[t, d] * Wr[e, d] as fp32.

    The router is learned and kept in fp32 (MoE panel, "Routing: learned").
    The dot product is evaluated in fp64 and rounded once, so each logit is
    the fp32 value nearest to the exact sum up to fp64 rounding.
    """
    return (np.asarray(h, F64) @ np.asarray(Wr, F64).T).astype(F32)


def sigmoid_scores(logits: np.ndarray) -> np.ndarray:
    """Sigmoid router scores s = 1 / (1 + exp(-l)) (MoE panel: "Sigmoid router scores").

    Evaluated in fp64 from the fp32 logit and rounded once to fp32.
    """
    x = np.asarray(logits, F32).astype(F64)
    if not np.all(np.isfinite(x)):
        raise ValueError("non-finite router logit")
    with np.errstate(over="ignore"):
        return (1.0 / (1.0 + np.exp(-x))).astype(F32)


def selection_keys(scores: np.ndarray, bias: np.ndarray) -> np.ndarray:
    """Selection key = score + correction bias, one fp32 add (MoE panel: the
    correction bias "affects top-k selection")."""
    return (np.asarray(scores, F32) + np.asarray(bias, F32)[None, :]).astype(F32)


def select_topk(keys: np.ndarray, k: int) -> np.ndarray:
    """The k experts that come first under (key descending, index ascending).

    Returned in that order (slot j = the j-th selected expert), int32 [T, k].
    A stable sort of the negated keys is exactly that order: equal keys keep
    their ascending index order.
    """
    keys = np.asarray(keys, F32)
    if not 1 <= k <= keys.shape[1]:
        raise ValueError("need 1 <= k <= E")
    order = np.argsort(-keys, axis=1, kind="stable")
    return order[:, :k].astype(np.int32)


def routing_weights(scores: np.ndarray, idx: np.ndarray, scale: float) -> np.ndarray:
    """w[t, j] = s[t, idx[t, j]] / (sum over the k selected s) * scale, fp32.

    MoE panel: the *un-biased* selected scores are renormalised and scaled by
    the routed scaling factor.  The sum runs over the slots in order, one fp32
    add at a time; then one fp32 division and one fp32 multiply per weight.
    """
    s_sel = np.take_along_axis(np.asarray(scores, F32), np.asarray(idx, np.int64), axis=1)
    total = np.zeros(s_sel.shape[0], F32)
    for j in range(s_sel.shape[1]):
        total = (total + s_sel[:, j]).astype(F32)
    if not np.all(total > 0):
        raise ValueError("renormalising sum is not positive")
    return ((s_sel / total[:, None]).astype(F32) * F32(scale)).astype(F32)


def route(logits: np.ndarray, bias: np.ndarray, k: int, scale: float
          ) -> Tuple[np.ndarray, np.ndarray]:
    """(idx [T, k] int32, w [T, k] fp32) from fp32 logits and the correction bias."""
    s = sigmoid_scores(logits)
    idx = select_topk(selection_keys(s, bias), k)
    return idx, routing_weights(s, idx, scale)


def group_scores(keys: np.ndarray, n_group: int) -> np.ndarray:
    """Score of each contiguous expert group: the sum of its two largest
    selection keys (one fp32 add), or its single key for one-expert groups.

    "GLM-4.5 Full Forward" (How it works) names sigmoid *group* routing
    without its rule or group counts; this is the reading taken: experts are
    cut into n_group equal contiguous groups ranked by their two best keys.
    """
    keys = np.asarray(keys, F32)
    T, E = keys.shape
    if n_group < 1 or E % n_group:
        raise ValueError("n_group must divide E")
    g = keys.reshape(T, n_group, E // n_group)
    if g.shape[2] == 1:
        return g[:, :, 0].astype(F32)
    top2 = -np.sort(-g, axis=2)[:, :, :2]
    return (top2[:, :, 0] + top2[:, :, 1]).astype(F32)


def route_grouped(logits: np.ndarray, bias: np.ndarray, k: int, scale: float, n_group: int,
                  topk_group: int) -> Tuple[np.ndarray, np.ndarray]:
    """Group-limited routing: keep the topk_group groups that come first under
    (group score descending, group index ascending), then select the top-k
    experts inside them exactly as route() does; weights from the un-biased
    scores.  n_group = 1 (or topk_group = n_group) is plain routing.
    """
    s = sigmoid_scores(logits)
    keys = selection_keys(s, bias)
    T, E = keys.shape
    if not 1 <= topk_group <= n_group:
        raise ValueError("need 1 <= topk_group <= n_group")
    if k > topk_group * (E // n_group):
        raise ValueError("k exceeds the experts of the kept groups")
    gs = group_scores(keys, n_group)
    keep = np.argsort(-gs, axis=1, kind="stable")[:, :topk_group]
    allowed = np.zeros((T, n_group), bool)
    np.put_along_axis(allowed, keep, True, axis=1)
    mask = np.repeat(allowed, E // n_group, axis=1)
    masked = np.where(mask, keys, F32(-np.inf)).astype(F32)
    idx = select_topk(masked, k)
    return idx, routing_weights(s, idx, scale)


def routing_alternatives(logits_row: np.ndarray, bias: np.ndarray, k: int, scale: float,
                         delta: float):
    """Every routing of one token that is correct up to a logit perturbation.

    Two implementations of the fp32 router sum the hidden dimension in
    different orders, so their logits (and hence keys) may differ in the last
    bits.  When the k-th and (k+1)-th selection keys lie within `delta` of
    each other, either choice is a correct top-k.  Returns a list of
    (idx [k] int32, w [k] fp32) candidates: the strict selection first, then
    every other choice of the boundary experts among those whose key lies
    within `delta` of the k-th key (at most 64 candidates).
    """
    s = sigmoid_scores(np.asarray(logits_row, F32)[None, :])
    keys = selection_keys(s, bias)[0]
    order = select_topk(keys[None, :], keys.shape[0])[0]
    kth = float(keys[order[k - 1]])
    near = [int(e) for e in order if abs(float(keys[e]) - kth) <= delta]
    sure = [int(e) for e in order[:k] if int(e) not in near]
    need = k - len(sure)
    cands = []
    from itertools import combinations
    for pick in combinations(near, need):
        chosen = set(sure) | set(pick)
        idx = np.array([int(e) for e in order if int(e) in chosen], np.int32)[None, :]
        cands.append((idx[0], routing_weights(s, idx, scale)[0]))
        if len(cands) >= 64:
            break
    strict = order[:k].astype(np.int32)
    cands.sort(key=lambda c: 0 if np.array_equal(c[0], strict) else 1)
    return cands


# ----------------------------------------------------------------------------
# experts
# ----------------------------------------------------------------------------

def swiglu_expert(x: np.ndarray, w1: np.ndarray, w3: np.ndarray, w2: np.ndarray) -> np.ndarray:
    """One gated expert MLP on rows x [n, D]: w2 (silu(w1 x) * (w3 x)), in fp64.

    w1 [F, D] is the gate projection, w3 [F, D] the up projection and
    w2 [D, F] the down projection (PocketLLM, Implemented execution path, names
    w1/w3 and w2; the gated form is the reading taken for the pages' silence).
    """
    x = np.asarray(x, F64)
    g = x @ np.asarray(w1, F64).T
    u = x @ np.asarray(w3, F64).T
    with np.errstate(over="ignore"):
        a = g / (1.0 + np.exp(-g)) * u
    return a @ np.asarray(w2, F64).T


# ----------------------------------------------------------------------------
# FP8 expert weights
# ----------------------------------------------------------------------------

def e4m3_value(code: np.ndarray) -> np.ndarray:
    """Value of an OCP E4M3 (float8_e4m3fn) code, from the format definition:
    sign bit, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 is
    subnormal (m * 2**-9); S.1111.111 is NaN; there is no infinity."""
    c = np.asarray(code, np.int64)
    sign = np.where(c >> 7, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def dequantize_fp8_blocks(codes: np.ndarray, exps: np.ndarray, block: int = 128) -> np.ndarray:
    """w = e4m3_value(code) * 2**e with one exponent per block x block tile
    of the last two dimensions (the weights an FP8 layer stands for)."""
    codes = np.asarray(codes)
    exps = np.asarray(exps, np.int64)
    R, K = codes.shape[-2:]
    scale = np.exp2(np.repeat(np.repeat(exps, block, axis=-2), block, axis=-1)[..., :R, :K])
    return e4m3_value(codes) * scale


# ----------------------------------------------------------------------------
# grouping by expert and merging
# ----------------------------------------------------------------------------

def group_by_expert(idx: np.ndarray, E: int):
    """Counting sort of the (token, slot) pairs by expert.

    Returns counts [E], offsets [E + 1] (exclusive prefix sum), perm [T*k]
    (the token of each grouped row: rows offsets[e]..offsets[e+1]-1 hold the
    tokens routed to e, in increasing (token, slot) order) and inv [T, k]
    (the grouped row of pair (t, j)).  A stable sort of the flattened expert
    ids is exactly that order.
    """
    idx = np.asarray(idx, np.int64)
    T, k = idx.shape
    flat = idx.reshape(-1)
    if flat.size and (flat.min() < 0 or flat.max() >= E):
        raise ValueError("expert index out of range")
    counts = np.bincount(flat, minlength=E).astype(np.int32)
    offsets = np.zeros(E + 1, np.int32)
    offsets[1:] = np.cumsum(counts)
    order = np.argsort(flat, kind="stable")
    perm = (order // k).astype(np.int32)
    inv = np.empty(T * k, np.int32)
    inv[order] = np.arange(T * k, dtype=np.int32)
    return counts, offsets, perm, inv.reshape(T, k)


def combine(y_routed: np.ndarray, w: np.ndarray, inv: np.ndarray,
            y_shared: Optional[np.ndarray]) -> np.ndarray:
    """out[t] = sum_s y_shared[s, t] + sum_j w[t, j] * y_routed[inv[t, j]], fp64.

    MoE panel: the weighted expert outputs are merged with the always-on
    shared expert ("Expert fan-out 8 + 1"); the shared expert has weight 1.
    """
    y = np.asarray(y_routed, F64)
    out = np.einsum("tj,tjd->td", np.asarray(w, F64), y[np.asarray(inv, np.int64)])
    if y_shared is not None:
        out = out + np.asarray(y_shared, F64).sum(axis=0)
    return out


# ----------------------------------------------------------------------------
# the layer
# ----------------------------------------------------------------------------

ExpertFn = Callable[[int], Tuple[np.ndarray, np.ndarray, np.ndarray]]


def routed_output_given_routing(h: np.ndarray, idx: np.ndarray, w: np.ndarray,
                                expert: ExpertFn) -> np.ndarray:
    """sum_j w[t, j] * expert_{idx[t, j]}(h[t]) for every row of h, fp64.

    ``expert(e)`` returns (w1, w3, w2) of routed expert e, so that only the
    experts some token selected are ever materialised.
    """
    h = np.asarray(h)
    idx = np.asarray(idx, np.int64)
    out = np.zeros((h.shape[0], h.shape[1]), F64)
    for e in np.unique(idx):
        rows, slots = np.nonzero(idx == e)
        y = swiglu_expert(h[rows], *expert(int(e)))
        out[rows] += np.asarray(w, F64)[rows, slots][:, None] * y
    return out


def shared_output(h: np.ndarray, shared: Sequence[Tuple[np.ndarray, np.ndarray, np.ndarray]]
                  ) -> np.ndarray:
    out = np.zeros((h.shape[0], h.shape[1]), F64)
    for w1, w3, w2 in shared:
        out += swiglu_expert(h, w1, w3, w2)
    return out


def moe_layer_tokens(h: np.ndarray, Wr: np.ndarray, bias: np.ndarray, k: int, scale: float,
                     expert: ExpertFn,
                     shared: Sequence[Tuple[np.ndarray, np.ndarray, np.ndarray]]):
    """The layer on the rows of h: returns (out fp64 [n, D], idx, w, logits).

    Steps, in the order the MoE panel gives them: fp32 router logits, sigmoid
    scores, biased top-k selection, un-biased renormalised and scaled weights,
    the weighted routed experts, plus the shared expert.
    """
    logits = router_logits(h, Wr)
    idx, w = route(logits, bias, k, scale)
    out = routed_output_given_routing(h, idx, w, expert) + shared_output(h, shared)
    return out, idx, w, logits


def moe_layer(h, Wr, bias, W1, W3, W2, Ws1, Ws3, Ws2, k: int, scale: float):
    """Whole layer with all weights given as arrays ([E, F, D], [E, F, D], [E, D, F], ...)."""
    W1, W3, W2 = np.asarray(W1), np.asarray(W3), np.asarray(W2)
    shared = [(Ws1[s], Ws3[s], Ws2[s]) for s in range(np.asarray(Ws1).shape[0])]
    return moe_layer_tokens(np.asarray(h), Wr, bias, k, scale,
                            lambda e: (W1[e], W3[e], W2[e]), shared)
