"""Host model of the selection order the routing kernels use (CPU only).

The kernels rank a selection key by an unsigned integer with the same order
(sign-magnitude float bits flipped into two's-complement order; -0 ranked as
+0; NaN as 0, below every key) and pick per warp the largest integer, ties to
the lowest expert index, then merge the per-warp lists the same way.  These
tests check that model against the oracle's definition of the order (key
descending, index ascending), including ties, signed zeros, infinities and
subnormals, so a wrong bit mapping or tie rule fails here before any GPU run.
"""
import numpy as np
import pytest

from oracle import moe_oracle as orc


def key_order(keys: np.ndarray) -> np.ndarray:
    u = np.asarray(keys, np.float32).view(np.uint32).copy()
    u[u == 0x80000000] = 0                     # -0 ranks as +0
    neg = (u & 0x80000000) != 0
    out = np.where(neg, ~u, u | 0x80000000).astype(np.uint32)
    out[np.isnan(np.asarray(keys, np.float32))] = 0
    return out


def model_topk(keys: np.ndarray, k: int, warp: int = 32) -> np.ndarray:
    """Per-warp top-k by (order max, index min), then the same over the union."""
    T, E = keys.shape
    out = np.zeros((T, k), np.int64)
    for t in range(T):
        u = key_order(keys[t]).astype(np.int64)
        cands = []
        for w0 in range(0, E, warp):
            uu = u[w0:w0 + warp].copy()
            for _ in range(min(k, len(uu))):
                m = uu.max()
                j = int(np.flatnonzero(uu == m)[0])
                if m > 0:
                    cands.append((m, w0 + j))
                uu[j] = -1
        cands.sort(key=lambda c: (-c[0], c[1]))
        out[t] = [e for _, e in cands[:k]]
    return out


def test_order_is_monotone_over_every_float_class():
    vals = np.array([-np.inf, -3.4e38, -1.0, -1e-38, -1e-45, -0.0, 0.0, 1e-45, 1e-38, 0.5, 1.0,
                     3.4e38, np.inf], np.float32)
    u = key_order(vals)
    assert np.all(np.diff(u[:5].astype(np.int64)) > 0)
    assert u[5] == u[6]                        # -0 and +0 tie
    assert np.all(np.diff(u[6:].astype(np.int64)) > 0)
    assert u[0] > 0                            # -inf is still a candidate
    assert key_order(np.array([np.nan], np.float32))[0] == 0


def test_order_matches_float_comparison_on_random_pairs():
    rng = np.random.default_rng(0)
    with np.errstate(over="ignore"):   # the widest draws round to +-inf on purpose
        a = (rng.standard_normal(20000) * 10.0 ** rng.integers(-40, 39, 20000)).astype(np.float32)
        b = (rng.standard_normal(20000) * 10.0 ** rng.integers(-40, 39, 20000)).astype(np.float32)
    ua, ub = key_order(a).astype(np.int64), key_order(b).astype(np.int64)
    assert np.array_equal(ua > ub, a > b)
    assert np.array_equal(ua == ub, a == b)


@pytest.mark.parametrize("E,k,grid", [(256, 8, False), (256, 8, True), (64, 6, True), (1000, 32, True),
                                      (8, 8, True), (40, 3, False)])
def test_model_selection_equals_the_oracle(E, k, grid):
    rng = np.random.default_rng(E * 100 + k)
    T = 50
    if grid:   # few distinct values: many exact ties, including signed zeros
        keys = rng.integers(-3, 4, (T, E)).astype(np.float32) * np.float32(0.25)
        keys[rng.random((T, E)) < 0.1] = -0.0
    else:
        keys = rng.standard_normal((T, E)).astype(np.float32)
    assert np.array_equal(model_topk(keys, k), orc.select_topk(keys, k))
