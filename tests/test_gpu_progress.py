"""Forward progress when the layer does not have the whole GPU.

A self-test kernel holds most of the SMs for about 1.5 s (it spins on its own
clock and waits on nothing else) while the whole layer runs on another
stream.  The layer must finish on the SMs that are left, with a clean device
status and the same output as when it runs alone: the expert FFN hands its
tiles out only to CTAs that are already running, so no down tile waits for a
gate/up tile of a CTA that has no SM.  (With a statically assigned first tile
per CTA, such a wait would outlast the one-second wait budget and end in
MOE_ERR_TIMEOUT.)  The output is also checked against the oracle on sampled
tokens.
"""
import time

import numpy as np
import pytest
import torch

import moe_inputs as mi
from tests.gpu_helpers import (MAX_ABS_TOL, REL_L2_TOL, HostExperts, layer_on_device, oracle_rows,
                               rel_l2)

pytestmark = pytest.mark.gpu

# SMs left to the layer while the occupier runs, and the occupier's hold:
# 3e9 SM cycles is 1.5 s at 1.965 GHz, longer than one bounded wait (2^31 cycles).
FREE_SMS = 40
HOLD_CYCLES = 3_000_000_000

CASES = {
    # 256-wide tiles (T > 512): ~40 row tiles x 8 or 4 column tiles per GEMM
    "wide": mi.custom_config("prefill", T=1024, D=2048, E=32, k=4, F=1024, S=1, Fs=1024,
                             name="progress_wide"),
    # 128-wide tiles with the shared expert's FFN beside the routing (25 MB of shared weights)
    "narrow_overlap": mi.custom_config("decode", T=128, D=4096, E=32, k=8, F=1024, S=1, Fs=1024,
                                       name="progress_narrow"),
}


class Fp8HostExperts:
    """The oracle's decoding of one expert's FP8 weights, on demand."""

    def __init__(self, q):
        self.q = q
        self.cache = {}

    def matrix(self, name, g):
        from oracle import moe_oracle as orc
        return orc.dequantize_fp8_blocks(self.q[name + "q"][g].cpu().numpy(),
                                         self.q[name + "e"][g].cpu().numpy())

    def __call__(self, e):
        if e not in self.cache:
            self.cache[e] = tuple(self.matrix(n, e) for n in ("W1", "W3", "W2"))
        return self.cache[e]


@pytest.fixture(scope="module")
def moe():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import sparse_moe_layer_04_b200 as m
    return m


def _forward(moe, cfg, inp, d, ws, out, idx, w8):
    if w8 is None:
        moe.moe_forward(inp["h"], inp["Wr"], inp["bias"], inp["W1"], inp["W3"], inp["W2"],
                        inp["Ws1"], inp["Ws3"], inp["Ws2"], d, out, ws, idx)
    else:
        moe.moe_forward_fp8(inp["h"], inp["Wr"], inp["bias"], w8, d, out, ws, idx)


@pytest.mark.parametrize("weights", ["bf16", "fp8"])
@pytest.mark.parametrize("name", list(CASES))
def test_layer_finishes_beside_an_sm_occupier(moe, name, weights):
    cfg = CASES[name]
    inp = layer_on_device(cfg)
    w8 = None
    if weights == "fp8":
        q = mi.fp8_layer_weights(inp)
        w8 = moe.fp8_weights(*(q[n + "q"] for n in ("W1", "W3", "W2", "Ws1", "Ws3", "Ws2")),
                             *(q[n + "e"] for n in ("W1", "W3", "W2", "Ws1", "Ws3", "Ws2")))
        w8._keep = q
    d = moe.dims_of(cfg)
    ws = moe.alloc_workspace(d)
    dev = "cuda"
    alone = torch.empty((cfg.T, cfg.D), device=dev)
    idx_alone = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=dev)
    _forward(moe, cfg, inp, d, ws, alone, idx_alone, w8)
    assert moe.moe_get_device_status(ws) == 0, moe.moe_last_error()

    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    side = torch.cuda.Stream()
    out = torch.full((cfg.T, cfg.D), float("nan"), device=dev)
    idx = torch.full((cfg.T, cfg.k), -1, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()
    moe.moe_selftest_occupy(nsm - FREE_SMS, HOLD_CYCLES, side)
    side.query()          # submit the occupier now
    time.sleep(0.05)      # it holds its SMs before the layer is enqueued
    _forward(moe, cfg, inp, d, ws, out, idx, w8)
    done = torch.cuda.Event()
    done.record()
    done.synchronize()
    held_throughout = not side.query()
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0, moe.moe_last_error()
    # the layer ran, and finished, while the occupier held all but FREE_SMS SMs
    assert held_throughout
    # the same tiles with the same arithmetic, whichever CTA ran them
    assert torch.equal(idx, idx_alone)
    assert torch.equal(out.view(torch.int32), alone.view(torch.int32))

    if weights == "bf16":
        experts = HostExperts(inp["W1"], inp["W3"], inp["W2"])
        ref_inp = inp
    else:
        experts = Fp8HostExperts(q)
        ref_inp = dict(inp, **{n: torch.from_numpy(Fp8HostExperts(q).matrix(n, 0))[None]
                               for n in ("Ws1", "Ws3", "Ws2")})
    tokens = np.unique(mi.uniform_int(24, cfg.T, 0, "sample/" + cfg.name).numpy())
    ref, flips, wrong = oracle_rows(ref_inp, cfg, tokens, idx.cpu().numpy()[tokens], experts)
    got = out.cpu().numpy()[tokens].astype(np.float64)
    assert wrong == 0 and flips <= 1
    assert rel_l2(got, ref) <= REL_L2_TOL
    assert np.max(np.abs(got - ref)) <= MAX_ABS_TOL
