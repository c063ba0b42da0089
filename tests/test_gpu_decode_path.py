"""The small-batch paths of moe_forward, against the oracle on every token.

* T <= 128 with bf16 weights: the router kernel that splits the fp32 router
  weight in shared memory (D % 64 == 0, E % 64 == 0), routing that only sets
  each token's bit in the rows of its experts, and an FFN that derives the
  groups from those bits and records inv; with the shared expert's FFN in the
  same launch and on the internal stream beside the routing.
* 128 < T <= 256: the routing kernel's last block groups the pairs from the
  bits.

Each case also checks the layer's routing statistics against the grouping of
the indices it returned, and that a second call on the same workspace gives
the same bits (the bits, counters and tickets are left clear for it).
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from tests.gpu_helpers import (MAX_ABS_TOL, REL_L2_TOL, HostExperts, layer_on_device, oracle_rows,
                               rel_l2)

pytestmark = pytest.mark.gpu

CASES = {
    "decode_T1": mi.custom_config("decode", T=1, D=512, E=64, k=6, F=256, S=1, Fs=256,
                                  hidden_std=1.0, name="dp_T1"),
    "decode_T77": mi.custom_config("decode", T=77, D=512, E=64, k=6, F=256, S=1, Fs=256,
                                   hidden_std=1.0, name="dp_T77"),
    "decode_T128_no_shared": mi.custom_config("decode", T=128, D=512, E=128, k=8, F=256, S=0,
                                              Fs=256, hidden_std=1.0, name="dp_T128s0"),
    # 3 * 2048 * 2048 * 2 bytes of shared weights: the shared FFN runs beside the routing
    "decode_T128_overlap": mi.custom_config("decode", T=128, D=2048, E=64, k=8, F=512, S=1,
                                            Fs=2048, hidden_std=1.0, name="dp_T128ov"),
    "grouped_T200": mi.custom_config("decode", T=200, D=512, E=128, k=8, F=256, S=1, Fs=256,
                                     hidden_std=1.0, name="dp_T200"),
}


@pytest.fixture(scope="module")
def moe():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import sparse_moe_layer_04_b200 as m
    return m


def _forward(moe, cfg, inp, d, ws):
    out = torch.empty((cfg.T, cfg.D), dtype=torch.float32, device="cuda")
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    w = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device="cuda")
    moe.moe_forward(inp["h"], inp["Wr"], inp["bias"], inp["W1"], inp["W3"], inp["W2"], inp["Ws1"],
                    inp["Ws3"], inp["Ws2"], d, out, ws, idx, w)
    assert moe.moe_get_device_status(ws) == 0, moe.moe_last_error()
    return out, idx, w


@pytest.mark.parametrize("name", list(CASES))
def test_small_batch_path(moe, name):
    cfg = CASES[name]
    inp = layer_on_device(cfg)
    d = moe.dims_of(cfg)
    ws = moe.alloc_workspace(d)
    out, idx, w = _forward(moe, cfg, inp, d, ws)

    tokens = np.arange(cfg.T)
    experts = HostExperts(inp["W1"], inp["W3"], inp["W2"])
    ref, flips, wrong = oracle_rows(inp, cfg, tokens, idx.cpu().numpy(), experts)
    got = out.cpu().numpy().astype(np.float64)
    assert wrong == 0
    assert flips <= max(1, 0.02 * cfg.T)
    assert rel_l2(got, ref) <= REL_L2_TOL
    assert np.max(np.abs(got - ref)) <= MAX_ABS_TOL

    # routing statistics: those of the returned indices
    counts = np.bincount(idx.cpu().numpy().reshape(-1), minlength=cfg.E)
    assert np.array_equal(moe.moe_ws_expert_counts(ws, d).cpu().numpy(), counts)
    assert int(moe.moe_ws_touched_experts(ws, d).item()) == int((counts > 0).sum())

    # the same call again on the same workspace: the same bits
    out2, idx2, w2 = _forward(moe, cfg, inp, d, ws)
    assert torch.equal(idx2, idx)
    assert torch.equal(w2.view(torch.int32), w.view(torch.int32))
    assert torch.equal(out2.view(torch.int32), out.view(torch.int32))
