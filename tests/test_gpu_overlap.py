"""The shared experts' FFN beside the routing (moe_forward with bf16 weights,
T <= 512, shared weights >= 16 MiB): it runs on an internal stream and the
routed FFN launch carries the routed experts only.  Its output must equal,
bit for bit, the same layer composed from the single-step entry points (one
FFN launch over all groups), and the oracle's within the layer tolerances."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from tests.gpu_helpers import (MAX_ABS_TOL, REL_L2_TOL, HostExperts, layer_on_device, oracle_rows,
                               rel_l2)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import sparse_moe_layer_04_b200 as m
    return m


CASES = {
    "decode": mi.CONFIGS["decode"],
    # ragged: 300 tokens, two shared experts of width 2048 (48 MiB), k = 6 of 64
    "ragged_two_shared": mi.custom_config("decode", T=300, D=2048, E=64, k=6, F=1024, S=2,
                                          Fs=2048, name="ragged_two_shared"),
}


def _composed(moe, cfg, inp):
    """The layer from the single-step entry points, one FFN launch over all groups."""
    d = moe.dims_of(cfg)
    ws = moe.alloc_workspace(d)
    T, E, k, D = cfg.T, cfg.E, cfg.k, cfg.D
    dev = "cuda"
    logits = torch.empty((T, E), device=dev)
    moe.moe_router_logits(inp["h"], inp["Wr"], d, logits, ws)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), device=dev)
    moe.moe_route(logits, inp["bias"], d, idx, w, ws)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(T * k, dtype=torch.int32, device=dev)
    inv = torch.empty((T, k), dtype=torch.int32, device=dev)
    moe.moe_permute(idx, d, counts, offsets, perm, inv, ws)
    y = torch.empty((T * k + cfg.S * T, D), device=dev)
    moe.moe_expert_ffn(inp["h"], perm, offsets, inp["W1"], inp["W3"], inp["W2"], inp["Ws1"],
                       inp["Ws3"], inp["Ws2"], d, y, ws)
    out = torch.empty((T, D), device=dev)
    moe.moe_combine(y, w, inv, d, out, ws)
    assert moe.moe_get_device_status(ws) == 0
    return out, idx


@pytest.mark.parametrize("name", list(CASES))
def test_overlapped_forward_equals_composed_layer(moe, name):
    cfg = CASES[name]
    d = moe.dims_of(cfg)
    assert moe.moe_forward_shared_overlap(d)
    inp = layer_on_device(cfg)
    ws = moe.alloc_workspace(d)
    out = torch.empty((cfg.T, cfg.D), device="cuda")
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    for _ in range(2):   # the second call reuses the internal stream and the workspace
        moe.moe_forward(inp["h"], inp["Wr"], inp["bias"], inp["W1"], inp["W3"], inp["W2"],
                        inp["Ws1"], inp["Ws3"], inp["Ws2"], d, out, ws, idx)
    assert moe.moe_get_device_status(ws) == 0
    ref, ref_idx = _composed(moe, cfg, inp)
    assert torch.equal(idx, ref_idx)
    assert torch.equal(out.view(torch.int32), ref.view(torch.int32))
    if name != "decode":   # the decode layer is pinned to the oracle in the parity suite
        tokens = np.unique(mi.uniform_int(24, cfg.T, 0, "sample/" + name).numpy())
        r, flips, wrong = oracle_rows(inp, cfg, tokens, idx.cpu().numpy()[tokens],
                                      HostExperts(inp["W1"], inp["W3"], inp["W2"]))
        got = out.cpu().numpy()[tokens].astype(np.float64)
        assert wrong == 0 and flips <= 1
        assert rel_l2(got, r) <= REL_L2_TOL
        assert np.max(np.abs(got - r)) <= MAX_ABS_TOL


def test_overlapped_forward_in_a_cuda_graph(moe):
    cfg = CASES["decode"]
    d = moe.dims_of(cfg)
    inp = layer_on_device(cfg)
    ws = moe.alloc_workspace(d)
    out = torch.empty((cfg.T, cfg.D), device="cuda")
    ref = torch.empty_like(out)
    args = (inp["h"], inp["Wr"], inp["bias"], inp["W1"], inp["W3"], inp["W2"], inp["Ws1"],
            inp["Ws3"], inp["Ws2"], d)
    moe.moe_forward(*args, ref, ws)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        moe.moe_forward(*args, out, ws)          # warm-up on the capture stream
        torch.cuda.current_stream().synchronize()
        with torch.cuda.graph(g, stream=s):
            moe.moe_forward(*args, out, ws)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    assert torch.equal(out.view(torch.int32), ref.view(torch.int32))
