"""Metamorphic properties of the CUDA path, bit for bit.  Every step's
arithmetic for one token is independent of where the token sits in the batch
(router and FFN dot products run over K in a fixed order whatever the row,
routing and merge are per token), and of the experts' labels (the selection
order is by key; the merge follows it).  So permuting the tokens permutes the
output, and relabelling the experts (router rows, bias and weights moved
together) leaves it unchanged, exactly, absent exact key ties."""
import pytest
import torch

import moe_inputs as mi
from tests.gpu_helpers import layer_on_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import sparse_moe_layer_04_b200 as m
    return m


def _forward(moe, cfg, inp, h, fp8=None):
    d = moe.dims_of(cfg)
    ws = moe.alloc_workspace(d)
    out = torch.empty((cfg.T, cfg.D), device="cuda")
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    if fp8 is None:
        moe.moe_forward(h.contiguous(), inp["Wr"], inp["bias"], inp["W1"], inp["W3"], inp["W2"],
                        inp["Ws1"], inp["Ws3"], inp["Ws2"], d, out, ws, idx)
    else:
        moe.moe_forward_fp8(h.contiguous(), inp["Wr"], inp["bias"], fp8, d, out, ws, idx)
    assert moe.moe_get_device_status(ws) == 0
    return out, idx


CASES = {
    # decode layer: shared expert beside the routing, grouping in the routing kernel
    "decode": mi.CONFIGS["decode"],
    # 700 tokens: single FFN launch, multi-block grouping, 256-wide tiles
    "mid700": mi.custom_config("decode", T=700, D=1024, E=32, k=4, F=512, S=1, Fs=512,
                               hidden_std=1.0, name="mid700"),
}


def _perm(T, name):
    return torch.argsort(mi.hash_u32(T, 0, "perm/" + name).to(torch.int64)).cuda()


@pytest.mark.parametrize("name", list(CASES))
def test_token_permutation_permutes_the_output(moe, name):
    cfg = CASES[name]
    inp = layer_on_device(cfg)
    p = _perm(cfg.T, name)
    out, idx = _forward(moe, cfg, inp, inp["h"])
    out_p, idx_p = _forward(moe, cfg, inp, inp["h"][p])
    assert torch.equal(idx_p, idx[p])
    assert torch.equal(out_p.view(torch.int32), out[p].view(torch.int32))


def test_token_permutation_fp8(moe):
    cfg = mi.custom_config("decode", T=200, D=512, E=16, k=4, F=256, S=1, Fs=256, hidden_std=1.0,
                           name="fp8_200")
    inp = layer_on_device(cfg)
    q = mi.fp8_layer_weights(inp)
    w8 = moe.fp8_weights(*(q[n + "q"] for n in ("W1", "W3", "W2", "Ws1", "Ws3", "Ws2")),
                         *(q[n + "e"] for n in ("W1", "W3", "W2", "Ws1", "Ws3", "Ws2")))
    p = _perm(cfg.T, "fp8_200")
    out, _ = _forward(moe, cfg, inp, inp["h"], fp8=w8)
    out_p, _ = _forward(moe, cfg, inp, inp["h"][p], fp8=w8)
    assert torch.equal(out_p.view(torch.int32), out[p].view(torch.int32))


def test_expert_relabelling_leaves_the_output_unchanged(moe):
    cfg = mi.custom_config("decode", T=300, D=1024, E=32, k=4, F=512, S=1, Fs=512, hidden_std=1.0,
                           name="relabel300")
    inp = layer_on_device(cfg)
    r = _perm(cfg.E, "relabel")          # new label i holds old expert r[i]
    moved = dict(inp)
    for n in ("Wr", "bias", "W1", "W3", "W2"):
        moved[n] = inp[n][r].contiguous()
    out, idx = _forward(moe, cfg, inp, inp["h"])
    out_m, idx_m = _forward(moe, cfg, moved, inp["h"])
    assert torch.equal(r[idx_m.long()], idx.long())
    assert torch.equal(out_m.view(torch.int32), out.view(torch.int32))
