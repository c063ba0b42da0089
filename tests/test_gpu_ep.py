"""Expert parallelism on the GPU at world size 1 (the only GPU count this
build has): sparse_moe_layer_04_b200.ep with the library's kernels and NCCL
collectives of one rank.  The layer must match the oracle like moe_forward
does, with routing identical to moe_forward's.  The exchange between several
ranks is checked on the CPU (tests/test_ep_gloo.py)."""
import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist

import moe_inputs as mi
from tests.gpu_helpers import (MAX_ABS_TOL, REL_L2_TOL, HostExperts, layer_on_device,
                               oracle_rows, rel_l2)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nccl_one_rank():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=timedelta(seconds=120), device_id=torch.device("cuda", 0))
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("T,D,E,F,k,S", [(64, 128, 8, 64, 2, 1), (300, 256, 16, 128, 4, 1),
                                         (700, 256, 12, 192, 3, 0), (1, 128, 4, 64, 4, 1)])
def test_ep_one_rank_matches_oracle_and_moe_forward(nccl_one_rank, T, D, E, F, k, S):
    import sparse_moe_layer_04_b200 as moe
    from sparse_moe_layer_04_b200 import ep
    cfg = mi.LayerConfig("ep1", T, D, E, k, F, S, F, 2.5, 1.0, f"ep1_{T}x{D}x{E}")
    inp = layer_on_device(cfg)
    d = moe.dims_of(cfg)
    sh = (inp["Ws1"], inp["Ws3"], inp["Ws2"]) if S else (None, None, None)
    out, idx, w = ep.ep_forward(inp["h"], inp["Wr"], inp["bias"], inp["W1"], inp["W3"], inp["W2"],
                                *sh, d)
    torch.cuda.synchronize()
    # routing: the same kernels as moe_forward, bit for bit
    ws = moe.alloc_workspace(d)
    o2 = torch.empty_like(out)
    i2 = torch.empty_like(idx)
    w2 = torch.empty_like(w)
    if S == 0:
        moe.moe_forward(inp["h"], inp["Wr"], inp["bias"], inp["W1"], inp["W3"], inp["W2"], None,
                        None, None, d, o2, ws, i2, w2)
    else:
        moe.moe_forward(inp["h"], inp["Wr"], inp["bias"], inp["W1"], inp["W3"], inp["W2"],
                        inp["Ws1"], inp["Ws3"], inp["Ws2"], d, o2, ws, i2, w2)
    assert torch.equal(idx, i2) and torch.equal(w.view(torch.int32), w2.view(torch.int32))
    assert moe.moe_get_device_status(ws) == 0
    # the layer against the oracle on the same inputs
    if S == 0:
        inp["Ws1"] = torch.empty((0, 8, D), dtype=torch.bfloat16, device="cuda")
        inp["Ws3"] = inp["Ws1"]
        inp["Ws2"] = torch.empty((0, D, 8), dtype=torch.bfloat16, device="cuda")
    tokens = np.arange(T)
    ref, flips, wrong = oracle_rows(inp, cfg, tokens, idx.cpu().numpy(),
                                    HostExperts(inp["W1"], inp["W3"], inp["W2"]))
    got = out.cpu().numpy().astype(np.float64)
    assert wrong == 0 and flips <= max(1, T // 50)
    assert rel_l2(got, ref) <= REL_L2_TOL
    assert np.max(np.abs(got - ref)) <= MAX_ABS_TOL
    # and close to moe_forward (the expert GEMMs tile the rows differently)
    assert rel_l2(got, o2.cpu().numpy().astype(np.float64)) < 2e-3


def test_gather_rows_bit_exact_and_bounds(nccl_one_rank):
    import sparse_moe_layer_04_b200 as moe
    src = torch.randn(50, 96, device="cuda").to(torch.bfloat16)
    idx = torch.tensor([3, 0, 49, 3, 17], dtype=torch.int32, device="cuda")
    dst = torch.empty(5, 96, dtype=torch.bfloat16, device="cuda")
    d = moe.dims(T=1, D=128, E=8, F=64, k=2)
    ws = moe.alloc_workspace(d)
    moe.moe_gather_rows(src, idx, dst, ws)
    assert torch.equal(dst, src[idx.long()])
    assert moe.moe_get_device_status(ws) == 0
    src32 = torch.randn(10, 12, device="cuda")
    bad = torch.tensor([1, 10, -1], dtype=torch.int32, device="cuda")
    dst32 = torch.full((3, 12), 7.0, device="cuda")
    moe.moe_gather_rows(src32, bad, dst32, ws)
    assert moe.moe_get_device_status(ws) == moe.MOE_ERR_BOUNDS
    assert torch.equal(dst32[0], src32[1]) and not dst32[1:].any()
