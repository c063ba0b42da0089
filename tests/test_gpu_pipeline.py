"""The host-buffer pipeline, through the C ABI: page-locked host input ->
layer -> page-locked host output, with the copies of neighbouring steps on
their own streams.  Every step's output must equal moe_forward's on the same
input bit for bit (same kernels, same arithmetic), whatever the overlap, and
the oracle's within the layer tolerances."""
import ctypes

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


def _pinned_batches(cfg, n, seed0=1):
    """n different seeded hidden batches of the workload, in page-locked host memory."""
    return [mi.hidden(cfg, seed0 + i).contiguous().pin_memory() for i in range(n)]


def _pinned_outputs(cfg, n):
    return [torch.full((cfg.T, cfg.D), float("nan"), dtype=torch.float32).pin_memory()
            for _ in range(n)]


def _bf16_pipeline(moe, cfg, inp):
    return moe.moe_pipeline_create(moe.dims_of(cfg), inp["Wr"], inp["bias"], inp["W1"], inp["W3"],
                                   inp["W2"], inp["Ws1"], inp["Ws3"], inp["Ws2"])


def _forward(moe, cfg, inp, h, fp8=None):
    d = moe.dims_of(cfg)
    ws = moe.alloc_workspace(d)
    out = torch.empty((cfg.T, cfg.D), dtype=torch.float32, device="cuda")
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    if fp8 is None:
        moe.moe_forward(h.cuda(), inp["Wr"], inp["bias"], inp["W1"], inp["W3"], inp["W2"],
                        inp["Ws1"], inp["Ws3"], inp["Ws2"], d, out, ws, idx)
    else:
        moe.moe_forward_fp8(h.cuda(), inp["Wr"], inp["bias"], fp8, d, out, ws, idx)
    assert moe.moe_get_device_status(ws) == 0
    return out.cpu(), idx


@pytest.mark.parametrize("name,steps", [("tiny", 7), ("decode", 5)])
def test_pipeline_matches_forward(moe, name, steps):
    cfg = mi.CONFIGS[name]
    inp = layer_on_device(cfg)
    p = _bf16_pipeline(moe, cfg, inp)
    hs, outs = _pinned_batches(cfg, steps), _pinned_outputs(cfg, steps)
    for h, o in zip(hs, outs):       # all submitted before any wait: both slots are reused
        moe.moe_pipeline_submit(p, h, o)
    moe.moe_pipeline_wait(p)
    moe.moe_pipeline_destroy(p)
    for h, o in zip(hs, outs):
        ref, _ = _forward(moe, cfg, inp, h)
        assert torch.equal(o, ref)


def test_pipeline_against_the_oracle(moe):
    cfg = mi.CONFIGS["tiny"]
    inp = layer_on_device(cfg)
    p = _bf16_pipeline(moe, cfg, inp)
    (h,), (o,) = _pinned_batches(cfg, 1, seed0=3), _pinned_outputs(cfg, 1)
    moe.moe_pipeline_submit(p, h, o)
    moe.moe_pipeline_wait(p)
    _, idx = _forward(moe, cfg, inp, h)
    step = dict(inp)
    step["h"] = h.cuda()
    tokens = np.arange(cfg.T)
    ref, flips, wrong = oracle_rows(step, cfg, tokens, idx.cpu().numpy(),
                                    HostExperts(inp["W1"], inp["W3"], inp["W2"]))
    got = o.numpy().astype(np.float64)
    assert wrong == 0 and flips <= 1
    assert rel_l2(got, ref) <= REL_L2_TOL
    assert np.max(np.abs(got - ref)) <= MAX_ABS_TOL


def test_pipeline_waits_between_submissions(moe):
    cfg = mi.CONFIGS["tiny"]
    inp = layer_on_device(cfg)
    p = _bf16_pipeline(moe, cfg, inp)
    hs, outs = _pinned_batches(cfg, 5, seed0=11), _pinned_outputs(cfg, 5)
    for i, (h, o) in enumerate(zip(hs, outs)):
        moe.moe_pipeline_submit(p, h, o)
        if i in (0, 3):
            moe.moe_pipeline_wait(p)
    moe.moe_pipeline_wait(p)
    for h, o in zip(hs, outs):
        assert torch.equal(o, _forward(moe, cfg, inp, h)[0])


def test_pipeline_fp8(moe):
    cfg = mi.CONFIGS["tiny"]
    inp = layer_on_device(cfg)
    q = mi.fp8_layer_weights(inp)
    w8 = moe.fp8_weights(*(q[n + "q"] for n in ("W1", "W3", "W2", "Ws1", "Ws3", "Ws2")),
                         *(q[n + "e"] for n in ("W1", "W3", "W2", "Ws1", "Ws3", "Ws2")))
    p = moe.moe_pipeline_create(moe.dims_of(cfg), inp["Wr"], inp["bias"], w8=w8, keep=(q,))
    hs, outs = _pinned_batches(cfg, 4, seed0=21), _pinned_outputs(cfg, 4)
    for h, o in zip(hs, outs):
        moe.moe_pipeline_submit(p, h, o)
    moe.moe_pipeline_wait(p)
    moe.moe_pipeline_destroy(p)
    for h, o in zip(hs, outs):
        assert torch.equal(o, _forward(moe, cfg, inp, h, fp8=w8)[0])


def test_pipeline_refuses_pageable_host_memory(moe):
    cfg = mi.CONFIGS["tiny"]
    inp = layer_on_device(cfg)
    p = _bf16_pipeline(moe, cfg, inp)
    h = mi.hidden(cfg, 1).contiguous()                       # pageable
    o = torch.empty((cfg.T, cfg.D), dtype=torch.float32).pin_memory()
    with pytest.raises(ValueError, match="pinned"):
        moe.moe_pipeline_submit(p, h, o)
    rc = moe._lib.moe_pipeline_submit(p.handle, ctypes.c_void_p(h.data_ptr()),
                                      ctypes.c_void_p(o.data_ptr()))
    assert rc == moe.MOE_ERR_INVALID_ARG and "page-locked" in moe.moe_last_error()
    moe.moe_pipeline_destroy(p)


def test_pipeline_empty_batch(moe):
    cfg = mi.custom_config("tiny", T=0)
    inp = layer_on_device(mi.CONFIGS["tiny"])
    p = moe.moe_pipeline_create(moe.dims_of(cfg), inp["Wr"], inp["bias"], inp["W1"], inp["W3"],
                                inp["W2"], inp["Ws1"], inp["Ws3"], inp["Ws2"])
    h = torch.empty((0, cfg.D), dtype=torch.bfloat16).pin_memory()
    o = torch.empty((0, cfg.D), dtype=torch.float32).pin_memory()
    moe.moe_pipeline_submit(p, h, o)
    moe.moe_pipeline_wait(p)
    moe.moe_pipeline_destroy(p)
