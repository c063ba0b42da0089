"""FP8 weights: the oracle's E4M3 decoding against torch's float8 cast, and
the block quantization of the shared input generator against its contract."""
import numpy as np
import torch

import moe_inputs as mi
from oracle import moe_oracle as orc


def test_e4m3_definition_matches_torch_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    got = orc.e4m3_value(codes)
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got)) and nan.sum() == 2      # 0x7F and 0xFF
    assert np.array_equal(got[~nan], ref[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x38] == 1.0


def test_block_quantization_contract():
    g = torch.Generator().manual_seed(3)
    w = (torch.randn(300, 200, generator=g) * 0.05).to(torch.bfloat16)
    w[128:256, 128:200] = 0                       # an all-zero block
    w[5, 7] = 3.0                                 # a block with a large entry
    codes, exps = mi.quantize_fp8_blocks(w)
    assert codes.shape == (300, 200) and codes.dtype == torch.uint8
    assert exps.shape == (3, 2) and exps.dtype == torch.int8
    deq = orc.dequantize_fp8_blocks(codes.numpy(), exps.numpy())
    wf = w.float().numpy().astype(np.float64)
    assert np.all(np.isfinite(deq))
    for rb in range(3):
        for kb in range(2):
            blk = np.s_[rb * 128:(rb + 1) * 128, kb * 128:(kb + 1) * 128]
            amax = np.abs(wf[blk]).max()
            e = int(exps[rb, kb])
            if amax == 0:
                assert e == 0 and np.all(deq[blk] == 0)
                continue
            assert amax <= 448.0 * 2.0 ** e and amax > 448.0 * 2.0 ** (e - 1)   # smallest e
            # round to nearest: error at most half an E4M3 step (2^-4 relative, or
            # half the subnormal step 2^-10 * 2^e)
            err = np.abs(deq[blk] - wf[blk])
            assert np.all(err <= np.maximum(np.abs(wf[blk]) * 2.0 ** -4, 2.0 ** (e - 10)))
    # the dequantized weights are exact bf16 values
    assert np.array_equal(torch.from_numpy(deq).to(torch.bfloat16).double().numpy(), deq)


def test_fp8_layer_weights_shapes():
    cfg = mi.CONFIGS["tiny"]
    q = mi.fp8_layer_weights(mi.layer_weights(cfg))
    assert q["W1q"].shape == (cfg.E, cfg.F, cfg.D) and q["W1e"].shape == (cfg.E, 1, 1)
    assert q["W2q"].shape == (cfg.E, cfg.D, cfg.F) and q["Ws2e"].shape == (cfg.S, 1, 1)


def test_dequantize_worked_example():
    """Values written out by hand from the E4M3 definition: 0x38 = 1.0,
    0x40 = 2.0, 0x7E = 448, 0x01 = 2^-9 (smallest subnormal), 0x08 = 2^-6
    (smallest normal), 0xB8 = -1.0, 0x80 = -0.0, each times 2^e of its block."""
    codes = np.zeros((130, 144), np.uint8)
    codes[0, :7] = [0x38, 0x40, 0x7E, 0x01, 0x08, 0xB8, 0x80]
    codes[129, 130] = 0x39              # 1.125, row block 1, K block 1
    codes[5, 140] = 0x30                # 0.5, row block 0, K block 1
    exps = np.array([[-12, 3], [0, -117]], np.int8)
    got = orc.dequantize_fp8_blocks(codes, exps)
    s = 2.0 ** -12
    assert list(got[0, :7]) == [s, 2 * s, 448 * s, 2.0 ** -9 * s, 2.0 ** -6 * s, -s, 0.0]
    assert np.signbit(got[0, 6])
    assert got[129, 130] == 1.125 * 2.0 ** -117
    assert got[5, 140] == 0.5 * 8
    assert np.count_nonzero(got) == 8
