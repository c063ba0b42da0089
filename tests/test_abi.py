"""The C ABI: the library loads, exports every declared entry point, and its
host-side argument checks reject bad calls before touching the device.

Only calls that must fail validation are made here (null or misaligned
pointers, bad dimensions, short workspaces), so nothing is ever launched and
no fake pointer is dereferenced, with or without a GPU.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


@pytest.fixture(scope="module")
def mod():
    import __graft_entry__
    __graft_entry__._build_module().build()   # no-op unless a source is newer
    import sparse_moe_layer_04_b200 as m
    return m


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(mod):
    names = _declared_functions()
    assert "moe_forward" in names and "moe_route" in names
    lib = ctypes.CDLL(mod.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_workspace_size(mod):
    d = mod.dims(T=128, D=6144, E=256, F=2048, k=8, S=1, Fs=2048, scale=2.5)
    n = mod.moe_workspace_size(d)
    # at least the fp32 expert outputs and the gathered rows
    assert n >= (128 * 8 + 128) * 6144 * 4 + 128 * 8 * 6144 * 2
    assert n % 256 == 0
    assert mod._lib.moe_workspace_size(ctypes.byref(mod.dims(T=4, D=12, E=8, F=64, k=2))) == 0
    assert mod._lib.moe_workspace_size(ctypes.byref(mod.dims(T=4, D=128, E=8, F=64, k=9))) == 0
    assert mod._lib.moe_workspace_size(ctypes.byref(mod.dims(T=-1, D=128, E=8, F=64, k=2))) == 0
    assert mod._lib.moe_workspace_size(ctypes.byref(mod.dims(T=4, D=128, E=2000, F=64, k=2))) == 0
    assert mod._lib.moe_workspace_size(ctypes.byref(mod.dims(T=4, D=128, E=64, F=64, k=33))) == 0
    assert mod._lib.moe_workspace_size(ctypes.byref(mod.dims(T=0, D=128, E=8, F=64, k=2))) > 0


FAKE = 0x7F0000000000  # never dereferenced: every call below fails validation first


def test_null_and_misaligned_pointers_rejected(mod):
    lib = mod._lib
    d = mod.dims(T=8, D=128, E=8, F=64, k=2)
    ws_n = mod.moe_workspace_size(d)
    rc = lib.moe_forward(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.byref(d),
                         FAKE, None, None, FAKE, ws_n, None)
    assert rc == mod.MOE_ERR_INVALID_ARG and "h is NULL" in mod.moe_last_error()
    rc = lib.moe_forward(FAKE + 4, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.byref(d),
                         FAKE, None, None, FAKE, ws_n, None)
    assert rc == mod.MOE_ERR_INVALID_ARG and "aligned" in mod.moe_last_error()
    rc = lib.moe_route(FAKE, None, ctypes.byref(d), FAKE, FAKE, None, None)
    assert rc == mod.MOE_ERR_INVALID_ARG and "bias" in mod.moe_last_error()
    rc = lib.moe_combine(FAKE, FAKE, None, ctypes.byref(d), FAKE, None, None)
    assert rc == mod.MOE_ERR_INVALID_ARG and "inv" in mod.moe_last_error()
    # shared weights are required when S > 0
    rc = lib.moe_expert_ffn(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, ctypes.byref(d),
                            FAKE, FAKE, ws_n, None)
    assert rc == mod.MOE_ERR_INVALID_ARG and "Ws1" in mod.moe_last_error()


def test_workspace_checks(mod):
    lib = mod._lib
    d = mod.dims(T=8, D=128, E=8, F=64, k=2)
    ws_n = mod.moe_workspace_size(d)
    args = [FAKE] * 9
    rc = lib.moe_forward(*args, ctypes.byref(d), FAKE, None, None, FAKE, ws_n - 256, None)
    assert rc == mod.MOE_ERR_WORKSPACE and "needs" in mod.moe_last_error()
    rc = lib.moe_forward(*args, ctypes.byref(d), FAKE, None, None, None, ws_n, None)
    assert rc == mod.MOE_ERR_WORKSPACE
    rc = lib.moe_forward(*args, ctypes.byref(d), FAKE, None, None, FAKE + 16, ws_n, None)
    assert rc == mod.MOE_ERR_WORKSPACE and "256-byte" in mod.moe_last_error()
    rc = lib.moe_permute(FAKE, ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, 100, None)
    assert rc == mod.MOE_ERR_WORKSPACE


def test_bad_dims_rejected(mod):
    lib = mod._lib
    for bad in (dict(T=8, D=100, E=8, F=64, k=2), dict(T=8, D=128, E=8, F=60, k=2),
                dict(T=8, D=128, E=8, F=64, k=0), dict(T=8, D=128, E=0, F=64, k=1),
                dict(T=8, D=128, E=8, F=64, k=2, S=1, Fs=4)):
        d = mod.dims(**bad)
        rc = lib.moe_forward(*([FAKE] * 9), ctypes.byref(d), FAKE, None, None, FAKE, 1 << 40, None)
        assert rc == mod.MOE_ERR_INVALID_ARG, bad
    d = mod.dims(T=8, D=128, E=8, F=64, k=2, scale=float("nan"))
    rc = lib.moe_route(FAKE, FAKE, ctypes.byref(d), FAKE, FAKE, None, None)
    assert rc == mod.MOE_ERR_INVALID_ARG and "scale" in mod.moe_last_error()
    rc = lib.moe_route(FAKE, FAKE, None, FAKE, FAKE, None, None)
    assert rc == mod.MOE_ERR_INVALID_ARG


def test_grouped_route_argument_checks(mod):
    lib = mod._lib
    d = mod.dims(T=8, D=128, E=12, F=64, k=4)
    for n_group, topk_group in [(5, 1), (0, 1), (33, 1), (4, 5), (4, 0), (6, 1)]:
        rc = lib.moe_route_grouped(FAKE, FAKE, ctypes.byref(d), n_group, topk_group, FAKE, FAKE,
                                   None, None)
        assert rc == mod.MOE_ERR_INVALID_ARG, (n_group, topk_group)


def test_binding_names_match_the_abi(mod):
    for n in _declared_functions():
        assert hasattr(mod, n), n


def _w8(mod, **over):
    w = mod.moe_fp8_weights_t()
    for n in ("W1", "W3", "W2", "Ws1", "Ws3", "Ws2", "W1e", "W3e", "W2e", "Ws1e", "Ws3e", "Ws2e"):
        setattr(w, n, over.get(n, FAKE))
    return w


def test_fp8_argument_checks(mod):
    lib = mod._lib
    d = mod.dims(T=8, D=128, E=8, F=64, k=2)
    ws_n = mod.moe_workspace_size(d)
    ok = _w8(mod)
    # D, F, Fs must be multiples of 16 for FP8 rows (TMA strides)
    for bad in (dict(D=136), dict(F=72), dict(Fs=40)):
        db = mod.dims(**{**dict(T=8, D=128, E=8, F=64, k=2), **bad})
        rc = lib.moe_expert_ffn_fp8(FAKE, FAKE, FAKE, ctypes.byref(ok), ctypes.byref(db), FAKE,
                                    FAKE, 1 << 40, None)
        assert rc == mod.MOE_ERR_INVALID_ARG and "multiple of 16" in mod.moe_last_error(), bad
    rc = lib.moe_expert_ffn_fp8(FAKE, FAKE, FAKE, None, ctypes.byref(d), FAKE, FAKE, ws_n, None)
    assert rc == mod.MOE_ERR_INVALID_ARG and "w8" in mod.moe_last_error()
    rc = lib.moe_expert_ffn_fp8(FAKE, FAKE, FAKE, ctypes.byref(_w8(mod, W2e=None)), ctypes.byref(d),
                                FAKE, FAKE, ws_n, None)
    assert rc == mod.MOE_ERR_INVALID_ARG and "W2e" in mod.moe_last_error()
    rc = lib.moe_expert_ffn_fp8(FAKE, FAKE, FAKE, ctypes.byref(_w8(mod, W3=FAKE + 8)),
                                ctypes.byref(d), FAKE, FAKE, ws_n, None)
    assert rc == mod.MOE_ERR_INVALID_ARG and "aligned" in mod.moe_last_error()
    rc = lib.moe_expert_ffn_fp8(FAKE, FAKE, FAKE, ctypes.byref(_w8(mod, Ws2e=None)),
                                ctypes.byref(d), FAKE, FAKE, ws_n, None)
    assert rc == mod.MOE_ERR_INVALID_ARG and "Ws" in mod.moe_last_error()
    # S = 0: shared members may be NULL (then the workspace check is reached)
    d0 = mod.dims(T=8, D=128, E=8, F=64, k=2, S=0, Fs=8)
    rc = lib.moe_expert_ffn_fp8(FAKE, FAKE, FAKE,
                                ctypes.byref(_w8(mod, Ws1=None, Ws3=None, Ws2=None, Ws1e=None,
                                                 Ws3e=None, Ws2e=None)),
                                ctypes.byref(d0), FAKE, FAKE, 0, None)
    assert rc == mod.MOE_ERR_WORKSPACE
    rc = lib.moe_forward_fp8(FAKE, FAKE, None, ctypes.byref(ok), ctypes.byref(d), FAKE, None, None,
                             FAKE, ws_n, None)
    assert rc == mod.MOE_ERR_INVALID_ARG and "bias" in mod.moe_last_error()
    rc = lib.moe_forward_fp8(FAKE, FAKE, FAKE, ctypes.byref(ok), ctypes.byref(d), FAKE, None, None,
                             FAKE, ws_n - 256, None)
    assert rc == mod.MOE_ERR_WORKSPACE
    # T = 0 is a no-op that launches nothing
    dz = mod.dims(T=0, D=128, E=8, F=64, k=2)
    assert lib.moe_forward_fp8(None, None, None, None, ctypes.byref(dz), None, None, None, None, 0,
                               None) == mod.MOE_OK


def test_fp8_dequantize_argument_checks(mod):
    lib = mod._lib
    assert lib.moe_fp8_dequantize(FAKE, FAKE, 1, 4, 24, FAKE, None, None) == mod.MOE_ERR_INVALID_ARG
    assert "multiple of 16" in mod.moe_last_error()
    assert lib.moe_fp8_dequantize(FAKE, FAKE, -1, 4, 16, FAKE, None, None) == mod.MOE_ERR_INVALID_ARG
    assert lib.moe_fp8_dequantize(FAKE, None, 1, 4, 16, FAKE, None, None) == mod.MOE_ERR_INVALID_ARG
    assert lib.moe_fp8_dequantize(FAKE + 1, FAKE, 1, 4, 16, FAKE, None, None) == mod.MOE_ERR_INVALID_ARG
    assert lib.moe_fp8_dequantize(FAKE, FAKE, 1, 4, 16, FAKE, FAKE + 16, None) == mod.MOE_ERR_WORKSPACE
    assert lib.moe_fp8_dequantize(None, None, 0, 4, 16, None, None, None) == mod.MOE_OK


def test_gather_rows_argument_checks(mod):
    lib = mod._lib
    assert lib.moe_gather_rows(FAKE, 10, FAKE, 4, 24, FAKE, None, None) == mod.MOE_ERR_INVALID_ARG
    assert "multiple of 16" in mod.moe_last_error()
    assert lib.moe_gather_rows(FAKE, -1, FAKE, 4, 32, FAKE, None, None) == mod.MOE_ERR_INVALID_ARG
    assert lib.moe_gather_rows(FAKE + 8, 10, FAKE, 4, 32, FAKE, None, None) == mod.MOE_ERR_INVALID_ARG
    assert lib.moe_gather_rows(FAKE, 10, None, 4, 32, FAKE, None, None) == mod.MOE_ERR_INVALID_ARG
    assert lib.moe_gather_rows(FAKE, 10, FAKE, 4, 32, FAKE, FAKE + 16, None) == mod.MOE_ERR_WORKSPACE
    assert lib.moe_gather_rows(None, 0, None, 0, 32, None, None, None) == mod.MOE_OK


def test_pipeline_argument_checks(mod):
    lib = mod._lib
    d = mod.dims(T=8, D=128, E=8, F=64, k=2)

    def a256(x):
        return (x + 255) // 256 * 256

    need = mod.moe_pipeline_device_bytes(d)
    assert need == 2 * a256(8 * 128 * 2) + 2 * a256(8 * 128 * 4) + a256(mod.moe_workspace_size(d))
    assert lib.moe_pipeline_device_bytes(ctypes.byref(mod.dims(T=4, D=12, E=8, F=64, k=2))) == 0
    h = ctypes.c_void_p(FAKE)
    P = ctypes.c_void_p

    def create(dd, Wr=FAKE, W1=FAKE, w8=None, dev=FAKE, n=None, out=True):
        handle = ctypes.c_void_p(FAKE)
        rc = lib.moe_pipeline_create(ctypes.byref(dd), Wr, FAKE, W1, FAKE, FAKE, FAKE, FAKE, FAKE,
                                     w8, dev, need if n is None else n, None,
                                     ctypes.byref(handle) if out else None)
        if out:
            assert handle.value is None   # cleared on failure
        return rc, mod.moe_last_error()

    rc, msg = create(d, out=False)
    assert rc == mod.MOE_ERR_INVALID_ARG and "out is NULL" in msg
    rc, msg = create(d, Wr=None)
    assert rc == mod.MOE_ERR_INVALID_ARG and "Wr" in msg
    rc, msg = create(d, W1=None)
    assert rc == mod.MOE_ERR_INVALID_ARG and "W1" in msg
    rc, msg = create(d, dev=None)
    assert rc == mod.MOE_ERR_WORKSPACE and "dev is NULL" in msg
    rc, msg = create(d, dev=FAKE + 16)
    assert rc == mod.MOE_ERR_WORKSPACE and "256-byte" in msg
    rc, msg = create(d, n=need - 1)
    assert rc == mod.MOE_ERR_WORKSPACE and "needs" in msg
    rc, msg = create(mod.dims(T=8, D=128, E=8, F=64, k=9))
    assert rc == mod.MOE_ERR_INVALID_ARG
    # FP8 weights: the bf16 pointers are ignored, the FP8 rules apply
    w8 = mod.moe_fp8_weights_t()
    rc, msg = create(d, w8=ctypes.byref(w8))          # bf16 W1 given, w8->W1 NULL
    assert rc == mod.MOE_ERR_INVALID_ARG and "W1 is NULL" in msg
    d24 = mod.dims(T=8, D=136, E=8, F=64, k=2)
    rc, msg = create(d24, W1=None, w8=ctypes.byref(w8))
    assert rc == mod.MOE_ERR_INVALID_ARG and "multiple of 16" in msg

    assert lib.moe_pipeline_submit(None, h, h) == mod.MOE_ERR_INVALID_ARG
    assert "pipeline is NULL" in mod.moe_last_error()
    assert lib.moe_pipeline_wait(None) == mod.MOE_ERR_INVALID_ARG
    assert lib.moe_pipeline_destroy(None) == mod.MOE_OK


def test_pipeline_binding_checks_host_tensors(mod):
    import torch
    d = mod.dims(T=2, D=16, E=8, F=16, k=2)
    p = mod.MoePipeline(ctypes.c_void_p(None), d, ())
    with pytest.raises(ValueError, match="T x D"):
        mod.moe_pipeline_submit(p, torch.zeros(3, 16, dtype=torch.bfloat16),
                                torch.zeros(2, 16, dtype=torch.float32))
    with pytest.raises((ValueError, RuntimeError)):
        # pageable (or, without a GPU, unpinnable) host memory is refused
        mod.moe_pipeline_submit(p, torch.zeros(2, 16, dtype=torch.bfloat16),
                                torch.zeros(2, 16, dtype=torch.float32))


def test_shared_overlap_rule(mod):
    f = mod.moe_forward_shared_overlap
    assert f(mod.dims(T=128, D=6144, E=256, F=2048, k=8, S=1))
    assert f(mod.dims(T=512, D=4096, E=8, F=64, k=2, S=1, Fs=1408))     # 33 MiB shared
    assert not f(mod.dims(T=128, D=6144, E=256, F=2048, k=8, S=1), fp8_weights=True)
    assert not f(mod.dims(T=513, D=6144, E=8, F=64, k=2, S=1, Fs=2048))
    assert not f(mod.dims(T=128, D=6144, E=8, F=64, k=2, S=0))
    assert not f(mod.dims(T=0, D=6144, E=8, F=64, k=2, S=1, Fs=2048))
    assert not f(mod.dims(T=64, D=128, E=8, F=64, k=2, S=1))           # 48 KiB shared
    assert not f(mod.dims(T=128, D=12, E=8, F=64, k=2, S=1))           # invalid dims
