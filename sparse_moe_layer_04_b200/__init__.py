"""Python binding of libmoe_b200.so, the B200 (sm_100a) GLM-5.2 MoE-layer forward.

Argument marshalling only: every function here checks dtypes, shapes and
devices of torch tensors, passes their device pointers and the current CUDA
stream to the C ABI of the same name (``include/moe_b200.h``) and raises on a
non-zero return code.  Every step of the layer runs in the library's CUDA
kernels; there is no fallback.  If the library is missing the import fails.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED = -2
MOE_ERR_CUDA = -3
MOE_ERR_WORKSPACE = -4
MOE_ERR_NONFINITE = -5
MOE_ERR_TIMEOUT = -6
MOE_ERR_BOUNDS = -7


class MoeError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[{code}] {msg}")
        self.code = code


class moe_dims_t(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("D", ctypes.c_int32), ("E", ctypes.c_int32),
                ("F", ctypes.c_int32), ("k", ctypes.c_int32), ("S", ctypes.c_int32),
                ("Fs", ctypes.c_int32), ("scale", ctypes.c_float)]

    def __repr__(self):
        return ("moe_dims_t(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_)
                + ")")


def dims(T: int, D: int, E: int, F: int, k: int, S: int = 1, Fs: Optional[int] = None,
         scale: float = 2.5) -> moe_dims_t:
    return moe_dims_t(T, D, E, F, k, S, F if Fs is None else Fs, scale)


def dims_of(cfg, T: Optional[int] = None) -> moe_dims_t:
    """moe_dims_t of a workload description with fields T, D, E, F, k, S, Fs, scale."""
    return moe_dims_t(cfg.T if T is None else T, cfg.D, cfg.E, cfg.F, cfg.k, cfg.S, cfg.Fs,
                      cfg.scale)


class moe_fp8_weights_t(ctypes.Structure):
    """FP8 expert weights: E4M3 code arrays and int8 block-exponent arrays
    (device pointers; see moe_fp8_weights_t in include/moe_b200.h)."""
    _fields_ = [(n, ctypes.c_void_p) for n in ("W1", "W3", "W2", "Ws1", "Ws3", "Ws2",
                                                "W1e", "W3e", "W2e", "Ws1e", "Ws3e", "Ws2e")]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python sparse_moe_layer_04_b200/build.py` (or "
                          "`python __graft_entry__.py`)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    D = ctypes.POINTER(moe_dims_t)
    W8 = ctypes.POINTER(moe_fp8_weights_t)
    sig = {
        "moe_workspace_size": (Z, [D]),
        "moe_router_logits": (I, [P, P, D, P, P, Z, P]),
        "moe_route": (I, [P, P, D, P, P, P, P]),
        "moe_route_grouped": (I, [P, P, D, I, I, P, P, P, P]),
        "moe_permute": (I, [P, D, P, P, P, P, P, Z, P]),
        "moe_permute_noalloc": (I, [P, D, P, P, P, P, P]),
        "moe_expert_ffn": (I, [P, P, P, P, P, P, P, P, P, D, P, P, Z, P]),
        "moe_combine": (I, [P, P, P, D, P, P, P]),
        "moe_forward": (I, [P, P, P, P, P, P, P, P, P, D, P, P, P, P, Z, P]),
        "moe_get_device_status": (I, [P, P]),
        "moe_selftest_bounded_wait": (I, [P, P]),
        "moe_selftest_occupy": (I, [I, ctypes.c_longlong, P]),
        "moe_ws_expert_counts": (P, [P, D]),
        "moe_ws_touched_experts": (P, [P, D]),
        "moe_last_error": (ctypes.c_char_p, []),
        "moe_last_launch_count": (I, []),
        "moe_set_profile_events": (I, [ctypes.POINTER(P), I]),
        "moe_expert_ffn_fp8": (I, [P, P, P, W8, D, P, P, Z, P]),
        "moe_forward_fp8": (I, [P, P, P, W8, D, P, P, P, P, Z, P]),
        "moe_fp8_dequantize": (I, [P, P, I, I, I, P, P, P]),
        "moe_gather_rows": (I, [P, I, P, I, I, P, P, P]),
        "moe_forward_shared_overlap": (I, [D, I]),
        "moe_pipeline_device_bytes": (Z, [D]),
        "moe_pipeline_create": (I, [D, P, P, P, P, P, P, P, P, W8, P, Z, P,
                                    ctypes.POINTER(ctypes.c_void_p)]),
        "moe_pipeline_submit": (I, [P, P, P]),
        "moe_pipeline_wait": (I, [P]),
        "moe_pipeline_destroy": (I, [P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def _check(rc: int) -> None:
    if rc != MOE_OK:
        raise MoeError(rc, _lib.moe_last_error().decode())


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _ptr(t: Optional[torch.Tensor], dtype=None, name: str = "tensor") -> Optional[int]:
    if t is None:
        return None
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name}: expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous tensor")
    return t.data_ptr()


def _ws(ws: Optional[torch.Tensor]):
    if ws is None:
        return None, 0
    return _ptr(ws, torch.uint8, "ws"), ws.numel()


def moe_workspace_size(d: moe_dims_t) -> int:
    n = _lib.moe_workspace_size(ctypes.byref(d))
    if n == 0:
        raise MoeError(MOE_ERR_INVALID_ARG, f"invalid dimensions {d}")
    return n


def alloc_workspace(d: moe_dims_t, device="cuda") -> torch.Tensor:
    """A zeroed workspace of moe_workspace_size(d) bytes (torch allocations are 256-B aligned)."""
    return torch.zeros(moe_workspace_size(d), dtype=torch.uint8, device=device)


def moe_router_logits(h, Wr, d, logits, ws=None, stream=None) -> None:
    wp, wn = _ws(ws)
    _check(_lib.moe_router_logits(_ptr(h, torch.bfloat16, "h"), _ptr(Wr, torch.float32, "Wr"),
                                  ctypes.byref(d), _ptr(logits, torch.float32, "logits"), wp, wn,
                                  _stream(stream)))


def moe_route(logits, bias, d, idx, w, ws=None, stream=None) -> None:
    wp, _ = _ws(ws)
    _check(_lib.moe_route(_ptr(logits, torch.float32, "logits"), _ptr(bias, torch.float32, "bias"),
                          ctypes.byref(d), _ptr(idx, torch.int32, "idx"),
                          _ptr(w, torch.float32, "w"), wp, _stream(stream)))


def moe_route_grouped(logits, bias, d, n_group, topk_group, idx, w, ws=None, stream=None) -> None:
    wp, _ = _ws(ws)
    _check(_lib.moe_route_grouped(_ptr(logits, torch.float32, "logits"),
                                  _ptr(bias, torch.float32, "bias"), ctypes.byref(d), n_group,
                                  topk_group, _ptr(idx, torch.int32, "idx"),
                                  _ptr(w, torch.float32, "w"), wp, _stream(stream)))


def moe_permute(idx, d, counts, offsets, perm, inv, ws, stream=None) -> None:
    wp, wn = _ws(ws)
    _check(_lib.moe_permute(_ptr(idx, torch.int32, "idx"), ctypes.byref(d),
                            _ptr(counts, torch.int32, "counts"),
                            _ptr(offsets, torch.int32, "offsets"), _ptr(perm, torch.int32, "perm"),
                            _ptr(inv, torch.int32, "inv"), wp, wn, _stream(stream)))


def moe_permute_noalloc(idx, d, counts, offsets, perm, inv, stream=None) -> None:
    """moe_permute without a workspace (scratch inside the library; T <= 16384, E <= 1024)."""
    _check(_lib.moe_permute_noalloc(_ptr(idx, torch.int32, "idx"), ctypes.byref(d),
                                    _ptr(counts, torch.int32, "counts"),
                                    _ptr(offsets, torch.int32, "offsets"),
                                    _ptr(perm, torch.int32, "perm"), _ptr(inv, torch.int32, "inv"),
                                    _stream(stream)))


def moe_expert_ffn(h, perm, offsets, W1, W3, W2, Ws1, Ws3, Ws2, d, y, ws, stream=None) -> None:
    wp, wn = _ws(ws)
    bf = torch.bfloat16
    _check(_lib.moe_expert_ffn(_ptr(h, bf, "h"), _ptr(perm, torch.int32, "perm"),
                               _ptr(offsets, torch.int32, "offsets"), _ptr(W1, bf, "W1"),
                               _ptr(W3, bf, "W3"), _ptr(W2, bf, "W2"), _ptr(Ws1, bf, "Ws1"),
                               _ptr(Ws3, bf, "Ws3"), _ptr(Ws2, bf, "Ws2"), ctypes.byref(d),
                               _ptr(y, torch.float32, "y"), wp, wn, _stream(stream)))


_CODE_DTYPES = (torch.uint8, torch.float8_e4m3fn)


def _code_ptr(t: Optional[torch.Tensor], name: str) -> Optional[int]:
    if t is not None and t.dtype not in _CODE_DTYPES:
        raise TypeError(f"{name}: expected uint8 or float8_e4m3fn codes, got {t.dtype}")
    return _ptr(t, None, name)


def fp8_weights(W1, W3, W2, Ws1, Ws3, Ws2, W1e, W3e, W2e, Ws1e, Ws3e, Ws2e) -> moe_fp8_weights_t:
    """Packs FP8 code tensors (uint8 or float8_e4m3fn) and their int8 block
    exponents into the struct the FP8 entry points take.  The struct holds raw
    pointers: keep the tensors alive while it is in use."""
    w = moe_fp8_weights_t()
    for name, t in (("W1", W1), ("W3", W3), ("W2", W2), ("Ws1", Ws1), ("Ws3", Ws3), ("Ws2", Ws2)):
        setattr(w, name, _code_ptr(t, name))
    for name, t in (("W1e", W1e), ("W3e", W3e), ("W2e", W2e), ("Ws1e", Ws1e), ("Ws3e", Ws3e),
                    ("Ws2e", Ws2e)):
        setattr(w, name, _ptr(t, torch.int8, name))
    return w


def moe_expert_ffn_fp8(h, perm, offsets, w8: moe_fp8_weights_t, d, y, ws, stream=None) -> None:
    wp, wn = _ws(ws)
    _check(_lib.moe_expert_ffn_fp8(_ptr(h, torch.bfloat16, "h"), _ptr(perm, torch.int32, "perm"),
                                   _ptr(offsets, torch.int32, "offsets"), ctypes.byref(w8),
                                   ctypes.byref(d), _ptr(y, torch.float32, "y"), wp, wn,
                                   _stream(stream)))


def moe_forward_fp8(h, Wr, bias, w8: moe_fp8_weights_t, d, out, ws, idx_out=None, w_out=None,
                    stream=None) -> None:
    wp, wn = _ws(ws)
    _check(_lib.moe_forward_fp8(_ptr(h, torch.bfloat16, "h"), _ptr(Wr, torch.float32, "Wr"),
                                _ptr(bias, torch.float32, "bias"), ctypes.byref(w8),
                                ctypes.byref(d), _ptr(out, torch.float32, "out"),
                                _ptr(idx_out, torch.int32, "idx_out"),
                                _ptr(w_out, torch.float32, "w_out"), wp, wn, _stream(stream)))


def moe_fp8_dequantize(codes, exps, out, ws=None, stream=None) -> None:
    """codes [G, R, K] (or [R, K]) E4M3, exps [G, ceil(R/128), ceil(K/128)]
    int8 -> out bf16 of the codes' shape."""
    if codes.dim() not in (2, 3):
        raise ValueError("codes: expected [R, K] or [G, R, K]")
    G, R, K = (1, *codes.shape) if codes.dim() == 2 else tuple(codes.shape)
    if tuple(out.shape) != tuple(codes.shape):
        raise ValueError("out: expected the shape of codes")
    wp, _ = _ws(ws)
    _check(_lib.moe_fp8_dequantize(_code_ptr(codes, "codes"), _ptr(exps, torch.int8, "exps"),
                                   G, R, K, _ptr(out, torch.bfloat16, "out"), wp,
                                   _stream(stream)))


def moe_gather_rows(src, idx, dst, ws=None, stream=None) -> None:
    """dst[i] = src[idx[i]] (rows of any dtype, a multiple of 16 bytes wide)."""
    if src.dim() != 2 or dst.dim() != 2 or src.shape[1] != dst.shape[1] or src.dtype != dst.dtype:
        raise ValueError("src [rows, W] and dst [n, W] with one dtype expected")
    if idx.numel() != dst.shape[0]:
        raise ValueError("idx must have one entry per dst row")
    wp, _ = _ws(ws)
    row_bytes = src.shape[1] * src.element_size()
    _check(_lib.moe_gather_rows(_ptr(src, None, "src"), src.shape[0], _ptr(idx, torch.int32, "idx"),
                                idx.numel(), row_bytes, _ptr(dst, None, "dst"), wp,
                                _stream(stream)))


def moe_combine(y, w, inv, d, out, ws=None, stream=None) -> None:
    wp, _ = _ws(ws)
    _check(_lib.moe_combine(_ptr(y, torch.float32, "y"), _ptr(w, torch.float32, "w"),
                            _ptr(inv, torch.int32, "inv"), ctypes.byref(d),
                            _ptr(out, torch.float32, "out"), wp, _stream(stream)))


def moe_forward(h, Wr, bias, W1, W3, W2, Ws1, Ws3, Ws2, d, out, ws, idx_out=None, w_out=None,
                stream=None) -> None:
    wp, wn = _ws(ws)
    bf = torch.bfloat16
    _check(_lib.moe_forward(_ptr(h, bf, "h"), _ptr(Wr, torch.float32, "Wr"),
                            _ptr(bias, torch.float32, "bias"), _ptr(W1, bf, "W1"),
                            _ptr(W3, bf, "W3"), _ptr(W2, bf, "W2"), _ptr(Ws1, bf, "Ws1"),
                            _ptr(Ws3, bf, "Ws3"), _ptr(Ws2, bf, "Ws2"), ctypes.byref(d),
                            _ptr(out, torch.float32, "out"), _ptr(idx_out, torch.int32, "idx_out"),
                            _ptr(w_out, torch.float32, "w_out"), wp, wn, _stream(stream)))


class MoePipeline:
    """Handle of a host-buffer pipeline (moe_pipeline_t).  It holds the
    tensors the library reads through raw pointers (weights, router, bias,
    the device buffer) so they outlive the pipeline."""

    def __init__(self, handle: ctypes.c_void_p, d: moe_dims_t, keep):
        self.handle = handle
        self.dims = d
        self._keep = keep

    def __del__(self):
        if getattr(self, "handle", None) and self.handle.value:
            try:
                _lib.moe_pipeline_destroy(self.handle)
            except Exception:
                pass
            self.handle = None


def moe_pipeline_device_bytes(d: moe_dims_t) -> int:
    n = _lib.moe_pipeline_device_bytes(ctypes.byref(d))
    if n == 0:
        raise MoeError(MOE_ERR_INVALID_ARG, f"invalid dimensions {d}")
    return n


def moe_pipeline_create(d, Wr, bias, W1=None, W3=None, W2=None, Ws1=None, Ws3=None, Ws2=None,
                        w8: Optional[moe_fp8_weights_t] = None, dev=None, stream=None,
                        keep=()) -> MoePipeline:
    """bf16 weights (W1..Ws2) or FP8 weights (w8, whose tensors the caller
    passes in `keep` or otherwise keeps alive).  `dev` defaults to a fresh
    device buffer of moe_pipeline_device_bytes(d) bytes."""
    if dev is None:
        dev = torch.empty(moe_pipeline_device_bytes(d), dtype=torch.uint8, device=Wr.device)
    bf = None if w8 is not None else torch.bfloat16
    handle = ctypes.c_void_p()
    _check(_lib.moe_pipeline_create(ctypes.byref(d), _ptr(Wr, torch.float32, "Wr"),
                                    _ptr(bias, torch.float32, "bias"), _ptr(W1, bf, "W1"),
                                    _ptr(W3, bf, "W3"), _ptr(W2, bf, "W2"), _ptr(Ws1, bf, "Ws1"),
                                    _ptr(Ws3, bf, "Ws3"), _ptr(Ws2, bf, "Ws2"),
                                    ctypes.byref(w8) if w8 is not None else None,
                                    _ptr(dev, torch.uint8, "dev"), dev.numel(), _stream(stream),
                                    ctypes.byref(handle)))
    return MoePipeline(handle, d, (Wr, bias, W1, W3, W2, Ws1, Ws3, Ws2, w8, dev, tuple(keep)))


def _host_ptr(t: torch.Tensor, dtype, name: str) -> int:
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if t.is_cuda or not t.is_pinned():
        raise ValueError(f"{name}: expected a page-locked (pinned) host tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous tensor")
    return t.data_ptr()


def moe_pipeline_submit(p: MoePipeline, h_host: torch.Tensor, out_host: torch.Tensor) -> None:
    """Enqueues h_host [T, D] bf16 -> out_host [T, D] fp32 (pinned host tensors)."""
    n = p.dims.T * p.dims.D
    if h_host.numel() != n or out_host.numel() != n:
        raise ValueError("h_host and out_host must hold T x D elements")
    if n == 0:
        _check(_lib.moe_pipeline_submit(p.handle, None, None))
        return
    _check(_lib.moe_pipeline_submit(p.handle, _host_ptr(h_host, torch.bfloat16, "h_host"),
                                    _host_ptr(out_host, torch.float32, "out_host")))


def moe_pipeline_wait(p: MoePipeline) -> None:
    _check(_lib.moe_pipeline_wait(p.handle))


def moe_pipeline_destroy(p: MoePipeline) -> None:
    handle, p.handle = p.handle, None
    if handle is not None and handle.value:
        _check(_lib.moe_pipeline_destroy(handle))


def moe_forward_shared_overlap(d: moe_dims_t, fp8_weights: bool = False) -> bool:
    """True if moe_forward (or, with fp8_weights, moe_forward_fp8) runs the
    shared experts' FFN beside the routing on an internal stream for these
    dims (then the routed FFN launch excludes them)."""
    return bool(_lib.moe_forward_shared_overlap(ctypes.byref(d), 1 if fp8_weights else 0))


def moe_get_device_status(ws, stream=None) -> int:
    """Synchronises the stream; returns (and clears) the first device-side error code."""
    return _lib.moe_get_device_status(_ptr(ws, torch.uint8, "ws"), _stream(stream))


def moe_ws_expert_counts(ws, d) -> torch.Tensor:
    """int32 [E] view of the per-expert load histogram kept in the workspace."""
    addr = _lib.moe_ws_expert_counts(_ptr(ws, torch.uint8, "ws"), ctypes.byref(d))
    return _view_int32(ws, addr, d.E)


def moe_ws_touched_experts(ws, d) -> torch.Tensor:
    """int32 [1] view of the touched-expert count kept in the workspace."""
    addr = _lib.moe_ws_touched_experts(_ptr(ws, torch.uint8, "ws"), ctypes.byref(d))
    return _view_int32(ws, addr, 1)


def _view_int32(ws: torch.Tensor, addr: int, n: int) -> torch.Tensor:
    if not addr:
        raise MoeError(MOE_ERR_INVALID_ARG, "invalid workspace or dims")
    off = addr - ws.data_ptr()
    return ws[off: off + 4 * n].view(torch.int32)


def moe_selftest_bounded_wait(ws, stream=None) -> None:
    """Runs the bounded-wait self-test; moe_get_device_status then reports MOE_ERR_TIMEOUT."""
    _check(_lib.moe_selftest_bounded_wait(_ptr(ws, torch.uint8, "ws"), _stream(stream)))


def moe_selftest_occupy(nctas: int, cycles: int, stream=None) -> None:
    """Holds `nctas` SMs for `cycles` SM clock cycles on `stream` (waits on nothing else)."""
    _check(_lib.moe_selftest_occupy(int(nctas), int(cycles), _stream(stream)))


def moe_last_error() -> str:
    return _lib.moe_last_error().decode()


def moe_last_launch_count() -> int:
    return _lib.moe_last_launch_count()


MOE_PROFILE_EVENTS = 7
_prof_keep = None


def moe_set_profile_events(events) -> None:
    """Record torch.cuda.Event objects at moe_forward's stage boundaries (None: stop)."""
    global _prof_keep
    if events is None:
        _check(_lib.moe_set_profile_events(None, 0))
        _prof_keep = None
        return
    if len(events) != MOE_PROFILE_EVENTS:
        raise ValueError(f"need {MOE_PROFILE_EVENTS} events")
    for ev in events:  # torch creates the underlying CUDA event on first record
        if not ev.cuda_event:
            ev.record()
    arr = (ctypes.c_void_p * MOE_PROFILE_EVENTS)(*[ev.cuda_event for ev in events])
    _check(_lib.moe_set_profile_events(arr, MOE_PROFILE_EVENTS))
    _prof_keep = (arr, events)
