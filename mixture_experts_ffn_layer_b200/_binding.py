"""ctypes binding of libmoe.so (include/moe.h). Argument marshalling only:
torch tensors supply device pointers, the current torch CUDA stream is passed
as the cudaStream_t, and every step of the layer runs in the library's
kernels. There is no fallback: if the library is missing or fails to load,
every call raises."""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe.so")

MOE_W_BF16, MOE_W_MXFP4 = 0, 1
MOE_ACT_SWIGLU, MOE_ACT_GPTOSS = 0, 1
STATUS = {
    0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE", 4: "MOE_ERR_CUDA",
    5: "MOE_ERR_TIMEOUT", 6: "MOE_ERR_DEVICE_BOUNDS",
}

# Every symbol include/moe.h declares.
EXPORTS = ("moe_workspace_bytes", "moe_check_dims", "moe_route", "moe_permute", "moe_gather", "moe_mlp1", "moe_mlp2",
           "moe_ffn_grouped", "moe_combine", "moe_forward", "moe_read_device_status", "moe_status_str",
           "moe_permute_noalloc", "moe_selftest_wait_timeout", "moe_mxfp4_prepared_bytes", "moe_mxfp4_prepare")


class MoeError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS.get(code, code)}")
        self.code = code


class Dims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("D", ctypes.c_int32), ("E", ctypes.c_int32), ("k", ctypes.c_int32),
                ("I", ctypes.c_int32), ("wfmt", ctypes.c_int32), ("act", ctypes.c_int32),
                ("act_alpha", ctypes.c_float), ("act_limit", ctypes.c_float)]


class Weight(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("prepared", ctypes.c_void_p)]


_lib = None
VP = ctypes.c_void_p


def load(path: str = LIB_PATH):
    """Load the library (building it first if it is missing or stale)."""
    global _lib
    if _lib is not None:
        return _lib
    from . import build as _build

    if _build.stale():
        _build.build()
    if not os.path.exists(path):
        raise RuntimeError(f"libmoe.so not found at {path}; run mixture_experts_ffn_layer_b200.build.build()")
    L = ctypes.CDLL(path)
    sig = {
        "moe_workspace_bytes": (ctypes.c_size_t, [Dims]),
        "moe_check_dims": (ctypes.c_int, [Dims]),
        "moe_route": (ctypes.c_int, [Dims, VP, VP, VP, VP, VP, VP, ctypes.c_size_t, VP]),
        "moe_permute": (ctypes.c_int, [Dims, VP, VP, VP, VP, VP, VP, ctypes.c_size_t, VP]),
        "moe_gather": (ctypes.c_int, [Dims, VP, VP, VP, VP, ctypes.c_size_t, VP]),
        "moe_mlp1": (ctypes.c_int, [Dims, VP, VP, Weight, VP, VP, VP, ctypes.c_size_t, VP]),
        "moe_mlp2": (ctypes.c_int, [Dims, VP, VP, VP, VP, Weight, VP, VP, VP, ctypes.c_size_t, VP]),
        "moe_ffn_grouped": (ctypes.c_int, [Dims, VP, VP, VP, VP, Weight, VP, Weight, VP, VP, VP, ctypes.c_size_t, VP]),
        "moe_combine": (ctypes.c_int, [Dims, VP, VP, VP, VP, ctypes.c_size_t, VP]),
        "moe_forward": (ctypes.c_int, [Dims, VP, VP, VP, Weight, VP, Weight, VP, VP, VP, ctypes.c_size_t, VP]),
        "moe_read_device_status": (ctypes.c_int, [VP, VP]),
        "moe_permute_noalloc": (ctypes.c_int, [Dims, VP, VP, VP, VP, VP, VP]),
        "moe_selftest_wait_timeout": (ctypes.c_int, [VP, ctypes.c_uint64, VP]),
        "moe_status_str": (ctypes.c_char_p, [ctypes.c_int]),
        "moe_mxfp4_prepared_bytes": (ctypes.c_size_t, [Dims, ctypes.c_int32]),
        "moe_mxfp4_prepare": (ctypes.c_int, [Dims, ctypes.c_int32, Weight, VP, ctypes.c_size_t, VP]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def dims(T, D, E, k, I, wfmt=MOE_W_BF16, act=MOE_ACT_SWIGLU, act_alpha=1.0, act_limit=float("inf")) -> Dims:
    return Dims(T, D, E, k, I, wfmt, act, act_alpha, act_limit)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _w(data: Optional[torch.Tensor], scales: Optional[torch.Tensor] = None,
       prepared: Optional[torch.Tensor] = None) -> Weight:
    # (data and scales may be None next to an MXFP4 prepared form)
    return Weight(None if data is None else data.data_ptr(), None if scales is None else scales.data_ptr(),
                  None if prepared is None else prepared.data_ptr())


def _check(rc: int, what: str):
    if rc != 0:
        raise MoeError(rc, what)


def workspace_bytes(d: Dims) -> int:
    n = load().moe_workspace_bytes(d)
    if n == 0:
        raise MoeError(load().moe_check_dims(d), "moe_workspace_bytes")
    return n


def alloc_workspace(d: Dims, device="cuda") -> torch.Tensor:
    return torch.zeros(workspace_bytes(d), dtype=torch.uint8, device=device)


def check_dims(d: Dims) -> int:
    return load().moe_check_dims(d)


def moe_route(d, x, Wr, br, topk_idx, topk_w, ws, stream=None):
    _check(load().moe_route(d, _p(x), _p(Wr), _p(br), _p(topk_idx), _p(topk_w), _p(ws), ws.numel(), _stream(stream)),
           "moe_route")


def moe_permute(d, topk_idx, counts, offsets, perm, inv, ws, stream=None):
    _check(load().moe_permute(d, _p(topk_idx), _p(counts), _p(offsets), _p(perm), _p(inv), _p(ws), ws.numel(),
                              _stream(stream)), "moe_permute")


def moe_gather(d, x, perm, x_perm, ws, stream=None):
    _check(load().moe_gather(d, _p(x), _p(perm), _p(x_perm), _p(ws), ws.numel(), _stream(stream)), "moe_gather")


def moe_mlp1(d, x_perm, offsets, W1, b1, h, ws, W1_scales=None, stream=None, W1_prepared=None):
    _check(load().moe_mlp1(d, _p(x_perm), _p(offsets), _w(W1, W1_scales, W1_prepared), _p(b1), _p(h), _p(ws), ws.numel(),
                           _stream(stream)), "moe_mlp1")


def moe_mlp2(d, h, perm, offsets, topk_w, W2, b2, o_perm, ws, W2_scales=None, stream=None, W2_prepared=None):
    _check(load().moe_mlp2(d, _p(h), _p(perm), _p(offsets), _p(topk_w), _w(W2, W2_scales, W2_prepared), _p(b2), _p(o_perm), _p(ws),
                           ws.numel(), _stream(stream)), "moe_mlp2")


def moe_ffn_grouped(d, x, perm, offsets, topk_w, W1, b1, W2, b2, o_perm, ws, W1_scales=None, W2_scales=None,
                    stream=None, W1_prepared=None, W2_prepared=None):
    _check(load().moe_ffn_grouped(d, _p(x), _p(perm), _p(offsets), _p(topk_w), _w(W1, W1_scales, W1_prepared), _p(b1),
                                  _w(W2, W2_scales, W2_prepared), _p(b2), _p(o_perm), _p(ws), ws.numel(), _stream(stream)),
           "moe_ffn_grouped")


def moe_combine(d, o_perm, inv, y, ws, stream=None):
    _check(load().moe_combine(d, _p(o_perm), _p(inv), _p(y), _p(ws), ws.numel(), _stream(stream)), "moe_combine")


def moe_forward(d, x, Wr, br, W1, b1, W2, b2, y, ws, W1_scales=None, W2_scales=None, stream=None, W1_prepared=None,
                W2_prepared=None):
    _check(load().moe_forward(d, _p(x), _p(Wr), _p(br), _w(W1, W1_scales, W1_prepared), _p(b1), _w(W2, W2_scales, W2_prepared), _p(b2), _p(y),
                              _p(ws), ws.numel(), _stream(stream)), "moe_forward")


def moe_permute_noalloc(d, topk_idx, counts, offsets, perm, inv, stream=None):
    """moe_permute without a workspace (scratch in a fixed library array)."""
    _check(load().moe_permute_noalloc(d, _p(topk_idx), _p(counts), _p(offsets), _p(perm), _p(inv), _stream(stream)),
           "moe_permute_noalloc")


def mxfp4_prepared_bytes(d, which: int) -> int:
    return load().moe_mxfp4_prepared_bytes(d, which)


def moe_mxfp4_prepare(d, which: int, W, W_scales, out, stream=None):
    """The prepare-once form of an MXFP4 expert weight (which = 1: W1, 2: W2) into out."""
    _check(load().moe_mxfp4_prepare(d, which, _w(W, W_scales), _p(out), out.numel(), _stream(stream)),
           "moe_mxfp4_prepare")


def mxfp4_prepare(d, which: int, W, W_scales, stream=None) -> torch.Tensor:
    """Allocate and fill the prepare-once form of an MXFP4 expert weight."""
    n = mxfp4_prepared_bytes(d, which)
    if n == 0:
        raise MoeError(2, "moe_mxfp4_prepared_bytes")
    out = torch.empty(n, dtype=torch.uint8, device=W.device)
    moe_mxfp4_prepare(d, which, W, W_scales, out, stream)
    return out


def moe_selftest_wait_timeout(ws, limit_ns: int, stream=None):
    _check(load().moe_selftest_wait_timeout(_p(ws), limit_ns, _stream(stream)), "moe_selftest_wait_timeout")


def moe_read_device_status(ws, stream=None) -> int:
    return load().moe_read_device_status(_p(ws), _stream(stream))


def status_str(code: int) -> str:
    return load().moe_status_str(code).decode()
