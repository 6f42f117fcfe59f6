"""Python wrapper of the plain C++ CPU oracle (``moe_oracle.cpp``).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg use it; the CUDA path never does. It shares no code with the
CUDA path (it imports nothing from the package).

Every function takes and returns CPU torch tensors; bf16 tensors cross the
boundary as their 16-bit patterns. ``build()`` compiles the library with g++
(OpenMP over tokens, -O2, nothing tuned).

Parity pins: every function here is pinned by the ``-m "not gpu"`` tests
(brute force, closed forms, library reductions, invariants, a hand-derived
golden example); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moe_oracle.cpp")
LIB = os.path.join(HERE, "liboracle.so")

_lib = None

c_i64, c_int, c_vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source if missing or stale."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared", SRC, "-o", tmp])
        os.replace(tmp, LIB)
    return LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB)
        L.oracle_num_threads.restype = c_int
        L.oracle_round_bf16.argtypes = [c_vp, c_i64, c_vp]
        L.oracle_dequant_mxfp4.argtypes = [c_vp, c_vp, c_i64, c_i64, c_vp]
        L.oracle_route.argtypes = [c_i64, c_int, c_int, c_int, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]
        L.oracle_permute.argtypes = [c_i64, c_int, c_int, c_vp, c_vp, c_vp, c_vp, c_vp]
        c_dbl = ctypes.c_double
        L.oracle_ffn_tokens.argtypes = [c_i64, c_int, c_int, c_int, c_int, c_int, c_int, c_dbl, c_dbl, c_vp, c_vp,
                                        c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_i64, c_vp, c_vp, c_vp]
        L.oracle_forward.argtypes = [c_i64, c_int, c_int, c_int, c_int, c_int, c_int, c_dbl, c_dbl, c_vp, c_vp,
                                     c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]
        for f in ("oracle_dequant_mxfp4", "oracle_route", "oracle_permute", "oracle_ffn_tokens", "oracle_forward"):
            getattr(L, f).restype = c_int
        _lib = L
    return _lib


def _cpu(t: Optional[torch.Tensor]) -> Optional[torch.Tensor]:
    if t is None:
        return None
    return t.detach().to("cpu").contiguous()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"{what}: oracle returned error {rc}")


def num_threads() -> int:
    return lib().oracle_num_threads()


def round_bf16(v: torch.Tensor) -> torch.Tensor:
    """Round float64 values to bf16 (one rounding, ties to even)."""
    v = _cpu(v).double()
    out = torch.empty(v.shape, dtype=torch.int16)
    lib().oracle_round_bf16(_ptr(v), v.numel(), _ptr(out))
    return out.view(torch.bfloat16)


def dequant_mxfp4(codes: torch.Tensor, scales: torch.Tensor) -> torch.Tensor:
    """(N, K/2) codes + (N, K/32) scales -> (N, K) float64 values."""
    codes, scales = _cpu(codes), _cpu(scales)
    N, K = codes.shape[0], codes.shape[1] * 2
    out = torch.empty((N, K), dtype=torch.float64)
    _check(lib().oracle_dequant_mxfp4(_ptr(codes), _ptr(scales), N, K, _ptr(out)), "dequant_mxfp4")
    return out


def route(x, Wr, br, k: int):
    """-> (logits (T,E) float32, topk_idx (T,k) int32, topk_w (T,k) float32)."""
    x, Wr, br = _cpu(x), _cpu(Wr), _cpu(br)
    T, D = x.shape
    E = Wr.shape[0]
    logits = torch.empty((T, E), dtype=torch.float32)
    idx = torch.empty((T, k), dtype=torch.int32)
    w = torch.empty((T, k), dtype=torch.float32)
    _check(lib().oracle_route(T, D, E, k, _ptr(x), _ptr(Wr), _ptr(br), _ptr(logits), _ptr(idx), _ptr(w)), "route")
    return logits, idx, w


def permute(topk_idx, E: int):
    """-> (counts (E,), offsets (E+1,), perm (R,), inv (R,)), all int32."""
    idx = _cpu(topk_idx).to(torch.int32)
    T, k = idx.shape
    R = T * k
    counts = torch.empty(E, dtype=torch.int32)
    offsets = torch.empty(E + 1, dtype=torch.int32)
    perm = torch.empty(R, dtype=torch.int32)
    inv = torch.empty(R, dtype=torch.int32)
    _check(lib().oracle_permute(T, E, k, _ptr(idx), _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(inv)), "permute")
    return counts, offsets, perm, inv


ACT_SWIGLU, ACT_GPTOSS = 0, 1


def ffn_tokens(x, topk_idx, topk_w, W1, b1, W2, b2, tokens: Optional[Sequence[int]] = None,
               W1_scales=None, W2_scales=None, return_o: bool = False, return_exact: bool = False,
               act=(ACT_SWIGLU, 1.0, float("inf"))):
    """Expert FFN + weighted combine for ``tokens`` (default all) -> y (n, D) bf16
    [and o (n, k, D) float64, the unweighted expert outputs]
    [and y_exact (n, D) float64, y before its final bf16 rounding].
    ``act`` = (kind, alpha, limit): plain SwiGLU (kind 0) or the GPT-OSS
    variant (kind 1, clamp at ``limit``, sigmoid(alpha * gate), up + 1)."""
    x, idx, w = _cpu(x), _cpu(topk_idx).to(torch.int32), _cpu(topk_w).float()
    W1, b1, W2, b2 = _cpu(W1), _cpu(b1), _cpu(W2), _cpu(b2)
    W1s, W2s = _cpu(W1_scales), _cpu(W2_scales)
    T, D = x.shape
    E = b1.shape[0]
    I = b1.shape[1] // 2
    k = idx.shape[1]
    wfmt = 0 if W1s is None else 1
    if tokens is None:
        tok = torch.arange(T, dtype=torch.int64)
    else:
        tok = torch.as_tensor(tokens, dtype=torch.int64).contiguous()
    n = tok.numel()
    y = torch.empty((n, D), dtype=torch.int16)
    o = torch.empty((n, k, D), dtype=torch.float64) if return_o else None
    ye = torch.empty((n, D), dtype=torch.float64) if return_exact else None
    _check(lib().oracle_ffn_tokens(T, D, E, k, I, wfmt, int(act[0]), float(act[1]), float(act[2]), _ptr(x), _ptr(idx),
                                   _ptr(w), _ptr(W1), _ptr(W1s), _ptr(b1), _ptr(W2), _ptr(W2s), _ptr(b2), _ptr(tok), n,
                                   _ptr(y), _ptr(o), _ptr(ye)),
           "ffn_tokens")
    out = [y.view(torch.bfloat16)]
    if return_o:
        out.append(o)
    if return_exact:
        out.append(ye)
    return tuple(out) if len(out) > 1 else out[0]


def forward(x, Wr, br, W1, b1, W2, b2, k: int, W1_scales=None, W2_scales=None, act=(ACT_SWIGLU, 1.0, float("inf"))):
    """The whole layer -> (y (T,D) bf16, topk_idx (T,k) int32, topk_w (T,k) float32)."""
    x, Wr, br = _cpu(x), _cpu(Wr), _cpu(br)
    W1, b1, W2, b2 = _cpu(W1), _cpu(b1), _cpu(W2), _cpu(b2)
    W1s, W2s = _cpu(W1_scales), _cpu(W2_scales)
    T, D = x.shape
    E = Wr.shape[0]
    I = b1.shape[1] // 2
    wfmt = 0 if W1s is None else 1
    y = torch.empty((T, D), dtype=torch.int16)
    idx = torch.empty((T, k), dtype=torch.int32)
    w = torch.empty((T, k), dtype=torch.float32)
    _check(lib().oracle_forward(T, D, E, k, I, wfmt, int(act[0]), float(act[1]), float(act[2]), _ptr(x), _ptr(Wr),
                                _ptr(br), _ptr(W1), _ptr(W1s), _ptr(b1), _ptr(W2), _ptr(W2s), _ptr(b2), _ptr(y), _ptr(idx),
                                _ptr(w)), "forward")
    return y.view(torch.bfloat16), idx, w


def gap_reject(min_gap: float = 1e-4):
    """A token-redraw predicate for ``synthetic.make_inputs``: rejects tokens
    whose top-(k+1) router logits (oracle logits) have an adjacent gap below
    ``min_gap``, so that the chosen experts and their order are unique."""

    def reject(x, Wr, br, k):
        logits, _, _ = route(x, Wr, br, k)
        E = logits.shape[1]
        m = min(k + 1, E)
        top = torch.sort(logits.double(), dim=1, descending=True).values[:, :m]
        if m < 2:
            return torch.zeros(logits.shape[0], dtype=torch.bool)
        gaps = top[:, :-1] - top[:, 1:]
        return (gaps < min_gap).any(dim=1)

    return reject
