"""Shared test helpers: run the CUDA path stage by stage through the C ABI,
and compare with the oracle."""
from __future__ import annotations

import dataclasses

import torch

import mixture_experts_ffn_layer_b200 as moe
import oracle
import synthetic

# max|y - y_ref| <= TOL * rms(y_ref): bf16 weights, MXFP4 weights.
TOL_BF16 = 2e-2
TOL_MXFP4 = 6e-2


@dataclasses.dataclass
class StageRun:
    topk_idx: torch.Tensor
    topk_w: torch.Tensor
    counts: torch.Tensor
    offsets: torch.Tensor
    perm: torch.Tensor
    inv: torch.Tensor
    x_perm: torch.Tensor
    h: torch.Tensor
    o_perm: torch.Tensor
    y: torch.Tensor
    status: int


SWIGLU = (moe.MOE_ACT_SWIGLU, 1.0, float("inf"))  # (act, alpha, limit); oracle.ACT_* use the same codes


def dims_of(inp: synthetic.LayerInputs, act=SWIGLU):
    s = inp.shape
    return moe.dims(s.T, s.D, s.E, s.k, s.I, moe.MOE_W_MXFP4 if s.wfmt == "mxfp4" else moe.MOE_W_BF16, *act)


def run_stages(inp: synthetic.LayerInputs, act=SWIGLU) -> StageRun:
    """Every stage through its own C-ABI entry point, intermediates kept."""
    s = inp.shape
    dev = inp.x.device
    d = dims_of(inp, act)
    ws = moe.alloc_workspace(d, device=dev)
    R = s.T * s.k
    i32 = dict(dtype=torch.int32, device=dev)
    topk_idx = torch.empty((s.T, s.k), **i32)
    topk_w = torch.empty((s.T, s.k), dtype=torch.float32, device=dev)
    counts = torch.empty(s.E, **i32)
    offsets = torch.empty(s.E + 1, **i32)
    perm = torch.empty(R, **i32)
    inv = torch.empty(R, **i32)
    x_perm = torch.empty((R, s.D), dtype=torch.bfloat16, device=dev)
    h = torch.empty((R, s.I), dtype=torch.bfloat16, device=dev)
    o_perm = torch.empty((R, s.D), dtype=torch.float32, device=dev)
    y = torch.empty((s.T, s.D), dtype=torch.bfloat16, device=dev)
    moe.moe_route(d, inp.x, inp.Wr, inp.br, topk_idx, topk_w, ws)
    moe.moe_permute(d, topk_idx, counts, offsets, perm, inv, ws)
    moe.moe_gather(d, inp.x, perm, x_perm, ws)
    moe.moe_mlp1(d, x_perm, offsets, inp.W1, inp.b1, h, ws, W1_scales=inp.W1_scales)
    moe.moe_mlp2(d, h, perm, offsets, topk_w, inp.W2, inp.b2, o_perm, ws, W2_scales=inp.W2_scales)
    moe.moe_combine(d, o_perm, inv, y, ws)
    status = moe.moe_read_device_status(ws)
    return StageRun(topk_idx, topk_w, counts, offsets, perm, inv, x_perm, h, o_perm, y, status)


def run_forward(inp: synthetic.LayerInputs, act=SWIGLU) -> torch.Tensor:
    s = inp.shape
    d = dims_of(inp, act)
    ws = moe.alloc_workspace(d, device=inp.x.device)
    y = torch.empty((s.T, s.D), dtype=torch.bfloat16, device=inp.x.device)
    moe.moe_forward(d, inp.x, inp.Wr, inp.br, inp.W1, inp.b1, inp.W2, inp.b2, y, ws, W1_scales=inp.W1_scales,
                    W2_scales=inp.W2_scales)
    st = moe.moe_read_device_status(ws)
    assert st == 0, moe.status_str(st)
    return y


def sample_tokens(idx: torch.Tensor, E: int, n: int, seed: int = 0, rare_rows: int = 64) -> torch.Tensor:
    """A seeded subset of tokens that includes every token routed to an
    expert with fewer than ``rare_rows`` rows, plus the first and last."""
    T = idx.shape[0]
    counts = torch.bincount(idx.flatten().long(), minlength=E)
    rare = (counts < rare_rows) & (counts > 0)
    rare_tok = torch.nonzero(rare[idx.long()].any(dim=1)).flatten()
    g = torch.Generator().manual_seed(seed)
    pick = torch.randperm(T, generator=g)[:n]
    toks = torch.unique(torch.cat([pick, rare_tok, torch.tensor([0, T - 1])]))
    return toks


def assert_close_rms(y: torch.Tensor, y_ref: torch.Tensor, tol: float, rms_ref: float | None = None):
    y, y_ref = y.double().cpu(), y_ref.double().cpu()
    rms = float(y_ref.pow(2).mean().sqrt()) if rms_ref is None else rms_ref
    err = float((y - y_ref).abs().max())
    assert err <= tol * rms, f"max|y-y_ref| = {err:.4g} > {tol} * rms {rms:.4g}"
    return err / rms
