"""B200 (sm_100a) GPT-OSS-style MoE feed-forward layer.

The compute lives in libmoe.so (C ABI in include/moe.h); this package is its
thin binding plus a convenience ``MoELayer`` that owns the workspace. The
library is loaded on first use; a missing library is an error, never a
fallback.
"""
from __future__ import annotations

from typing import Optional

import torch

from ._binding import (  # noqa: F401
    MOE_W_BF16, MOE_W_MXFP4, MOE_ACT_SWIGLU, MOE_ACT_GPTOSS, EXPORTS, MoeError, Dims, dims, load, workspace_bytes,
    alloc_workspace, check_dims,
    moe_route, moe_permute, moe_gather, moe_mlp1, moe_mlp2, moe_ffn_grouped, moe_combine, moe_forward,
    moe_read_device_status, status_str, moe_permute_noalloc, moe_selftest_wait_timeout, mxfp4_prepared_bytes,
    moe_mxfp4_prepare, mxfp4_prepare,
)
from .ep import CudaLocalOps, ExpertParallelMoE, ep_forward  # noqa: F401,E402


class MoELayer:
    """One MoE FFN layer's weights on the device plus its workspace.

    ``forward(x)`` enqueues the whole layer (moe_forward) on the current
    stream and returns y (T, D) bf16. Weights: Wr (E,D), br (E), W1 (E,2I,D),
    b1 (E,2I), W2 (E,D,I), b2 (E,D) bf16 -- or W1/W2 as MXFP4 codes with
    ``W1_scales``/``W2_scales``. ``act`` is MOE_ACT_SWIGLU or MOE_ACT_GPTOSS
    (with the caller's ``act_alpha`` and ``act_limit``)."""

    def __init__(self, Wr, br, W1, b1, W2, b2, k: int, W1_scales=None, W2_scales=None, act=MOE_ACT_SWIGLU,
                 act_alpha: float = 1.0, act_limit: float = float("inf")):
        self.Wr, self.br, self.W1, self.b1, self.W2, self.b2 = Wr, br, W1, b1, W2, b2
        self.W1_scales, self.W2_scales = W1_scales, W2_scales
        self.k = k
        self.E, self.D = Wr.shape
        self.I = b1.shape[1] // 2
        self.wfmt = MOE_W_BF16 if W1_scales is None else MOE_W_MXFP4
        self.act, self.act_alpha, self.act_limit = act, act_alpha, act_limit
        self._ws: Optional[torch.Tensor] = None
        self._ws_T = 0
        # MXFP4 weights: their prepare-once form (scale layout of the
        # block-scaled MMAs), made here so that no call repeats it
        self.W1_prepared = self.W2_prepared = None
        if self.wfmt == MOE_W_MXFP4:
            d1 = self.dims(1)
            self.W1_prepared = mxfp4_prepare(d1, 1, W1, W1_scales)
            self.W2_prepared = mxfp4_prepare(d1, 2, W2, W2_scales)

    def dims(self, T: int) -> Dims:
        return dims(T, self.D, self.E, self.k, self.I, self.wfmt, self.act, self.act_alpha, self.act_limit)

    def workspace(self, T: int) -> torch.Tensor:
        if self._ws is None or self._ws_T < T:
            self._ws = alloc_workspace(self.dims(T), device=self.Wr.device)
            self._ws_T = T
        return self._ws

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        T = x.shape[0]
        y = out if out is not None else torch.empty((T, self.D), dtype=torch.bfloat16, device=x.device)
        moe_forward(self.dims(T), x, self.Wr, self.br, self.W1, self.b1, self.W2, self.b2, y, self.workspace(T),
                    W1_scales=self.W1_scales, W2_scales=self.W2_scales, stream=stream, W1_prepared=self.W1_prepared,
                    W2_prepared=self.W2_prepared)
        return y

    __call__ = forward

    def device_status(self) -> int:
        return 0 if self._ws is None else moe_read_device_status(self._ws)
