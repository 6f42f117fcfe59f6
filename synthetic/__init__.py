"""Seeded synthetic inputs for the GPT-OSS-style MoE feed-forward layer.

This module only draws random tensors. It holds none of the layer's
arithmetic: no router product, no top-k, no softmax, no expert FFN. Both the
CPU oracle (through the tests) and the CUDA path (through the tests and the
benchmark) take their inputs from here.

Distributions (the workloads of the layer's descriptions; the pages print no
data, so every tensor is synthetic):

* x ~ N(0, 1), router weight Wr ~ N(0, std D^-0.5), router bias br ~ N(0, 0.02),
  expert weights W1, W2 and biases b1, b2 ~ N(0, 0.02). Every tensor is drawn
  in fp32 and rounded to bf16 (round-to-nearest-even, torch's conversion).
  "std dim^-0.5" follows the torchtitan GPT-OSS guide's initialisation
  section, which gives the lm_head that std; "N(0, 0.02)" the same section's
  embedding init.
* Skewed routing (the 120B-shaped layer): br[e] = 0.75 * ln p_{pi(e)} +
  N(0, 0.02) with p_r proportional to r^-s over ranks r = 1..E and pi a seeded
  permutation, so expert popularity roughly follows Zipf(s) and is not
  monotone in the expert index.
* MXFP4 expert weights: E2M1 codes uniform over the 16 codes (two per byte,
  low nibble first along the reduction dim) and one E8M0 scale byte per 32
  consecutive reduction elements, uniform in [127-8, 127].

Token redraw ("gap rejection"): a caller may pass ``reject(x, Wr, br, k)``
returning a bool mask of tokens to redraw; this module redraws exactly those
rows of x from a fresh seeded stream until the mask is empty. The test suite
passes a predicate computed by the oracle, so that the top-(k+1) router logits
of every token are separated by at least 1e-4 and the expert order is unique
under fp32 reassociation. The benchmark passes none (the redrawn tokens are a
handful out of thousands and do not change the timed work).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Callable, Optional

import torch

BF16 = torch.bfloat16


@dataclasses.dataclass(frozen=True)
class LayerShape:
    """Sizes of one MoE layer workload (T tokens, model dim D, E experts,
    top-k, expert intermediate dim I) and its expert-weight format."""

    name: str
    T: int
    D: int
    E: int
    k: int
    I: int
    wfmt: str = "bf16"  # "bf16" or "mxfp4"
    zipf_s: float = 0.0  # > 0: skewed routing bias

    @property
    def R(self) -> int:
        return self.T * self.k

    @property
    def flops(self) -> int:
        """Expert FLOPs of one forward, 6*T*k*D*I (router excluded)."""
        return 6 * self.T * self.k * self.D * self.I


# The synthetic workloads: a tiny parity case, a debug-model-sized layer,
# the GPT-OSS-20B expert shape (hidden 2880, 32 experts, top-4, per the
# from-scratch GPT-OSS write-up's parameter list), the 120B shape with skewed
# routing, and the 20B shape with MXFP4 expert weights at prefill and decode
# token counts.
SHAPES = {
    "tiny": LayerShape("tiny", T=64, D=64, E=4, k=2, I=64),
    "debug": LayerShape("debug", T=2048, D=256, E=8, k=2, I=512),
    "gptoss20b": LayerShape("gptoss20b", T=8192, D=2880, E=32, k=4, I=2880),
    "gptoss120b_zipf": LayerShape("gptoss120b_zipf", T=16384, D=2880, E=128, k=4, I=2880, zipf_s=1.1),
    "gptoss20b_mxfp4": LayerShape("gptoss20b_mxfp4", T=8192, D=2880, E=32, k=4, I=2880, wfmt="mxfp4"),
    "gptoss20b_mxfp4_decode": LayerShape("gptoss20b_mxfp4_decode", T=64, D=2880, E=32, k=4, I=2880, wfmt="mxfp4"),
}

SEEDS = {name: 1234 + i for i, name in enumerate(SHAPES)}


@dataclasses.dataclass
class LayerInputs:
    """One layer's tensors. bf16 tensors are torch.bfloat16; MXFP4 weights are
    uint8 codes (E, N, K/2) plus uint8 E8M0 scales (E, N, K/32)."""

    shape: LayerShape
    x: torch.Tensor  # (T, D) bf16
    Wr: torch.Tensor  # (E, D) bf16
    br: torch.Tensor  # (E,) bf16
    W1: torch.Tensor  # (E, 2I, D) bf16, or (E, 2I, D/2) uint8 codes
    b1: torch.Tensor  # (E, 2I) bf16
    W2: torch.Tensor  # (E, D, I) bf16, or (E, D, I/2) uint8 codes
    b2: torch.Tensor  # (E, D) bf16
    W1_scales: Optional[torch.Tensor] = None  # (E, 2I, D/32) uint8
    W2_scales: Optional[torch.Tensor] = None  # (E, D, I/32) uint8
    redrawn_tokens: int = 0

    def to(self, device) -> "LayerInputs":
        def mv(t):
            return None if t is None else t.to(device)

        return dataclasses.replace(
            self,
            x=mv(self.x), Wr=mv(self.Wr), br=mv(self.br), W1=mv(self.W1), b1=mv(self.b1),
            W2=mv(self.W2), b2=mv(self.b2), W1_scales=mv(self.W1_scales), W2_scales=mv(self.W2_scales),
        )


def _normal(shape, std, g, device):
    return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(BF16)


def _expert_normal(E, rows, cols, std, g, device):
    # One expert at a time keeps the fp32 temporary small for the large shapes.
    out = torch.empty((E, rows, cols), dtype=BF16, device=device)
    for e in range(E):
        out[e] = _normal((rows, cols), std, g, device)
    return out


def _mxfp4(E, rows, cols, g, device):
    if cols % 32:
        raise ValueError("MXFP4 reduction dim must be a multiple of 32")
    codes = torch.randint(0, 256, (E, rows, cols // 2), generator=g, device=device, dtype=torch.int32).to(torch.uint8)
    scales = torch.randint(127 - 8, 128, (E, rows, cols // 32), generator=g, device=device, dtype=torch.int32).to(torch.uint8)
    return codes, scales


def zipf_router_bias(E: int, s: float, g: torch.Generator, device) -> torch.Tensor:
    ranks = torch.arange(1, E + 1, dtype=torch.float64)
    p = ranks.pow(-s)
    p = p / p.sum()
    pi = torch.randperm(E, generator=g, device=device).cpu()
    base = 0.75 * torch.log(p[pi])
    noise = torch.randn(E, generator=g, device=device, dtype=torch.float32).cpu().double() * 0.02
    return (base + noise).float().to(BF16).to(device)


RejectFn = Callable[[torch.Tensor, torch.Tensor, torch.Tensor, int], torch.Tensor]


def make_inputs(shape: LayerShape | str, seed: Optional[int] = None, device="cpu",
                reject: Optional[RejectFn] = None, T: Optional[int] = None,
                max_redraw_rounds: int = 64) -> LayerInputs:
    """Draw one layer's inputs. ``T`` overrides the token count (same weights'
    distribution, fewer or more tokens)."""
    if isinstance(shape, str):
        if seed is None:
            seed = SEEDS[shape]
        shape = SHAPES[shape]
    if T is not None:
        shape = dataclasses.replace(shape, T=T)
    if seed is None:
        seed = 1234
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    T_, D, E, k, I = shape.T, shape.D, shape.E, shape.k, shape.I

    Wr = _normal((E, D), D ** -0.5, g, device)
    if shape.zipf_s > 0:
        br = zipf_router_bias(E, shape.zipf_s, g, device)
    else:
        br = _normal((E,), 0.02, g, device)
    b1 = _normal((E, 2 * I), 0.02, g, device)
    b2 = _normal((E, D), 0.02, g, device)
    W1s = W2s = None
    if shape.wfmt == "bf16":
        W1 = _expert_normal(E, 2 * I, D, 0.02, g, device)
        W2 = _expert_normal(E, D, I, 0.02, g, device)
    elif shape.wfmt == "mxfp4":
        W1, W1s = _mxfp4(E, 2 * I, D, g, device)
        W2, W2s = _mxfp4(E, D, I, g, device)
    else:
        raise ValueError(f"unknown weight format {shape.wfmt}")
    # x is drawn last from its own stream so that a different T keeps the weights.
    gx = torch.Generator(device=device)
    gx.manual_seed(seed * 7919 + 17)
    x = _normal((T_, D), 1.0, gx, device)

    redrawn = 0
    if reject is not None:
        for rnd in range(max_redraw_rounds):
            bad = reject(x, Wr, br, k).to(device)
            n_bad = int(bad.sum())
            if n_bad == 0:
                break
            redrawn += n_bad
            gr = torch.Generator(device=device)
            gr.manual_seed(seed * 104729 + 31 * rnd + 1)
            x[bad] = _normal((n_bad, D), 1.0, gr, device)
        else:
            raise RuntimeError("token redraw did not converge")
    return LayerInputs(shape, x, Wr, br, W1, b1, W2, b2, W1s, W2s, redrawn)


def make_custom(T, D, E, k, I, seed=0, device="cpu", wfmt="bf16", reject=None,
                x_std=1.0) -> LayerInputs:
    """Inputs of arbitrary sizes with the standard distributions (edge cases)."""
    shape = LayerShape("custom", T=T, D=D, E=E, k=k, I=I, wfmt=wfmt)
    inp = make_inputs(shape, seed=seed, device=device, reject=reject)
    if x_std != 1.0:
        inp.x = (inp.x.float() * x_std).to(BF16)
    return inp
