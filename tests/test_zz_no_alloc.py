"""moe_permute_noalloc: the permutation entry point for callers that cannot
allocate device memory (a host framework or serving runtime that fixes the
memory budget up front, or a latency-critical path that must not call
cudaMalloc). Its scratch is a fixed array inside the library, so this checks,
through the C ABI, that two calls in a row (different sizes, so the second
overwrites what the first left in the shared array) give exactly what the
oracle's stable counting sort gives and what the workspace-based moe_permute
gives, and that a size that fills the whole array is still exact. Sizes one
block beyond the array are refused on the host (tests/test_abi.py)."""
import pytest
import torch

import mixture_experts_ffn_layer_b200 as moe
import oracle

pytestmark = pytest.mark.gpu


def _routing(T, E, k, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    scores = torch.rand((T, E), generator=g, device="cuda")
    return torch.topk(scores, k, dim=1).indices.to(torch.int32).contiguous()


def _buffers(T, E, k):
    i32 = dict(dtype=torch.int32, device="cuda")
    return (torch.full((E,), -7, **i32), torch.full((E + 1,), -7, **i32), torch.full((T * k,), -7, **i32),
            torch.full((T * k,), -7, **i32))


def _check(T, E, k, seed):
    idx = _routing(T, E, k, seed)
    out = _buffers(T, E, k)
    moe.moe_permute_noalloc(moe.dims(T, 64, E, k, 64), idx, *out)
    torch.cuda.synchronize()
    ref = oracle.permute(idx.cpu(), E)
    for a, b in zip(out, ref):
        assert torch.equal(a.cpu(), b)
    return idx, out


def test_noalloc_permute_matches_oracle_and_workspace_permute_twice():
    for T, E, k, seed in [(5000, 32, 4, 1), (777, 8, 2, 2)]:
        idx, out = _check(T, E, k, seed)
        d = moe.dims(T, 64, E, k, 64)
        ws = moe.alloc_workspace(d)
        ref = _buffers(T, E, k)
        moe.moe_permute(d, idx, *ref, ws)
        assert moe.moe_read_device_status(ws) == 0
        for a, b in zip(out, ref):
            assert torch.equal(a, b)


def test_noalloc_permute_at_the_scratch_limit():
    # ceil(T*k / 2048) * E = 256 * 256 = 65536: every entry of the fixed
    # array is used; then a small call reuses the array
    _check(256 * 2048 // 8, 256, 8, 3)
    _check(300, 16, 3, 4)
