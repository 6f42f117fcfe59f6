"""moe_permute_noalloc: the permutation entry point for callers that cannot
allocate device memory (a host framework or serving runtime that fixes the
memory budget up front, or a latency-critical path that must not call
cudaMalloc). Its scratch is a fixed array inside the library, so this checks,
through the C ABI, that two calls in a row (different sizes, so the second
overwrites what the first left in the shared array) give exactly what the
workspace-based moe_permute gives, and that sizes beyond the array are
refused before anything is enqueued."""
import ctypes

import pytest
import torch

import mixture_experts_ffn_layer_b200 as moe

pytestmark = pytest.mark.gpu


def _routing(T, E, k, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    scores = torch.rand((T, E), generator=g, device="cuda")
    return torch.topk(scores, k, dim=1).indices.to(torch.int32).contiguous()


def _buffers(T, E, k):
    i32 = dict(dtype=torch.int32, device="cuda")
    return (torch.full((E,), -7, **i32), torch.full((E + 1,), -7, **i32), torch.full((T * k,), -7, **i32),
            torch.full((T * k,), -7, **i32))


def test_noalloc_permute_matches_workspace_permute_twice():
    for T, E, k, seed in [(5000, 32, 4, 1), (777, 8, 2, 2)]:
        idx = _routing(T, E, k, seed)
        d = moe.dims(T, 64, E, k, 64)
        ws = moe.alloc_workspace(d)
        ref = _buffers(T, E, k)
        moe.moe_permute(d, idx, *ref, ws)
        out = _buffers(T, E, k)
        moe.moe_permute_noalloc(d, idx, *out)
        torch.cuda.synchronize()
        assert moe.moe_read_device_status(ws) == 0
        for a, b in zip(out, ref):
            assert torch.equal(a, b)
        counts, offsets, perm, inv = out
        assert int(offsets[-1]) == T * k
        assert torch.equal(inv[perm.long()], torch.arange(T * k, dtype=torch.int32, device="cuda"))


def test_noalloc_permute_rejects_sizes_beyond_its_scratch():
    lib = moe.load()
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the size check comes first
    # ceil(600000 / 2048) * 256 = 75008 histogram entries > 65536
    d = moe.dims(600000, 64, 256, 1, 64)
    assert lib.moe_permute_noalloc(d, fake, fake, fake, fake, fake, None) == 2
