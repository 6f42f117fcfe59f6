"""The C-ABI library: it builds, loads, exports every symbol include/moe.h
declares, and its host-side logic (size validation, workspace sizing,
synchronous argument errors) works without a GPU."""
import ctypes
import os
import re

import pytest

import mixture_experts_ffn_layer_b200 as moe
from mixture_experts_ffn_layer_b200 import _binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = moe.load()
    names = _declared()
    assert len(names) >= 12
    assert sorted(_binding.EXPORTS) == names
    for n in names:
        assert hasattr(lib, n), n
    # nothing but the C ABI is exported
    out = os.popen(f"nm -D --defined-only {_binding.LIB_PATH}").read()
    exported = sorted(set(re.findall(r" T (moe_\w+)", out)))
    assert exported == names


def test_check_dims_supported_set():
    ok = moe.dims(8192, 2880, 32, 4, 2880)
    assert moe.check_dims(ok) == 0
    assert moe.check_dims(moe.dims(0, 64, 4, 2, 64)) == 1  # T = 0
    assert moe.check_dims(moe.dims(8, 64, 4, 5, 64)) == 1  # k > E
    assert moe.check_dims(moe.dims(8, 64, 4, 2, 64, wfmt=7)) == 1
    assert moe.check_dims(moe.dims(8, 64, 300, 2, 64)) == 2  # E > 256
    assert moe.check_dims(moe.dims(8, 64, 16, 9, 64)) == 2  # k > 8
    assert moe.check_dims(moe.dims(8, 96, 4, 2, 64)) == 2  # D % 64
    assert moe.check_dims(moe.dims(8, 64, 4, 2, 100)) == 2  # I % 64
    # activation: plain SwiGLU or the GPT-OSS variant with a finite alpha and a limit > 0 (inf allowed)
    G = moe.MOE_ACT_GPTOSS
    assert moe.check_dims(moe.dims(8, 64, 4, 2, 64, act=G, act_alpha=1.702, act_limit=7.0)) == 0
    assert moe.check_dims(moe.dims(8, 64, 4, 2, 64, act=G, act_alpha=1.0, act_limit=float("inf"))) == 0
    assert moe.check_dims(moe.dims(8, 64, 4, 2, 64, act=2)) == 1
    assert moe.check_dims(moe.dims(8, 64, 4, 2, 64, act=G, act_alpha=float("nan"), act_limit=7.0)) == 1
    assert moe.check_dims(moe.dims(8, 64, 4, 2, 64, act=G, act_alpha=1.0, act_limit=0.0)) == 1
    assert moe.check_dims(moe.dims(8, 64, 4, 2, 64, act=G, act_alpha=1.0, act_limit=float("nan"))) == 1


def test_workspace_bytes_cover_the_decode_paths():
    # 64 tokens at the 20B shape: the router splits K over 45 CTAs (fp32
    # partial logits, splits * T * E); MXFP4 weights add the block-scaled
    # GEMMs' operands -- routed rows and h as hi/lo E4M3 pairs and their
    # scales -- and never an expanded copy of the weights
    T, D, E, k, I = 64, 2880, 32, 4, 2880
    R = T * k
    base = R * D * (2 + 4) + R * I * 2 + R * 4 * 4
    splits = 45
    n = moe.workspace_bytes(moe.dims(T, D, E, k, I))
    assert base + splits * T * E * 4 <= n <= base + splits * T * E * 4 + 1024 * 1024
    nq = moe.workspace_bytes(moe.dims(T, D, E, k, I, wfmt=moe.MOE_W_MXFP4))
    mtiles = -(-R // 128) + E
    sf = mtiles * -(-D // 128) * 2048 + mtiles * -(-I // 128) * 2048  # 2 KB of scales per (128-row tile, 128-K stage)
    # the weights' scales in the MMA's atom layout for both kernels (mlp1: E x
    # 30 column tiles x 23 stages x 1 KB, E x 45 weight tiles x 23 stages x
    # 512 B) and the padded last 64 codes of every mlp1 weight row
    nst = -(-D // 128)
    prep = E * (I // 96) * nst * 1024 + E * (I // 64) * nst * 512 + E * 2 * I * 64
    assert R * (D + I) * 2 + sf + prep <= nq - n <= R * (D + I) * 2 + sf + prep + 8192
    assert nq - n < 128 * 1024 * 1024  # no expanded weights (1.59 GB at this shape)


def test_workspace_bytes_covers_intermediates():
    d = moe.dims(8192, 2880, 32, 4, 2880)
    R = 8192 * 4
    n = moe.workspace_bytes(d)
    need = R * 2880 * (2 + 2 + 4) + R * 4 * 4  # x_perm, h (bf16), o_perm (fp32) + idx, w, perm, inv
    assert need <= n <= need + 4 * 1024 * 1024
    dq = moe.dims(8192, 2880, 32, 4, 2880, wfmt=moe.MOE_W_MXFP4)
    extra = moe.workspace_bytes(dq) - n
    assert R * 2880 * 4 <= extra <= R * 2880 * 4 + 128 * 1024 * 1024  # hi/lo operands + scales, no weight copies
    with pytest.raises(moe.MoeError):
        moe.workspace_bytes(moe.dims(8, 64, 4, 5, 64))


class _Arena:
    """Addresses for the argument-error tests. On a machine with a GPU every
    address lies inside one real device buffer large enough for the tiny
    layer below (so even a check that regressed could only touch memory that
    exists); on a machine without one no kernel can run at all, and plain
    integers stand in for device addresses."""

    def __init__(self, size=32 << 20):
        import torch

        self.SIZE = size
        if torch.cuda.is_available():
            self.buf = torch.zeros(self.SIZE, dtype=torch.uint8, device="cuda")
            self.base = self.buf.data_ptr()
        else:
            self.buf = None
            self.base = 1 << 32
        self.next = 0

    def take(self, nbytes=1 << 20):
        """A 256-byte aligned address with `nbytes` of the buffer behind it."""
        at = self.next
        self.next += (nbytes + 255) // 256 * 256
        assert self.next <= self.SIZE
        return self.base + at


def test_argument_errors_are_synchronous():
    lib = moe.load()
    d = moe.dims(64, 64, 4, 2, 64)
    ar = _Arena()
    vp = ctypes.c_void_p
    ws_n = moe.workspace_bytes(d)
    ws = vp(ar.take(ws_n))
    p = [vp(ar.take()) for _ in range(8)]  # each 1 MB: more than any tensor of this layer
    mis8 = vp(ar.take() + 8)  # inside the buffer, not 32-byte aligned
    assert lib.moe_route(d, None, p[0], p[1], p[2], p[3], ws, ws_n, None) == 1
    assert lib.moe_route(d, mis8, p[0], p[1], p[2], p[3], ws, ws_n, None) == 1  # misaligned x
    assert lib.moe_route(d, p[0], p[1], p[2], p[3], p[4], ws, 16, None) == 3  # workspace too small
    assert lib.moe_permute(d, p[0], p[1], p[2], p[3], p[4], ws, 16, None) == 3
    assert lib.moe_permute(d, p[0], p[1], p[2], p[3], p[4], vp(ar.take() + 4), ws_n, None) == 1  # misaligned ws
    w = _binding.Weight(None, None)
    assert lib.moe_mlp1(d, p[0], p[1], w, p[2], p[3], ws, ws_n, None) == 1
    dq = moe.dims(64, 64, 4, 2, 64, wfmt=moe.MOE_W_MXFP4)
    wsq_n = moe.workspace_bytes(dq)
    wsq = vp(ar.take(wsq_n))
    wq = _binding.Weight(p[5].value, None)  # MXFP4 without scales
    assert lib.moe_mlp1(dq, p[0], p[1], wq, p[2], p[3], wsq, wsq_n, None) == 1
    wq_mis = _binding.Weight(p[5].value, p[6].value + 16)  # scales not 32-byte aligned
    assert lib.moe_mlp1(dq, p[0], p[1], wq_mis, p[2], p[3], wsq, wsq_n, None) == 1
    assert lib.moe_mlp2(dq, p[0], p[1], p[2], p[3], wq_mis, p[4], p[7], wsq, wsq_n, None) == 1
    # the GPT-OSS activation with an invalid limit fails every entry point's dims check
    dbad = moe.dims(64, 64, 4, 2, 64, act=moe.MOE_ACT_GPTOSS, act_alpha=1.0, act_limit=-1.0)
    assert lib.moe_mlp1(dbad, p[0], p[1], _binding.Weight(p[5].value, None), p[2], p[3], ws, ws_n, None) == 1
    assert lib.moe_forward(moe.dims(64, 64, 4, 9, 64), p[0], p[1], p[2], w, p[3], w, p[4], p[5], ws, 0, None) == 1
    assert lib.moe_read_device_status(None, None) == 1
    assert lib.moe_selftest_wait_timeout(None, 1000, None) == 1
    assert lib.moe_selftest_wait_timeout(ws, 0, None) == 1
    assert lib.moe_selftest_wait_timeout(ws, 3_000_000_000, None) == 1
    assert moe.status_str(6) == "device: index or offset out of range"


def test_noalloc_permute_size_limit_boundary():
    # The workspace-free permutation keeps one int32 per (block of 2048
    # assignments, expert) in a fixed 65536-entry array: exactly 65536 entries
    # are accepted (checked on the GPU against the oracle in its own test
    # file), one block more is refused before anything is enqueued.
    lib = moe.load()
    ar = _Arena(80 << 20)  # the largest case's perm array is 67 MB
    vp = ctypes.c_void_p
    for T, E, k in [(256 * 2048 + 1, 256, 1), (2048 * 2048 + 1, 32, 1), (8192 * 2048 // 4 + 1, 8, 4)]:
        blocks = -(-(T * k) // 2048)
        assert blocks * E == 65536 + E
        d = moe.dims(T, 64, E, k, 64)
        assert lib.moe_permute_noalloc(d, *[vp(ar.base)] * 5, None) == 2
    # invalid dims are refused by the dims check first
    assert lib.moe_permute_noalloc(moe.dims(8, 64, 4, 5, 64), *[vp(ar.base)] * 5, None) == 1
    assert lib.moe_permute_noalloc(moe.dims(8, 64, 4, 2, 64), None, *[vp(ar.base)] * 4, None) == 1


def test_mxfp4_prepare_arguments():
    # the prepare-once form of an MXFP4 weight: sizes for each weight, and
    # synchronous refusals (bf16 weights, an unknown weight, a null pointer,
    # a short buffer, a prepared form on a bf16 call)
    lib = moe.load()
    dq = moe.dims(64, 2880, 32, 4, 2880, wfmt=moe.MOE_W_MXFP4)
    n1, n2 = moe.mxfp4_prepared_bytes(dq, 1), moe.mxfp4_prepared_bytes(dq, 2)
    nst = -(-2880 // 128)
    # scale atoms of both kernels, then the codes K-block-major (every block of
    # 128 K padded to 64 bytes per row)
    assert n1 >= 32 * 30 * nst * 1024 + 32 * 45 * nst * 512 + 32 * nst * 5760 * 64
    assert n2 >= 32 * 12 * nst * 1024 + 32 * 23 * nst * 512 + 32 * nst * 2880 * 64
    assert moe.mxfp4_prepared_bytes(moe.dims(64, 2880, 32, 4, 2880), 1) == 0  # bf16 weights
    assert moe.mxfp4_prepared_bytes(dq, 3) == 0
    ar = _Arena(n1 + (64 << 20))
    vp = ctypes.c_void_p
    w = _binding.Weight(ar.take(), ar.take(), None)
    out = vp(ar.take(n1))
    assert lib.moe_mxfp4_prepare(moe.dims(64, 2880, 32, 4, 2880), 1, w, out, n1, None) == 1
    assert lib.moe_mxfp4_prepare(dq, 3, w, out, n1, None) == 1
    assert lib.moe_mxfp4_prepare(dq, 1, w, None, n1, None) == 1
    assert lib.moe_mxfp4_prepare(dq, 1, w, vp(ar.take() + 32), n1, None) == 1  # not 256-byte aligned
    assert lib.moe_mxfp4_prepare(dq, 1, _binding.Weight(ar.take(), None, None), out, n1, None) == 1  # no scales
    assert lib.moe_mxfp4_prepare(dq, 1, w, out, n1 - 1, None) == 3
    d = moe.dims(64, 64, 4, 2, 64)
    ws_n = moe.workspace_bytes(d)
    ws = vp(ar.take(ws_n))
    wp = _binding.Weight(ar.take(), None, ar.take())  # prepared form on bf16 weights
    assert lib.moe_mlp1(d, vp(ar.take()), vp(ar.take()), wp, vp(ar.take()), vp(ar.take()), ws, ws_n, None) == 1
