"""Edge cases of the CUDA path against the oracle, through the C ABI:
a single expert (a dense SwiGLU MLP), k = E, one token, empty experts, exact
ties, the largest supported E and k, ragged tails, and device-side range
errors reported through the status word without faulting."""
import dataclasses

import pytest
import torch

import mixture_experts_ffn_layer_b200 as moe
import oracle
import synthetic
from helpers import TOL_BF16, TOL_MXFP4, assert_close_rms, dims_of, run_forward, run_stages

pytestmark = pytest.mark.gpu

BF16 = torch.bfloat16


def _check_full(inp, tol=TOL_BF16, act=None):
    act = act or (moe.MOE_ACT_SWIGLU, 1.0, float("inf"))
    run = run_stages(inp, act)
    assert run.status == 0, moe.status_str(run.status)
    s = inp.shape
    _, idx_ref, w_ref = oracle.route(inp.x, inp.Wr, inp.br, s.k)
    assert torch.equal(run.topk_idx.cpu(), idx_ref)
    assert float((run.topk_w.cpu() - w_ref).abs().max()) <= 1e-5
    counts, offsets, perm, inv = oracle.permute(idx_ref, s.E)
    for a, b in ((run.counts, counts), (run.offsets, offsets), (run.perm, perm), (run.inv, inv)):
        assert torch.equal(a.cpu(), b)
    _, y_ref = oracle.ffn_tokens(inp.x, idx_ref, w_ref, inp.W1, inp.b1, inp.W2, inp.b2, return_exact=True,
                                 W1_scales=inp.W1_scales, W2_scales=inp.W2_scales, act=act)
    assert_close_rms(run.y, y_ref, tol)
    return run


@pytest.mark.parametrize("T,D,E,k,I", [
    (300, 64, 1, 1, 64),     # one expert: a dense SwiGLU MLP, ragged 300-row tail
    (130, 128, 4, 4, 192),   # k = E: every token visits every expert
    (1, 256, 8, 2, 128),     # one token
    (517, 192, 256, 8, 64),  # largest supported E and k
    (1000, 64, 3, 2, 320),   # non-power-of-two E, N tiles of 64 / 160
    (4200, 128, 4, 2, 192),  # >= 2048 rows per expert: SM-pair (256-row) GEMM tiles
    (8500, 64, 2, 1, 128),   # pair tiles, ragged segments
])
def test_shapes(T, D, E, k, I):
    inp = synthetic.make_custom(T, D, E, k, I, seed=T + E, device="cuda", reject=oracle.gap_reject())
    _check_full(inp)


@pytest.mark.parametrize("T,D,E,k,I", [
    (8, 64, 4, 2, 64),      # one 64-element K step, a partial 128-row weight block
    (40, 192, 8, 2, 320),   # three K steps, 2.5 weight blocks per expert
    (1, 128, 32, 4, 64),    # one token
    (96, 256, 24, 1, 192),  # non-power-of-two E
    (100, 128, 256, 8, 128),  # largest E and k: ~3 rows per expert, some experts empty
])
def test_mxfp4_small_batch_shapes(T, D, E, k, I):
    # a few routed rows per expert (decode-like): most of each 128-row tile is padding
    inp = synthetic.make_custom(T, D, E, k, I, seed=T + 7 * E, device="cuda", wfmt="mxfp4",
                                reject=oracle.gap_reject())
    _check_full(inp, TOL_MXFP4)


def test_mxfp4_hot_expert_several_tiles():
    # one expert takes most tokens: its rows span several 128-row tiles, the
    # last one ragged, while the other experts keep a few rows
    T, D, E, k, I = 400, 128, 16, 2, 128
    base = synthetic.make_custom(T, D, E, k, I, seed=11, wfmt="mxfp4")
    br = torch.zeros(E)
    br[5] = 6.0
    br = br.to(BF16)
    keep = ~oracle.gap_reject()(base.x, base.Wr, br, k)
    x = base.x[keep].contiguous()
    shape = synthetic.LayerShape("custom", x.shape[0], D, E, k, I, wfmt="mxfp4")
    inp = dataclasses.replace(base, shape=shape, x=x, br=br).to("cuda")
    run = _check_full(inp, TOL_MXFP4)
    assert int(run.counts.max()) > 256


@pytest.mark.parametrize("T,D,E,k,I,wfmt", [
    (512, 256, 8, 2, 512, "bf16"),   # single-SM tcgen05 GEMM tiles
    (4200, 128, 4, 2, 192, "bf16"),  # SM-pair GEMM tiles
    (40, 192, 8, 2, 320, "mxfp4"),   # MXFP4, block-scaled MMA, a few rows per expert
    (600, 128, 4, 2, 128, "mxfp4"),  # MXFP4, block-scaled MMA, several tiles per expert
])
def test_gptoss_activation(T, D, E, k, I, wfmt):
    # the GPT-OSS SwiGLU variant in every mlp1 epilogue; a small limit so that
    # both clamps act on a good share of the elements
    act = (moe.MOE_ACT_GPTOSS, 1.702, 0.25)
    inp = synthetic.make_custom(T, D, E, k, I, seed=T + 3 * E, device="cuda", wfmt=wfmt, reject=oracle.gap_reject())
    _check_full(inp, TOL_MXFP4 if wfmt == "mxfp4" else TOL_BF16, act=act)


@pytest.mark.parametrize("T,D,E,k,I", [
    (600, 128, 4, 2, 128),
    (1024, 256, 8, 4, 192),
    (40, 192, 8, 2, 320),
    (64, 2880, 32, 4, 2880),
])
def test_forward_mxfp4_matches_stages(T, D, E, k, I):
    # the one-call MXFP4 path (the gather writes the hi/lo E4M3 operands, mlp1
    # writes h in that form) is bitwise the staged path (bf16 x_perm and h,
    # each quantised by its own pass), call after call
    inp = synthetic.make_custom(T, D, E, k, I, seed=T + E, device="cuda", wfmt="mxfp4", reject=oracle.gap_reject())
    run = run_stages(inp)
    assert run.status == 0
    y1 = run_forward(inp)
    y2 = run_forward(inp)
    assert torch.equal(y1.view(torch.int16), run.y.view(torch.int16))
    assert torch.equal(y2.view(torch.int16), y1.view(torch.int16))


@pytest.mark.parametrize("T,D,E,k,I", [
    (64, 2880, 32, 4, 2880),  # decode-sized: the small-expert kernel
    (600, 128, 4, 2, 192),    # several 128-row tiles per expert: the big-tile kernel
    (300, 192, 16, 2, 320),   # both kernels in one call (hot and cold experts), ragged K
])
def test_mxfp4_prepared_weights_match_per_call(T, D, E, k, I):
    # weights prepared once (moe_mxfp4_prepare) give bitwise the result of the
    # per-call preparation, through the staged and the one-call entry points
    inp = synthetic.make_custom(T, D, E, k, I, seed=T + 5 * E, device="cuda", wfmt="mxfp4", reject=oracle.gap_reject())
    if T == 300:
        br = torch.zeros(E)
        br[2] = 3.0
        inp.br = br.to(BF16).to("cuda")
    run = run_stages(inp)
    assert run.status == 0
    d = dims_of(inp)
    p1 = moe.mxfp4_prepare(d, 1, inp.W1, inp.W1_scales)
    p2 = moe.mxfp4_prepare(d, 2, inp.W2, inp.W2_scales)
    s = inp.shape
    ws = moe.alloc_workspace(d)
    h = torch.empty((s.T * s.k, s.I), dtype=BF16, device="cuda")
    o = torch.empty((s.T * s.k, s.D), dtype=torch.float32, device="cuda")
    moe.moe_mlp1(d, run.x_perm, run.offsets, inp.W1, inp.b1, h, ws, W1_scales=inp.W1_scales, W1_prepared=p1)
    moe.moe_mlp2(d, h, run.perm, run.offsets, run.topk_w, inp.W2, inp.b2, o, ws, W2_scales=inp.W2_scales,
                 W2_prepared=p2)
    assert moe.moe_read_device_status(ws) == 0
    assert torch.equal(h.view(torch.int16), run.h.view(torch.int16))
    assert torch.equal(o, run.o_perm)
    # with the prepared forms the GEMMs read nothing else: codes and scales omitted
    y = torch.empty((s.T, s.D), dtype=BF16, device="cuda")
    moe.moe_forward(d, inp.x, inp.Wr, inp.br, None, inp.b1, None, inp.b2, y, ws, W1_prepared=p1, W2_prepared=p2)
    assert moe.moe_read_device_status(ws) == 0
    assert torch.equal(y.view(torch.int16), run.y.view(torch.int16))


@pytest.mark.parametrize("T", [40, 700])
def test_mxfp4_wide_weight_scales(T):
    # mlp2 weight rows whose E8M0 scales sit anywhere in a 60-binade range:
    # every block of output row dd (all experts) is offset by the same o_dd in
    # [-40, 20] binades (the synthetic workloads span 9 binades), and b2 = 0, so
    # output column dd scales with 2^o_dd. Each column must match the oracle
    # relative to its own magnitude: no block is flushed or rescaled against
    # the other rows' or blocks' scales.
    D, E, k, I = 256, 8, 2, 192
    inp = synthetic.make_custom(T, D, E, k, I, seed=T + 1, wfmt="mxfp4", reject=oracle.gap_reject())
    g = torch.Generator().manual_seed(T)
    off = torch.randint(-40, 21, (1, D, 1), generator=g)
    inp.W2_scales = (inp.W2_scales.long() + off).to(torch.uint8)
    inp.b2 = torch.zeros_like(inp.b2)
    inp = inp.to("cuda")
    run = run_stages(inp)
    assert run.status == 0
    _, idx_ref, w_ref = oracle.route(inp.x, inp.Wr, inp.br, k)
    assert torch.equal(run.topk_idx.cpu(), idx_ref)
    _, y_ref = oracle.ffn_tokens(inp.x, idx_ref, w_ref, inp.W1, inp.b1, inp.W2, inp.b2, return_exact=True,
                                 W1_scales=inp.W1_scales, W2_scales=inp.W2_scales)
    y = run.y.double().cpu()
    rms_col = y_ref.pow(2).mean(dim=0).sqrt()
    err_col = (y - y_ref).abs().max(dim=0).values
    assert bool((rms_col > 0).all())
    worst = float((err_col / rms_col).max())
    assert worst <= TOL_MXFP4, worst


@pytest.mark.parametrize("x_scale", [3.0e5, 1.0e-25])
def test_mxfp4_activation_range(x_scale):
    # routed rows far above f16's range (|x| ~ 1e6) and far below it: the
    # activations are quantised per 32-element block with their own E8M0
    # scale, so any bf16 magnitude is carried (router weights scaled back so
    # the routing is the usual one)
    T, D, E, k, I = 300, 128, 8, 2, 128
    base = synthetic.make_custom(T, D, E, k, I, seed=21, wfmt="mxfp4")
    x = (base.x.float() * x_scale).to(BF16)
    Wr = (base.Wr.float() / x_scale).to(BF16)
    keep = ~oracle.gap_reject()(x, Wr, base.br, k)
    x = x[keep].contiguous()
    shape = synthetic.LayerShape("custom", x.shape[0], D, E, k, I, wfmt="mxfp4")
    inp = dataclasses.replace(base, shape=shape, x=x, Wr=Wr).to("cuda")
    run = _check_full(inp, TOL_MXFP4)
    assert bool(torch.isfinite(run.y.float()).all())


def test_empty_experts():
    T, D, E, k, I = 200, 64, 16, 2, 64
    base = synthetic.make_custom(T, D, E, k, I, seed=3)
    # a strong bias on experts 3 and 11 leaves most experts with no rows
    br = torch.full((E,), -8.0)
    br[3] = br[11] = 8.0
    br[7] = 0.0
    br = br.to(BF16)
    keep = ~oracle.gap_reject()(base.x, base.Wr, br, k)
    x = base.x[keep].contiguous()
    shape = synthetic.LayerShape("custom", x.shape[0], D, E, k, I)
    inp = dataclasses.replace(base, shape=shape, x=x, br=br).to("cuda")
    run = _check_full(inp)
    assert int((run.counts == 0).sum()) >= 10


@pytest.mark.parametrize("D", [64, 256])  # 256: the router's K-split path (partial logits + reduce)
def test_exact_ties_pick_lower_index(D):
    T, E, k, I = 96, 6, 3, 64
    g = torch.Generator().manual_seed(5)
    x = torch.randint(-2, 3, (T, D), generator=g).to(BF16)
    base = torch.randint(-1, 2, (3, D), generator=g)
    Wr = torch.cat([base, base]).to(BF16)  # experts e and e+3 tie exactly
    inp = synthetic.make_custom(T, D, E, k, I, seed=6)
    inp.x, inp.Wr, inp.br = x, Wr, torch.zeros(E, dtype=BF16)
    inp = inp.to("cuda")
    run = run_stages(inp)
    _, idx_ref, _ = oracle.route(inp.x, inp.Wr, inp.br, k)
    assert torch.equal(run.topk_idx.cpu(), idx_ref)
    # ties are real: some token has an expert e and its twin e+3 both chosen, e first
    pairs = [(r.index(e), r.index(e + 3)) for r in idx_ref.tolist() for e in range(3) if e in r and e + 3 in r]
    assert pairs and all(a < b for a, b in pairs)


def test_out_of_range_indices_are_reported_not_faulted():
    T, E, k = 300, 8, 2
    d = moe.dims(T, 64, E, k, 64)
    ws = moe.alloc_workspace(d)
    idx = torch.randint(0, E, (T, k), dtype=torch.int32, device="cuda")
    idx[5, 1] = E + 3
    idx[77, 0] = -1
    i32 = dict(dtype=torch.int32, device="cuda")
    counts, offsets = torch.empty(E, **i32), torch.empty(E + 1, **i32)
    perm, inv = torch.empty(T * k, **i32), torch.empty(T * k, **i32)
    moe.moe_permute(d, idx, counts, offsets, perm, inv, ws)
    assert moe.moe_read_device_status(ws) == 6
    assert moe.moe_read_device_status(ws) == 0  # read clears
    assert int(inv[5 * k + 1]) == -1 and int(inv[77 * k]) == -1
    assert int(offsets[-1]) == T * k - 2


def test_bad_offsets_are_reported_and_skipped():
    T, D, E, k, I = 256, 64, 4, 2, 64
    R = T * k
    d = moe.dims(T, D, E, k, I)
    ws = moe.alloc_workspace(d)
    x_perm = torch.zeros((R, D), dtype=BF16, device="cuda")
    W1 = torch.zeros((E, 2 * I, D), dtype=BF16, device="cuda")
    b1 = torch.zeros((E, 2 * I), dtype=BF16, device="cuda")
    h = torch.full((R, I), 7.0, dtype=BF16, device="cuda")
    offsets = torch.tensor([0, 100, 50, 400, R], dtype=torch.int32, device="cuda")  # not monotone
    moe.moe_mlp1(d, x_perm, offsets, W1, b1, h, ws)
    assert moe.moe_read_device_status(ws) == 6
    assert bool((h == 7.0).all())  # nothing written


def test_bounded_wait_times_out_and_reports():
    # a wait on an mbarrier nothing arrives on gives up after 20 ms and reports
    # MOE_ERR_TIMEOUT; the context stays usable afterwards
    import time

    d = moe.dims(64, 64, 4, 2, 64)
    ws = moe.alloc_workspace(d)
    t0 = time.perf_counter()
    moe.moe_selftest_wait_timeout(ws, 20_000_000)
    assert moe.moe_read_device_status(ws) == 5
    assert 0.015 < time.perf_counter() - t0 < 1.5
    assert moe.moe_read_device_status(ws) == 0
    inp = synthetic.make_inputs("tiny", device="cuda", reject=oracle.gap_reject())
    assert run_stages(inp).status == 0


def _random_shapes(n, seed):
    g = torch.Generator().manual_seed(seed)

    def ri(lo, hi):
        return int(torch.randint(lo, hi + 1, (1,), generator=g))

    out = []
    for i in range(n):
        E = ri(1, 64)
        k = ri(1, min(8, E))
        D, I = 64 * ri(1, 7), 64 * ri(1, 7)
        T = ri(1, 320)
        wfmt = "mxfp4" if i % 2 else "bf16"
        out.append((T, D, E, k, I, wfmt))
    return out


@pytest.mark.parametrize("T,D,E,k,I,wfmt", _random_shapes(10, 2026))
def test_random_shapes(T, D, E, k, I, wfmt):
    # seeded random sizes (odd multiples of 64, odd E, k up to 8, ragged T):
    # every path the sizes select -- single-SM GEMM tiles, MXFP4 expanded or
    # streamed, the router with or without its K split -- against the oracle
    inp = synthetic.make_custom(T, D, E, k, I, seed=T * 7 + E, device="cuda", wfmt=wfmt, reject=oracle.gap_reject())
    _check_full(inp, TOL_MXFP4 if wfmt == "mxfp4" else TOL_BF16)


@pytest.mark.parametrize("T,k,E", [
    (256, 4, 32),    # T*k = 1024: the whole permutation in one block
    (205, 5, 64),    # 1025: the three-launch path
    (128, 8, 256),   # 1024 at the largest E and k
    (1, 1, 1),       # one assignment
])
def test_permutation_on_both_sides_of_the_one_block_limit(T, k, E):
    # the one-block and the multi-block permutation give the oracle's stable
    # counting sort exactly (torchtitan GPT-OSS guide, "grouped matrix
    # multiplication": counts, offsets = cumsum), with and without a workspace
    g = torch.Generator().manual_seed(T * 31 + E)
    idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32)
    counts, offsets, perm, inv = oracle.permute(idx, E)
    d = moe.dims(T, 64, E, k, 64)
    ws = moe.alloc_workspace(d)
    i32 = dict(dtype=torch.int32, device="cuda")
    for noalloc in (False, True):
        out = [torch.full((E,), -7, **i32), torch.full((E + 1,), -7, **i32), torch.full((T * k,), -7, **i32),
               torch.full((T * k,), -7, **i32)]
        if noalloc:
            moe.moe_permute_noalloc(d, idx.cuda(), *out)
        else:
            moe.moe_permute(d, idx.cuda(), *out, ws)
            assert moe.moe_read_device_status(ws) == 0
        for a, b in zip(out, (counts, offsets, perm, inv)):
            assert torch.equal(a.cpu(), b)


def test_one_block_permutation_reports_out_of_range_indices():
    T, E, k = 100, 8, 2  # T*k = 200: the one-block path
    d = moe.dims(T, 64, E, k, 64)
    ws = moe.alloc_workspace(d)
    idx = torch.randint(0, E, (T, k), dtype=torch.int32, device="cuda")
    idx[5, 1] = E
    idx[77, 0] = -3
    i32 = dict(dtype=torch.int32, device="cuda")
    counts, offsets = torch.empty(E, **i32), torch.empty(E + 1, **i32)
    perm, inv = torch.empty(T * k, **i32), torch.empty(T * k, **i32)
    moe.moe_permute(d, idx, counts, offsets, perm, inv, ws)
    assert moe.moe_read_device_status(ws) == 6
    assert int(inv[5 * k + 1]) == -1 and int(inv[77 * k]) == -1
    assert int(offsets[-1]) == T * k - 2 and int(counts.sum()) == T * k - 2
