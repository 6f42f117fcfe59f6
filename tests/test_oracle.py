"""Pins of the CPU oracle against things other than itself: hand-derived
golden examples, closed forms, library reductions (torch softmax, a dense
SwiGLU MLP written with torch.nn.functional), dense-mask brute force,
invariants and exact special cases. CPU only."""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
BF16 = torch.bfloat16


def bf16(a):
    return torch.as_tensor(np.asarray(a, dtype=np.float32)).to(BF16)


# ---------------------------------------------------------------- rounding
def test_round_bf16_matches_torch_on_float32_values():
    g = torch.Generator().manual_seed(0)
    v = torch.randn(200000, generator=g) * torch.exp(torch.randn(200000, generator=g) * 20)
    v = torch.cat([v, torch.tensor([0.0, -0.0, 1e-40, -3e-39, 3.3e38, -3.39e38, float("inf"), float("-inf")])])
    ours = oracle.round_bf16(v.double())
    ref = v.to(BF16)  # float32 -> bf16 is a single RNE rounding in torch
    assert torch.equal(ours.view(torch.int16), ref.view(torch.int16))


def test_round_bf16_ties_and_single_rounding():
    cases = {
        1 + 2.0 ** -8: 1.0,  # halfway, ties to even (down)
        1 + 3 * 2.0 ** -8: 1 + 2.0 ** -6,  # halfway, ties to even (up)
        1 + 2.0 ** -8 + 2.0 ** -40: 1 + 2.0 ** -7,  # just above halfway: a float first step would lose this
        -(1 + 2.0 ** -8 + 2.0 ** -40): -(1 + 2.0 ** -7),
        2.0 ** -133: 2.0 ** -133,  # smallest bf16 subnormal
        2.0 ** -134: 0.0,  # halfway to the smallest subnormal -> even (0)
    }
    inp = torch.tensor(list(cases.keys()), dtype=torch.float64)
    out = oracle.round_bf16(inp).double()
    assert out.tolist() == list(cases.values())


# ---------------------------------------------------------------- golden
def _golden_inputs(ex):
    x, Wr, br = bf16(ex["x"]), bf16(ex["Wr"]), bf16(ex["br"])
    W1, b1, W2, b2 = bf16(ex["W1"]), bf16(ex["b1"]), bf16(ex["W2"]), bf16(ex["b2"])
    return x, Wr, br, W1, b1, W2, b2


@pytest.mark.parametrize("name", ["top1_swiglu", "top2_softmax", "tie_lower_index"])
def test_golden_worked_examples(name):
    data = json.load(open(os.path.join(GOLDEN, "worked_examples.json")))
    ex = next(e for e in data["examples"] if e["name"] == name)
    x, Wr, br, W1, b1, W2, b2 = _golden_inputs(ex)
    y, idx, w = oracle.forward(x, Wr, br, W1, b1, W2, b2, ex["k"])
    assert idx.tolist() == ex["topk_idx"]
    np.testing.assert_allclose(w.numpy(), np.asarray(ex["topk_w"]), rtol=1e-7, atol=0)
    assert y.float().tolist() == ex["y"]


def test_e2m1_table():
    data = json.load(open(os.path.join(GOLDEN, "e2m1_table.json")))
    for s_str, scale in data["scales"].items():
        s = int(s_str)
        codes = torch.tensor([[c | (c << 4) for c in range(0, 16, 1)] * 2], dtype=torch.uint8)  # 32 bytes = 64 values
        codes = codes[:, :32]
        scales = torch.full((1, 2), s, dtype=torch.uint8)
        vals = oracle.dequant_mxfp4(codes, scales)[0]
        for i in range(64):
            code = i // 2 % 16
            expect = data["codes"][str(code)] * scale
            assert vals[i].item() == expect, (s, i, code)
            if code == 8:
                assert math.copysign(1.0, vals[i].item()) == -1.0


# ---------------------------------------------------------------- router
def _rank_mask(logits64_f32, k):
    """Dense brute force: expert e is chosen iff fewer than k experts beat it
    under (logit desc, index asc)."""
    L = logits64_f32
    T, E = L.shape
    mask = np.zeros((T, E), dtype=bool)
    rank = np.zeros((T, E), dtype=np.int64)
    for e in range(E):
        beats = (L > L[:, e:e + 1]) | ((L == L[:, e:e + 1]) & (np.arange(E)[None, :] < e))
        rank[:, e] = beats.sum(axis=1)
    mask = rank < k
    return mask, rank


@pytest.mark.parametrize("T,D,E,k", [(37, 48, 6, 2), (16, 64, 4, 4), (50, 32, 16, 5), (9, 8, 3, 1)])
def test_route_matches_dense_mask_brute_force(T, D, E, k):
    inp = synthetic.make_custom(T, D, E, k, 8, seed=T + D)
    logits, idx, w = oracle.route(inp.x, inp.Wr, inp.br, k)
    L = inp.x.double().numpy() @ inp.Wr.double().numpy().T + inp.br.double().numpy()[None, :]
    np.testing.assert_allclose(logits.numpy(), L, rtol=1e-6, atol=1e-6)
    Lf = logits.numpy().astype(np.float64)
    mask, rank = _rank_mask(Lf, k)
    # softmax restricted to the chosen experts (others get -inf)
    masked = np.where(mask, Lf, -np.inf)
    p = np.exp(masked - masked.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    for t in range(T):
        chosen = sorted(np.nonzero(mask[t])[0], key=lambda e: rank[t, e])
        assert idx[t].tolist() == chosen
        np.testing.assert_allclose(w[t].numpy(), p[t, chosen], rtol=2e-7, atol=1e-9)


def test_route_k_equals_E_is_plain_softmax():
    inp = synthetic.make_custom(64, 32, 8, 8, 8, seed=3)
    logits, idx, w = oracle.route(inp.x, inp.Wr, inp.br, 8)
    ref = torch.softmax(logits.double(), dim=1)
    for t in range(64):
        np.testing.assert_allclose(w[t].numpy(), ref[t, idx[t].long()].numpy(), rtol=2e-7)
        assert sorted(idx[t].tolist()) == list(range(8))


def test_route_exact_ties_pick_lower_index():
    # integer-valued inputs; duplicated router rows make exact ties
    T, D, E, k = 12, 4, 6, 3
    g = torch.Generator().manual_seed(5)
    x = torch.randint(-3, 4, (T, D), generator=g).to(BF16)
    base = torch.randint(-2, 3, (3, D), generator=g)
    Wr = torch.cat([base, base]).to(BF16)  # expert e and e+3 share weights
    br = torch.zeros(E, dtype=BF16)
    logits, idx, w = oracle.route(x, Wr, br, k)
    L = logits.double().numpy()
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-L[t, e], e))[:k]
        assert idx[t].tolist() == order
        for j in range(k - 1):
            if L[t, idx[t, j]] == L[t, idx[t, j + 1]]:
                assert idx[t, j] < idx[t, j + 1]
                assert w[t, j] == w[t, j + 1]


def test_route_invariants():
    inp = synthetic.make_inputs("debug", T=512)
    logits, idx, w = oracle.route(inp.x, inp.Wr, inp.br, 2)
    assert torch.all((idx >= 0) & (idx < 8))
    assert all(len(set(r)) == 2 for r in idx.tolist())
    np.testing.assert_allclose(w.double().sum(1).numpy(), 1.0, atol=1e-6)
    assert torch.all(w[:, 0] >= w[:, 1])
    # the chosen logits are the two largest
    top = torch.topk(logits, 2, dim=1).values
    assert torch.equal(torch.gather(logits, 1, idx.long()), top)


# ---------------------------------------------------------------- permutation
@pytest.mark.parametrize("T,E,k", [(100, 7, 3), (1, 4, 4), (257, 16, 2), (64, 128, 4)])
def test_permute_is_stable_sort_by_expert(T, E, k):
    g = torch.Generator().manual_seed(T * E)
    idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32)
    counts, offsets, perm, inv = oracle.permute(idx, E)
    flat = idx.flatten().numpy()
    ref_perm = np.argsort(flat, kind="stable")
    assert perm.numpy().tolist() == ref_perm.tolist()
    assert counts.numpy().tolist() == np.bincount(flat, minlength=E).tolist()
    assert offsets.numpy().tolist() == [0] + np.cumsum(np.bincount(flat, minlength=E)).tolist()
    assert int(counts.sum()) == T * k
    assert torch.equal(inv[perm.long()], torch.arange(T * k, dtype=torch.int32))
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]].numpy()
        assert np.all(np.diff(seg) > 0)
        assert np.all(flat[seg] == e)


def test_permute_rejects_out_of_range_index():
    idx = torch.tensor([[0, 5]], dtype=torch.int32)
    with pytest.raises(ValueError):
        oracle.permute(idx, 4)


# ---------------------------------------------------------------- expert FFN
def _dense_swiglu_reference(x, W1, b1, W2, b2, I):
    """A dense SwiGLU MLP with torch.nn.functional (float64), h rounded to bf16."""
    u = F.linear(x.double(), W1.double(), b1.double())
    h = (F.silu(u[:, :I]) * u[:, I:]).float().to(BF16).double()
    return F.linear(h, W2.double(), b2.double())


def test_ffn_single_expert_is_dense_swiglu_mlp():
    T, D, I = 24, 64, 48
    inp = synthetic.make_custom(T, D, 1, 1, I, seed=11)
    y, idx, w = oracle.forward(inp.x, inp.Wr, inp.br, inp.W1, inp.b1, inp.W2, inp.b2, 1)
    assert torch.all(idx == 0) and torch.all(w == 1.0)
    ref = _dense_swiglu_reference(inp.x, inp.W1[0], inp.b1[0], inp.W2[0], inp.b2[0], I)
    # one bf16 rounding of y (and h rounding through float here) -> within 2 bf16 ulps
    np.testing.assert_allclose(y.double().numpy(), ref.numpy(), rtol=2 ** -7, atol=1e-6)


@pytest.mark.parametrize("T,D,E,k,I", [(20, 32, 5, 2, 16), (8, 64, 3, 3, 32)])
def test_ffn_matches_dense_all_expert_brute_force(T, D, E, k, I):
    inp = synthetic.make_custom(T, D, E, k, I, seed=7 * T + E, reject=oracle.gap_reject())
    y, o = None, None
    logits, idx, w = oracle.route(inp.x, inp.Wr, inp.br, k)
    y, o = oracle.ffn_tokens(inp.x, idx, w, inp.W1, inp.b1, inp.W2, inp.b2, return_o=True)
    # brute force: every expert on every token, then a dense gate mask
    mask, rank = _rank_mask(logits.double().numpy(), k)
    gate = np.zeros((T, E))
    for t in range(T):
        for j in range(k):
            gate[t, idx[t, j]] = w[t, j].item()
    assert np.all((gate > 0) == mask)
    y_dense = np.zeros((T, D))
    for e in range(E):
        o_e = _dense_swiglu_reference(inp.x, inp.W1[e], inp.b1[e], inp.W2[e], inp.b2[e], I).numpy()
        y_dense += gate[:, e:e + 1] * o_e
        for t in range(T):
            for j in range(k):
                if idx[t, j] == e:
                    np.testing.assert_allclose(o[t, j].numpy(), o_e[t], rtol=1e-2, atol=1e-5)
    np.testing.assert_allclose(y.double().numpy(), y_dense, rtol=2 ** -7, atol=1e-5)


def test_exact_output_rounds_to_output():
    T, D, E, k, I = 16, 64, 4, 2, 32
    inp = synthetic.make_custom(T, D, E, k, I, seed=12)
    _, idx, w = oracle.route(inp.x, inp.Wr, inp.br, k)
    y, o, ye = oracle.ffn_tokens(inp.x, idx, w, inp.W1, inp.b1, inp.W2, inp.b2, return_o=True, return_exact=True)
    assert torch.equal(oracle.round_bf16(ye).view(torch.int16), y.view(torch.int16))
    # y_exact is the gate-weighted sum of the expert outputs
    ref = (w.double()[:, :, None] * o).sum(1)
    assert torch.allclose(ye, ref, rtol=1e-14, atol=1e-15)


def test_w2_zero_gives_weighted_bias_sum():
    T, D, E, k, I = 16, 32, 6, 3, 16
    inp = synthetic.make_custom(T, D, E, k, I, seed=2)
    W2 = torch.zeros_like(inp.W2)
    y, idx, w = oracle.forward(inp.x, inp.Wr, inp.br, inp.W1, inp.b1, W2, inp.b2, k)
    ref = (w.double()[:, :, None] * inp.b2.double()[idx.long()]).sum(1)
    assert torch.equal(y, oracle.round_bf16(ref))


def test_equivariance_under_token_and_expert_relabelling():
    T, D, E, k, I = 24, 32, 6, 2, 16
    inp = synthetic.make_custom(T, D, E, k, I, seed=9, reject=oracle.gap_reject())
    y, idx, w = oracle.forward(inp.x, inp.Wr, inp.br, inp.W1, inp.b1, inp.W2, inp.b2, k)
    pt = torch.randperm(T, generator=torch.Generator().manual_seed(1))
    y2, _, _ = oracle.forward(inp.x[pt], inp.Wr, inp.br, inp.W1, inp.b1, inp.W2, inp.b2, k)
    assert torch.equal(y2, y[pt])
    pe = torch.randperm(E, generator=torch.Generator().manual_seed(2))
    y3, idx3, _ = oracle.forward(inp.x, inp.Wr[pe], inp.br[pe], inp.W1[pe], inp.b1[pe], inp.W2[pe], inp.b2[pe], k)
    assert torch.equal(y3, y)
    assert torch.equal(pe[idx3.long()].int(), idx)


# ---------------------------------------------------------------- MXFP4
def test_mxfp4_layer_equals_bf16_layer_with_dequantized_weights():
    T, D, E, k, I = 16, 64, 4, 2, 64
    inp = synthetic.make_custom(T, D, E, k, I, seed=4, wfmt="mxfp4")
    y4, idx4, w4 = oracle.forward(inp.x, inp.Wr, inp.br, inp.W1, inp.b1, inp.W2, inp.b2, k,
                                  W1_scales=inp.W1_scales, W2_scales=inp.W2_scales)
    W1d = torch.stack([oracle.dequant_mxfp4(inp.W1[e], inp.W1_scales[e]) for e in range(E)])
    W2d = torch.stack([oracle.dequant_mxfp4(inp.W2[e], inp.W2_scales[e]) for e in range(E)])
    W1b, W2b = W1d.to(BF16), W2d.to(BF16)
    assert torch.equal(W1b.double(), W1d) and torch.equal(W2b.double(), W2d)  # exact in bf16
    yb, idxb, wb = oracle.forward(inp.x, inp.Wr, inp.br, W1b, inp.b1, W2b, inp.b2, k)
    assert torch.equal(idx4, idxb)
    assert torch.equal(y4.view(torch.int16), yb.view(torch.int16))


def test_mxfp4_nibble_order_and_scale_blocks():
    # one row, K=64: element 2m is the low nibble of byte m; scale block b covers 32b..32b+31
    codes = torch.zeros((1, 32), dtype=torch.uint8)
    codes[0, 0] = 0x72  # element 0 -> code 2 (1.0), element 1 -> code 7 (6.0)
    codes[0, 16] = 0x0b  # element 32 -> code 11 (-1.5)
    scales = torch.tensor([[127, 125]], dtype=torch.uint8)
    v = oracle.dequant_mxfp4(codes, scales)[0]
    assert v[0].item() == 1.0 and v[1].item() == 6.0 and v[32].item() == -1.5 * 0.25
    assert torch.count_nonzero(v).item() == 3


# ---- GPT-OSS SwiGLU variant (torchtitan GPT-OSS guide, paragraph on the
# grouped experts' SwiGLU variant): gate clamped from above at `limit` and
# multiplied by sigmoid(alpha * gate); up clipped to [-limit, limit], plus 1.

def _one_expert_case(T=8, D=32, I=16, seed=21, x_scale=1.0):
    g = torch.Generator().manual_seed(seed)
    x = bf16(torch.randn(T, D, generator=g) * x_scale)
    W1 = bf16(torch.randn(1, 2 * I, D, generator=g) * 0.2)
    W2 = bf16(torch.randn(1, D, I, generator=g) * 0.2)
    # biases on a 2^-6 grid in [-1/4, 1/4]: b1 + 1 is exact in bf16
    b1 = bf16(torch.randint(-16, 17, (1, 2 * I), generator=g).float() / 64)
    b2 = bf16(torch.randint(-16, 17, (1, D), generator=g).float() / 64)
    idx = torch.zeros(T, 1, dtype=torch.int32)
    w = torch.ones(T, 1)
    return x, idx, w, W1, b1, W2, b2


def test_gptoss_act_with_unit_alpha_and_no_limit_is_swiglu_with_up_offset():
    # alpha = 1, limit = inf: gc = g, uc = u, act = silu(g) * (u + 1), i.e. the
    # plain SwiGLU layer with 1 added to the up half of b1
    x, idx, w, W1, b1, W2, b2 = _one_expert_case()
    I = b1.shape[1] // 2
    b1_up = b1.clone().float()
    b1_up[:, I:] += 1.0
    _, y_var = oracle.ffn_tokens(x, idx, w, W1, b1, W2, b2, return_exact=True, act=(oracle.ACT_GPTOSS, 1.0, math.inf))
    _, y_ref = oracle.ffn_tokens(x, idx, w, W1, bf16(b1_up), W2, b2, return_exact=True)
    assert torch.equal(bf16(b1_up).float(), b1_up)  # the offset bias is exact
    rms = y_ref.pow(2).mean().sqrt()
    assert float((y_var - y_ref).abs().max()) <= 1e-3 * float(rms)
    # and it is not the plain layer (the +1 is there)
    _, y_plain = oracle.ffn_tokens(x, idx, w, W1, b1, W2, b2, return_exact=True)
    assert float((y_var - y_plain).abs().max()) > 0.1 * float(rms)


def test_gptoss_act_with_huge_alpha_is_clamped_relu_glu():
    # alpha -> inf turns sigmoid(alpha * gc) into a step: act = max(gc, 0) * (uc + 1)
    # (a ReLU-gated GLU), checked against a dense float64 computation
    limit = 0.75
    x, idx, w, W1, b1, W2, b2 = _one_expert_case(seed=22)
    I = b1.shape[1] // 2
    u = x.double() @ W1[0].double().T + b1[0].double()
    assert float(u[:, :I].abs().min()) > 1e-4  # alpha * |g| > 100: the sigmoid is 0 or 1 to double precision
    gc = u[:, :I].clamp(max=limit)
    uc = u[:, I:].clamp(-limit, limit)
    h = (gc.clamp(min=0) * (uc + 1)).to(torch.bfloat16).double()
    y_dense = h @ W2[0].double().T + b2[0].double()
    _, y = oracle.ffn_tokens(x, idx, w, W1, b1, W2, b2, return_exact=True, act=(oracle.ACT_GPTOSS, 1e6, limit))
    assert torch.allclose(y, y_dense, rtol=1e-12, atol=1e-12)
    assert bool((u[:, :I] > limit).any()) and bool((u[:, I:].abs() > limit).any())  # both clamps are exercised


def test_gptoss_act_clamps_gate_only_from_above():
    # W2 = identity, b2 = 0, one expert, k = 1: y is h itself (bf16). Doubling a
    # token leaves h unchanged wherever the gate is above the limit and the up
    # value outside [-limit, limit] at both scales; where the gate is below
    # -limit it is not clamped, so h changes.
    D = I = 32
    limit, alpha = 0.5, 1.702
    x, idx, w, W1, b1, _, _ = _one_expert_case(D=D, I=I, seed=23, x_scale=4.0)
    b1 = torch.zeros_like(b1)
    W2 = bf16(torch.eye(D).unsqueeze(0))
    b2 = torch.zeros(1, D, dtype=torch.bfloat16)
    act = (oracle.ACT_GPTOSS, alpha, limit)
    y1 = oracle.ffn_tokens(x, idx, w, W1, b1, W2, b2, act=act).float()
    y2 = oracle.ffn_tokens(bf16(2 * x.float()), idx, w, W1, b1, W2, b2, act=act).float()
    u = x.double() @ W1[0].double().T
    g, up = u[:, :I], u[:, I:]
    sat = (g > limit) & (up.abs() > limit)  # g > limit and |u| > limit at x, hence at 2x too
    low = g < -limit
    assert bool(sat.any()) and bool(low.any())
    assert torch.equal(y1[sat], y2[sat])
    assert bool((y1[low] != y2[low]).all())
