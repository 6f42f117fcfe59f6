"""Expert-parallel layer: the exchange and its bookkeeping on CPU ranks.

torchtitan PR "gpt-oss model enablement" (expert parallelism with all-to-all
token dispatch) and the torchtitan GPT-OSS guide, "expert-parallel sharding".
Each rank holds E / W experts; the per-rank compute here is the oracle (a
test backend), so the layer on W gloo ranks must reproduce the oracle's
single-process layer on the same tokens bit for bit: the exchange moves rows
and sizes and never changes a value.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synthetic
from mixture_experts_ffn_layer_b200 import ep


class OracleOps:
    """LocalOps on CPU through the oracle (float64 expert outputs)."""

    def __init__(self, inp, rank, world, k):
        E = inp.Wr.shape[0]
        self.E_local = E // world
        e0 = rank * self.E_local
        sl = slice(e0, e0 + self.E_local)
        self.Wr, self.br, self.k, self.E = inp.Wr, inp.br, k, E
        self.W1, self.b1, self.W2, self.b2 = inp.W1[sl], inp.b1[sl], inp.W2[sl], inp.b2[sl]
        self.W1s = None if inp.W1_scales is None else inp.W1_scales[sl]
        self.W2s = None if inp.W2_scales is None else inp.W2_scales[sl]

    def route(self, x):
        _, idx, w = oracle.route(x, self.Wr, self.br, self.k)
        return idx, w

    def permute(self, topk_idx):
        return oracle.permute(topk_idx, self.E)

    def gather(self, x, perm):
        return x[perm.long() // self.k]

    def expert_ffn(self, rows, offsets, w):
        N, D = rows.shape
        o = torch.zeros((N, D), dtype=torch.float64)
        if N == 0:
            return o
        off = offsets.tolist()
        local = torch.zeros((N, 1), dtype=torch.int32)
        for j in range(self.E_local):
            local[off[j]:off[j + 1]] = j
        _, ou = oracle.ffn_tokens(rows, local, torch.ones((N, 1)), self.W1, self.b1, self.W2, self.b2,
                                  W1_scales=self.W1s, W2_scales=self.W2s, return_o=True)
        return w.double()[:, None] * ou[:, 0, :]

    def combine(self, o_perm, inv):
        T = inv.numel() // self.k
        y = torch.zeros((T, o_perm.shape[1]), dtype=torch.float64)
        rows = inv.long().view(T, self.k)
        for j in range(self.k):
            y += o_perm[rows[:, j]]
        return oracle.round_bf16(y)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, case, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.set_num_threads(1)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        T, D, E, k, I, wfmt, splits, hot = case
        inp = synthetic.make_custom(T, D, E, k, I, seed=11 + T, device="cpu", wfmt=wfmt, reject=oracle.gap_reject())
        if hot:
            # every token prefers experts 0 and 1: the other ranks' experts get no rows
            br = torch.zeros(E)
            br[:2] = 20.0
            inp.br = br.to(torch.bfloat16)
        bounds = [0]
        for n in splits:
            bounds.append(bounds[-1] + n)
        x = inp.x[bounds[rank]:bounds[rank + 1]]
        y = ep.ep_forward(x, OracleOps(inp, rank, world, k), E)
        torch.save(y, os.path.join(out_dir, f"y{rank}.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", [
    # T, D, E, k, I, weights, tokens per rank, hot experts
    (24, 64, 4, 2, 64, "bf16", (10, 14), False),
    (30, 64, 6, 2, 64, "bf16", (7, 0, 23), False),      # a rank with no tokens of its own
    (20, 64, 4, 2, 64, "bf16", (9, 11), True),          # rank 1's experts receive no rows
    (16, 64, 4, 2, 64, "mxfp4", (8, 8), False),
])
def test_ep_matches_single_process_layer(case, tmp_path):
    T, D, E, k, I, wfmt, splits, hot = case
    world = len(splits)
    assert sum(splits) == T
    mp.spawn(_rank_main, args=(world, _free_port(), case, str(tmp_path)), nprocs=world, join=True)
    y = torch.cat([torch.load(os.path.join(tmp_path, f"y{r}.pt")) for r in range(world)])
    inp = synthetic.make_custom(T, D, E, k, I, seed=11 + T, device="cpu", wfmt=wfmt, reject=oracle.gap_reject())
    if hot:
        br = torch.zeros(E)
        br[:2] = 20.0
        inp.br = br.to(torch.bfloat16)
    y_ref, _, _ = oracle.forward(inp.x, inp.Wr, inp.br, inp.W1, inp.b1, inp.W2, inp.b2, k,
                                 W1_scales=inp.W1_scales, W2_scales=inp.W2_scales)
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))


def test_recv_layout_orders_blocks_by_expert_then_source():
    # recv[s][j]: rows rank s sends to local expert j
    recv = [[2, 0, 1], [3, 4, 0]]
    start, off = ep.recv_layout(recv)
    assert off == [0, 5, 9, 10]
    assert start == [[0, 2], [5, 5], [9, 10]]


def test_blocks_pair_every_send_with_a_receive():
    # two ranks, E = 4 (2 local each): counts on each rank and what each receives
    counts = {0: [1, 0, 2, 3], 1: [4, 1, 0, 2]}
    world, E_local = 2, 2
    recv = {d: [[counts[s][d * E_local + j] for j in range(E_local)] for s in range(world)] for d in range(world)}
    runs = {}
    for r in range(world):
        offs = [0]
        for c in counts[r]:
            offs.append(offs[-1] + c)
        runs[r] = ep._blocks(counts[r], offs, recv[r], world, r)
    for s in range(world):
        out_runs, _ = runs[s]
        for d in range(world):
            sent = [(j, n) for dd, j, _, n in out_runs if dd == d]
            got = [(j, n) for ss, j, _, n in runs[d][1] if ss == s]
            assert sent == got  # same blocks, same order: point-to-point messages match up
    # a rank's runs cover its routed rows exactly once
    for r in range(world):
        out_runs, _ = runs[r]
        assert sum(n for *_, n in out_runs) == sum(counts[r])


def test_ep_refuses_experts_that_do_not_shard_evenly(monkeypatch):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1)
    try:
        inp = synthetic.make_custom(4, 64, 3, 1, 64, seed=1, device="cpu")
        ops = OracleOps(inp, 0, 1, 1)
        y = ep.ep_forward(inp.x, ops, 3)  # one rank holds all three experts
        assert y.shape == (4, 64)
        # two ranks cannot hold three experts evenly: refused before any exchange
        monkeypatch.setattr(ep, "_group_info", lambda group: (2, 0))
        with pytest.raises(ValueError):
            ep.ep_forward(inp.x, ops, 3)
    finally:
        dist.destroy_process_group()
