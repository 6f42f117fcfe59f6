"""Expert-parallel MoE FFN layer over the ranks of a process group.

torchtitan PR "gpt-oss model enablement" (expert parallelism with an
all-to-all token dispatch) and the torchtitan GPT-OSS guide, "expert-parallel
sharding" (the expert weights sharded along their expert dimension,
mlp1_weight_EGD / mlp2_weight_EDF): every rank of `group` holds E / W
experts (rank d holds experts [d*E/W, (d+1)*E/W)) plus the replicated router,
and its own batch of tokens. Per layer and rank:

1. route, permute and gather the rank's own tokens (the single-GPU kernels,
   over all E experts): x_perm holds the routed rows sorted by expert, so the
   rows for rank d's experts form one contiguous run per expert;
2. exchange the per-expert row counts (one all-to-all of E integers per
   rank) and copy them to the host: the only device-to-host transfer of the
   layer, needed for the message sizes;
3. send every (expert, destination) run of routed rows and their routing
   weights to the expert's rank. The receiver posts one receive per
   (local expert j, source s) block and lays the blocks out expert by expert,
   sources in rank order, so the received rows arrive already grouped by
   local expert: no re-sort pass;
4. run the unchanged local grouped FFN on them (mlp1 + activation, mlp2 +
   bias, each row's expert output times its routing weight, fp32);
5. send every block back; it lands in the source's o_perm at the run it came
   from, so the source's own combine (its inverse permutation) finishes the
   layer exactly as on one GPU.

The data plane is point-to-point messages of whole row runs between local
buffers (NCCL on GPUs, batched into one group call per direction; gloo on
CPU). Blocks a rank keeps are copied, not sent. No rank reads another
rank's memory, and no tensor-core operand or TMA load ever refers to peer
memory. Each row's expert output depends only on that row, so the layer's
result on W ranks equals the single-GPU layer's on the same tokens (bitwise
where both runs pick the same GEMM kernel for the expert; the MXFP4 path
picks by rows per expert, within its tolerance otherwise).

The per-rank compute is an object with the methods of `LocalOps`;
`CudaLocalOps` runs it through the C ABI. Every step that computes runs in
the library's kernels; this module moves buffers and sizes.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

from . import _binding as B


class LocalOps:
    """The per-rank compute the exchange wraps (all tensors on the ops' device).

    route(x) -> (topk_idx (T,k) int32, topk_w (T,k) float32)
    permute(topk_idx) -> (counts (E,), offsets (E+1,), perm (R,), inv (R,)) int32
    gather(x, perm) -> x_perm (R,D): row r = x[perm[r] // k]
    expert_ffn(rows (N,D), offsets (E_local+1,), w (N,) float32) -> o (N,D), float32 or wider:
        o[r] = w[r] * (W2[e] . act(W1[e] . rows[r] + b1[e]) + b2[e]) for the
        local expert e whose segment holds r (N may be 0)
    combine(o_perm (R,D) of expert_ffn's type, inv (R,)) -> y (T,D) bf16
    """


def _group_info(group) -> Tuple[int, int]:
    if group is None:
        group = dist.group.WORLD
    return dist.get_world_size(group), dist.get_rank(group)


def exchange_counts(counts: torch.Tensor, world: int, group=None) -> Tuple[List[int], List[List[int]]]:
    """Per-expert row counts of this rank's routed rows (E,) -> (counts on the
    host, recv[s][j] = rows rank s routes to this rank's local expert j)."""
    E = counts.numel()
    E_local = E // world
    send = counts.to(torch.int64).contiguous()
    recv = torch.empty_like(send)  # row s: rank s's counts for this rank's experts
    if world > 1:
        dist.all_to_all_single(recv, send, group=group)
    else:
        recv.copy_(send)
    counts_h = send.cpu().tolist()
    recv_h = recv.cpu().view(world, E_local).tolist()
    return counts_h, recv_h


def recv_layout(recv_h: Sequence[Sequence[int]]) -> Tuple[List[List[int]], List[int]]:
    """Where block (local expert j, source s) starts in the receive buffer
    (experts in order, sources in rank order within an expert), and the
    local expert offsets for the grouped GEMM (E_local + 1 entries)."""
    world = len(recv_h)
    E_local = len(recv_h[0]) if world else 0
    start = [[0] * world for _ in range(E_local)]
    offsets = [0] * (E_local + 1)
    at = 0
    for j in range(E_local):
        offsets[j] = at
        for s in range(world):
            start[j][s] = at
            at += recv_h[s][j]
    offsets[E_local] = at
    return start, offsets


def _blocks(counts_h: Sequence[int], offsets_h: Sequence[int], recv_h, world: int, rank: int):
    """Yield (peer, local expert j, rows run in x_perm / o_perm, rows in the
    receive buffer) for every non-empty block this rank sends and receives."""
    E_local = len(counts_h) // world
    start, _ = recv_layout(recv_h)
    out_runs = []  # (dest, j, first row in x_perm, n)
    for d in range(world):
        for j in range(E_local):
            e = d * E_local + j
            n = counts_h[e]
            if n:
                out_runs.append((d, j, offsets_h[e], n))
    in_runs = []  # (source, j, first row in the receive buffer, n)
    for j in range(E_local):
        for s in range(world):
            n = recv_h[s][j]
            if n:
                in_runs.append((s, j, start[j][s], n))
    return out_runs, in_runs


def _exchange(sends, recvs, group):
    """Post every send and receive of one direction as one batch and wait."""
    ops = [dist.P2POp(dist.isend, t, peer, group) for peer, t in sends]
    ops += [dist.P2POp(dist.irecv, t, peer, group) for peer, t in recvs]
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()


def ep_forward(x: torch.Tensor, ops, E: int, group=None) -> torch.Tensor:
    """The layer on this rank's tokens x (T,D) bf16 with experts sharded over
    `group` (E divisible by its size) -> y (T,D) bf16. Every rank of the group
    calls it once per layer, in the same order."""
    world, rank = _group_info(group)
    if E % world:
        raise ValueError(f"E={E} experts do not shard evenly over {world} ranks")
    E_local = E // world
    T, D = x.shape
    if T > 0:
        topk_idx, topk_w = ops.route(x)
        counts, offsets, perm, inv = ops.permute(topk_idx)
        x_perm = ops.gather(x, perm)
        w_perm = topk_w.reshape(-1).index_select(0, perm.long())  # each routed row's routing weight
    else:  # no tokens of its own: the rank still serves its experts
        counts = torch.zeros(E, dtype=torch.int32, device=x.device)
        x_perm = torch.empty((0, D), dtype=x.dtype, device=x.device)
        w_perm = torch.empty(0, dtype=torch.float32, device=x.device)
        inv = None
    counts_h, recv_h = exchange_counts(counts, world, group)
    offsets_h = [0]
    for c in counts_h:
        offsets_h.append(offsets_h[-1] + c)
    start, loff = recv_layout(recv_h)
    N = loff[-1]
    rows = torch.empty((N, D), dtype=x_perm.dtype, device=x.device)
    w_rows = torch.empty(N, dtype=torch.float32, device=x.device)
    out_runs, in_runs = _blocks(counts_h, offsets_h, recv_h, world, rank)

    # dispatch: routed rows and their weights to the experts' ranks
    sends, recvs = [], []
    for d, j, r0, n in out_runs:
        if d == rank:
            b0 = start[j][rank]
            rows[b0:b0 + n].copy_(x_perm[r0:r0 + n])
            w_rows[b0:b0 + n].copy_(w_perm[r0:r0 + n])
        else:
            sends += [(d, x_perm[r0:r0 + n]), (d, w_perm[r0:r0 + n])]
    for s, j, b0, n in in_runs:
        if s != rank:
            recvs += [(s, rows[b0:b0 + n]), (s, w_rows[b0:b0 + n])]
    _exchange(sends, recvs, group)

    # the local experts' grouped FFN
    loff_t = torch.tensor(loff, dtype=torch.int32, device=x.device)
    o_rows = ops.expert_ffn(rows, loff_t, w_rows)

    # combine: each block back to the run of o_perm it was routed from
    R = x_perm.shape[0]
    o_perm = torch.empty((R, D), dtype=o_rows.dtype, device=x.device)
    sends, recvs = [], []
    for s, j, b0, n in in_runs:
        if s == rank:
            r0 = offsets_h[rank * E_local + j]
            o_perm[r0:r0 + n].copy_(o_rows[b0:b0 + n])
        else:
            sends.append((s, o_rows[b0:b0 + n]))
    for d, j, r0, n in out_runs:
        if d != rank:
            recvs.append((d, o_perm[r0:r0 + n]))
    _exchange(sends, recvs, group)
    if T == 0:
        return torch.empty((0, D), dtype=torch.bfloat16, device=x.device)
    return ops.combine(o_perm, inv)


class CudaLocalOps(LocalOps):
    """The per-rank compute through the C ABI (bf16 or MXFP4 expert weights).

    Wr (E,D), br (E) bf16: the replicated router; W1 (E_local,2I,D),
    b1 (E_local,2I), W2 (E_local,D,I), b2 (E_local,D): this rank's experts
    (bf16, or MXFP4 codes with W1_scales / W2_scales, prepared once here)."""

    def __init__(self, Wr, br, W1, b1, W2, b2, k: int, W1_scales=None, W2_scales=None, act=B.MOE_ACT_SWIGLU,
                 act_alpha: float = 1.0, act_limit: float = float("inf")):
        self.Wr, self.br, self.b1, self.b2 = Wr, br, b1, b2
        self.E, self.D = Wr.shape
        self.E_local = b1.shape[0]
        self.I = b1.shape[1] // 2
        self.k = k
        self.wfmt = B.MOE_W_BF16 if W1_scales is None else B.MOE_W_MXFP4
        self.act, self.act_alpha, self.act_limit = act, act_alpha, act_limit
        self.device = Wr.device
        self._ws = {}
        if self.wfmt == B.MOE_W_MXFP4:
            dl = self._dims(1, self.E_local, 1)
            # the GEMMs read only the prepared forms
            self.W1, self.W1_scales, self.W2, self.W2_scales = None, None, None, None
            self.W1p = B.mxfp4_prepare(dl, 1, W1, W1_scales)
            self.W2p = B.mxfp4_prepare(dl, 2, W2, W2_scales)
        else:
            self.W1, self.W2 = W1, W2
            self.W1_scales = self.W2_scales = self.W1p = self.W2p = None

    def _dims(self, T: int, E: int, k: int) -> B.Dims:
        return B.dims(T, self.D, E, k, self.I, self.wfmt, self.act, self.act_alpha, self.act_limit)

    def _workspace(self, d: B.Dims, key: str) -> torch.Tensor:
        n = B.workspace_bytes(d)
        ws = self._ws.get(key)
        if ws is None or ws.numel() < n:
            ws = B.alloc_workspace(d, device=self.device)
            self._ws[key] = ws
        return ws

    def _src(self, T: int):
        d = self._dims(T, self.E, self.k)
        return d, self._workspace(d, "src")

    def route(self, x):
        T = x.shape[0]
        d, ws = self._src(T)
        idx = torch.empty((T, self.k), dtype=torch.int32, device=x.device)
        w = torch.empty((T, self.k), dtype=torch.float32, device=x.device)
        B.moe_route(d, x, self.Wr, self.br, idx, w, ws)
        return idx, w

    def permute(self, topk_idx):
        T = topk_idx.shape[0]
        d, ws = self._src(T)
        R = T * self.k
        i32 = dict(dtype=torch.int32, device=topk_idx.device)
        counts, offsets = torch.empty(self.E, **i32), torch.empty(self.E + 1, **i32)
        perm, inv = torch.empty(R, **i32), torch.empty(R, **i32)
        B.moe_permute(d, topk_idx, counts, offsets, perm, inv, ws)
        return counts, offsets, perm, inv

    def gather(self, x, perm):
        T = x.shape[0]
        d, ws = self._src(T)
        x_perm = torch.empty((T * self.k, self.D), dtype=torch.bfloat16, device=x.device)
        B.moe_gather(d, x, perm, x_perm, ws)
        return x_perm

    def expert_ffn(self, rows, offsets, w):
        N = rows.shape[0]
        o = torch.empty((N, self.D), dtype=torch.float32, device=rows.device)
        if N == 0:
            return o
        d = self._dims(N, self.E_local, 1)  # every received row is one (row, expert) pair
        ws = self._workspace(d, "experts")
        h = torch.empty((N, self.I), dtype=torch.bfloat16, device=rows.device)
        ident = torch.arange(N, dtype=torch.int32, device=rows.device)
        B.moe_mlp1(d, rows, offsets, self.W1, self.b1, h, ws, W1_scales=self.W1_scales, W1_prepared=self.W1p)
        B.moe_mlp2(d, h, ident, offsets, w, self.W2, self.b2, o, ws, W2_scales=self.W2_scales, W2_prepared=self.W2p)
        return o

    def combine(self, o_perm, inv):
        T = inv.shape[0] // self.k
        d, ws = self._src(T)
        y = torch.empty((T, self.D), dtype=torch.bfloat16, device=o_perm.device)
        B.moe_combine(d, o_perm, inv, y, ws)
        return y

    def device_status(self) -> int:
        """Read and clear the device status words of this rank's workspaces."""
        st = 0
        for ws in self._ws.values():
            st = st or B.moe_read_device_status(ws)
        return st


class ExpertParallelMoE:
    """The layer with its experts sharded over `group`: construct it on every
    rank with the replicated router and that rank's E / W experts, then call
    it on each rank's own tokens."""

    def __init__(self, Wr, br, W1, b1, W2, b2, k: int, group=None, **kw):
        self.group = group
        self.ops = CudaLocalOps(Wr, br, W1, b1, W2, b2, k, **kw)
        world, _ = _group_info(group)
        if self.ops.E_local * world != self.ops.E:
            raise ValueError(f"{self.ops.E_local} local experts x {world} ranks != E = {self.ops.E}")

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        return ep_forward(x, self.ops, self.ops.E, self.group)

    __call__ = forward
