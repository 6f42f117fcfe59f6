"""Expert-parallel layer on the GPU through the C ABI (one rank, NCCL).

torchtitan PR "gpt-oss model enablement" (expert parallelism) and the
torchtitan GPT-OSS guide, "expert-parallel sharding". A one-rank group runs
the whole exchange path (count exchange, block layout, local grouped FFN
with k = 1 on the received rows, return into o_perm, combine) with every
block kept locally; the result must be bitwise the single-GPU layer's. The
multi-rank exchange is covered on CPU ranks (test_ep.py); runs on several
GPUs are not part of this suite.
"""
import datetime
import socket

import pytest
import torch
import torch.distributed as dist

import oracle
import synthetic
import mixture_experts_ffn_layer_b200 as moe
from helpers import dims_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nccl_group():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    yield dist.group.WORLD
    dist.destroy_process_group()


@pytest.mark.parametrize("T,D,E,k,I,wfmt", [
    (300, 256, 8, 2, 512, "bf16"),
    (64, 2880, 32, 4, 2880, "mxfp4"),   # decode-sized: the small-expert MXFP4 kernel
    (600, 192, 4, 2, 320, "mxfp4"),     # big-tile MXFP4 kernel, ragged K
])
def test_ep_one_rank_matches_single_gpu_layer(nccl_group, T, D, E, k, I, wfmt):
    inp = synthetic.make_custom(T, D, E, k, I, seed=3 * T + E, device="cuda", wfmt=wfmt, reject=oracle.gap_reject())
    d = dims_of(inp)
    ws = moe.alloc_workspace(d)
    y_ref = torch.empty((T, D), dtype=torch.bfloat16, device="cuda")
    moe.moe_forward(d, inp.x, inp.Wr, inp.br, inp.W1, inp.b1, inp.W2, inp.b2, y_ref, ws,
                    W1_scales=inp.W1_scales, W2_scales=inp.W2_scales)
    layer = moe.ExpertParallelMoE(inp.Wr, inp.br, inp.W1, inp.b1, inp.W2, inp.b2, k, group=nccl_group,
                                  W1_scales=inp.W1_scales, W2_scales=inp.W2_scales)
    y = layer(inp.x)
    torch.cuda.synchronize()
    assert layer.ops.device_status() == 0
    assert moe.moe_read_device_status(ws) == 0
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    # a rank without tokens of its own returns an empty result and still serves its experts
    assert layer(inp.x[:0]).shape == (0, D)
