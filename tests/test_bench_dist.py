"""The multi-rank logic of bench.py on CPU: two gloo ranks, each with its own
step time; the job's step time is the slowest rank's and the throughput counts
every rank's tokens (replicas, no collective on the data path)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        assert bench.dist_env()[:2] == (world, rank)
        mine = [100.0 + 10 * rank, 300.0 - rank, 50.0 * (rank + 1)]
        times = bench.max_over_ranks(mine, world)
        ms, value = bench.step_throughput(times[0], 20, 8192, world)
        out[rank] = (times, ms, value)
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_takes_the_slowest_rank():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == res[1]  # every rank agrees
    times, ms, value = res[0]
    assert times == [110.0, 300.0, 100.0]
    assert ms == pytest.approx(110.0 / 20)
    assert value == pytest.approx(2 * 8192 / (110.0 / 20 / 1e3))


def test_single_rank_is_identity():
    assert bench.max_over_ranks([1.0, 2.0], 1) == [1.0, 2.0]
    ms, value = bench.step_throughput(1000.0, 10, 8192, 1)
    assert ms == 100.0 and value == pytest.approx(81920.0)


@pytest.mark.parametrize("workload", ["gptoss20b", "gptoss20b_mxfp4", "gptoss20b_mxfp4_decode"])
def test_profile_traffic_is_read_for_the_profiled_kernel_sources(tmp_path, monkeypatch, workload):
    # each committed ncu summary carries the hash of the kernel sources it was
    # taken on; the bench reports its DRAM bytes only while that hash matches
    name, sources = bench.PROFILE_OF[workload]
    text = open(os.path.join(bench.ROOT, "profiles", name)).read()
    fake = tmp_path / "profiles"
    fake.mkdir()
    (fake / name).write_text(text)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    import re

    sha = re.search(r"kernel_sources_sha256_16: `([0-9a-f]{16})`", text).group(1)
    nbytes = int(re.search(r"dram_bytes_per_launch: `(\d+)`", text).group(1))
    monkeypatch.setattr(bench, "source_hash", lambda srcs: sha if srcs == sources else "0" * 16)
    assert bench.traffic_from_profile(workload) == nbytes
    # a summary taken on other kernel sources is ignored
    monkeypatch.setattr(bench, "source_hash", lambda srcs: "f" * 16)
    assert bench.traffic_from_profile(workload) is None
    assert bench.traffic_from_profile("gptoss120b_zipf") is None  # no summary for this workload
