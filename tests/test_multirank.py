"""The benchmark's multi-rank plumbing on CPU: two gloo ranks, replicas only.

The decode path has no exchange step, so N GPUs run N independent replicas; the
job time is the slowest rank's and the job throughput counts every rank's tokens.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        times = [10.0 + rank, 3.0 - rank]     # rank 1 is slower on the first value, faster on the second
        got = bench.max_over_ranks(times, dist)
        q.put((rank, got, bench.job_throughput(world, 64, got[0])))
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_take_the_slowest_rank():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, tput in results:
        assert got == [11.0, 3.0]
        assert tput == 2 * 64 / (11.0 / 1e3)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert bench.job_throughput(1, 64, 0.4) == 64 / 0.0004


def test_profiled_traffic_comes_only_from_the_same_workload(tmp_path):
    """roofline.traffic scales a capture by tokens only when the capture is of the
    same workload (bytes per token depend on the head counts) and the sources its
    kernels are built from are the ones it was taken on."""
    import bench
    per_token_7b = 629657088 / 37801
    assert bench.profiled_traffic(1000, "llama7b") == pytest.approx(1000 * per_token_7b)
    assert bench.profiled_traffic(1000, "llama13b") is None
    assert bench.profiled_traffic(1000, "gqa70b", bench.GQA_PROFILE_SUMMARY) == pytest.approx(
        1000 * 203340544 / 47015)
    assert bench.profiled_traffic(1000, "gqa70b") is None           # the 7B capture does not serve gqa70b
    assert bench.profiled_traffic(1000, "beam", bench.SHARED_PROFILE_SUMMARY) is not None
    # a summary whose recorded digest no longer matches its sources gives no traffic
    stale = tmp_path / "stale.md"
    text = open(bench.PROFILE_SUMMARY).read()
    line = next(ln for ln in text.splitlines() if ln.startswith("- source_sha256_16: "))
    stale.write_text(text.replace(line, "- source_sha256_16: 0000000000000000"))
    assert bench.profiled_traffic(1000, "llama7b", str(stale)) is None
