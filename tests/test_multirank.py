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
    text = open(bench.PROFILE_SUMMARY).read()
    fields = dict(ln[2:].split(": ", 1) for ln in text.splitlines() if ln.startswith("- ") and ": " in ln)
    sources = [os.path.join(bench.ROOT, "paged_kv_cache_374_b200", "csrc", n.strip())
               for n in fields["sources"].split(",")]
    old = "- source_sha256_16: " + fields["source_sha256_16"]

    def summary(name, sha):
        f = tmp_path / name
        f.write_text(text.replace(old, "- source_sha256_16: " + sha))
        return str(f)

    current = summary("current.md", bench.source_digest(sources))
    per_token = int(fields["dram_bytes_per_launch"]) / int(fields["tokens_per_launch"])
    assert bench.profiled_traffic(1000, fields["workload"], current) == pytest.approx(1000 * per_token)
    assert bench.profiled_traffic(1000, "gqa70b", current) is None      # another workload's capture
    assert bench.profiled_traffic(1000, fields["workload"], summary("stale.md", "0" * 16)) is None
    assert bench.profiled_traffic(1000, fields["workload"], str(tmp_path / "missing.md")) is None
