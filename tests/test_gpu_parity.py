"""GPU parity: the library's kernels against the fp64 oracle on the five workloads.

Every workload runs at its full size in the launch configuration the benchmark
times (default partitioning).  Cache writes are compared bit for bit over the
whole pool; decode outputs are compared with the oracle on every (sequence, head)
pair where the oracle finishes in seconds, else on a seeded sample of pairs that
always includes the longest and the shortest sequence.
"""
import numpy as np
import pytest
import torch

from gpu_cases import DT, Step, assert_close, bits, device_inputs, oracle_decode, run_library
import oracle as oracle_pkg
from paged_kv_cache_374_b200 import binding as pa

pytestmark = pytest.mark.gpu


def _pairs(step, n, rng):
    s, h = step.spec.num_seqs, step.spec.num_heads
    lens = step.lens
    must = [(int(np.argmax(lens)), 0), (int(np.argmin(lens)), h - 1)]
    picks = [(int(rng.integers(0, s)), int(rng.integers(0, h))) for _ in range(n)]
    return np.array(must + picks, dtype=np.int32)


def _parity(name, sample_pairs=None, num_seqs=None):
    step = Step(name, num_seqs=num_seqs)
    t = step.tensors()
    kc_host, vc_host = bits(t["k_cache"]), bits(t["v_cache"])
    q_host, k_host, v_host = bits(t["q"]), bits(t["k"]), bits(t["v"])
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = run_library(step, t, err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    # K1: bit-exact over the whole pool
    o = oracle_pkg.get()
    skipped = o.reshape_and_cache(k_host, v_host, step.slots, kc_host, vc_host)
    assert skipped == 0
    assert np.array_equal(bits(t["k_cache"]), kc_host) and np.array_equal(bits(t["v_cache"]), vc_host)
    # K2 + K3
    if sample_pairs is None:
        ref = oracle_decode(step, q_host, kc_host, vc_host)
        got = out
    else:
        pairs = _pairs(step, sample_pairs, np.random.default_rng(123))
        ref = oracle_decode(step, q_host, kc_host, vc_host, pairs=pairs)
        got = out[torch.from_numpy(pairs[:, 0]).long(), torch.from_numpy(pairs[:, 1]).long()]
    return assert_close(got, ref, step.dtype, name)


def test_tiny():
    _parity("tiny")


def test_llama7b_full_size():
    _parity("llama7b")


def test_gqa70b_full_size():
    _parity("gqa70b", sample_pairs=96)


def test_beam_prefix_sharing_full_size():
    step = Step("beam")
    npre = 512 // step.bs
    # every sequence maps its first 8 logical blocks to the same physical blocks
    assert (step.tables[:, :npre] == step.tables[0, :npre]).all()
    assert all(step.alloc.refcount(int(b)) == 1 + step.spec.num_seqs for b in step.tables[0, :npre])
    _parity("beam", sample_pairs=128)


def test_llama13b_32_steps():
    """32 consecutive steps: each appends one token per sequence (a new block at
    16-token boundaries, from the library's allocator), writes it with K1 and
    attends with K2(+K3).  The oracle replays every step on its own copy."""
    step = Step("llama13b")
    t = step.tensors()
    kc_host, vc_host = bits(t["k_cache"]), bits(t["v_cache"])
    o = oracle_pkg.get()
    rng = np.random.default_rng(7)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(99)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for i in range(step.spec.steps):
        if i > 0:
            step.slots = step.append()
            for key in ("q", "k", "v"):
                t[key] = torch.randn(t[key].shape, generator=gen, device="cuda").to(t[key].dtype)
        out = run_library(step, t, err=err)
        torch.cuda.synchronize()
        o.reshape_and_cache(bits(t["k"]), bits(t["v"]), step.slots, kc_host, vc_host)
        q_host = bits(t["q"])
        if i == step.spec.steps - 1:
            ref = oracle_decode(step, q_host, kc_host, vc_host)
            assert_close(out, ref, step.dtype, f"step {i}")
            assert np.array_equal(bits(t["k_cache"]), kc_host) and np.array_equal(bits(t["v_cache"]), vc_host)
        else:
            pairs = _pairs(step, 8, rng)
            ref = oracle_decode(step, q_host, kc_host, vc_host, pairs=pairs)
            got = out[torch.from_numpy(pairs[:, 0]).long(), torch.from_numpy(pairs[:, 1]).long()]
            assert_close(got, ref, step.dtype, f"step {i}")
    assert err.item() == 0
