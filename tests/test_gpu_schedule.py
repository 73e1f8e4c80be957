"""The engine's claim order on the GPU.  Full partitions run sequence-major,
then every sequence's last partition, longest first; how many units each warp
gets, and so which units run beside which, depends on how many (sequence, head
slot) pairs a launch has.  The cases below take both extremes, a few sequences
(fewer units than warps) and 700 (several units per warp), with lengths on and
around the partition boundaries of 64, 128, 256 and 512 tokens, on the
CUDA-core and tensor-core paths, plus a shared prefix of two partitions.  Each
is checked against the oracle, and repeated calls (one of them on a reused
workspace) must agree bit for bit: the merge order is fixed."""
import math

import numpy as np
import pytest
import torch

from gpu_cases import assert_close
from pins import BF16, F16, PagedCase
from test_gpu_shared_prefix import share
import oracle as oracle_pkg
from paged_kv_cache_374_b200 import binding as pa

pytestmark = pytest.mark.gpu

TDT = {F16: torch.float16, BF16: torch.bfloat16}
WK = {F16: "f16", BF16: "bf16"}

# on and around multiples of 64 tokens
BOUNDARY_LENS = [1, 63, 64, 65, 127, 128, 129, 191, 192, 193, 255, 256, 257, 383, 384, 385, 511, 512, 513,
                 640, 1023, 1024, 1025, 2047, 2049, 3000]


def dev(bits_arr, dtype):
    return torch.from_numpy(np.ascontiguousarray(bits_arr).view(np.int16)).view(TDT[dtype]).cuda()


def decode(c, partition_tokens, ws=None):
    q = dev(c.q, c.dtype)
    kc, vc = dev(c.k_cache, c.dtype), dev(c.v_cache, c.dtype)
    tb, ln = torch.from_numpy(c.tables).cuda(), torch.from_numpy(c.lens).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    pa.pa_decode(q, kc, vc, tb, ln, c.scale, c.Hk, out, partition_tokens=partition_tokens, err_word=err,
                 workspace=ws)
    torch.cuda.synchronize()
    assert err.item() == 0
    return out


@pytest.mark.parametrize("g,dtype", [(1, F16), (1, BF16), (8, BF16), (4, F16)])
@pytest.mark.parametrize("pt", [0, 128, 256, 512])
def test_few_sequences_boundary_lengths(g, dtype, pt):
    rng = np.random.default_rng(400 + g * 10 + dtype + pt)
    hk = 2
    c = PagedCase(rng, BOUNDARY_LENS, hk * g, hk, 128, 16, dtype, 1 / math.sqrt(128), extra_blocks=6)
    ref = c.run(oracle_pkg.get(), nthreads=8)
    a = decode(c, pt)
    assert_close(a, ref, WK[dtype], f"g{g} pt{pt}")
    assert torch.equal(a, decode(c, pt)), "repeated call differs"


@pytest.mark.parametrize("g,dtype,bs", [(1, F16, 16), (8, BF16, 32)])
def test_many_sequences_several_units_per_warp(g, dtype, bs):
    """700 sequences x 4 head slots, lengths up to 1800 tokens: several units per
    warp, and the last partitions of 700 sequences sorted at the end."""
    rng = np.random.default_rng(500 + g)
    hk = 4
    lens = rng.integers(1, 1800, size=700).tolist()
    lens[:len(BOUNDARY_LENS)] = BOUNDARY_LENS
    c = PagedCase(rng, lens, hk * g, hk, 128, bs, dtype, 1 / math.sqrt(128), extra_blocks=8)
    ref = c.run(oracle_pkg.get(), nthreads=16)
    a = decode(c, 0)
    assert_close(a, ref, WK[dtype], f"g{g} 700 seqs")
    # the same workspace, reused: counters are left zero by every call
    ws_bytes = pa.pa_decode_workspace_size(len(lens), hk * g, hk, 128, bs, c.tables.shape[1], 0)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    b1 = decode(c, 0, ws)
    b2 = decode(c, 0, ws)
    assert torch.equal(a, b1) and torch.equal(b1, b2)


def test_shared_prefix_of_two_partitions():
    """Four sequences share a 512-token prefix (two partitions of the default
    256 tokens); their suffixes end on and around 128-token boundaries.  The
    prefix kernel leaves the prefix partials, the engine the rest."""
    rng = np.random.default_rng(600)
    lens = [512 + 1, 512 + 128, 512 + 129, 512 + 700]
    c = PagedCase(rng, lens, 8, 8, 128, 16, F16, 1 / math.sqrt(128), extra_blocks=4)
    share(c, [0, 1, 2, 3], 512)
    ref = c.run(oracle_pkg.get(), nthreads=8)
    P = pa.pa_decode_partition_tokens(len(lens), 8, 8, 128, 16, c.tables.shape[1])
    g = pa.pa_find_shared_prefixes(c.tables, c.lens, 16, P)
    assert g.num_groups == 1 and g.max_shared_tokens == 512
    q = dev(c.q, c.dtype)
    kc, vc = dev(c.k_cache, c.dtype), dev(c.v_cache, c.dtype)
    tb, ln = torch.from_numpy(c.tables).cuda(), torch.from_numpy(c.lens).cuda()
    start, offs, mem = g.to("cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    pa.pa_decode_shared_prefix(q, kc, vc, tb, ln, c.scale, c.Hk, out, start, offs, mem, g.num_groups,
                               g.max_group_size, g.max_shared_tokens, partition_tokens=P, err_word=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert_close(out, ref, "f16", "shared prefix of two partitions")
