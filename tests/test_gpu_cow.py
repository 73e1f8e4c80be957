"""Copy-on-write after a beam fork, on the GPU, against the oracle.

A 500-token prompt (block size 64: seven full blocks and one holding 52 tokens)
is forked into 4 beams that share every block.  Each decode step then runs the
library's copy-on-write step (pa_cow_prepare) and block copy (pa_copy_blocks)
before slot resolution, K1 and K2; the oracle side replays the same steps with the
allocator model and its own block copy.  Cache contents are compared bit for bit
and every beam's output within the decode tolerance.
"""
import math

import numpy as np
import pytest
import torch

from gpu_cases import assert_close, bits
import oracle as oracle_pkg
from oracle.block_pool import ManagerModel
from paged_kv_cache_374_b200 import binding as pa

pytestmark = pytest.mark.gpu


def test_beam_copy_on_write_three_steps():
    rng = np.random.default_rng(44)
    bs, hk, d, beams, prompt = 64, 8, 128, 4, 500
    nb = 40
    order = rng.permutation(nb).astype(np.int32)
    alloc = pa.BlockAllocator(nb, order)
    model = ManagerModel(nb, bs, order)
    mb = 10
    tables = np.full((beams, mb), -1, dtype=np.int32)
    npre = pa.pa_num_required_blocks(prompt, bs)
    tables[0, :npre] = alloc.alloc_n(npre)
    model.allocate_for_request(0, prompt)
    for b in range(1, beams):
        tables[b, :npre] = alloc.fork(tables[0, :npre])
        model.share_prefix_blocks(0, b, prompt)
    kc = torch.randn(nb, bs, hk, d, device="cuda").to(torch.float16)
    vc = torch.randn(nb, bs, hk, d, device="cuda").to(torch.float16)
    kh, vh = bits(kc), bits(vc)
    o = oracle_pkg.get()
    lens = np.full(beams, prompt, dtype=np.int32)  # stored tokens
    for step in range(3):
        stored = {b: int(lens[b]) for b in range(beams)}
        pairs = alloc.cow_prepare(tables, lens, bs)
        want = model.cow_prepare(stored)
        assert [tuple(p) for p in pairs.tolist()] == want
        if step == 0:
            assert len(pairs) == beams - 1          # three beams copy; the last keeps the shared block
        else:
            assert len(pairs) == 0                  # every beam now appends into its own block
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        if len(pairs):
            pa.pa_copy_blocks(kc, vc, torch.from_numpy(pairs).cuda(), err_word=err)
            o.copy_blocks(kh, vh, pairs)
        slots = alloc.append_slots(tables, lens, bs)
        for b in range(beams):
            model.append_slot(b, stored[b])
            assert list(tables[b, :len(model.tables[b])]) == model.tables[b]
        q = torch.randn(beams, 4 * hk, d, device="cuda").to(torch.float16)   # GQA group 4
        k = torch.randn(beams, hk, d, device="cuda").to(torch.float16)
        v = torch.randn(beams, hk, d, device="cuda").to(torch.float16)
        pa.pa_reshape_and_cache(k, v, torch.from_numpy(slots).cuda(), kc, vc, err_word=err)
        out = torch.empty_like(q)
        pa.pa_decode(q, kc, vc, torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda(),
                     1 / math.sqrt(d), hk, out, err_word=err)
        torch.cuda.synchronize()
        assert err.item() == 0
        o.reshape_and_cache(bits(k), bits(v), slots, kh, vh)
        assert np.array_equal(bits(kc), kh) and np.array_equal(bits(vc), vh)
        ref = o.decode(bits(q), kh, vh, tables, lens, 1 / math.sqrt(d), 0, nthreads=8)
        assert_close(out, ref, "f16", f"step {step}")
    # the seven full prompt blocks stay shared by all four beams
    for blk in tables[0, :npre - 1]:
        assert alloc.refcount(int(blk)) == beams
    assert all((tables[b, :npre - 1] == tables[0, :npre - 1]).all() for b in range(beams))


def test_copy_blocks_bad_ids_and_bit_exactness():
    rng = np.random.default_rng(45)
    for dtype in (torch.float16, torch.bfloat16):
        nb, bs, hk, d = 12, 32, 4, 64
        kc = torch.randn(nb, bs, hk, d, device="cuda").to(dtype)
        vc = torch.randn(nb, bs, hk, d, device="cuda").to(dtype)
        kh, vh = bits(kc), bits(vc)
        pairs = np.array([[1, 9], [4, 2], [7, nb + 3], [0, 11]], dtype=np.int32)
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        pa.pa_copy_blocks(kc, vc, torch.from_numpy(pairs).cuda(), err_word=err)
        torch.cuda.synchronize()
        assert oracle_pkg.get().copy_blocks(kh, vh, pairs) == 1
        assert err.item() == pa.PA_DEVERR_TABLE_RANGE
        assert np.array_equal(bits(kc), kh) and np.array_equal(bits(vc), vh)


def test_copy_blocks_refuses_overlapping_pairs():
    """The pairs are copied all at once, so pairs that overlap are skipped with
    PA_DEVERR_PAIR_CONFLICT instead of being copied in some order: a chain
    (1->2, 2->3), two pairs into one block (8->9, 10->9), and a destination that is
    another pair's source (4->12, 12->13).  Pairs that share a source (5->6, 5->7),
    a pair onto itself and the pairs beside them are copied; an id out of range is
    skipped with PA_DEVERR_TABLE_RANGE and conflicts with nothing.  The result is
    the oracle's sequential copy of the non-overlapping pairs alone."""
    nb, bs, hk, d = 16, 16, 4, 128
    kc = torch.randn(nb, bs, hk, d, device="cuda").to(torch.float16)
    vc = torch.randn(nb, bs, hk, d, device="cuda").to(torch.float16)
    kh, vh = bits(kc), bits(vc)
    pairs = np.array([[1, 2], [2, 3], [5, 6], [8, 9], [10, 9], [5, 7], [11, 11], [4, 12], [12, 13], [0, 15],
                      [14, nb + 1]], dtype=np.int32)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_copy_blocks(kc, vc, torch.from_numpy(pairs).cuda(), err_word=err)
    torch.cuda.synchronize()
    assert err.item() == pa.PA_DEVERR_PAIR_CONFLICT | pa.PA_DEVERR_TABLE_RANGE
    oracle_pkg.get().copy_blocks(kh, vh, np.array([[5, 6], [5, 7], [11, 11], [0, 15]], dtype=np.int32))
    assert np.array_equal(bits(kc), kh) and np.array_equal(bits(vc), vh)


@pytest.mark.parametrize("num_pairs,bs,hk,d,overlap", [(3, 64, 5, 64, False), (701, 16, 2, 128, False),
                                                       (2100, 16, 1, 64, False), (2100, 16, 1, 64, True)])
def test_copy_blocks_chunks_and_many_pairs(num_pairs, bs, hk, d, overlap):
    """A few large blocks (several 16 KiB chunks each, the last one partial), many
    small ones (one partial chunk each), and more pairs than the kernel stages in
    shared memory (2048), with and without two pairs into one block.  Bit-exact
    against the oracle's copy of the pairs that do not overlap."""
    rng = np.random.default_rng(46 + num_pairs)
    nb = 2 * num_pairs + 5
    kc = torch.randn(nb, bs, hk, d, device="cuda").to(torch.bfloat16)
    vc = torch.randn(nb, bs, hk, d, device="cuda").to(torch.bfloat16)
    kh, vh = bits(kc), bits(vc)
    perm = rng.permutation(nb).astype(np.int32)
    pairs = np.stack([perm[:num_pairs], perm[num_pairs:2 * num_pairs]], axis=1).copy()
    keep = np.ones(num_pairs, dtype=bool)
    if overlap:
        pairs[2077, 1] = pairs[3, 1]     # two pairs into one block: both refused
        keep[[3, 2077]] = False
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_copy_blocks(kc, vc, torch.from_numpy(pairs).cuda(), err_word=err)
    torch.cuda.synchronize()
    assert err.item() == (pa.PA_DEVERR_PAIR_CONFLICT if overlap else 0)
    oracle_pkg.get().copy_blocks(kh, vh, np.ascontiguousarray(pairs[keep]))
    assert np.array_equal(bits(kc), kh) and np.array_equal(bits(vc), vh)
