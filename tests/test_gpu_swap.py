"""Swap-out / swap-in of a preempted sequence between the device pool and a pinned
host pool, on the GPU.

Sequence 1 is swapped out (its blocks copied to host memory and freed on the
device), the freed device blocks are taken by other work and overwritten, then
the sequence is swapped back in to fresh device blocks.  The round trip is bit
exact (checked against the oracle's own block copy), and decode over the swapped-
in table gives the same output, bit for bit, as before the swap (the computation
does not depend on physical ids), and matches the oracle.
"""
import math

import numpy as np
import pytest
import torch

from gpu_cases import assert_close, bits
import oracle as oracle_pkg
from paged_kv_cache_374_b200 import binding as pa

pytestmark = pytest.mark.gpu


def test_swap_out_overwrite_swap_in():
    rng = np.random.default_rng(46)
    bs, hk, d, h = 16, 4, 128, 8
    nd, nh = 48, 16
    dev = pa.BlockAllocator(nd, rng.permutation(nd).astype(np.int32))
    host = pa.BlockAllocator(nh, rng.permutation(nh).astype(np.int32))
    lens = np.array([70, 150, 33], dtype=np.int32)
    mb = 12
    tables = np.full((3, mb), -1, dtype=np.int32)
    for s in range(3):
        n = pa.pa_num_required_blocks(int(lens[s]), bs)
        tables[s, :n] = dev.alloc_n(n)
    kc = torch.randn(nd, bs, hk, d, device="cuda").to(torch.bfloat16)
    vc = torch.randn(nd, bs, hk, d, device="cuda").to(torch.bfloat16)
    kh_pool = torch.zeros(nh, bs, hk, d, dtype=torch.bfloat16).pin_memory()   # the host pool
    vh_pool = torch.zeros_like(kh_pool).pin_memory()
    q = torch.randn(3, h, d, device="cuda").to(torch.bfloat16)
    scale = 1 / math.sqrt(d)

    def decode():
        out = torch.empty_like(q)
        pa.pa_decode(q, kc, vc, torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda(), scale, hk, out)
        torch.cuda.synchronize()
        return out

    before = decode()
    o = oracle_pkg.get()
    # the oracle's view of both pools, updated by its own block copies
    k_dev, v_dev = bits(kc), bits(vc)
    k_host, v_host = bits(kh_pool), bits(vh_pool)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")

    # swap out sequence 1
    nblk = pa.pa_num_required_blocks(int(lens[1]), bs)
    out_pairs = pa.pa_swap_plan(dev.handle, host.handle, tables[1], nblk)
    pa.pa_swap_blocks(kc, vc, kh_pool, vh_pool, torch.from_numpy(out_pairs).cuda(), err_word=err)
    torch.cuda.synchronize()
    for (src, dst) in out_pairs:
        k_host[dst], v_host[dst] = k_dev[src], v_dev[src]
    assert np.array_equal(bits(kh_pool), k_host) and np.array_equal(bits(vh_pool), v_host)
    assert dev.num_free() == nd - sum(pa.pa_num_required_blocks(int(n), bs) for n in lens) + nblk

    # other work takes the freed device blocks and overwrites them
    grabbed = dev.alloc_n(dev.num_free())
    idx = torch.from_numpy(grabbed.astype(np.int64)).cuda()
    kc[idx] = torch.randn(len(grabbed), bs, hk, d, device="cuda").to(torch.bfloat16)
    vc[idx] = float("nan")
    dev.free_n(grabbed)

    # swap back in to fresh device blocks
    in_pairs = pa.pa_swap_plan(host.handle, dev.handle, tables[1], nblk)
    pa.pa_swap_blocks(kh_pool, vh_pool, kc, vc, torch.from_numpy(in_pairs).cuda(), err_word=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    k_dev, v_dev = bits(kc), bits(vc)
    for (src, dst) in in_pairs:
        assert np.array_equal(k_dev[dst], k_host[src]) and np.array_equal(v_dev[dst], v_host[src])
    assert host.num_free() == nh

    after = decode()
    assert torch.equal(before, after)
    ref = o.decode(bits(q), k_dev, v_dev, tables, lens, scale, 1, nthreads=8)
    assert_close(after, ref, "bf16", "after the swap round trip")
