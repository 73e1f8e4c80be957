"""Paged prefill on the GPU against the oracle: chunks with and without cached
context before them, MHA and GQA, block sizes 16/32/64, head_dim 64/128, fp16 and
bf16, a full allocator -> cache write -> prefill -> decode flow, and error rows."""
import math

import numpy as np
import pytest
import torch

from gpu_cases import assert_close, bits
from pins import BF16, F16, PagedCase, to_bits
import oracle as oracle_pkg
from paged_kv_cache_374_b200 import binding as pa

pytestmark = pytest.mark.gpu

TDT = {F16: torch.float16, BF16: torch.bfloat16}
WK = {F16: "f16", BF16: "bf16"}


def dev(bits_arr, dtype):
    return torch.from_numpy(np.ascontiguousarray(bits_arr).view(np.int16)).view(TDT[dtype]).cuda()


def run_prefill(c, q_bits, qs, err=None, tables=None):
    q = dev(q_bits, c.dtype)
    out = torch.full_like(q, float("nan"))
    pa.pa_prefill(q, dev(c.k_cache, c.dtype), dev(c.v_cache, c.dtype),
                  torch.from_numpy(c.tables if tables is None else tables).cuda(), torch.from_numpy(c.lens).cuda(),
                  torch.from_numpy(qs).cuda(), c.scale, c.Hk, out, int(np.max(np.diff(qs))), err_word=err)
    torch.cuda.synchronize()
    return out


CASES = [(128, 16, 1, F16), (128, 64, 4, BF16), (64, 32, 1, BF16), (64, 16, 2, F16), (128, 32, 8, F16)]


@pytest.mark.parametrize("d,bs,g,dtype", CASES)
def test_prefill_matches_oracle(d, bs, g, dtype):
    rng = np.random.default_rng(60 + d + bs + g)
    hk = 2
    lens = [37, 200, 64, 513, 9]
    n_new = [37, 70, 1, 200, 9]      # whole prompts, chunks after cached context, a single token
    c = PagedCase(rng, lens, hk * g, hk, d, bs, dtype, 1 / math.sqrt(d), extra_blocks=3)
    qs = np.concatenate([[0], np.cumsum(n_new)]).astype(np.int32)
    q = to_bits(rng.normal(0, 1, (int(qs[-1]), hk * g, d)), dtype)
    ref = oracle_pkg.get().prefill(q, c.k_cache, c.v_cache, c.tables, c.lens, qs, c.scale, dtype, nthreads=8)
    out = run_prefill(c, q, qs)
    assert_close(out, ref, WK[dtype], f"prefill d{d} bs{bs} g{g}")


def test_prefill_flow_then_decode():
    """Allocate and write a chunk through the library (pa_prefill_slots, K1), attend
    with pa_prefill, then take one decode step; the oracle replays every step."""
    rng = np.random.default_rng(61)
    bs, hk, h, d, nb = 16, 4, 8, 128, 200
    order = rng.permutation(nb).astype(np.int32)
    alloc = pa.BlockAllocator(nb, order)
    cached = np.array([0, 300, 45], dtype=np.int32)      # tokens already in the cache
    new = np.array([120, 64, 33], dtype=np.int32)
    mb = 40
    tables = np.full((3, mb), -1, dtype=np.int32)
    for s in range(3):
        k = pa.pa_num_required_blocks(int(cached[s]), bs)
        tables[s, :k] = alloc.alloc_n(k)
    kc = torch.randn(nb, bs, hk, d, device="cuda").to(torch.float16)
    vc = torch.randn(nb, bs, hk, d, device="cuda").to(torch.float16)
    lens = cached.copy()
    slots = alloc.prefill_slots(tables, lens, new, bs)
    total = int(new.sum())
    k = torch.randn(total, hk, d, device="cuda").to(torch.float16)
    v = torch.randn(total, hk, d, device="cuda").to(torch.float16)
    q = torch.randn(total, h, d, device="cuda").to(torch.float16)
    qs = np.concatenate([[0], np.cumsum(new)]).astype(np.int32)
    kh, vh = bits(kc), bits(vc)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_reshape_and_cache(k, v, torch.from_numpy(slots).cuda(), kc, vc, err_word=err)
    out = torch.empty_like(q)
    tb = torch.from_numpy(tables).cuda()
    pa.pa_prefill(q, kc, vc, tb, torch.from_numpy(lens).cuda(), torch.from_numpy(qs).cuda(), 1 / math.sqrt(d), hk,
                  out, int(new.max()), err_word=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    o = oracle_pkg.get()
    o.reshape_and_cache(bits(k), bits(v), slots, kh, vh)
    assert np.array_equal(bits(kc), kh) and np.array_equal(bits(vc), vh)
    ref = o.prefill(bits(q), kh, vh, tables, lens, qs, 1 / math.sqrt(d), 0, nthreads=8)
    assert_close(out, ref, "f16", "prefill flow")
    # one decode step after the chunk
    slots1 = alloc.append_slots(tables, lens, bs)
    k1 = torch.randn(3, hk, d, device="cuda").to(torch.float16)
    v1 = torch.randn(3, hk, d, device="cuda").to(torch.float16)
    q1 = torch.randn(3, h, d, device="cuda").to(torch.float16)
    pa.pa_reshape_and_cache(k1, v1, torch.from_numpy(slots1).cuda(), kc, vc)
    out1 = torch.empty_like(q1)
    pa.pa_decode(q1, kc, vc, torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda(), 1 / math.sqrt(d), hk,
                 out1)
    torch.cuda.synchronize()
    o.reshape_and_cache(bits(k1), bits(v1), slots1, kh, vh)
    ref1 = o.decode(bits(q1), kh, vh, tables, lens, 1 / math.sqrt(d), 0, nthreads=8)
    assert_close(out1, ref1, "f16", "decode after prefill")


def test_prefill_bad_entries_give_nan_rows():
    rng = np.random.default_rng(62)
    c = PagedCase(rng, [100, 100], 4, 4, 128, 16, F16, 0.1)
    qs = np.array([0, 40, 80], dtype=np.int32)
    q = to_bits(rng.normal(0, 1, (80, 4, 128)), F16)
    tables = c.tables.copy()
    tables[1, 2] = c.NB + 7
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = run_prefill(c, q, qs, err=err, tables=tables)
    assert err.item() & pa.PA_DEVERR_TABLE_RANGE
    assert torch.isnan(out[40:]).all()
    ref = oracle_pkg.get().prefill(q[:40].copy(), c.k_cache, c.v_cache, c.tables[:1].copy(), c.lens[:1].copy(),
                                   qs[:2].copy(), c.scale, F16)
    assert_close(out[:40], ref, "f16", "unaffected sequence")
