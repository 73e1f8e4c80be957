"""Paged prefill on the GPU against the oracle: chunks with and without cached
context before them, MHA and GQA, block sizes 16/32/64, head_dim 64/128, fp16 and
bf16, a full allocator -> cache write -> prefill -> decode flow, and error rows."""
import math

import numpy as np
import pytest
import torch

from gpu_cases import assert_close, bits
from pins import BF16, F16, PagedCase, from_bits, to_bits
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


@pytest.mark.parametrize("dtype", [F16, BF16])
def test_prefill_negative_scale(dtype):
    """A negative scale: the kernel takes the tile max over -x.  Covers query tiles
    of 128 rows (copied by TMA) and partial ones (stored by the row threads)."""
    rng = np.random.default_rng(68)
    d, bs, hk, g = 128, 16, 2, 2
    lens = [256, 600, 129]
    n_new = [256, 300, 129]    # two full tiles; a full and a ragged CTA; a tile and one row
    c = PagedCase(rng, lens, hk * g, hk, d, bs, dtype, -0.7 / math.sqrt(d), extra_blocks=3)
    qs = np.concatenate([[0], np.cumsum(n_new)]).astype(np.int32)
    q = to_bits(rng.normal(0, 1, (int(qs[-1]), hk * g, d)), dtype)
    ref = oracle_pkg.get().prefill(q, c.k_cache, c.v_cache, c.tables, c.lens, qs, c.scale, dtype, nthreads=8)
    out = run_prefill(c, q, qs)
    assert_close(out, ref, WK[dtype], "prefill, negative scale")


def test_prefill_empty_chunks():
    """Sequences with no new rows (query_start[s] == query_start[s+1]) launch CTAs that
    find no rows and leave; the others match the oracle."""
    rng = np.random.default_rng(69)
    d, bs, hk, g = 128, 16, 2, 2
    lens = [100, 300, 50, 257]
    n_new = [0, 300, 0, 1]     # the grid is sized by the 300-row chunk
    c = PagedCase(rng, lens, hk * g, hk, d, bs, F16, 1 / math.sqrt(d), extra_blocks=3)
    qs = np.concatenate([[0], np.cumsum(n_new)]).astype(np.int32)
    q = to_bits(rng.normal(0, 1, (int(qs[-1]), hk * g, d)), F16)
    ref = oracle_pkg.get().prefill(q, c.k_cache, c.v_cache, c.tables, c.lens, qs, c.scale, F16, nthreads=8)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = run_prefill(c, q, qs, err=err)
    assert err.item() == 0
    assert_close(out, ref, "f16", "prefill with empty chunks")


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


@pytest.mark.parametrize("bad_block,bad_id", [(2, "past"), (10, "negative"), (20, "past")])
def test_prefill_bad_entries_give_nan_rows(bad_block, bad_id):
    """A bad table entry in the first K/V tile (its copy goes out before the range
    check, so the box is skipped and the CTA waits for its other copies), in the
    second, or in a later one: NaN rows for that sequence only, the error bit, and
    the other sequence unchanged."""
    rng = np.random.default_rng(62 + bad_block)
    c = PagedCase(rng, [400, 400], 4, 4, 128, 16, F16, 0.1)
    qs = np.array([0, 300, 600], dtype=np.int32)
    q = to_bits(rng.normal(0, 1, (600, 4, 128)), F16)
    tables = c.tables.copy()
    tables[1, bad_block] = c.NB + 7 if bad_id == "past" else -3
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = run_prefill(c, q, qs, err=err, tables=tables)
    assert err.item() & pa.PA_DEVERR_TABLE_RANGE
    assert torch.isnan(out[300:]).all()
    ref = oracle_pkg.get().prefill(q[:300].copy(), c.k_cache, c.v_cache, c.tables[:1].copy(), c.lens[:1].copy(),
                                   qs[:2].copy(), c.scale, F16, nthreads=8)
    assert_close(out[:300], ref, "f16", "unaffected sequence")


# ------------------------------------------------- large logits: the rescale path
#
# The kernel keeps the running max it exponentiates against until a row's tile max
# grows past it by more than 2^8 (in log2 units), then rescales O and the row sum
# in tensor memory.  N(0,1) inputs at scale 1/sqrt(d) never get there after the
# first tile, so these cases make the scores grow along the sequence: keys scaled
# by (1 + t / 24) at position t, or a large scale.  rescale_events() counts, from
# fp64 scores on the host, the (row, head) pairs that must take that path, so each
# case shows it is reached.

LOG2E = 1.4426950408889634


def ramp_keys(c, rate=24.0):
    """Scale every sequence's key at position t by (1 + t / rate)."""
    for s in range(c.S):
        k = from_bits(c.seq_k[s], c.dtype)
        k *= (1.0 + np.arange(k.shape[0]) / rate)[:, None, None]
        c.seq_k[s] = to_bits(k, c.dtype)
    c._assemble()


def _events(x_row, t_lo, t_hi):
    """Rescales of one row over tokens [t_lo, t_hi), walked in 64-token tiles."""
    m, n = None, 0
    for t0 in range(t_lo, t_hi, 64):
        mt = float(np.max(x_row[t0:min(t0 + 64, t_hi)]))
        if m is None:
            m = mt
        elif mt > m + 8.0:
            n, m = n + 1, mt
    return n


def rescale_events(c, q_bits, qs):
    q = from_bits(q_bits, c.dtype)
    g = c.H // c.Hk
    total = 0
    for s in range(c.S):
        n, L = int(qs[s + 1] - qs[s]), int(c.lens[s])
        k = from_bits(c.seq_k[s], c.dtype)
        for h in range(c.H):
            x = q[qs[s]:qs[s + 1], h] @ k[:, h // g].T * (c.scale * LOG2E)
            total += sum(_events(x[i], 0, L - n + i + 1) for i in range(n))
    return total


LARGE = [(128, 16, 1, F16, "ramp"), (128, 32, 4, BF16, "ramp"), (64, 64, 2, BF16, "ramp"),
         (128, 16, 1, F16, "scale"), (64, 32, 2, BF16, "scale")]


@pytest.mark.parametrize("d,bs,g,dtype,kind", LARGE)
def test_prefill_large_logits_take_the_rescale_path(d, bs, g, dtype, kind):
    rng = np.random.default_rng(63 + d + bs + g)
    hk = 2
    lens = [37, 200, 64, 513, 9]
    n_new = [37, 70, 1, 200, 9]
    scale = 2.0 if kind == "scale" else 1 / math.sqrt(d)
    c = PagedCase(rng, lens, hk * g, hk, d, bs, dtype, scale, extra_blocks=3)
    if kind == "ramp":
        ramp_keys(c)
    qs = np.concatenate([[0], np.cumsum(n_new)]).astype(np.int32)
    q = to_bits(rng.normal(0, 1, (int(qs[-1]), hk * g, d)), dtype)
    assert rescale_events(c, q, qs) >= 100
    ref = oracle_pkg.get().prefill(q, c.k_cache, c.v_cache, c.tables, c.lens, qs, c.scale, dtype, nthreads=8)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = run_prefill(c, q, qs, err=err)
    assert err.item() == 0
    assert_close(out, ref, WK[dtype], f"large logits ({kind}) d{d} bs{bs} g{g}")


@pytest.mark.parametrize("dtype,kind", [(F16, "ramp"), (BF16, "ramp"), (BF16, "scale")])
def test_shared_prefix_large_logits_take_the_rescale_path(dtype, kind):
    """The same kernel in its shared-prefix mode (pa_decode_shared_prefix): each CTA
    walks one 256-token partition of the shared prefix in four tiles with no mask."""
    rng = np.random.default_rng(64)
    d, bs, hk, g, P = 128, 32, 2, 4, 256
    scale = 2.0 if kind == "scale" else 1 / math.sqrt(d)
    c = PagedCase(rng, [700, 650, 600, 520, 300, 513], hk * g, hk, d, bs, dtype, scale, extra_blocks=4)
    if kind == "ramp":
        ramp_keys(c)
    members = [0, 1, 2, 3]
    nb = 512 // bs
    for s in members[1:]:
        c.tables[s, :nb] = c.tables[0, :nb]
        c.seq_k[s][:512] = c.seq_k[0][:512]
        c.seq_v[s][:512] = c.seq_v[0][:512]
    c._assemble()
    grp = pa.pa_find_shared_prefixes(c.tables, c.lens, c.bs, P)
    assert grp.num_groups == 1 and grp.max_shared_tokens == 512
    q = from_bits(c.q, dtype)
    k0 = from_bits(c.seq_k[0], dtype)
    events = sum(_events(q[s, h] @ k0[:, h // g].T * (c.scale * LOG2E), p * P, (p + 1) * P)
                 for s in members for h in range(hk * g) for p in range(2))
    assert events >= 8
    qd = torch.from_numpy(np.ascontiguousarray(c.q).view(np.int16)).view(TDT[dtype]).cuda()
    out = torch.empty_like(qd)
    start, offs, mem = grp.to("cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_decode_shared_prefix(qd, dev(c.k_cache, dtype), dev(c.v_cache, dtype), torch.from_numpy(c.tables).cuda(),
                               torch.from_numpy(c.lens).cuda(), c.scale, hk, out, start, offs, mem, grp.num_groups,
                               grp.max_group_size, grp.max_shared_tokens, partition_tokens=P, err_word=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    ref = oracle_pkg.get().decode(c.q, c.k_cache, c.v_cache, c.tables, c.lens, c.scale, dtype, nthreads=8)
    assert_close(out, ref, WK[dtype], f"shared prefix, large logits ({kind})")


# --------------------------------------------------------- the benchmarked size

def test_prefill_at_bench_size_on_sampled_rows():
    """8 whole 2048-token prompts at the 7B layer shape (32 heads, head_dim 128,
    block size 16, fp16): the configuration the prefill benchmark times.  Checked
    on sampled query rows -- the first two and the last of every 128-row tile, plus
    random ones, every head -- each against the oracle's decode of that row over its
    visible prefix (a query row at position p attends exactly as a decode over
    p + 1 tokens does)."""
    s, chunk, h, d, bs = 8, 2048, 32, 128, 16
    nblk = chunk // bs
    nb = s * nblk + 8
    g = torch.Generator(device="cuda").manual_seed(65)
    kc = torch.randn(nb, bs, h, d, generator=g, device="cuda").to(torch.float16)
    vc = torch.randn(nb, bs, h, d, generator=g, device="cuda").to(torch.float16)
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(66))[: s * nblk]
    tables = perm.view(s, nblk).to(torch.int32).numpy().copy()
    lens = np.full(s, chunk, dtype=np.int32)
    qs = (np.arange(s + 1) * chunk).astype(np.int32)
    q = torch.randn(s * chunk, h, d, generator=g, device="cuda").to(torch.float16)
    out = torch.empty_like(q)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_prefill(q, kc, vc, torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda(),
                  torch.from_numpy(qs).cuda(), 1 / math.sqrt(d), h, out, chunk, err_word=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    rng = np.random.default_rng(67)
    rows = sorted({0, 1} | {t * 128 + 127 for t in range(chunk // 128)} | set(rng.integers(0, chunk, 6).tolist()))
    seq_of = np.repeat(np.arange(s), len(rows))
    pos = np.tile(np.array(rows), s)
    q_rows = bits(q.view(s, chunk, h, d)[torch.from_numpy(seq_of).long(), torch.from_numpy(pos).long()])
    ref = oracle_pkg.get().decode(np.ascontiguousarray(q_rows), bits(kc), bits(vc),
                                  np.ascontiguousarray(tables[seq_of]), (pos + 1).astype(np.int32),
                                  1 / math.sqrt(d), F16, nthreads=8)
    got = out.view(s, chunk, h, d)[torch.from_numpy(seq_of).long(), torch.from_numpy(pos).long()]
    assert_close(got, ref, "f16", "prefill 8 x 2048, sampled rows")
