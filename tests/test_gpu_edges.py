"""GPU parity on small paged problems that sweep the supported shapes, plus the
degenerate and error cases: empty contexts, single tokens, lengths on block and
partition boundaries, the longest context a table can hold, bad table entries,
bad lengths and bad slots (reported through the error word, never a fault)."""
import itertools
import math

import numpy as np
import pytest
import torch

from gpu_cases import assert_close
from pins import BF16, F16, PagedCase
import oracle as oracle_pkg
from paged_kv_cache_374_b200 import binding as pa

pytestmark = pytest.mark.gpu

TDT = {F16: torch.float16, BF16: torch.bfloat16}
WK = {F16: "f16", BF16: "bf16"}


def dev(bits_arr, dtype):
    return torch.from_numpy(np.ascontiguousarray(bits_arr).view(np.int16)).view(TDT[dtype]).cuda()


def run_case(c, partition_tokens=0, err=None, tables=None, lens=None):
    q = dev(c.q, c.dtype)
    kc, vc = dev(c.k_cache, c.dtype), dev(c.v_cache, c.dtype)
    tb = torch.from_numpy(c.tables if tables is None else tables).cuda()
    ln = torch.from_numpy(c.lens if lens is None else lens).cuda()
    out = torch.empty_like(q)
    pa.pa_decode(q, kc, vc, tb, ln, c.scale, c.Hk, out, partition_tokens=partition_tokens, err_word=err)
    torch.cuda.synchronize()
    return out


# groups 1 (CUDA-core path), 2..16 (tensor-core path), 32 (CUDA-core path again)
SHAPES = list(itertools.product([64, 128], [16, 32, 64], [1, 2, 4, 8, 16], [F16, BF16])) + [(128, 16, 32, F16)]


@pytest.mark.parametrize("d,bs,g,dtype", SHAPES)
def test_shape_sweep(d, bs, g, dtype):
    rng = np.random.default_rng(d * 1000 + bs * 10 + g + dtype)
    hk = 2
    lens = [0, 1, bs - 1, bs, bs + 1, 64, 511, 512, 513, 1000 + bs // 2]
    c = PagedCase(rng, lens, hk * g, hk, d, bs, dtype, 1 / math.sqrt(d), extra_blocks=4)
    ref = c.run(oracle_pkg.get(), nthreads=8)
    for pt in (0, 64, 192):
        out = run_case(c, partition_tokens=pt)
        assert_close(out, ref, WK[dtype], f"d{d} bs{bs} g{g} pt{pt}")
        assert torch.count_nonzero(out[0]) == 0            # empty context: zeros


def test_split_invariance_and_relabelling():
    rng = np.random.default_rng(31)
    c = PagedCase(rng, [3000, 1500, 64, 4096], 8, 8, 128, 16, F16, 0.088, extra_blocks=10)
    outs = [run_case(c, partition_tokens=pt).double() for pt in (64, 512, 4096)]
    assert (outs[0] - outs[2]).abs().max().item() <= 2e-3
    assert (outs[1] - outs[2]).abs().max().item() <= 2e-3
    a = run_case(c)
    c.relabel(rng.permutation(c.NB).astype(np.int32))
    b = run_case(c)
    assert torch.equal(a, b), "relabelling physical blocks changed the output"


def test_longest_context_and_large_scores():
    rng = np.random.default_rng(32)
    c = PagedCase(rng, [64 * 40, 7], 4, 4, 128, 64, BF16, 0.5, extra_blocks=1)   # table exactly full for seq 0
    ref = c.run(oracle_pkg.get(), nthreads=8)
    assert_close(run_case(c), ref, "bf16", "full table, large scores")


def test_bad_table_entry_gives_nan_row_and_error_bit():
    rng = np.random.default_rng(33)
    c = PagedCase(rng, [40, 40, 900], 4, 4, 64, 16, F16, 0.125)
    ref = c.run(oracle_pkg.get())
    for bad in (c.NB + 3, -2):
        tables = c.tables.copy()
        tables[1, 1] = bad
        tables[2, 40] = bad          # inside a later partition of sequence 2
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = run_case(c, err=err, tables=tables)
        assert err.item() & pa.PA_DEVERR_TABLE_RANGE
        assert torch.isnan(out[1]).all() and torch.isnan(out[2]).all()
        assert_close(out[0], ref[0], "f16", "unaffected row")


def test_bad_context_len_gives_nan_row_and_error_bit():
    rng = np.random.default_rng(34)
    c = PagedCase(rng, [20, 20], 2, 2, 64, 16, F16, 0.125)
    lens = c.lens.copy()
    lens[0] = c.MB * 16 + 1
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = run_case(c, err=err, lens=lens)
    assert err.item() & pa.PA_DEVERR_LEN_RANGE
    assert torch.isnan(out[0]).all() and not torch.isnan(out[1]).any()


def test_reshape_and_cache_slots():
    """Negative slots are skipped in silence; slots past the pool set an error bit
    and are skipped; the rest is a bit-exact copy (compared with the oracle)."""
    rng = np.random.default_rng(35)
    nb, bs, hk, d, n = 8, 16, 4, 128, 12
    for dtype in (torch.float16, torch.bfloat16):
        kc = torch.randn(nb, bs, hk, d, device="cuda").to(dtype)
        vc = torch.randn(nb, bs, hk, d, device="cuda").to(dtype)
        k = torch.randn(n, hk, d, device="cuda").to(dtype)
        v = torch.randn(n, hk, d, device="cuda").to(dtype)
        slots = rng.choice(nb * bs, size=n, replace=False).astype(np.int64)
        slots[2] = -1
        slots[5] = nb * bs
        kh, vh = kc.view(torch.int16).cpu().numpy().view(np.uint16), vc.view(torch.int16).cpu().numpy().view(np.uint16)
        skipped = oracle_pkg.get().reshape_and_cache(k.view(torch.int16).cpu().numpy().view(np.uint16),
                                                     v.view(torch.int16).cpu().numpy().view(np.uint16),
                                                     slots, kh, vh)
        assert skipped == 2
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        pa.pa_reshape_and_cache(k, v, torch.from_numpy(slots).cuda(), kc, vc, err_word=err)
        torch.cuda.synchronize()
        assert err.item() == pa.PA_DEVERR_SLOT_RANGE
        assert np.array_equal(kc.view(torch.int16).cpu().numpy().view(np.uint16), kh)
        assert np.array_equal(vc.view(torch.int16).cpu().numpy().view(np.uint16), vh)


def test_empty_batch_and_binding_checks():
    q = torch.empty(0, 4, 64, dtype=torch.float16, device="cuda")
    kc = torch.zeros(4, 16, 4, 64, dtype=torch.float16, device="cuda")
    tb = torch.zeros(0, 2, dtype=torch.int32, device="cuda")
    ln = torch.zeros(0, dtype=torch.int32, device="cuda")
    pa.pa_decode(q, kc, kc, tb, ln, 0.125, 4, torch.empty_like(q))
    q1 = torch.zeros(1, 4, 64, dtype=torch.bfloat16, device="cuda")
    tb1 = torch.zeros(1, 2, dtype=torch.int32, device="cuda")
    ln1 = torch.ones(1, dtype=torch.int32, device="cuda")
    with pytest.raises(TypeError):                       # q bf16, caches fp16
        pa.pa_decode(q1, kc, kc, tb1, ln1, 0.125, 4, torch.empty_like(q1))
    with pytest.raises(pa.PAError) as e:
        pa.pa_decode(torch.zeros(1, 4, 96, dtype=torch.float16, device="cuda"),
                     torch.zeros(4, 16, 4, 96, dtype=torch.float16, device="cuda"),
                     torch.zeros(4, 16, 4, 96, dtype=torch.float16, device="cuda"),
                     torch.zeros(1, 2, dtype=torch.int32, device="cuda"),
                     torch.ones(1, dtype=torch.int32, device="cuda"), 0.1, 4,
                     torch.zeros(1, 4, 96, dtype=torch.float16, device="cuda"))
    assert e.value.status == pa.PA_ERR_UNSUPPORTED


def test_bounded_wait_gives_up_and_reports():
    """A wait on a barrier that nothing completes runs out by itself, reports
    PA_DEVERR_TIMEOUT, and the context keeps working afterwards."""
    import time
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    outcome = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    pa.pa_selftest_bounded_wait(err, outcome)
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 30
    assert outcome.item() == 0 and err.item() == pa.PA_DEVERR_TIMEOUT
    c = PagedCase(np.random.default_rng(80), [100, 300], 4, 4, 128, 16, F16, 0.1)
    assert_close(run_case(c), c.run(oracle_pkg.get()), "f16", "decode after the self-test")


@pytest.mark.parametrize("mode", ["mha", "gqa", "fp8", "shared_prefix", "two_launches"])
def test_many_calls_on_one_workspace_leave_the_counters_zero(mode):
    """Decode calls in a row on one workspace, with split contexts: the merge of
    each (sequence, head) runs in the engine's tail from a completion queue whose
    counters live at the start of the workspace.  Every call must leave them zero
    (the next call starts from them) and give the same output bit for bit, which
    must match the oracle."""
    rng = np.random.default_rng(35)
    lens = [700, 2100, 257, 1024, 33, 1500, 513, 3000]
    if mode == "two_launches":   # more sequences than one engine launch schedules (1024)
        lens = rng.integers(200, 700, size=1100).tolist()
    g = 4 if mode == "gqa" else 1
    hk = 2 if mode in ("gqa", "two_launches") else 4
    c = PagedCase(rng, lens, hk * g, hk, 128, 16, BF16 if mode == "gqa" else F16, 1 / math.sqrt(128))
    if mode == "shared_prefix":
        members, nb = [1, 3, 5, 7], 512 // 16
        for s in members[1:]:
            c.tables[s, :nb] = c.tables[1, :nb]
            c.seq_k[s][:512] = c.seq_k[1][:512]
            c.seq_v[s][:512] = c.seq_v[1][:512]
        c._assemble()
    P = 256
    s_, h_ = c.S, c.H
    need = pa.pa_decode_workspace_size(s_, h_, hk, 128, 16, c.MB, P)
    up = lambda x: (x + 255) // 256 * 256
    counters = 256 + 2 * up(s_ * h_ * 4)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    q = dev(c.q, c.dtype)
    tb, ln = torch.from_numpy(c.tables).cuda(), torch.from_numpy(c.lens).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    if mode == "fp8":
        codes = lambda bits: (torch.from_numpy(bits.view(np.int16)).view(torch.float16).float() * 32).clamp(
            -448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
        kc, vc = codes(c.k_cache).cuda(), codes(c.v_cache).cuda()
        call = lambda out: pa.pa_decode_fp8(q, kc, vc, tb, ln, c.scale, 1 / 32, 1 / 32, hk, out, workspace=ws,
                                            partition_tokens=P, err_word=err)
        ref = oracle_pkg.get().decode_fp8(c.q, kc.cpu().numpy(), vc.cpu().numpy(), c.tables, c.lens, c.scale,
                                          1 / 32, 1 / 32, F16, nthreads=8)
    else:
        kc, vc = dev(c.k_cache, c.dtype), dev(c.v_cache, c.dtype)
        if mode == "shared_prefix":
            grp = pa.pa_find_shared_prefixes(c.tables, c.lens, c.bs, P)
            assert grp.num_groups == 1 and grp.max_shared_tokens == 512
            start, offs, mem = grp.to("cuda")
            call = lambda out: pa.pa_decode_shared_prefix(q, kc, vc, tb, ln, c.scale, hk, out, start, offs, mem,
                                                          grp.num_groups, grp.max_group_size, grp.max_shared_tokens,
                                                          workspace=ws, partition_tokens=P, err_word=err)
        else:
            call = lambda out: pa.pa_decode(q, kc, vc, tb, ln, c.scale, hk, out, workspace=ws, partition_tokens=P,
                                            err_word=err)
        ref = c.run(oracle_pkg.get(), nthreads=8)
    outs = [torch.full_like(q, float("nan")) for _ in range(8 if mode == "two_launches" else 40)]
    for out in outs:
        call(out)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert int(ws[:counters].count_nonzero()) == 0
    for out in outs[1:]:
        assert torch.equal(out, outs[0])
    assert_close(outs[0], ref, WK[c.dtype], mode)
