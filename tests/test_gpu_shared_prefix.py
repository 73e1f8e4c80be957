"""Two-level decode of sequences that share a prefix through the same blocks
(pa_decode_shared_prefix), on the GPU against the oracle: the shared part is
attended once per group, the suffix per sequence, and the result must be the
oracle's decode of every sequence over all of its tokens."""
import math

import numpy as np
import pytest
import torch

from gpu_cases import Step, assert_close, bits
from pins import BF16, F16, PagedCase
import oracle as oracle_pkg
from paged_kv_cache_374_b200 import binding as pa

pytestmark = pytest.mark.gpu

TDT = {F16: torch.float16, BF16: torch.bfloat16}
WK = {F16: "f16", BF16: "bf16"}


def dev(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(TDT[dtype]).cuda()


def share(c: PagedCase, members, tokens):
    """Members of a group use the lead's blocks (and data) for their first ``tokens``."""
    lead, nb = members[0], tokens // c.bs
    for s in members[1:]:
        c.tables[s, :nb] = c.tables[lead, :nb]
        c.seq_k[s][:tokens] = c.seq_k[lead][:tokens]
        c.seq_v[s][:tokens] = c.seq_v[lead][:tokens]
    c._assemble()


def run_both(c, P, err=None, groups=None):
    q = dev(c.q, c.dtype)
    kc, vc = dev(c.k_cache, c.dtype), dev(c.v_cache, c.dtype)
    tb, ln = torch.from_numpy(c.tables).cuda(), torch.from_numpy(c.lens).cuda()
    g = groups or pa.pa_find_shared_prefixes(c.tables, c.lens, c.bs, P)
    start, offs, mem = g.to("cuda")
    out = torch.empty_like(q)
    pa.pa_decode_shared_prefix(q, kc, vc, tb, ln, c.scale, c.Hk, out, start, offs, mem, g.num_groups,
                               g.max_group_size, g.max_shared_tokens, partition_tokens=P, err_word=err)
    ref = torch.empty_like(q)
    pa.pa_decode(q, kc, vc, tb, ln, c.scale, c.Hk, ref, partition_tokens=P)
    torch.cuda.synchronize()
    return out, ref, g


CASES = [(128, 16, 1, F16), (128, 32, 4, BF16), (64, 64, 1, BF16), (64, 16, 8, F16), (128, 64, 2, F16)]


@pytest.mark.parametrize("d,bs,g,dtype", CASES)
def test_shared_prefix_matches_oracle(d, bs, g, dtype):
    rng = np.random.default_rng(70 + d + bs + g)
    P = 64
    lens = [300, 200, 193, 257, 140, 129, 130, 400, 90, 1]
    hk = 2
    c = PagedCase(rng, lens, hk * g, hk, d, bs, dtype, 1 / math.sqrt(d), extra_blocks=4)
    share(c, [0, 1, 2, 3], 192)        # three partitions
    share(c, [0, 4], 64)               # 4 shares only the first with 0
    share(c, [5, 6, 7], 128)           # two partitions
    out, ref_gpu, grp = run_both(c, P)
    assert grp.num_groups == 2
    assert list(grp.seq_start) == [192, 192, 192, 192, 0, 128, 128, 128, 0, 0]
    ref = oracle_pkg.get().decode(c.q, c.k_cache, c.v_cache, c.tables, c.lens, c.scale, dtype, nthreads=8)
    assert_close(out, ref, WK[dtype], f"shared d{d} bs{bs} g{g}")
    assert_close(ref_gpu, ref, WK[dtype], "pa_decode")


def test_shared_prefix_negative_scale():
    """A negative scale through the prefix kernel (its tile max is taken over -x)."""
    rng = np.random.default_rng(79)
    c = PagedCase(rng, [300, 200, 193, 257, 70], 4, 2, 128, 16, F16, -1 / math.sqrt(128), extra_blocks=4)
    share(c, [0, 1, 2, 3], 192)
    out, _, grp = run_both(c, 64)
    assert grp.num_groups == 1
    ref = oracle_pkg.get().decode(c.q, c.k_cache, c.v_cache, c.tables, c.lens, c.scale, F16, nthreads=8)
    assert_close(out, ref, "f16", "shared prefix, negative scale")


def test_no_groups_is_pa_decode():
    rng = np.random.default_rng(71)
    c = PagedCase(rng, [100, 300, 64], 4, 4, 128, 16, F16, 0.1)
    out, ref, grp = run_both(c, 64)
    assert grp.num_groups == 0
    assert torch.equal(out, ref)


def test_bad_start_is_reported_and_ignored():
    """A member whose start is not a multiple of the partition runs whole in the
    per-sequence kernel (and gets no shared partials): still the oracle's result."""
    rng = np.random.default_rng(72)
    c = PagedCase(rng, [300, 280, 290], 8, 8, 128, 16, BF16, 1 / math.sqrt(128))
    share(c, [0, 1, 2], 256)
    grp = pa.pa_find_shared_prefixes(c.tables, c.lens, c.bs, 64)
    assert list(grp.seq_start) == [256, 256, 256]
    grp.seq_start = grp.seq_start.copy()
    grp.seq_start[2] = 200
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, _, _ = run_both(c, 64, err=err, groups=grp)
    assert err.item() & pa.PA_DEVERR_LEN_RANGE
    ref = oracle_pkg.get().decode(c.q, c.k_cache, c.v_cache, c.tables, c.lens, c.scale, BF16)
    assert_close(out, ref, "bf16", "bad start")


def test_beam_full_size():
    """The beam workload (128 sequences forked from one 512-token prompt, block
    size 64): one group sharing the prompt; compared with the oracle on sampled
    (sequence, head) pairs and with pa_decode everywhere."""
    step = Step("beam")
    t = step.tensors()
    P = pa.pa_decode_partition_tokens(step.spec.num_seqs, 32, 32, 128, step.bs, step.tables.shape[1])
    grp = pa.pa_find_shared_prefixes(step.tables, step.lens, step.bs, P)
    assert grp.num_groups >= 1 and grp.max_shared_tokens == step.spec.prefix_tokens // P * P
    start, offs, mem = grp.to("cuda")
    tb, ln = torch.from_numpy(step.tables).cuda(), torch.from_numpy(step.lens).cuda()
    pa.pa_reshape_and_cache(t["k"], t["v"], torch.from_numpy(step.slots).cuda(), t["k_cache"], t["v_cache"])
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(t["q"])
    pa.pa_decode_shared_prefix(t["q"], t["k_cache"], t["v_cache"], tb, ln, step.spec.scale, 32, out, start, offs,
                               mem, grp.num_groups, grp.max_group_size, grp.max_shared_tokens, err_word=err)
    ref_gpu = torch.empty_like(out)
    pa.pa_decode(t["q"], t["k_cache"], t["v_cache"], tb, ln, step.spec.scale, 32, ref_gpu)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert (out.float() - ref_gpu.float()).abs().max().item() <= 2e-3
    o = oracle_pkg.get()
    kh, vh = bits(t["k_cache"]), bits(t["v_cache"])
    rng = np.random.default_rng(73)
    pairs = np.array([(int(rng.integers(0, step.spec.num_seqs)), int(rng.integers(0, 32))) for _ in range(64)],
                     dtype=np.int32)
    ref = o.decode(bits(t["q"]), kh, vh, step.tables, step.lens, step.spec.scale, F16, pairs=pairs, nthreads=8)
    got = out[torch.from_numpy(pairs[:, 0]).long(), torch.from_numpy(pairs[:, 1]).long()]
    assert_close(got, ref, "f16", "beam shared")


def test_more_sequences_than_one_launch():
    """1100 sequences in four groups: the engine runs in two launches (at most
    1024 sequences each); every sequence's start and partials must line up."""
    rng = np.random.default_rng(74)
    S, P, bs = 1100, 64, 16
    lens = rng.integers(65, 400, size=S).astype(np.int32)
    c = PagedCase(rng, lens, 2, 2, 64, bs, F16, 0.125, extra_blocks=2)
    groups = [list(range(0, 300)), list(range(300, 700)), list(range(700, 1050, 2)), [1098, 1099]]
    for g in groups:
        share(c, g, 64 * int(min(-(-int(min(lens[g])) // 64) - 1, 3)))
    out, ref_gpu, grp = run_both(c, P)
    assert grp.num_groups >= 4
    assert torch.equal(torch.isnan(out), torch.isnan(ref_gpu))
    ref = oracle_pkg.get().decode(c.q, c.k_cache, c.v_cache, c.tables, c.lens, c.scale, F16, nthreads=8)
    assert_close(out, ref, "f16", "1100 sequences shared")


def test_launch_bounds_too_small_are_reported():
    rng = np.random.default_rng(75)
    c = PagedCase(rng, [300] * 6, 4, 4, 128, 16, F16, 0.1)
    share(c, list(range(6)), 256)
    g = pa.pa_find_shared_prefixes(c.tables, c.lens, c.bs, 64)
    assert g.max_shared_tokens == 256 and g.max_group_size == 6
    for mg, mt in ((6, 128), (6, 256)):
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        q = dev(c.q, F16)
        out = torch.empty_like(q)
        start, offs, mem = g.to("cuda")
        pa.pa_decode_shared_prefix(q, dev(c.k_cache, F16), dev(c.v_cache, F16), torch.from_numpy(c.tables).cuda(),
                                   torch.from_numpy(c.lens).cuda(), c.scale, 4, out, start, offs, mem,
                                   g.num_groups, mg, mt, partition_tokens=64, err_word=err)
        torch.cuda.synchronize()
        assert bool(err.item() & pa.PA_DEVERR_LEN_RANGE) == (mt < 256)


@pytest.mark.parametrize("bad", ["member", "end_past_batch", "end_before_start"])
def test_group_arrays_out_of_range_are_skipped(bad):
    """group_offsets and group_members come from the caller.  A group whose
    offsets leave [0, num_seqs] or run backwards, or that lists a member outside
    the batch, is skipped whole with PA_DEVERR_GROUP_RANGE (no access outside the
    arrays the caller passed); every sequence outside it still gets the oracle's
    result."""
    rng = np.random.default_rng(76)
    c = PagedCase(rng, [300, 280, 290, 200, 210, 150], 8, 8, 128, 16, F16, 1 / math.sqrt(128))
    share(c, [0, 1, 2], 256)
    share(c, [3, 4], 192)
    start = np.array([256, 256, 256, 192, 192, 0], dtype=np.int32)
    offs = np.array([0, 3, 5], dtype=np.int32)
    members = np.array([0, 1, 2, 3, 4], dtype=np.int32)
    if bad == "member":
        members[4] = 1 << 20
    elif bad == "end_past_batch":
        offs[2] = 6 + 9
        members = np.concatenate([members, np.zeros(16, dtype=np.int32)])  # the array is long enough; offsets are not
    else:
        offs[2] = 2
    grp = pa.SharedPrefixes(start, offs, members, 2, 3, 256)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, _, _ = run_both(c, 64, err=err, groups=grp)
    assert err.item() == pa.PA_DEVERR_GROUP_RANGE
    keep = [0, 1, 2, 5]
    pairs = np.array([(s, h) for s in keep for h in range(8)], dtype=np.int32)
    ref = oracle_pkg.get().decode(c.q, c.k_cache, c.v_cache, c.tables, c.lens, c.scale, F16, pairs=pairs)
    got = out[torch.from_numpy(pairs[:, 0]).long(), torch.from_numpy(pairs[:, 1]).long()]
    assert_close(got, ref, "f16", f"groups beside a bad one ({bad})")


def same_bits(a, b):
    """Bit-for-bit equality (unused cache rows hold NaN, which compares unequal)."""
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


def _new_tokens(c, rng):
    """Each sequence's new K/V row [S, Hk, d] and its slot: position L-1, which lies
    past every shared prefix (in a block private to the sequence)."""
    slots = np.array([c.tables[s, (n - 1) // c.bs] * c.bs + (n - 1) % c.bs for s, n in enumerate(c.lens)],
                     dtype=np.int64)
    shape = (len(c.lens), c.Hk, c.d)
    k = torch.from_numpy(rng.standard_normal(shape).astype(np.float32)).to(TDT[c.dtype]).cuda()
    v = torch.from_numpy(rng.standard_normal(shape).astype(np.float32)).to(TDT[c.dtype]).cuda()
    return k, v, torch.from_numpy(slots).cuda()


@pytest.mark.parametrize("dtype", [F16, BF16])
def test_decode_step_shared_prefix_is_write_then_decode(dtype):
    """pa_decode_step_shared_prefix (the prefix kernel a programmatic dependent of the
    cache write) equals pa_reshape_and_cache then pa_decode_shared_prefix bit for bit,
    caches and output, over nested groups and three back-to-back steps; the output
    is the oracle's decode over the written caches."""
    rng = np.random.default_rng(80)
    P = 64
    c = PagedCase(rng, [300, 200, 193, 257, 140, 129, 130, 400, 90, 1], 8, 2, 128, 16, dtype, 1 / math.sqrt(128),
                  extra_blocks=4)
    share(c, [0, 1, 2, 3], 192)
    share(c, [0, 4], 64)
    share(c, [5, 6, 7], 128)
    grp = pa.pa_find_shared_prefixes(c.tables, c.lens, c.bs, P)
    assert grp.num_groups == 2
    start, offs, mem = grp.to("cuda")
    q = dev(c.q, dtype)
    tb, ln = torch.from_numpy(c.tables).cuda(), torch.from_numpy(c.lens).cuda()
    k, v, slots = _new_tokens(c, rng)
    kc_a, vc_a = dev(c.k_cache, dtype), dev(c.v_cache, dtype)
    kc_b, vc_b = kc_a.clone(), vc_a.clone()
    err_a = torch.zeros(1, dtype=torch.int32, device="cuda")
    err_b = torch.zeros(1, dtype=torch.int32, device="cuda")
    out_a, out_b = torch.empty_like(q), torch.empty_like(q)
    pa.pa_reshape_and_cache(k, v, slots, kc_a, vc_a, err_word=err_a)
    pa.pa_decode_shared_prefix(q, kc_a, vc_a, tb, ln, c.scale, c.Hk, out_a, start, offs, mem, grp.num_groups,
                               grp.max_group_size, grp.max_shared_tokens, partition_tokens=P, err_word=err_a)
    for _ in range(3):
        pa.pa_decode_step_shared_prefix(k, v, slots, q, kc_b, vc_b, tb, ln, c.scale, c.Hk, out_b, start, offs, mem,
                                        grp.num_groups, grp.max_group_size, grp.max_shared_tokens,
                                        partition_tokens=P, err_word=err_b)
    torch.cuda.synchronize()
    assert err_a.item() == 0 and err_b.item() == 0
    assert same_bits(kc_a, kc_b) and same_bits(vc_a, vc_b)
    assert same_bits(out_a, out_b)
    kh, vh = bits(kc_b), bits(vc_b)
    ref = oracle_pkg.get().decode(c.q, kh, vh, c.tables, c.lens, c.scale, dtype, nthreads=8)
    assert_close(out_b, ref, WK[dtype], "fused shared-prefix step")


def test_decode_step_shared_prefix_without_groups_is_decode_step():
    """With no groups the call is pa_decode_step, bit for bit."""
    rng = np.random.default_rng(81)
    c = PagedCase(rng, [100, 300, 64], 4, 4, 128, 16, F16, 0.1)
    grp = pa.pa_find_shared_prefixes(c.tables, c.lens, c.bs, 64)
    assert grp.num_groups == 0
    start, offs, mem = grp.to("cuda")
    q = dev(c.q, F16)
    tb, ln = torch.from_numpy(c.tables).cuda(), torch.from_numpy(c.lens).cuda()
    k, v, slots = _new_tokens(c, rng)
    kc_a, vc_a = dev(c.k_cache, F16), dev(c.v_cache, F16)
    kc_b, vc_b = kc_a.clone(), vc_a.clone()
    out_a, out_b = torch.empty_like(q), torch.empty_like(q)
    pa.pa_decode_step(k, v, slots, q, kc_a, vc_a, tb, ln, c.scale, c.Hk, out_a, partition_tokens=64)
    pa.pa_decode_step_shared_prefix(k, v, slots, q, kc_b, vc_b, tb, ln, c.scale, c.Hk, out_b, start, offs, mem,
                                    grp.num_groups, grp.max_group_size, grp.max_shared_tokens, partition_tokens=64)
    torch.cuda.synchronize()
    assert same_bits(kc_a, kc_b) and same_bits(vc_a, vc_b) and same_bits(out_a, out_b)


def test_beam_decode_step_shared_prefix():
    """The beam workload's step through pa_decode_step_shared_prefix: bitwise the
    two-call step, and the oracle's decode on sampled (sequence, head) pairs."""
    step = Step("beam")
    t = step.tensors()
    grp = pa.pa_find_shared_prefixes(step.tables, step.lens, step.bs, 256)
    start, offs, mem = grp.to("cuda")
    tb, ln = torch.from_numpy(step.tables).cuda(), torch.from_numpy(step.lens).cuda()
    slots = torch.from_numpy(step.slots).cuda()
    kc_b, vc_b = t["k_cache"].clone(), t["v_cache"].clone()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out_a, out_b = torch.empty_like(t["q"]), torch.empty_like(t["q"])
    pa.pa_reshape_and_cache(t["k"], t["v"], slots, t["k_cache"], t["v_cache"], err_word=err)
    pa.pa_decode_shared_prefix(t["q"], t["k_cache"], t["v_cache"], tb, ln, step.spec.scale, 32, out_a, start, offs,
                               mem, grp.num_groups, grp.max_group_size, grp.max_shared_tokens, err_word=err)
    pa.pa_decode_step_shared_prefix(t["k"], t["v"], slots, t["q"], kc_b, vc_b, tb, ln, step.spec.scale, 32, out_b,
                                    start, offs, mem, grp.num_groups, grp.max_group_size, grp.max_shared_tokens,
                                    err_word=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert same_bits(t["k_cache"], kc_b) and same_bits(t["v_cache"], vc_b) and same_bits(out_a, out_b)
    rng = np.random.default_rng(82)
    pairs = np.array([(int(rng.integers(0, step.spec.num_seqs)), int(rng.integers(0, 32))) for _ in range(32)],
                     dtype=np.int32)
    ref = oracle_pkg.get().decode(bits(t["q"]), bits(kc_b), bits(vc_b), step.tables, step.lens, step.spec.scale, F16,
                                  pairs=pairs, nthreads=8)
    got = out_b[torch.from_numpy(pairs[:, 0]).long(), torch.from_numpy(pairs[:, 1]).long()]
    assert_close(got, ref, "f16", "beam fused step")


def test_decode_step_shared_prefix_more_sequences_than_one_launch():
    """The fused step with 1100 sequences in four groups (two engine launches, which
    start only once the cache write is complete): bit for bit the two calls."""
    rng = np.random.default_rng(83)
    S, P, bs = 1100, 64, 16
    lens = rng.integers(65, 400, size=S).astype(np.int32)
    c = PagedCase(rng, lens, 2, 2, 64, bs, F16, 0.125, extra_blocks=2)
    for g in [list(range(0, 300)), list(range(300, 700)), list(range(700, 1050, 2)), [1098, 1099]]:
        share(c, g, 64 * int(min(-(-int(min(lens[g])) // 64) - 1, 3)))
    grp = pa.pa_find_shared_prefixes(c.tables, c.lens, c.bs, P)
    assert grp.num_groups >= 4
    start, offs, mem = grp.to("cuda")
    q = dev(c.q, F16)
    tb, ln = torch.from_numpy(c.tables).cuda(), torch.from_numpy(c.lens).cuda()
    k, v, slots = _new_tokens(c, rng)
    kc_a, vc_a = dev(c.k_cache, F16), dev(c.v_cache, F16)
    kc_b, vc_b = kc_a.clone(), vc_a.clone()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out_a, out_b = torch.empty_like(q), torch.empty_like(q)
    pa.pa_reshape_and_cache(k, v, slots, kc_a, vc_a, err_word=err)
    pa.pa_decode_shared_prefix(q, kc_a, vc_a, tb, ln, c.scale, c.Hk, out_a, start, offs, mem, grp.num_groups,
                               grp.max_group_size, grp.max_shared_tokens, partition_tokens=P, err_word=err)
    for _ in range(2):
        pa.pa_decode_step_shared_prefix(k, v, slots, q, kc_b, vc_b, tb, ln, c.scale, c.Hk, out_b, start, offs, mem,
                                        grp.num_groups, grp.max_group_size, grp.max_shared_tokens,
                                        partition_tokens=P, err_word=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert same_bits(kc_a, kc_b) and same_bits(vc_a, vc_b) and same_bits(out_a, out_b)


def test_bad_table_entry_in_a_shared_prefix():
    """A table entry out of range inside a group's shared prefix: the prefix kernel
    copies nothing from it and reports PA_DEVERR_TABLE_RANGE, and the prefix partial
    is NaN, so every member's rows come out NaN; the sequence outside the group
    still gets the oracle's result."""
    rng = np.random.default_rng(84)
    c = PagedCase(rng, [300, 280, 290, 200], 4, 4, 128, 16, F16, 1 / math.sqrt(128))
    share(c, [0, 1, 2], 256)
    ref = oracle_pkg.get().decode(c.q, c.k_cache, c.v_cache, c.tables, c.lens, c.scale, F16)
    for s in (0, 1, 2):  # the members' common entry 3 (tokens 48-63) points past the pool
        c.tables[s, 3] = c.NB + 7
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, _, grp = run_both(c, 64, err=err)
    assert grp.num_groups == 1 and list(grp.seq_start) == [256, 256, 256, 0]
    assert err.item() & pa.PA_DEVERR_TABLE_RANGE
    assert torch.isnan(out[:3].float()).all()
    assert_close(out[3:], ref[3:], "f16", "sequence outside the group")
