"""The C++ host allocator against the Python model of the pages' block pool, id for id
(P3 = "LLM 推理中的 PageAttention 实现原理：虚拟内存管理在 KV Cache 中的创新应用")."""
import json
import os

import numpy as np
import pytest

from oracle.block_pool import BlockPoolModel, ManagerModel, OutOfBlocks, RefcountError, swap_plan
from pins import GOLDEN


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_374_b200 import binding
    return binding


def _expect_error(pa, fn, status):
    with pytest.raises(pa.PAError) as e:
        fn()
    assert e.value.status == status


def test_random_operation_sequences_match_the_model(pa):
    rng = np.random.default_rng(5)
    for trial in range(20):
        n = int(rng.integers(1, 40))
        order = rng.permutation(n).astype(np.int32) if trial % 2 else None
        a = pa.BlockAllocator(n, order)
        m = BlockPoolModel(n, order)
        held = []  # one entry per reference held
        for _ in range(400):
            op = rng.integers(0, 6)
            if op == 0:
                k = int(rng.integers(0, 5))
                try:
                    want = m.allocate_n(k)
                except OutOfBlocks:
                    _expect_error(pa, lambda: a.alloc_n(k), pa.PA_ERR_OUT_OF_BLOCKS)
                    continue
                assert list(a.alloc_n(k)) == want
                held += want
            elif op == 1 and held:
                b = held.pop(int(rng.integers(0, len(held))))
                m.free(b)
                a.free(b)
            elif op == 2 and held:
                b = held[int(rng.integers(0, len(held)))]
                m.add_ref(b)
                a.add_ref(b)
                held.append(b)
            elif op == 3 and held:
                src = [held[int(i)] for i in rng.integers(0, len(held), size=int(rng.integers(1, 4)))]
                assert list(a.fork(np.array(src, dtype=np.int32))) == m.fork(src)
                held += src
            elif op == 4:
                b = int(rng.integers(0, n))
                if m.ref[b] == 0:
                    with pytest.raises(RefcountError):
                        m.free(b)
                    _expect_error(pa, lambda: a.free(b), pa.PA_ERR_REFCOUNT)
                    _expect_error(pa, lambda: a.add_ref(b), pa.PA_ERR_REFCOUNT)
            elif op == 5:
                try:
                    want = m.allocate()
                except OutOfBlocks:
                    _expect_error(pa, a.alloc, pa.PA_ERR_OUT_OF_BLOCKS)
                    continue
                assert a.alloc() == want
                held.append(want)
            assert a.num_free() == m.num_free()
            assert a.usage() == pytest.approx(m.usage_ratio(), abs=0)
            for b in range(n):
                assert a.refcount(b) == m.ref[b]
        # drain: the free queue order must match too
        for b in held:
            a.free(b)
            m.free(b)
        assert list(a.alloc_n(n)) == list(m.allocate_n(n))


def test_free_n_and_fork_are_all_or_nothing(pa):
    a = pa.BlockAllocator(6)
    ids = a.alloc_n(4)
    _expect_error(pa, lambda: a.free_n([ids[0], ids[1], 5]), pa.PA_ERR_REFCOUNT)   # 5 is free
    assert [a.refcount(int(b)) for b in ids] == [1, 1, 1, 1]
    _expect_error(pa, lambda: a.free_n([ids[0], ids[0]]), pa.PA_ERR_REFCOUNT)      # second drop would underflow
    assert a.refcount(int(ids[0])) == 1
    _expect_error(pa, lambda: a.fork(np.array([ids[0], 4], dtype=np.int32)), pa.PA_ERR_REFCOUNT)
    assert a.refcount(int(ids[0])) == 1
    _expect_error(pa, lambda: a.alloc_n(3), pa.PA_ERR_OUT_OF_BLOCKS)
    assert a.num_free() == 2
    _expect_error(pa, lambda: a.free(99), pa.PA_ERR_INVALID_ARG)
    assert a.refcount(99) == -1


def test_create_rejects_non_permutations(pa):
    with pytest.raises(pa.PAError):
        pa.BlockAllocator(3, np.array([0, 0, 1], dtype=np.int32))
    with pytest.raises(pa.PAError):
        pa.BlockAllocator(3, np.array([0, 1, 3], dtype=np.int32))


def test_demo_program_through_the_library(pa):
    """P3 §三 main(), with per-request tables kept by the caller."""
    with open(os.path.join(GOLDEN, "allocator_demo.json")) as f:
        demo = json.load(f)
    bs = demo["block_size"]
    a = pa.BlockAllocator(demo["num_blocks"])
    tables = {}
    for st in demo["steps"]:
        if st["op"] == "allocate_for_request":
            n = pa.pa_num_required_blocks(st["prompt_len"], bs)
            assert n == st["returns"]
            tables[st["rid"]] = list(a.alloc_n(n))
        elif st["op"] == "append_slot":
            # append_slot allocates only on a block boundary
            if st["current_len"] % bs == 0:
                tables[st["rid"]].append(a.alloc())
        elif st["op"] == "share_prefix_blocks":
            n = pa.pa_num_required_blocks(st["shared_len"], bs)
            tables[st["dst"]] = list(a.fork(np.array(tables[st["src"]][:n], dtype=np.int32)))
        elif st["op"] == "free_request":
            a.free_n(np.array(tables.pop(st["rid"]), dtype=np.int32))
        if "table" in st:
            rid = st.get("rid", st.get("dst"))
            assert tables[rid] == st["table"]
        for b, r in st.get("refcounts", {}).items():
            assert a.refcount(int(b)) == r
    assert a.num_free() == demo["final_num_free"] and a.usage() == demo["final_usage"]
    # the freed blocks were requeued at the back in the order the demo frees them
    assert list(a.alloc_n(1024))[-4:] == [2, 3, 0, 1]


def test_append_slots_matches_model_and_oracle(pa, oracle):
    rng = np.random.default_rng(9)
    bs, s, mb = 16, 12, 12
    nb = 200
    order = rng.permutation(nb).astype(np.int32)
    a = pa.BlockAllocator(nb, order)
    mgr = ManagerModel(nb, bs, order)
    lens = rng.integers(0, 100, size=s).astype(np.int32)
    tables = np.full((s, mb), -1, dtype=np.int32)
    for i in range(s):
        n = pa.pa_num_required_blocks(int(lens[i]), bs)
        mgr.allocate_for_request(i, int(lens[i]))
        tables[i, :n] = a.alloc_n(n)
        assert list(tables[i, :n]) == mgr.tables[i]
    for step in range(40):
        before = lens.copy()
        slots = a.append_slots(tables, lens, bs)
        for i in range(s):
            mgr.append_slot(i, int(before[i]))
            assert list(tables[i, :len(mgr.tables[i])]) == mgr.tables[i]
        assert np.array_equal(lens, before + 1)
        assert np.array_equal(slots, oracle.slot_mapping(tables, lens, bs))
        assert a.num_free() == mgr.pool.num_free()


def test_append_slots_is_all_or_nothing(pa):
    bs = 16
    a = pa.BlockAllocator(3)
    tables = np.full((3, 4), -1, dtype=np.int32)
    lens = np.array([16, 32, 5], dtype=np.int32)
    tables[0, 0] = a.alloc()
    tables[1, :2] = a.alloc_n(2)
    tables[2, 0] = -1   # token 5 would land in a block the table does not hold
    t0, l0 = tables.copy(), lens.copy()
    _expect_error(pa, lambda: a.append_slots(tables, lens, bs), pa.PA_ERR_INVALID_ARG)
    assert np.array_equal(tables, t0) and np.array_equal(lens, l0) and a.num_free() == 0
    lens[2] = 0        # now two sequences need a block and none is free: "preemption required"
    l0 = lens.copy()
    _expect_error(pa, lambda: a.append_slots(tables, lens, bs), pa.PA_ERR_OUT_OF_BLOCKS)
    assert np.array_equal(tables, t0) and np.array_equal(lens, l0)
    full = np.full((1, 1), 0, dtype=np.int32)
    _expect_error(pa, lambda: a.append_slots(full, np.array([16], dtype=np.int32), bs), pa.PA_ERR_INVALID_ARG)


def test_cow_prepare_matches_model(pa):
    """Random forks and appends: the library's copy-on-write step equals the model's,
    id for id, including the tables and every reference count."""
    rng = np.random.default_rng(10)
    for trial in range(30):
        bs = int(rng.choice([4, 16]))
        nb = 64
        order = rng.permutation(nb).astype(np.int32)
        a = pa.BlockAllocator(nb, order)
        mgr = ManagerModel(nb, bs, order)
        nreq, mb = 6, 12
        tables = np.full((nreq, mb), -1, dtype=np.int32)
        prompt = int(rng.integers(1, 3 * bs))
        mgr.allocate_for_request(0, prompt)
        n0 = pa.pa_num_required_blocks(prompt, bs)
        tables[0, :n0] = a.alloc_n(n0)
        stored = {0: prompt}
        for rid in range(1, nreq):           # forks of request 0's prompt, some of them partial
            shared = int(rng.integers(1, prompt + 1))
            mgr.share_prefix_blocks(0, rid, shared)
            k = pa.pa_num_required_blocks(shared, bs)
            tables[rid, :k] = a.fork(tables[0, :k])
            stored[rid] = shared
        lens = np.array([stored[r] for r in range(nreq)], dtype=np.int32)
        try:
            want = mgr.cow_prepare(dict(stored))
        except OutOfBlocks:
            with pytest.raises(pa.PAError):
                a.cow_prepare(tables, lens, bs)
            continue
        got = a.cow_prepare(tables, lens, bs)
        assert [tuple(x) for x in got.tolist()] == want
        for r in range(nreq):
            assert list(tables[r, :len(mgr.tables[r])]) == mgr.tables[r]
        for b in range(nb):
            assert a.refcount(b) == mgr.pool.ref[b]


def test_swap_plan_matches_model(pa):
    """Preempting a sequence moves its blocks to the other pool; a block it shares
    with another sequence stays allocated in the source pool for that sequence."""
    rng = np.random.default_rng(12)
    for trial in range(30):
        nd, nh = 24, 10
        od, oh = rng.permutation(nd).astype(np.int32), rng.permutation(nh).astype(np.int32)
        dev, host = pa.BlockAllocator(nd, od), pa.BlockAllocator(nh, oh)
        mdev, mhost = BlockPoolModel(nd, od), BlockPoolModel(nh, oh)
        k = int(rng.integers(1, 8))
        row = dev.alloc_n(k)
        assert list(row) == mdev.allocate_n(k)
        shared = [int(b) for b in row[: int(rng.integers(0, k + 1))]]   # another sequence holds a prefix
        dev.fork(np.array(shared, dtype=np.int32))
        mdev.fork(shared)
        other = host.alloc_n(int(rng.integers(0, 5)))
        mhost.allocate_n(len(other))
        mrow = [int(b) for b in row]
        try:
            want = swap_plan(mdev, mhost, mrow)
        except OutOfBlocks:
            with pytest.raises(pa.PAError) as e:
                pa.pa_swap_plan(dev.handle, host.handle, row, k)
            assert e.value.status == pa.PA_ERR_OUT_OF_BLOCKS
            continue
        got = pa.pa_swap_plan(dev.handle, host.handle, row, k)
        assert [tuple(x) for x in got.tolist()] == want and list(row) == mrow
        assert dev.num_free() == mdev.num_free() and host.num_free() == mhost.num_free()
        for b in range(nd):
            assert dev.refcount(b) == mdev.ref[b]
        # and back again
        back = swap_plan(mhost, mdev, mrow)
        got = pa.pa_swap_plan(host.handle, dev.handle, row, k)
        assert [tuple(x) for x in got.tolist()] == back and list(row) == mrow
        assert host.num_free() == mhost.num_free()


def test_prefill_slots_match_model_and_oracle(pa, oracle):
    """A chunk of new tokens per sequence: blocks open exactly as repeated appends
    would open them (the model), and every new token's slot is the oracle's
    physical location of its position."""
    rng = np.random.default_rng(13)
    for bs in (16, 64):
        nb, s, mb = 300, 6, 40
        order = rng.permutation(nb).astype(np.int32)
        a = pa.BlockAllocator(nb, order)
        mgr = ManagerModel(nb, bs, order)
        lens = rng.integers(0, 3 * bs, size=s).astype(np.int32)
        tables = np.full((s, mb), -1, dtype=np.int32)
        for i in range(s):
            n = pa.pa_num_required_blocks(int(lens[i]), bs)
            tables[i, :n] = a.alloc_n(n)
            mgr.allocate_for_request(i, int(lens[i]))
        new = rng.integers(0, 5 * bs, size=s).astype(np.int32)
        before = lens.copy()
        slots = a.prefill_slots(tables, lens, new, bs)
        k = 0
        for i in range(s):
            for pos in range(int(before[i]), int(before[i] + new[i])):
                mgr.append_slot(i, pos)
                phys, off = oracle.physical_location(tables[i], pos, bs)
                assert slots[k] == phys * bs + off
                k += 1
            assert list(tables[i, :len(mgr.tables[i])]) == mgr.tables[i]
        assert np.array_equal(lens, before + new) and a.num_free() == mgr.pool.num_free()


# ------------------------------------------------------------- shared prefixes

def _check_groups(tables, lens, bs, P, g):
    """Invariants of pa_find_shared_prefixes' result."""
    S = len(lens)
    seen = set()
    for k in range(g.num_groups):
        mem = list(g.group_members[g.group_offsets[k]:g.group_offsets[k + 1]])
        assert len(mem) >= 2 and not (set(mem) & seen)
        seen |= set(mem)
        st = {int(g.seq_start[m]) for m in mem}
        assert len(st) == 1
        st = st.pop()
        assert st > 0 and st % P == 0 and all(st < lens[m] for m in mem)
        for m in mem:  # same physical blocks below the start
            assert np.array_equal(tables[m, :st // bs], tables[mem[0], :st // bs])
    for s in range(S):
        if s not in seen:
            assert g.seq_start[s] == 0
    assert g.max_shared_tokens == max([int(x) for x in g.seq_start] + [0])


@pytest.mark.parametrize("seed", range(6))
def test_find_shared_prefixes_on_random_forks(pa, seed):
    rng = np.random.default_rng(seed)
    bs = int(rng.choice([16, 32, 64]))
    P = bs * int(rng.choice([1, 2, 4]))
    S, MB = 40, 40
    tables = np.full((S, MB), -1, np.int32)
    lens = np.zeros(S, np.int32)
    nxt = 0
    for s in range(S):
        L = int(rng.integers(1, MB * bs + 1))
        nb = -(-L // bs)
        if s > 0 and rng.random() < 0.7:  # fork from an earlier sequence: share a random number of its blocks
            src = int(rng.integers(0, s))
            k = int(rng.integers(0, -(-int(lens[src]) // bs) + 1))
            k = min(k, nb)
            tables[s, :k] = tables[src, :k]
        else:
            k = 0
        tables[s, k:nb] = np.arange(nxt, nxt + nb - k)
        nxt += nb - k
        lens[s] = L
    g = pa.pa_find_shared_prefixes(tables, lens, bs, P)
    _check_groups(tables, lens, bs, P, g)


def test_find_shared_prefixes_beam_fork(pa):
    """Every beam holds the prompt's blocks: one group sharing the whole prompt."""
    bs, P = 64, 256
    prompt = np.arange(8, dtype=np.int32)       # 512 tokens
    tables = np.full((12, 16), -1, np.int32)
    lens = np.zeros(12, np.int32)
    for s in range(12):
        tables[s, :8] = prompt
        tables[s, 8:10] = [100 + 2 * s, 101 + 2 * s]
        lens[s] = 512 + 1 + 7 * s
    g = pa.pa_find_shared_prefixes(tables, lens, bs, P)
    assert g.num_groups == 1 and list(g.group_members) == list(range(12))
    assert list(g.seq_start) == [512] * 12 and g.max_group_size == 12 and g.max_shared_tokens == 512
    _check_groups(tables, lens, bs, P, g)
    lens[3] = 512  # its last token sits in the prompt: it can share only 256 tokens, the others keep 512
    g = pa.pa_find_shared_prefixes(tables, lens, bs, P)
    assert g.seq_start[3] == 0 and g.num_groups == 1
    _check_groups(tables, lens, bs, P, g)
    with pytest.raises(pa.PAError):
        pa.pa_find_shared_prefixes(tables, lens, bs, 100)  # not a multiple of the block size
