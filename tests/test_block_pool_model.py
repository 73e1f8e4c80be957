"""The allocator model against the demo program of P3 ("LLM 推理中的 PageAttention 实现原理：虚拟内存管理在
KV Cache 中的创新应用") §三 (main) and its own rules."""
import json
import os

import pytest

from oracle.block_pool import BlockPoolModel, ManagerModel, OutOfBlocks, RefcountError, swap_plan
from pins import GOLDEN


def test_demo_program():
    with open(os.path.join(GOLDEN, "allocator_demo.json")) as f:
        demo = json.load(f)
    m = ManagerModel(demo["num_blocks"], demo["block_size"])
    for st in demo["steps"]:
        if st["op"] == "allocate_for_request":
            assert m.allocate_for_request(st["rid"], st["prompt_len"]) == st["returns"]
            assert m.tables[st["rid"]] == st["table"]
        elif st["op"] == "append_slot":
            assert m.append_slot(st["rid"], st["current_len"]) == st["returns"]
            assert m.tables[st["rid"]] == st["table"]
        elif st["op"] == "share_prefix_blocks":
            m.share_prefix_blocks(st["src"], st["dst"], st["shared_len"])
            assert m.tables[st["dst"]] == st["table"]
        elif st["op"] == "free_request":
            m.free_request(st["rid"])
        for b, r in st.get("refcounts", {}).items():
            assert m.pool.ref[int(b)] == r, (st, b)
        if "free_tail" in st:
            tail = st["free_tail"]
            assert list(m.pool.free_queue)[-len(tail):] == tail
    assert m.pool.num_free() == demo["final_num_free"]
    assert m.pool.usage_ratio() == demo["final_usage"]


def test_all_or_nothing_and_errors():
    p = BlockPoolModel(4, initial_order=[2, 0, 3, 1])
    assert p.allocate_n(3) == [2, 0, 3]
    with pytest.raises(OutOfBlocks):
        p.allocate_n(2)
    assert p.num_free() == 1 and p.usage_ratio() == 0.75
    p.free(0)
    with pytest.raises(RefcountError):
        p.free(0)                      # double free is an error here, not a silent no-op
    with pytest.raises(RefcountError):
        p.add_ref(0)
    t = p.fork([2, 3])
    assert t == [2, 3] and p.ref[2] == 2 and p.ref[3] == 2
    p.free(2)
    assert p.ref[2] == 1 and 2 not in p.free_queue   # back to the queue only at zero
    p.free(2)
    assert list(p.free_queue) == [1, 0, 2]


def test_copy_on_write_after_a_beam_fork():
    """Four beams share a 40-token prompt (block size 16: two full blocks and one
    holding 8 tokens).  Before appending, each beam still sharing the partly filled
    block takes a private copy, in request order; the last holder keeps the original.
    The full blocks stay shared."""
    m = ManagerModel(20, 16)
    m.allocate_for_request(0, 40)
    a, b, c = m.tables[0]
    for rid in (1, 2, 3):
        m.share_prefix_blocks(0, rid, 40)
    assert [m.pool.ref[x] for x in (a, b, c)] == [4, 4, 4]
    pairs = m.cow_prepare({0: 40, 1: 40, 2: 40, 3: 40})
    fresh = [3, 4, 5]                      # FIFO: the next free ids
    assert pairs == [(c, f) for f in fresh]
    assert [m.tables[r][2] for r in range(4)] == fresh + [c]
    assert m.pool.ref[c] == 1 and all(m.pool.ref[f] == 1 for f in fresh)
    assert m.pool.ref[a] == m.pool.ref[b] == 4
    # nothing left to copy; a request on a block boundary never copies
    assert m.cow_prepare({0: 40, 3: 40}) == []
    assert m.cow_prepare({1: 48}) == []


def test_copy_on_write_is_all_or_nothing():
    m = ManagerModel(4, 16)
    m.allocate_for_request(0, 20)          # 2 blocks, 2 free
    for rid in (1, 2, 3):
        m.share_prefix_blocks(0, rid, 20)  # refs 4
    with pytest.raises(OutOfBlocks):
        m.cow_prepare({0: 20, 1: 20, 2: 20, 3: 20})   # needs 3 copies, 2 free
    assert m.pool.num_free() == 2 and m.pool.ref[m.tables[0][1]] == 4


# ---------------------------------------------------------------- swap plan
#
# Preemption (P3 §三, append_slot's "Preemption required") sends a sequence's KV
# blocks to host memory and P3 §五 brings them back.  The trace below was worked
# out by hand from the pool rules (FIFO front allocation, back-of-queue return at
# count zero, all-or-nothing):
#
#   device pool, 6 blocks, free queue 4 1 5 0 3 2; host pool, 4 blocks, queue 2 0 3 1
#   request A allocates 3 blocks -> row [4, 1, 5], device queue 0 3 2
#   request B holds A's first block by reference (a shared prefix) -> ref[4] = 2
#   swap A out: host allocates 2, 0, 3 in row order; device drops one reference
#     of 4 (2 -> 1, still held by B, stays out of the queue), 1 and 5 (-> 0, to the
#     back of the queue in row order): pairs (4,2) (1,0) (5,3), row [2, 0, 3],
#     device queue 0 3 2 1 5, host queue 1
#   swap A back in: device allocates from the front 0, 3, 2 (never 4, which B still
#     holds); host frees 2, 0, 3 to its back: pairs (2,0) (0,3) (3,2), row [0, 3, 2],
#     device queue 1 5, host queue 1 2 0 3

def _swap_trace(plan):
    """Run the hand-traced swap-out / swap-in through ``plan`` (a swap_plan with the
    model's signature) and assert every value of the trace; then the two refusals:
    a row holding a block more often than its count allows, and a target pool
    too small -- each must leave both pools and the row exactly as they were."""
    dev = BlockPoolModel(6, initial_order=[4, 1, 5, 0, 3, 2])
    host = BlockPoolModel(4, initial_order=[2, 0, 3, 1])
    row = dev.allocate_n(3)
    assert row == [4, 1, 5]
    dev.add_ref(4)                                   # request B shares the first block
    pairs = plan(dev, host, row)
    assert [tuple(p) for p in pairs] == [(4, 2), (1, 0), (5, 3)]
    assert row == [2, 0, 3]
    assert [dev.ref[b] for b in range(6)] == [0, 0, 0, 0, 1, 0]
    assert list(dev.free_queue) == [0, 3, 2, 1, 5]
    assert [host.ref[b] for b in range(4)] == [1, 0, 1, 1]
    assert list(host.free_queue) == [1]
    assert dev.usage_ratio() == 1 / 6 and host.usage_ratio() == 3 / 4
    pairs = plan(host, dev, row)
    assert [tuple(p) for p in pairs] == [(2, 0), (0, 3), (3, 2)]
    assert row == [0, 3, 2]
    assert [dev.ref[b] for b in range(6)] == [1, 0, 1, 1, 1, 0]
    assert list(dev.free_queue) == [1, 5]
    assert [host.ref[b] for b in range(4)] == [0, 0, 0, 0]
    assert list(host.free_queue) == [1, 2, 0, 3]

    # refusals change nothing
    def snapshot():
        return (list(dev.ref), list(dev.free_queue), dev.allocated, list(host.ref), list(host.free_queue),
                host.allocated)
    before, twice = snapshot(), [0, 0, 3]            # block 0 listed twice, held once
    with pytest.raises(RefcountError):
        plan(dev, host, twice)
    assert snapshot() == before and twice == [0, 0, 3]
    big = BlockPoolModel(6, initial_order=[0, 1, 2, 3, 4, 5])
    grown = big.allocate_n(5)                        # host pool has 4 free: too few
    host_before, big_before = snapshot(), (list(big.ref), list(big.free_queue))
    with pytest.raises(OutOfBlocks):
        plan(big, host, grown)
    assert snapshot() == host_before and (list(big.ref), list(big.free_queue)) == big_before
    assert grown == [0, 1, 2, 3, 4]


def test_swap_plan_hand_traced():
    _swap_trace(swap_plan)


# Planted mistakes in the model's swap_plan (its own source with one line changed,
# compiled on the CPU): each must fail the hand-traced pin above.
SWAP_MUTANTS = {
    "row not rewritten": ("table[i] = fresh", "pass"),
    "source reference not dropped": ("src.free(b)", "pass"),
    "pair reversed": ("pairs.append((b, fresh))", "pairs.append((fresh, b))"),
    "held-count check dropped": ("if src.ref[b] < held[b]:", "if False:"),
    "not all or nothing": ("if dst.num_free() < len(table):", "if False:"),
    "target taken from the back": ("fresh = dst.allocate()", "fresh = dst.free_queue.pop(); dst.ref[fresh] = 1; "
                                                              "dst.allocated += 1"),
}


@pytest.mark.parametrize("name", sorted(SWAP_MUTANTS))
def test_swap_plan_pin_catches_planted_mistake(name):
    import inspect
    import textwrap

    import oracle.block_pool as bp
    old, new = SWAP_MUTANTS[name]
    src = textwrap.dedent(inspect.getsource(bp.swap_plan))
    assert src.count(old) == 1, f"mutation site for {name!r} not found"
    scope = dict(vars(bp))
    exec(compile(src.replace(old, new), "<swap_plan mutant>", "exec"), scope)
    with pytest.raises((AssertionError, OutOfBlocks, RefcountError, IndexError)):
        _swap_trace(scope["swap_plan"])
