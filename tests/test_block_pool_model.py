"""The allocator model against the demo program of P3 ("LLM 推理中的 PageAttention 实现原理：虚拟内存管理在
KV Cache 中的创新应用") §三 (main) and its own rules."""
import json
import os

import pytest

from oracle.block_pool import BlockPoolModel, ManagerModel, OutOfBlocks, RefcountError
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
