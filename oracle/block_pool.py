"""Pure-Python model of the host block allocator -- TEST INFRASTRUCTURE ONLY.

Follows the block pool of P3 ("LLM 推理中的 PageAttention 实现原理：虚拟内存管理在
KV Cache 中的创新应用", §三, BlockPool / BlockTable / PageAttentionManager) step
by step, in Python, as the oracle the C++ allocator is compared with id for id:

  allocate      pop the FRONT of the free queue, set its reference count to 1
  free          decrement the count; at zero push the id to the BACK of the queue
  add_ref       increment the count (prefix sharing)
  usage_ratio   allocated / total
  allocate_n    all-or-nothing: check the free count first, then pop n ids
                (PageAttentionManager::allocate_for_request)
  append_slot   a new block only when current_len % B == 0
                (PageAttentionManager::append_slot)
  fork          copy a table's ids, each add_ref'd (P3 §四, beam search: "fork copies
                the block references, reference count + 1")
  swap_plan     move a preempted request's blocks to another pool (device <-> host):
                allocate there, drop one reference here (P3 §三 "Preemption
                required", P3 §五 swap to CPU memory and back)
  cow_prepare   before appending into a partly filled block that is still shared,
                take a private copy: allocate, drop one reference of the shared
                block, record (shared, fresh) -- the completion of the fork that the
                pages leave implicit

One deliberate difference from the listing: its ``free`` saturates at zero in
silence; here freeing (or add_ref-ing) a block whose count is already zero is an
error, so that a double free shows up.
"""
from __future__ import annotations

from collections import deque


class AllocatorError(Exception):
    pass


class OutOfBlocks(AllocatorError):
    pass


class RefcountError(AllocatorError):
    pass


class BlockPoolModel:
    def __init__(self, num_blocks: int, initial_order=None):
        self.total = num_blocks
        order = list(range(num_blocks)) if initial_order is None else [int(i) for i in initial_order]
        if sorted(order) != list(range(num_blocks)):
            raise ValueError("initial_order must be a permutation of 0..num_blocks-1")
        self.free_queue = deque(order)
        self.ref = [0] * num_blocks
        self.allocated = 0

    def allocate(self) -> int:
        if not self.free_queue:
            raise OutOfBlocks("no free blocks")
        b = self.free_queue.popleft()
        self.ref[b] = 1
        self.allocated += 1
        return b

    def allocate_n(self, n: int) -> list[int]:
        if n < 0:
            raise ValueError("n < 0")
        if len(self.free_queue) < n:
            raise OutOfBlocks(f"need {n}, available {len(self.free_queue)}")
        return [self.allocate() for _ in range(n)]

    def free(self, b: int) -> None:
        self._check(b)
        if self.ref[b] == 0:
            raise RefcountError(f"block {b} is already free")
        self.ref[b] -= 1
        if self.ref[b] == 0:
            self.free_queue.append(b)
            self.allocated -= 1

    def add_ref(self, b: int) -> None:
        self._check(b)
        if self.ref[b] == 0:
            raise RefcountError(f"block {b} is free")
        self.ref[b] += 1

    def fork(self, table: list[int]) -> list[int]:
        for b in table:
            self._check(b)
            if self.ref[b] == 0:
                raise RefcountError(f"block {b} is free")
        for b in table:
            self.ref[b] += 1
        return list(table)

    def usage_ratio(self) -> float:
        return self.allocated / self.total if self.total else 0.0

    def num_free(self) -> int:
        return len(self.free_queue)

    def _check(self, b: int) -> None:
        if not 0 <= b < self.total:
            raise ValueError(f"block id {b} out of range")


def swap_plan(src: BlockPoolModel, dst: BlockPoolModel, table: list[int]) -> list[tuple[int, int]]:
    """Move the blocks of ``table`` (in place) from pool ``src`` to pool ``dst``:
    all or nothing; returns the (old, new) pairs in table order."""
    held = {}
    for b in table:
        src._check(b)
        held[b] = held.get(b, 0) + 1
        if src.ref[b] < held[b]:
            raise RefcountError(f"block {b} is not held often enough")
    if dst.num_free() < len(table):
        raise OutOfBlocks(f"need {len(table)}, available {dst.num_free()}")
    pairs = []
    for i, b in enumerate(table):
        fresh = dst.allocate()
        src.free(b)
        pairs.append((b, fresh))
        table[i] = fresh
    return pairs


def num_required_blocks(num_tokens: int, block_size: int) -> int:
    """P3 §三, BlockTable::num_required_blocks."""
    return -(-num_tokens // block_size)


class ManagerModel:
    """Per-request tables over one pool (P3 §三, PageAttentionManager)."""

    def __init__(self, num_blocks: int, block_size: int, initial_order=None):
        self.pool = BlockPoolModel(num_blocks, initial_order)
        self.block_size = block_size
        self.tables: dict[int, list[int]] = {}

    def allocate_for_request(self, rid: int, prompt_len: int) -> int:
        n = num_required_blocks(prompt_len, self.block_size)
        self.tables[rid] = self.pool.allocate_n(n)
        return n

    def append_slot(self, rid: int, current_len: int):
        """Allocate a block when ``current_len`` sits on a block boundary; else None."""
        if current_len % self.block_size != 0:
            return None
        b = self.pool.allocate()
        self.tables[rid].append(b)
        return b

    def free_request(self, rid: int) -> None:
        for b in self.tables.pop(rid, []):
            self.pool.free(b)

    def cow_prepare(self, stored_lens: dict[int, int]) -> list[tuple[int, int]]:
        """Copy-on-write for the requests about to append (request id -> stored tokens),
        handled in ascending request order; returns the (src, dst) copies."""
        pairs = []
        pending = []
        for rid in sorted(stored_lens):
            n = stored_lens[rid]
            if n % self.block_size == 0:
                continue  # the next token opens a fresh block
            pending.append((rid, n // self.block_size))
        # all or nothing: simulate the counts first
        need, ref = 0, list(self.pool.ref)
        for rid, j in pending:
            b = self.tables[rid][j]
            if ref[b] > 1:
                ref[b] -= 1
                need += 1
        if need > self.pool.num_free():
            raise OutOfBlocks(f"copy-on-write needs {need}, available {self.pool.num_free()}")
        for rid, j in pending:
            b = self.tables[rid][j]
            if self.pool.ref[b] > 1:
                fresh = self.pool.allocate()
                self.pool.ref[b] -= 1
                self.tables[rid][j] = fresh
                pairs.append((b, fresh))
        return pairs

    def share_prefix_blocks(self, src: int, dst: int, shared_len: int) -> None:
        n = num_required_blocks(shared_len, self.block_size)
        table = self.tables[src]
        if len(table) < n:
            raise AllocatorError("source has fewer blocks than the shared length needs")
        self.tables[dst] = self.pool.fork(table[:n])
