"""Block manager model: free list, reference counts, fork and copy-on-write.

TEST INFRASTRUCTURE ONLY (tests and the smoke check).  A plain Python model of
what the pages ask of the KV block manager, used to check the library's native
allocator operation by operation, bit for bit.

What the pages fix:
  - blocks are handed out on demand as a sequence grows and a sequence holds
    only the blocks it has filled plus part of the last one ("What is
    PagedAttention ..." §How it works; "pagedattention vllm" §Memory
    Management: a free list, allocate on demand, return blocks on completion);
  - sequences with a common start share physical blocks; each block carries a
    reference count and is freed when the count reaches zero; a sequence about
    to write into a shared block first copies it and points its table at the
    copy, and the other holders are unaffected ("pagedattention vllm"
    §Copy-on-Write Sharing; lastdictionary "PagedAttention").

What the pages leave open, and the reading taken here (one rule each, so the
native allocator's tables can be compared exactly):
  - the free list is a LIFO stack that first pops 0, 1, 2, ...;
  - add_seq(n) pops ceil(n / block_size) blocks in logical order, all or none;
  - append_slot: if the last block is full (or there is none) pop a new block;
    else if the last block is shared (count > 1) pop a block dst, report the
    copy (last, dst), drop one reference to last and put dst in its place;
    the sole holder of a block writes in place.  Then the slot is
    table[-1] * block_size + len % block_size and len grows by one;
  - fork(parent, child): the child gets a copy of the parent's table and length
    and every block in it gains a reference;
  - free_seq walks the table in logical order, drops one reference per entry
    and pushes each block whose count reaches zero;
  - a failed call (no free block, unknown or existing sequence) changes nothing.
"""
from __future__ import annotations

OK, EINVAL, ENOMEM, ENOSEQ, EEXIST = 0, -1, -2, -3, -4


class BlockManagerModel:
    def __init__(self, num_blocks: int, block_size: int):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("bad sizes")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free = list(range(num_blocks - 1, -1, -1))   # top of stack = end
        self.ref = [0] * num_blocks
        self.tables: dict[int, list[int]] = {}
        self.lens: dict[int, int] = {}

    # -- operations -------------------------------------------------------
    def add_seq(self, seq_id: int, num_tokens: int) -> int:
        if num_tokens < 0:
            return EINVAL
        if seq_id in self.tables:
            return EEXIST
        need = (num_tokens + self.block_size - 1) // self.block_size
        if need > len(self.free):
            return ENOMEM
        table = []
        for _ in range(need):
            blk = self.free.pop()
            self.ref[blk] = 1
            table.append(blk)
        self.tables[seq_id] = table
        self.lens[seq_id] = num_tokens
        return OK

    def fork(self, parent: int, child: int) -> int:
        if parent not in self.tables:
            return ENOSEQ
        if child in self.tables:
            return EEXIST
        table = list(self.tables[parent])
        for blk in table:
            self.ref[blk] += 1
        self.tables[child] = table
        self.lens[child] = self.lens[parent]
        return OK

    def append_slot(self, seq_id: int):
        """-> (status, slot, cow_src, cow_dst); cow_* = -1 when no copy."""
        if seq_id not in self.tables:
            return ENOSEQ, -1, -1, -1
        table = self.tables[seq_id]
        n = self.lens[seq_id]
        src = dst = -1
        if n % self.block_size == 0:
            if not self.free:
                return ENOMEM, -1, -1, -1
            blk = self.free.pop()
            self.ref[blk] = 1
            table.append(blk)
        elif self.ref[table[-1]] > 1:
            if not self.free:
                return ENOMEM, -1, -1, -1
            dst = self.free.pop()
            self.ref[dst] = 1
            src = table[-1]
            self.ref[src] -= 1
            table[-1] = dst
        slot = table[-1] * self.block_size + n % self.block_size
        self.lens[seq_id] = n + 1
        return OK, slot, src, dst

    def free_seq(self, seq_id: int) -> int:
        if seq_id not in self.tables:
            return ENOSEQ
        for blk in self.tables.pop(seq_id):
            self.ref[blk] -= 1
            if self.ref[blk] == 0:
                self.free.append(blk)
        del self.lens[seq_id]
        return OK

    # -- queries ----------------------------------------------------------
    def block_table(self, seq_id: int) -> list[int]:
        return list(self.tables[seq_id])

    def seq_len(self, seq_id: int) -> int:
        return self.lens[seq_id]

    def refcount(self, blk: int) -> int:
        return self.ref[blk]

    def stats(self) -> dict:
        used = sum(1 for r in self.ref if r > 0)
        return dict(
            num_blocks=self.num_blocks,
            block_size=self.block_size,
            free_blocks=len(self.free),
            used_blocks=used,
            shared_blocks=sum(1 for r in self.ref if r > 1),
            num_seqs=len(self.tables),
            refcount_sum=sum(self.ref),
            logical_tokens=sum(self.lens.values()),
        )

    def free_list(self) -> list[int]:
        """Free blocks, next to be handed out first."""
        return list(reversed(self.free))

    def apply(self, op):
        """Run one scripted op (see workloads.random_alloc_ops)."""
        kind = op[0]
        if kind == "add":
            return self.add_seq(op[1], op[2])
        if kind == "fork":
            return self.fork(op[1], op[2])
        if kind == "append":
            return self.append_slot(op[1])
        if kind == "free":
            return self.free_seq(op[1])
        raise ValueError(kind)
