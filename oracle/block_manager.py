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

Swapping ("pagedattention vllm" §Memory Management: blocks can be swapped to
CPU memory to serve more sequences than the GPU holds), with a host pool of
its own (LIFO free stack popping 0, 1, 2, ... first):
  - swap_out(seq): for each table entry in logical order take a host block,
    report (device block, host block) and drop one reference to the device
    block (a block still shared stays on the device); the table holds host
    ids and the sequence is swapped;
  - swap_in(seq): for each entry take a device block, report (host block,
    device block) and push the host block back, in logical order;
  - a swapped sequence cannot be appended to, forked or decoded until it is
    swapped in; freeing it returns its host blocks.

Sliding window ("pagedattention vllm" §Advanced Features: sliding-window models
keep only recent blocks): slide_window(seq, W) releases, in logical order,
every block j with (j + 1) * block_size <= len - W (one reference dropped, the
entry becomes -1); fork, free and swap skip -1 entries.
"""
from __future__ import annotations

OK, EINVAL, ENOMEM, ENOSEQ, EEXIST = 0, -1, -2, -3, -4


class BlockManagerModel:
    def __init__(self, num_blocks: int, block_size: int, num_host_blocks: int = 0):
        if num_blocks <= 0 or block_size <= 0 or num_host_blocks < 0:
            raise ValueError("bad sizes")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.num_host_blocks = num_host_blocks
        self.free = list(range(num_blocks - 1, -1, -1))   # top of stack = end
        self.host_free = list(range(num_host_blocks - 1, -1, -1))
        self.ref = [0] * num_blocks
        self.tables: dict[int, list[int]] = {}
        self.lens: dict[int, int] = {}
        self.swapped: set[int] = set()

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
        if parent in self.swapped:
            return EINVAL
        table = list(self.tables[parent])
        for blk in table:
            if blk >= 0:
                self.ref[blk] += 1
        self.tables[child] = table
        self.lens[child] = self.lens[parent]
        return OK

    def append_slot(self, seq_id: int):
        """-> (status, slot, cow_src, cow_dst); cow_* = -1 when no copy."""
        if seq_id not in self.tables:
            return ENOSEQ, -1, -1, -1
        if seq_id in self.swapped:
            return EINVAL, -1, -1, -1
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
        if seq_id in self.swapped:
            self.host_free.extend(h for h in self.tables.pop(seq_id) if h >= 0)
            self.swapped.discard(seq_id)
        else:
            for blk in self.tables.pop(seq_id):
                if blk < 0:
                    continue
                self.ref[blk] -= 1
                if self.ref[blk] == 0:
                    self.free.append(blk)
        del self.lens[seq_id]
        return OK

    def swap_out(self, seq_id: int):
        """-> (status, [(device block, host block), ...])"""
        if seq_id not in self.tables:
            return ENOSEQ, []
        if seq_id in self.swapped:
            return EINVAL, []
        table = self.tables[seq_id]
        if sum(1 for b in table if b >= 0) > len(self.host_free):
            return ENOMEM, []
        pairs = []
        for i, blk in enumerate(table):
            if blk < 0:
                continue
            h = self.host_free.pop()
            pairs.append((blk, h))
            self.ref[blk] -= 1
            if self.ref[blk] == 0:
                self.free.append(blk)
            table[i] = h
        self.swapped.add(seq_id)
        return OK, pairs

    def swap_in(self, seq_id: int):
        """-> (status, [(host block, device block), ...])"""
        if seq_id not in self.tables:
            return ENOSEQ, []
        if seq_id not in self.swapped:
            return EINVAL, []
        table = self.tables[seq_id]
        if sum(1 for h in table if h >= 0) > len(self.free):
            return ENOMEM, []
        pairs = []
        for i, h in enumerate(table):
            if h < 0:
                continue
            d = self.free.pop()
            self.ref[d] = 1
            pairs.append((h, d))
            self.host_free.append(h)
            table[i] = d
        self.swapped.discard(seq_id)
        return OK, pairs

    def slide_window(self, seq_id: int, window: int):
        """-> (status, number of entries released)"""
        if window <= 0:
            return EINVAL, 0
        if seq_id not in self.tables:
            return ENOSEQ, 0
        if seq_id in self.swapped:
            return EINVAL, 0
        table = self.tables[seq_id]
        keep_from = self.lens[seq_id] - window
        released = 0
        for j in range(len(table)):
            if (j + 1) * self.block_size > keep_from:
                break
            if table[j] < 0:
                continue
            self.ref[table[j]] -= 1
            if self.ref[table[j]] == 0:
                self.free.append(table[j])
            table[j] = -1
            released += 1
        return OK, released

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
            num_host_blocks=self.num_host_blocks,
            free_host_blocks=len(self.host_free),
            swapped_seqs=len(self.swapped),
            reserved=0,
        )

    def host_free_list(self) -> list[int]:
        return list(reversed(self.host_free))

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
        if kind == "swap_out":
            return self.swap_out(op[1])
        if kind == "swap_in":
            return self.swap_in(op[1])
        if kind == "slide":
            return self.slide_window(op[1], op[2])
        raise ValueError(kind)
