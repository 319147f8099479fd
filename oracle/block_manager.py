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

Prefix cache ("pagedattention vllm" §vLLM Integration, §Advanced Features:
prefix caching; lastdictionary "PagedAttention": prompt caching lets requests
that begin the same way skip that part):
  - add_seq_prefix(seq, tokens): full block j of the prompt has the key
    (registration id of block j - 1, or 0 for j = 0; its block_size tokens).
    Walking j = 0, 1, ... while a registered block has that key, the sequence
    takes those blocks (one more reference; an evictable one comes back);
    the first miss ends the walk.  The remaining blocks are taken in logical
    order and each full one is registered under its key with the next
    registration id (1, 2, ...); the partial last block is never registered.
    It reports the number of prompt tokens found (hits * block_size); all or
    nothing;
  - a registered block whose count reaches zero is not pushed on the free
    stack but appended to the evictable list; taking a block pops the free
    stack, or, when that is empty, evicts the head of the evictable list
    (least recently released), unregistering it;
  - capacity of an allocation = free stack + evictable list (minus evictable
    blocks the same call takes back as hits).
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
        # prefix cache
        self.key_of: dict[int, tuple] = {}      # registered block -> (parent id, tokens)
        self.reg_of: dict[int, int] = {}        # registered block -> registration id
        self.block_of: dict[tuple, int] = {}    # key -> registered block
        self.next_reg = 1
        self.evictable: list[int] = []          # least recently released first

    # -- block supply -----------------------------------------------------
    def _available(self) -> int:
        return len(self.free) + len(self.evictable)

    def _take(self) -> int:
        if self.free:
            blk = self.free.pop()
        else:
            blk = self.evictable.pop(0)
            del self.block_of[self.key_of.pop(blk)]
            del self.reg_of[blk]
        self.ref[blk] = 1
        return blk

    def _release(self, blk: int) -> None:
        self.ref[blk] -= 1
        if self.ref[blk] == 0:
            if blk in self.reg_of:
                self.evictable.append(blk)
            else:
                self.free.append(blk)

    # -- operations -------------------------------------------------------
    def add_seq(self, seq_id: int, num_tokens: int) -> int:
        if num_tokens < 0:
            return EINVAL
        if seq_id in self.tables:
            return EEXIST
        need = (num_tokens + self.block_size - 1) // self.block_size
        if need > self._available():
            return ENOMEM
        self.tables[seq_id] = [self._take() for _ in range(need)]
        self.lens[seq_id] = num_tokens
        return OK

    def add_seq_prefix(self, seq_id: int, tokens):
        """-> (status, prompt tokens found in the cache)"""
        tokens = [int(t) for t in tokens]
        if seq_id in self.tables:
            return EEXIST, 0
        bs = self.block_size
        nfull = len(tokens) // bs
        need = (len(tokens) + bs - 1) // bs
        hits, parent = [], 0
        for j in range(nfull):
            blk = self.block_of.get((parent, tuple(tokens[j * bs:(j + 1) * bs])))
            if blk is None:
                break
            hits.append(blk)
            parent = self.reg_of[blk]
        back = sum(1 for b in hits if self.ref[b] == 0)
        if need - len(hits) > self._available() - back:
            return ENOMEM, 0
        table = []
        for blk in hits:
            if self.ref[blk] == 0:
                self.evictable.remove(blk)
            self.ref[blk] += 1
            table.append(blk)
        for j in range(len(hits), need):
            blk = self._take()
            table.append(blk)
            if j < nfull:
                key = (parent, tuple(tokens[j * bs:(j + 1) * bs]))
                self.key_of[blk] = key
                self.block_of[key] = blk
                self.reg_of[blk] = self.next_reg
                self.next_reg += 1
                parent = self.reg_of[blk]
        self.tables[seq_id] = table
        self.lens[seq_id] = len(tokens)
        return OK, len(hits) * bs

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
            if not self._available():
                return ENOMEM, -1, -1, -1
            table.append(self._take())
        elif self.ref[table[-1]] > 1:
            if not self._available():
                return ENOMEM, -1, -1, -1
            dst = self._take()
            src = table[-1]
            self._release(src)   # stays > 0: another sequence still holds it
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
                if blk >= 0:
                    self._release(blk)
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
            self._release(blk)
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
        if sum(1 for h in table if h >= 0) > self._available():
            return ENOMEM, []
        pairs = []
        for i, h in enumerate(table):
            if h < 0:
                continue
            d = self._take()
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
            self._release(table[j])
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

    def cache_stats(self) -> tuple[int, int]:
        """(registered blocks, evictable blocks)"""
        return len(self.reg_of), len(self.evictable)

    def evictable_list(self) -> list[int]:
        return list(self.evictable)

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
        if kind == "prefix":
            return self.add_seq_prefix(op[1], op[2])
        raise ValueError(kind)
