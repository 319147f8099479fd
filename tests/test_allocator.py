"""The native block allocator against the Python model, operation by
operation: statuses, slots, copy-on-write pairs, tables, reference counts,
free lists and stats must all be identical."""
import numpy as np
import pytest

from oracle import block_manager as bm
from paged_kv_cache_346_b200 import BlockAllocator
from workloads import draw_cow_recipe, random_alloc_ops


def same_state(native: BlockAllocator, model: bm.BlockManagerModel):
    assert native.free_list() == model.free_list()
    for blk in range(model.num_blocks):
        assert native.refcount(blk) == model.refcount(blk)
    for sid in model.tables:
        assert native.block_table(sid) == model.block_table(sid)
        assert native.seq_len(sid) == model.seq_len(sid)
    assert native.stats() == model.stats()


@pytest.mark.parametrize("seed", range(10))
@pytest.mark.parametrize("bs", [1, 4, 16])
def test_random_scripts_bit_exact(seed, bs):
    N = 40
    nat, mod = BlockAllocator(N, bs), bm.BlockManagerModel(N, bs)
    for i, op in enumerate(random_alloc_ops(seed, 300, max_len=50)):
        r_nat, r_mod = nat.apply(op), mod.apply(op)
        assert r_nat == r_mod, (i, op)
        if i % 25 == 0:
            same_state(nat, mod)
    same_state(nat, mod)


def test_batch_append_matches_single_appends():
    nat, mod = BlockAllocator(64, 4), bm.BlockManagerModel(64, 4)
    for x in (nat, mod):
        x.add_seq(0, 6)
        x.fork(0, 1)
        x.fork(0, 2)
        x.add_seq(3, 8)
    st, slots, pairs, done = nat.append_slots([1, 2, 0, 3, 1])
    assert st == 0 and done == 5
    want_slots, want_pairs = [], []
    for sid in [1, 2, 0, 3, 1]:
        s, slot, src, dst = mod.append_slot(sid)
        want_slots.append(slot)
        if src >= 0:
            want_pairs.append((src, dst))
    assert slots.tolist() == want_slots
    assert [tuple(p) for p in pairs.tolist()] == want_pairs
    same_state(nat, mod)


def test_batch_append_stops_at_first_failure():
    nat = BlockAllocator(2, 4)
    nat.add_seq(0, 4)
    nat.add_seq(1, 4)
    st, slots, pairs, done = nat.append_slots([0, 1])
    assert st == -2 and done == 0        # no free block for seq 0's next token
    assert nat.seq_len(0) == 4


def test_build_block_tables():
    nat = BlockAllocator(32, 4)
    nat.add_seq(10, 9)
    nat.add_seq(11, 0)
    nat.add_seq(12, 4)
    tables, lens = nat.build_block_tables([12, 10, 11], max_blocks=4, fill=-1)
    assert lens.tolist() == [4, 9, 0]
    assert tables.tolist() == [[3, -1, -1, -1], [0, 1, 2, -1], [-1, -1, -1, -1]]
    with pytest.raises(Exception):
        nat.build_block_tables([10], max_blocks=2)


def test_cow_sampling_setup_matches_model():
    # the copy-on-write sampling workload's allocator history, on both sides
    rec = draw_cow_recipe(seed=5, num_prompts=4, samples=8, prefix=64, tail_hi=40)
    bs = 16
    N = 4 * 8 * 8 + 64
    nat, mod = BlockAllocator(N, bs), bm.BlockManagerModel(N, bs)
    for x in (nat, mod):
        sid = 0
        for p in range(rec.num_prompts):
            assert x.add_seq(1000 + p, int(rec.shared_lens[p])) == 0
            for s in range(rec.samples):
                assert x.fork(1000 + p, sid) == 0
                sid += 1
            assert x.free_seq(1000 + p) == 0
    same_state(nat, mod)
    for sid in range(rec.num_prompts * rec.samples):
        assert nat.append_slot(sid) == mod.append_slot(sid)
    same_state(nat, mod)
    st = nat.stats()
    # per prompt: samples - 1 copies of the shared partial block
    assert st["used_blocks"] == sum(int(np.ceil(L / bs)) for L in rec.shared_lens) + \
        rec.num_prompts * (rec.samples - 1)


@pytest.mark.parametrize("seed", range(6))
def test_random_scripts_with_swapping_bit_exact(seed):
    nat = BlockAllocator(40, 4, num_host_blocks=30)
    mod = bm.BlockManagerModel(40, 4, num_host_blocks=30)
    for i, op in enumerate(random_alloc_ops(seed, 400, max_len=50, swap=True)):
        r_nat, r_mod = nat.apply(op), mod.apply(op)
        assert r_nat == r_mod, (i, op, r_nat, r_mod)
        if i % 20 == 0:
            same_state(nat, mod)
            for sid in mod.tables:
                assert nat.is_swapped(sid) == (sid in mod.swapped)
    same_state(nat, mod)


def test_swapped_sequence_cannot_join_a_decode_batch():
    nat = BlockAllocator(8, 4, num_host_blocks=8)
    nat.add_seq(0, 5)
    assert nat.swap_out(0)[0] == 0
    with pytest.raises(Exception):
        nat.build_block_tables([0], max_blocks=4)


@pytest.mark.parametrize("seed", range(6))
def test_random_scripts_with_windows_bit_exact(seed):
    nat = BlockAllocator(40, 4, num_host_blocks=30)
    mod = bm.BlockManagerModel(40, 4, num_host_blocks=30)
    for i, op in enumerate(random_alloc_ops(seed, 400, max_len=50, swap=True, slide=True)):
        r_nat, r_mod = nat.apply(op), mod.apply(op)
        assert r_nat == r_mod, (i, op, r_nat, r_mod)
        if i % 20 == 0:
            same_state(nat, mod)
    same_state(nat, mod)


# ---------------------------------------------------------------------------
# prefix cache

def same_cache_state(native: BlockAllocator, model: bm.BlockManagerModel):
    same_state(native, model)
    assert native.cache_stats() == model.cache_stats()
    assert native.evictable_list() == model.evictable_list()


@pytest.mark.parametrize("seed", range(12))
@pytest.mark.parametrize("bs", [1, 4, 16])
def test_random_scripts_with_prefix_cache_bit_exact(seed, bs):
    N = {1: 240, 4: 64, 16: 24}[bs]   # tight enough that evictions happen
    nat, mod = BlockAllocator(N, bs, num_host_blocks=24), bm.BlockManagerModel(N, bs, 24)
    ops = random_alloc_ops(seed, 400, max_len=60, prefix=True, swap=seed % 3 == 0,
                           slide=seed % 3 == 1)
    assert any(op[0] == "prefix" for op in ops)
    hits = 0
    for i, op in enumerate(ops):
        r_nat, r_mod = nat.apply(op), mod.apply(op)
        assert r_nat == r_mod, (i, op)
        if op[0] == "prefix" and r_mod[0] == 0:
            hits += r_mod[1]
        if i % 20 == 0:
            same_cache_state(nat, mod)
    same_cache_state(nat, mod)
    assert hits > 0          # the scripts do reuse cached prefixes


def _invariants(model: bm.BlockManagerModel):
    st = model.stats()
    cached, evictable = model.cache_stats()
    assert st["free_blocks"] + evictable + st["used_blocks"] == model.num_blocks
    assert set(model.free) .isdisjoint(model.evictable)
    assert all(model.ref[b] == 0 for b in model.evictable)
    assert all(b in model.reg_of for b in model.evictable)
    assert cached == len(model.block_of)
    # a registered block is full and holds exactly the tokens of its key
    for blk, (parent, toks) in model.key_of.items():
        assert len(toks) == model.block_size


@pytest.mark.parametrize("seed", range(6))
def test_prefix_model_invariants(seed):
    mod = bm.BlockManagerModel(40, 4, 16)
    for op in random_alloc_ops(seed, 400, max_len=60, prefix=True, swap=True, slide=True):
        mod.apply(op)
        _invariants(mod)


def test_prefix_sharing_by_hand():
    """Worked example: block size 4, prompts A = 0..9, B = A[:8] + others."""
    for x in (BlockAllocator(8, 4), bm.BlockManagerModel(8, 4)):
        A = list(range(10))
        B = list(range(8)) + [70, 71, 72]
        C = [0, 1, 2, 3, 99, 5, 6, 7]      # differs inside block 1
        assert x.add_seq_prefix(0, A) == (0, 0)        # nothing cached yet
        tA = x.block_table(0)
        assert tA == [0, 1, 2]
        assert x.add_seq_prefix(1, B) == (0, 8)        # blocks 0, 1 reused
        tB = x.block_table(1)
        assert tB[:2] == tA[:2] and tB[2] not in tA
        assert x.refcount(tA[0]) == 2 and x.refcount(tA[2]) == 1
        assert x.add_seq_prefix(2, C) == (0, 4)        # only block 0 matches
        assert x.block_table(2)[0] == tA[0] and x.block_table(2)[1] not in tA + tB
        # the partial last blocks were never registered: A's third block has 2
        # tokens, B's 3; registered = A's 2 full blocks + C's second block
        assert x.cache_stats() == (3, 0)
        # free everything: registered blocks become evictable in the order
        # their counts reach zero (B frees A's block 1, C frees block 0, then
        # its own registered block 1)
        c1 = x.block_table(2)[1]
        for sid in (0, 1, 2):
            assert x.free_seq(sid) == 0
        assert x.cache_stats() == (3, 3)
        assert x.evictable_list() == [tA[1], tA[0], c1]
        # a new prompt with A's start takes the evictable blocks back
        assert x.add_seq_prefix(3, A[:8]) == (0, 8)
        assert x.block_table(3) == tA[:2]
        assert x.cache_stats() == (3, 1)


def test_prefix_eviction_order_and_capacity():
    for x in (BlockAllocator(4, 2), bm.BlockManagerModel(4, 2)):
        assert x.add_seq_prefix(0, [1, 2, 3, 4]) == (0, 0)   # blocks 0, 1 registered
        assert x.free_seq(0) == 0                              # both evictable: 0 then 1
        assert x.evictable_list() == [0, 1]
        assert x.stats()["free_blocks"] == 2
        # 4 blocks needed: 2 from the free stack, then evict 0, then 1
        assert x.add_seq(1, 8) == 0
        assert x.block_table(1) == [2, 3, 0, 1]
        assert x.cache_stats() == (0, 0)
        assert x.add_seq_prefix(2, [1, 2]) == (-2, 0)        # ENOMEM, nothing changed
        assert x.free_seq(1) == 0
        assert x.add_seq_prefix(2, [1, 2, 3, 4]) == (0, 0)   # nothing cached any more


def test_prefix_hit_needs_whole_prefix():
    """Equal tokens at an equal position but a different earlier block do not
    match: a hit means the entire prefix is identical."""
    for x in (BlockAllocator(16, 2), bm.BlockManagerModel(16, 2)):
        assert x.add_seq_prefix(0, [5, 5, 7, 7]) == (0, 0)
        assert x.add_seq_prefix(1, [6, 6, 7, 7]) == (0, 0)
        assert x.block_table(1)[1] != x.block_table(0)[1]
        assert x.add_seq_prefix(2, [6, 6, 7, 7, 8]) == (0, 4)
        assert x.block_table(2)[:2] == x.block_table(1)


def test_prefix_capacity_counts_evictable_hits():
    """An evictable block that the same call takes back as a hit cannot also
    be evicted to satisfy the call's fresh blocks."""
    for x in (BlockAllocator(3, 2), bm.BlockManagerModel(3, 2)):
        assert x.add_seq_prefix(0, [1, 1, 2, 2]) == (0, 0)
        assert x.free_seq(0) == 0                 # 2 evictable + 1 free
        # hits 2 blocks (both evictable) + needs 2 fresh: only 1 free -> ENOMEM
        assert x.add_seq_prefix(1, [1, 1, 2, 2, 3, 3, 4]) == (-2, 0)
        assert x.cache_stats() == (2, 2)
        assert x.add_seq_prefix(1, [1, 1, 2, 2, 3]) == (0, 4)
