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
