"""Pins for the block manager model: invariants the pages state, the worked
fragmentation example, and copy-on-write behaviour checked on the data."""
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import block_manager as bm
from oracle.cache_ops import copy_blocks, kv_cache_append
from workloads import random_alloc_ops

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                     "page_figures.json")))


def check_invariants(m: bm.BlockManagerModel):
    bs = m.block_size
    held = []
    for sid, table in m.tables.items():
        # a sequence holds the blocks it filled plus part of the last one
        # (entries released by a sliding window are -1)
        assert len(table) == (m.lens[sid] + bs - 1) // bs
        held.extend(b for b in table if b >= 0)
    assert sum(m.ref) == len(held)                        # one reference per table entry
    for blk in range(m.num_blocks):
        assert m.ref[blk] == held.count(blk)
    free = set(m.free)
    assert len(free) == len(m.free)                       # no duplicates on the free list
    assert free.isdisjoint(held)                          # never free and in use
    assert len(free) + len(set(held)) == m.num_blocks     # nothing leaks


@pytest.mark.parametrize("seed", range(8))
def test_random_scripts_keep_invariants(seed):
    m = bm.BlockManagerModel(num_blocks=48, block_size=int([1, 4, 16][seed % 3]))
    for op in random_alloc_ops(seed, 400, max_len=60):
        m.apply(op)
        check_invariants(m)


def test_fragmentation_worked_example():
    ex = GOLDEN["fragmentation_example"]
    bs = GOLDEN["default_block_size"]["tokens"]
    n, L, maxlen = ex["num_sequences"], ex["average_length"], ex["max_length"]
    m = bm.BlockManagerModel(num_blocks=n * maxlen // bs, block_size=bs)
    for s in range(n):
        assert m.add_seq(s, L) == bm.OK
    st = m.stats()
    assert st["used_blocks"] == n * math.ceil(L / bs) == 416
    assert st["logical_tokens"] == n * L
    naive_reserved = n * maxlen
    assert abs(naive_reserved - ex["naive_reserved_tokens_approx"]) / naive_reserved < 0.01
    assert abs(n * L - ex["actual_tokens_approx"]) / (n * L) < 0.01
    naive_waste = 1 - n * L / naive_reserved
    assert abs(naive_waste - ex["naive_waste_fraction_approx"]) < 0.01
    paged_waste = 1 - st["logical_tokens"] / (st["used_blocks"] * bs)
    assert paged_waste < GOLDEN["paged_waste_bound"]["max_waste_fraction"]
    # waste per sequence is below one block (the last block's unused tail)
    assert st["used_blocks"] * bs - st["logical_tokens"] < n * bs


def test_free_list_order_and_reuse():
    m = bm.BlockManagerModel(8, 4)
    assert m.add_seq(1, 9) == bm.OK
    assert m.block_table(1) == [0, 1, 2]
    assert m.add_seq(2, 4) == bm.OK
    assert m.block_table(2) == [3]
    assert m.free_seq(1) == bm.OK
    assert m.free_list()[:3] == [2, 1, 0]          # LIFO: last pushed comes first
    assert m.add_seq(3, 5) == bm.OK
    assert m.block_table(3) == [2, 1]


def test_errors_leave_state_unchanged():
    m = bm.BlockManagerModel(4, 4)
    assert m.add_seq(1, 12) == bm.OK
    before = (list(m.free), list(m.ref), {k: list(v) for k, v in m.tables.items()})
    assert m.add_seq(2, 8) == bm.ENOMEM            # needs 2, one free
    assert m.add_seq(1, 1) == bm.EEXIST
    assert m.fork(7, 8) == bm.ENOSEQ
    assert m.free_seq(9) == bm.ENOSEQ
    assert m.append_slot(9)[0] == bm.ENOSEQ
    assert m.add_seq(3, -1) == bm.EINVAL
    assert (list(m.free), list(m.ref), {k: list(v) for k, v in m.tables.items()}) == before
    m.add_seq(2, 4)                                 # takes the last block
    assert m.append_slot(1)[0] == bm.ENOMEM        # 12 tokens: next needs a new block
    assert m.seq_len(1) == 12


def test_fork_and_copy_on_write_rules():
    m = bm.BlockManagerModel(16, 4)
    m.add_seq(0, 6)                                 # blocks [0, 1], last half full
    m.fork(0, 1)
    m.fork(0, 2)
    assert m.refcount(0) == 3 and m.refcount(1) == 3
    # first writer of the shared partial block copies it
    st, slot, src, dst = m.append_slot(1)
    assert (st, src, dst) == (bm.OK, 1, 2) and slot == 2 * 4 + 2
    assert m.block_table(1) == [0, 2] and m.refcount(1) == 2
    st, slot, src, dst = m.append_slot(2)
    assert (src, dst) == (1, 3) and slot == 3 * 4 + 2
    # the last holder writes in place
    st, slot, src, dst = m.append_slot(0)
    assert (src, dst) == (-1, -1) and slot == 1 * 4 + 2
    # full shared block: a new block, no copy
    m2 = bm.BlockManagerModel(8, 4)
    m2.add_seq(0, 4)
    m2.fork(0, 1)
    st, slot, src, dst = m2.append_slot(1)
    assert (src, dst) == (-1, -1) and m2.block_table(1) == [0, 1] and slot == 4


def test_copy_on_write_on_data_matches_private_history():
    """Run forks and appends through the model and the cache ops; every
    sequence's decode output equals attention over its own token history, and
    sequences that did not write are unaffected by the others' copies."""
    g = np.random.default_rng(11)
    H, bs, D, N = 2, 4, 8, 40
    K = g.standard_normal((N, H, bs, D)).astype(np.float32)
    V = g.standard_normal((N, H, bs, D)).astype(np.float32)
    m = bm.BlockManagerModel(N, bs)
    hist = {}                                          # seq -> list of (k, v) tokens

    def append(sid):
        st, slot, src, dst = m.append_slot(sid)
        assert st == bm.OK
        if src >= 0:
            copy_blocks(K, V, [(src, dst)])
        k = g.standard_normal((1, H, D)).astype(np.float32)
        v = g.standard_normal((1, H, D)).astype(np.float32)
        kv_cache_append(K, V, k, v, np.array([slot]))
        hist[sid].append((k[0], v[0]))

    m.add_seq(0, 0)
    hist[0] = []
    for _ in range(6):
        append(0)
    for c in (1, 2, 3):
        m.fork(0, c)
        hist[c] = list(hist[0])
    for step in range(7):
        for sid in (1, 2, 3):
            if step < sid * 2:
                append(sid)
    seqs = [0, 1, 2, 3]
    lens = np.array([m.seq_len(s) for s in seqs], dtype=np.int32)
    maxb = max(len(m.block_table(s)) for s in seqs)
    tables = np.full((4, maxb), -1, dtype=np.int32)
    for i, s in enumerate(seqs):
        t = m.block_table(s)
        tables[i, :len(t)] = t
    q = g.standard_normal((4, H, D)).astype(np.float32)
    out = oracle.paged_decode(q, K, V, tables, lens, scale=0.5, dtype="f32")
    for i, s in enumerate(seqs):
        ks = np.array([kv[0] for kv in hist[s]], np.float64)   # [L, H, D]
        vs = np.array([kv[1] for kv in hist[s]], np.float64)
        for h in range(H):
            logits = 0.5 * ks[:, h] @ q[i, h].astype(np.float64)
            w = np.exp(logits - logits.max())
            np.testing.assert_allclose(out[i, h], (w @ vs[:, h]) / w.sum(), rtol=0, atol=1e-12)


def check_swap_invariants(m: bm.BlockManagerModel):
    bs = m.block_size
    resident, host = [], []
    for sid, table in m.tables.items():
        assert len(table) == (m.lens[sid] + bs - 1) // bs
        (host if sid in m.swapped else resident).extend(b for b in table if b >= 0)
    assert sum(m.ref) == len(resident)
    assert len(set(host)) == len(host)                       # host blocks are never shared
    assert set(host).isdisjoint(m.host_free)
    assert len(host) + len(m.host_free) == m.num_host_blocks
    assert set(m.free).isdisjoint(resident)
    assert len(m.free) + len(set(resident)) == m.num_blocks


@pytest.mark.parametrize("seed", range(6))
def test_random_scripts_with_swapping_keep_invariants(seed):
    m = bm.BlockManagerModel(num_blocks=40, block_size=4, num_host_blocks=30)
    for op in random_alloc_ops(seed, 400, max_len=50, swap=True):
        m.apply(op)
        check_swap_invariants(m)


def test_swap_rules():
    m = bm.BlockManagerModel(8, 4, num_host_blocks=4)
    m.add_seq(0, 6)                                   # blocks [0, 1]
    m.fork(0, 1)                                      # shared
    st, pairs = m.swap_out(1)
    assert st == bm.OK and pairs == [(0, 0), (1, 1)]
    assert m.refcount(0) == 1 and m.refcount(1) == 1  # still held by seq 0
    assert m.block_table(1) == [0, 1]                 # now host ids
    assert m.append_slot(1)[0] == bm.EINVAL and m.fork(1, 2) == bm.EINVAL
    assert m.swap_out(1)[0] == bm.EINVAL
    st, pairs = m.swap_in(1)
    assert st == bm.OK and pairs == [(0, 2), (1, 3)]  # fresh device blocks
    assert m.host_free_list() == [1, 0, 2, 3]
    m.add_seq(5, 16)                                  # 4 blocks: device now full but two
    assert m.swap_out(5)[0] == bm.OK
    assert m.swap_out(0)[0] == bm.ENOMEM              # host pool exhausted: nothing changes
    assert 0 not in m.swapped and m.block_table(0) == [0, 1]
    assert m.free_seq(5) == bm.OK and m.stats()["free_host_blocks"] == 4


@pytest.mark.parametrize("seed", range(6))
def test_random_scripts_with_windows_and_swapping_keep_invariants(seed):
    m = bm.BlockManagerModel(num_blocks=40, block_size=4, num_host_blocks=30)
    for op in random_alloc_ops(seed, 400, max_len=50, swap=True, slide=True):
        m.apply(op)
        check_swap_invariants(m)


def test_slide_window_rules():
    m = bm.BlockManagerModel(16, 4)
    m.add_seq(0, 18)                                  # blocks 0..4, last one half full
    m.fork(0, 1)
    assert m.slide_window(0, 7) == (bm.OK, 2)         # tokens 0..10 gone: blocks 0, 1
    assert m.block_table(0) == [-1, -1, 2, 3, 4]
    assert m.refcount(0) == 1 and m.refcount(1) == 1  # still held by the fork
    assert m.slide_window(0, 7) == (bm.OK, 0)         # idempotent
    assert m.slide_window(0, 1) == (bm.OK, 2)         # keep only the last token's block
    assert m.slide_window(0, 0)[0] == bm.EINVAL
    m.free_seq(1)
    assert m.free_list()[:4] == [3, 2, 1, 0]          # freed once their last holder left
