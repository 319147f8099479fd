"""Host grouping for the shared-prefix decode (pkv_decode_prefix_groups),
checked by hand and by its defining properties on random forked batches."""
import numpy as np
import pytest

import paged_kv_cache_346_b200 as pkv
from paged_kv_cache_346_b200 import _binding as b


def test_by_hand():
    bt = np.array([[5, 6, 7, 9], [5, 6, 7, 10], [5, 6, 8, 11], [1, 2, 3, 4], [1, 2, 3, 4],
                   [0, -1, -1, -1], [1, 2, 3, 4]], np.int32)
    lens = np.array([60, 64, 50, 64, 40, 10, 64], np.int32)
    spl, members = pkv.pkv_decode_prefix_groups(bt, lens, 16)
    # 0, 1, 2 share blocks 5, 6 (seq 2 holds 8 at position 2); 3, 4, 6 share
    # 1, 2 (seq 4 has only two full blocks); 5 has no full block
    assert spl.tolist() == [32, 32, 32, 32, 32, 0, 32]
    assert members.tolist() == [[0, 1, 2], [3, 4, 6]]
    # groups of at most 2: the leftover member of each bucket stays out
    spl, members = pkv.pkv_decode_prefix_groups(bt, lens, 16, max_group_size=2)
    assert members.tolist() == [[0, 1], [3, 4]]
    assert spl.tolist() == [48, 48, 0, 32, 32, 0, 0]
    # a prefix of at least 3 blocks: 0, 1, 2 share only two; seq 4 has only
    # two full blocks, so 3 and 6 share all four of theirs
    spl, members = pkv.pkv_decode_prefix_groups(bt, lens, 16, min_prefix_blocks=3)
    assert members.tolist() == [[3, 6]]
    assert spl.tolist() == [0, 0, 0, 64, 0, 0, 64]


@pytest.mark.parametrize("seed", range(6))
def test_random_forks_properties(seed):
    g = np.random.default_rng(seed)
    bs = 16
    al = pkv.BlockAllocator(4000, bs)
    sid = 0
    for _ in range(int(g.integers(3, 9))):                 # prompts
        root = 100_000 + sid
        assert al.add_seq(root, int(g.integers(1, 300))) == 0
        kids = []
        for _ in range(int(g.integers(1, 20))):            # samples (some forked from samples)
            parent = root if not kids or g.random() < 0.6 else kids[g.integers(len(kids))]
            assert al.fork(parent, sid) == 0
            kids.append(sid)
            for _ in range(int(g.integers(0, 70))):
                assert al.append_slot(sid)[0] == 0
            sid += 1
        assert al.free_seq(root) == 0
    for _ in range(5):                                     # unrelated sequences
        assert al.add_seq(sid, int(g.integers(0, 200))) == 0
        sid += 1
    seqs = np.arange(sid)
    tables, lens = al.build_block_tables(seqs, 256)
    mgs = int(g.integers(2, 17))
    spl, members = pkv.pkv_decode_prefix_groups(tables, lens, bs, max_group_size=mgs)
    seen = set()
    for row in members:
        mem = [int(x) for x in row if x >= 0]
        assert 2 <= len(mem) <= mgs and (row[len(mem):] == -1).all()
        assert not (seen & set(mem))
        seen |= set(mem)
        S = int(spl[mem[0]])
        nb = S // bs
        assert S > 0 and S % bs == 0 and all(int(spl[m]) == S for m in mem)
        for m in mem:
            assert lens[m] >= S and (tables[m, :nb] == tables[mem[0], :nb]).all()
        # maximal: one more block is not a full block shared by every member
        full = min(int(lens[m]) // bs for m in mem)
        if nb < full:
            assert len({int(tables[m, nb]) for m in mem}) > 1
    assert all(spl[i] == 0 for i in range(sid) if i not in seen)
    assert len(members) > 0


def test_bad_arguments():
    bt = np.zeros((2, 4), np.int32)
    lens = np.array([32, 32], np.int32)
    ng = b._c.c_int(0)
    spl = np.zeros(2, np.int32)
    mem = np.zeros((1, 4), np.int32)
    f = b.lib.pkv_decode_prefix_groups
    args = [bt.ctypes.data, lens.ctypes.data, 2, 4, 16, 4, 1, spl.ctypes.data, mem.ctypes.data, 1,
            b._c.byref(ng)]
    assert f(*args) == b.PKV_OK and ng.value == 1
    for i, bad in ((5, 1), (5, b.PKV_MAX_PREFIX_GROUP + 1), (6, 0), (4, 0)):
        a = list(args)
        a[i] = bad
        assert f(*a) == b.PKV_EINVAL
    a = list(args)
    a[9] = 0                                  # no room for the one group
    assert f(*a) == b.PKV_EBOUNDS
