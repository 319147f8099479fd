"""The decode's work list (pkv_decode_schedule_items): every (sequence,
partition) pair with tokens, longest partition first.  Checked against the
partition count written out from its definition (attended tokens [lo, L),
lo = max(0, L - W) under a window; partitions from the block holding lo),
by hand and on random batches."""
import numpy as np
import pytest

import paged_kv_cache_346_b200 as pkv
from paged_kv_cache_346_b200 import _binding as b


def _partitions(L, bs, P, W):
    """(partition index, tokens) of one sequence, by the definition."""
    if L == 0:
        return [(0, 0)]
    lo = L - W if W > 0 and L > W else 0
    first = (lo // bs) * bs
    out, t, p = [], first, 0
    while t < L:
        out.append((p, min(P, L - t)))
        t += P
        p += 1
    return out


def test_by_hand():
    lens = np.array([0, 10, 5000, 4096, 4097, 300, 8192], np.int32)
    it = pkv.pkv_decode_schedule_items(lens, 16, 4096)
    assert it.tolist() == [[2, 0], [3, 0], [4, 0], [6, 0], [6, 1], [2, 1], [5, 0], [1, 0],
                           [4, 1], [0, 0]]
    # window 1500, partitions of 1024: 5000 attends [3500, 5000), its first
    # partition starts at 3488 (the block holding 3500): 1024 + 488 tokens
    it = pkv.pkv_decode_schedule_items(lens, 16, 1024, sliding_window=1500)
    assert it.tolist() == [[2, 0], [3, 0], [4, 0], [6, 0], [2, 1], [4, 1], [3, 1], [6, 1],
                           [5, 0], [1, 0], [0, 0]]


@pytest.mark.parametrize("seed", range(8))
def test_random_batches_against_the_definition(seed):
    g = np.random.default_rng(seed)
    B = int(g.integers(1, 300))
    lens = np.exp(g.normal(np.log(500), 1.2, size=B)).astype(np.int32).clip(0, 20000)
    lens[g.random(B) < 0.05] = 0
    bs = int(g.choice([16, 32, 64]))
    P = int(g.choice([64, 256, 1024, 4096]))
    W = int(g.choice([0, 0, 100, 3000]))
    it = pkv.pkv_decode_schedule_items(lens, bs, P, sliding_window=W)
    want = {(bi, p): n for bi in range(B) for p, n in _partitions(int(lens[bi]), bs, P, W)}
    got = [tuple(x) for x in it.tolist()]
    assert len(got) == len(set(got)) == len(want)          # every pair once
    assert set(got) == set(want)
    sizes = [want[x] for x in got]
    assert all(sizes[i] >= sizes[i + 1] for i in range(len(sizes) - 1))   # longest first
    for i in range(len(got) - 1):                            # ties in (sequence, partition) order
        if sizes[i] == sizes[i + 1]:
            assert got[i] < got[i + 1]


def test_bad_arguments_and_capacity():
    lens = np.array([100, 5000], np.int32)
    n = b._c.c_int(0)
    items = np.zeros((4, 2), np.int32)
    f = b.lib.pkv_decode_schedule_items
    assert f(lens.ctypes.data, 2, 16, 4096, 0, items.ctypes.data, 4, b._c.byref(n)) == b.PKV_OK
    assert n.value == 3 and items[:3].tolist() == [[1, 0], [1, 1], [0, 0]]
    assert f(lens.ctypes.data, 2, 16, 4096, 0, items.ctypes.data, 2, b._c.byref(n)) == \
        b.PKV_EBOUNDS and n.value == 3
    for args in ((2, 16, 100, 0), (2, 16, 0, 0), (2, 16, 16384, 0), (2, 0, 4096, 0),
                 (2, 16, 4096, -1), (-1, 16, 4096, 0)):
        assert f(lens.ctypes.data, *args, items.ctypes.data, 4, b._c.byref(n)) == b.PKV_EINVAL
    neg = np.array([100, -3], np.int32)
    assert f(neg.ctypes.data, 2, 16, 4096, 0, items.ctypes.data, 4, b._c.byref(n)) == b.PKV_EINVAL


def test_decode_items_host_checks():
    f = b.lib.pkv_paged_attention_decode_items
    p = b._c.c_void_p(1 << 20)
    base = [p, p, p, p, p, p, p, 1, 1, 8, 8, 128, 16, 4, 100, 64, 1.0, 0, b.PKV_F16, 64, None,
            0, 0, None]
    # each call below is refused by the host checks, before any launch (the
    # pointers are placeholders, never dereferenced)
    a = list(base); a[19] = 0                # partition size left to the library: refused
    assert f(*a) == b.PKV_EINVAL
    a = list(base); a[7] = 0                 # no items
    assert f(*a) == b.PKV_EINVAL
    a = list(base); a[7] = 70000             # more than a grid dimension holds
    assert f(*a) == b.PKV_EINVAL
    a = list(base); a[6] = None              # null list
    assert f(*a) == b.PKV_EINVAL
