"""The planned decode's host plan (pkv_decode_plan): every unit's attended
tokens are covered exactly once by pieces no longer than the piece size,
every piece of a unit names the unit, its first slot and piece count, the
units' slot ranges tile the workspace, and the CTAs' loads are balanced as
list scheduling (largest first) guarantees."""
import numpy as np
import pytest

import paged_kv_cache_346_b200 as pkv
from paged_kv_cache_346_b200 import _binding as b

HW, IW = b.PKV_PLAN_HEADER_WORDS, b.PKV_PLAN_ITEM_WORDS


def _parse(plan):
    h = pkv.plan_header(plan)
    C, n = h["num_ctas"], h["num_items"]
    cta = plan[HW:HW + C + 1]
    items = plan[HW + C + 1:HW + C + 1 + n * IW].reshape(n, IW)
    assert h["words"] == plan.size == HW + C + 1 + n * IW
    return h, cta, items


@pytest.mark.parametrize("seed", range(8))
def test_plan_covers_every_token_once(seed):
    g = np.random.default_rng(seed)
    B = int(g.integers(1, 40))
    lens = np.exp(g.normal(np.log(300), 1.2, size=B)).astype(np.int32)
    lens[g.random(B) < 0.1] = 0
    Hkv = int(g.choice([1, 2, 4, 8]))
    G = int(g.choice([1, 3, 8, 12, 16]))
    D = int(g.choice([128, 256]))
    bs = int(g.choice([16, 32, 64]))
    W = int(g.choice([0, 0, 40, 500]))
    C = int(g.integers(1, 300))
    pt = int(g.choice([0, 64, 256, 1024]))
    order = g.permutation(B).astype(np.int32) if seed % 2 else None
    plan = pkv.pkv_decode_plan(lens, G * Hkv, Hkv, D, bs, num_ctas=C, sliding_window=W,
                               seq_order=order, piece_tokens=pt)
    h, cta, items = _parse(plan)
    NH = 8 if G <= 8 else 16
    chunks = -(-G // NH)
    NW = 2 if (D == 128 and G == 1) else 4
    assert (h["heads_per_cta"], h["head_chunks"], h["warps_per_cta"]) == (NH, chunks, NW)
    P = h["piece_tokens"]
    assert P % 64 == 0 and (pt == 0 or P == pt) and P <= 512 * NW
    assert cta[0] == 0 and cta[-1] == len(items) and (np.diff(cta) >= 0).all()
    units = {}
    for it in items:
        units.setdefault((int(it[0]), int(it[1])), []).append(it)
    assert set(units) == {(bb, y) for bb in range(B) for y in range(Hkv * chunks)}
    slot_ranges = []
    unit_ids = set()
    for (bb, y), its in units.items():
        L = int(lens[bb])
        lo = max(0, L - W) if W > 0 else 0
        base = lo - lo % bs
        its = sorted(its, key=lambda r: r[2])
        assert its[0][2] == base and its[-1][3] == L
        for a_, b_ in zip(its, its[1:]):
            assert a_[3] == b_[2]                      # no gap, no overlap
        for k, it in enumerate(its):
            assert it[3] - it[2] <= P and it[2] % bs == 0
            assert it[4] == (lo - base if k == 0 else 0)
            # unit, first slot, pieces, index; zeros after
            assert it[5] == its[0][5] and it[6] == its[0][6] and it[7] == len(its) and it[8] == k
            assert not it[9:].any()
        unit_ids.add(int(its[0][5]))
        slot_ranges.append((int(its[0][6]), len(its) * NW))
    assert sorted(unit_ids) == list(range(B * Hkv * chunks))
    slot_ranges.sort()
    pos = 0
    for s0, n in slot_ranges:                          # the units' slots tile [0, num_slots)
        assert s0 == pos
        pos += n
    assert pos == h["num_slots"]
    # list scheduling: no CTA above the average load plus the largest piece
    cost = (items[:, 3] - items[:, 2]).astype(np.int64) + 32
    load = np.array([cost[cta[c]:cta[c + 1]].sum() for c in range(C)])
    assert load.max() == h["max_cta_tokens"]
    assert load.max() <= cost.sum() / C + cost.max()


def test_plan_bad_arguments():
    lens = np.array([10, 20], np.int32)
    hdr = np.zeros(HW, np.int32)
    f = b.lib.pkv_decode_plan
    good = [lens.ctypes.data, None, 2, 8, 2, 128, 16, 0, 4, 0, None, 0, hdr.ctypes.data]
    assert f(*good) == b.PKV_OK and hdr[0] == b.PKV_PLAN_MAGIC
    for i, bad in ((3, 7), (3, 2 * 17), (5, 64), (6, 8), (8, 0), (9, 100), (9, 4096)):
        a = list(good)
        a[i] = bad
        assert f(*a) == b.PKV_EINVAL, (i, bad)
    small = np.zeros(8, np.int32)
    a = list(good)
    a[10], a[11] = small.ctypes.data, small.size
    assert f(*a) == b.PKV_EBOUNDS
