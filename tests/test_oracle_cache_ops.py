"""Pins for the oracle's cache write / block copy definitions."""
import numpy as np

from oracle.cache_ops import copy_blocks, kv_cache_append


def _pool(seed, N=6, H=3, bs=4, D=5):
    g = np.random.default_rng(seed)
    return (g.standard_normal((N, H, bs, D)).astype(np.float32),
            g.standard_normal((N, H, bs, D)).astype(np.float32))


def test_append_round_trip_and_untouched_slots():
    K, V = _pool(0)
    K0, V0 = K.copy(), V.copy()
    g = np.random.default_rng(1)
    T = 7
    k = g.standard_normal((T, 3, 5)).astype(np.float32)
    v = g.standard_normal((T, 3, 5)).astype(np.float32)
    slots = np.array([0, 5, -1, 23, 9, -7, 12], dtype=np.int64)
    kv_cache_append(K, V, k, v, slots)
    written = set()
    for t, s in enumerate(slots):
        if s < 0:
            continue
        written.add(int(s))
        # reading the slot back by (block, offset) = divmod(s, bs) gives the token
        assert np.array_equal(K[s // 4, :, s % 4], k[t])
        assert np.array_equal(V[s // 4, :, s % 4], v[t])
    for s in range(6 * 4):
        if s not in written:
            assert np.array_equal(K[s // 4, :, s % 4], K0[s // 4, :, s % 4])
            assert np.array_equal(V[s // 4, :, s % 4], V0[s // 4, :, s % 4])


def test_copy_blocks_whole_block_every_head():
    K, V = _pool(2)
    K0, V0 = K.copy(), V.copy()
    copy_blocks(K, V, [(1, 4), (3, 0)])
    assert np.array_equal(K[4], K0[1]) and np.array_equal(V[4], V0[1])
    assert np.array_equal(K[0], K0[3]) and np.array_equal(V[0], V0[3])
    for b in (1, 2, 3, 5):
        assert np.array_equal(K[b], K0[b]) and np.array_equal(V[b], V0[b])
