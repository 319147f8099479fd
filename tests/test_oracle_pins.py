"""Pins for the CPU oracle: it must agree with things other than itself.

Each test ties the float64 oracle to a fact the pages or the mathematics fix:
paged attention equals attention over the contiguous cache (checked against
torch's float64 scaled_dot_product_attention on the contiguous keys and
values), permuting physical blocks changes nothing, closed forms (one token,
identical keys, zero scale, two tokens), the GQA head grouping, a pure-Python
brute force, and the bit decoders against numpy / torch casts.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from workloads import DecodeConfig, make_decode_inputs, round_to_dtype

ATOL = 1e-12


def _bf16_bits_to_f64_torch(bits: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(bits.astype(np.uint16).view(np.int16)).view(torch.bfloat16)
    return t.to(torch.float64).numpy()


def test_f16_decoder_all_bit_patterns():
    bits = np.arange(1 << 16, dtype=np.uint16)
    got = oracle.decode_bits(bits.view(np.float16), "f16")
    want = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(want[~nan]))


def test_bf16_decoder_all_bit_patterns():
    bits = np.arange(1 << 16, dtype=np.uint16)
    got = oracle.decode_bits(bits, "bf16")
    want = _bf16_bits_to_f64_torch(bits)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(want[~nan]))


def test_f32_decoder_sampled_bit_patterns():
    g = np.random.default_rng(1)
    bits = np.concatenate([
        g.integers(0, 1 << 32, size=1 << 20, dtype=np.uint64).astype(np.uint32),
        np.array([0, 1, 0x7FFFFF, 0x800000, 0x7F7FFFFF, 0x7F800000, 0xFF800000,
                  0x80000000, 0x80000001, 0x3F800000], dtype=np.uint32)])
    got = oracle.decode_bits(bits.view(np.float32), "f32")
    with np.errstate(invalid="ignore"):
        want = bits.view(np.float32).astype(np.float64)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])


def test_bf16_rounding_of_generator_matches_torch():
    # the input generator's float32 -> bf16 rounding (round to nearest even)
    x = np.random.default_rng(2).standard_normal(1 << 16).astype(np.float32) * 37.0
    mine = round_to_dtype(x, "bf16")
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, ref)


# ---------------------------------------------------------------------------
# paged == contiguous, against a library routine

def _scatter_contiguous(Kc, Vc, bs, num_blocks, seed):
    """Write contiguous per-sequence caches Kc[b][g] ([L_b, D]) into a paged
    pool at random physical blocks; returns pool arrays and tables."""
    g = np.random.default_rng(seed)
    B = len(Kc)
    Hkv = len(Kc[0])
    D = Kc[0][0].shape[1]
    lens = np.array([Kc[b][0].shape[0] for b in range(B)], dtype=np.int32)
    nb = (lens + bs - 1) // bs
    perm = g.permutation(num_blocks)
    maxb = max(1, int(nb.max()))
    tables = np.full((B, maxb), -1, dtype=np.int32)
    K = g.standard_normal((num_blocks, Hkv, bs, D)).astype(np.float32)  # garbage
    V = g.standard_normal((num_blocks, Hkv, bs, D)).astype(np.float32)
    pos = 0
    for b in range(B):
        for j in range(int(nb[b])):
            phys = int(perm[pos]); pos += 1
            tables[b, j] = phys
            for o in range(bs):
                t = j * bs + o
                if t >= lens[b]:
                    break
                for kv in range(Hkv):
                    K[phys, kv, o] = Kc[b][kv][t]
                    V[phys, kv, o] = Vc[b][kv][t]
    return K, V, tables, lens


@pytest.mark.parametrize("seed", range(6))
def test_paged_equals_contiguous_sdpa(seed):
    g = np.random.default_rng(100 + seed)
    B = int(g.integers(1, 5))
    Hkv = int(g.integers(1, 4))
    G = int(g.choice([1, 2, 4]))
    D = int(g.choice([8, 16, 64]))
    bs = int(g.choice([1, 4, 16]))
    lens = g.integers(0, 70, size=B)
    lens[0] = max(lens[0], 1)
    Kc = [[g.standard_normal((int(lens[b]), D)).astype(np.float32) for _ in range(Hkv)]
          for b in range(B)]
    Vc = [[g.standard_normal((int(lens[b]), D)).astype(np.float32) for _ in range(Hkv)]
          for b in range(B)]
    nblocks = int(((lens + bs - 1) // bs).sum()) + 5
    K, V, tables, lens32 = _scatter_contiguous(Kc, Vc, bs, nblocks, seed)
    q = g.standard_normal((B, Hkv * G, D)).astype(np.float32)
    scale = 1.0 / math.sqrt(D)
    got = oracle.paged_decode(q, K, V, tables, lens32, scale=scale, dtype="f32")
    for b in range(B):
        for h in range(Hkv * G):
            L = int(lens[b])
            if L == 0:
                assert np.all(got[b, h] == 0.0)
                continue
            qq = torch.from_numpy(q[b, h].astype(np.float64)).view(1, 1, D)
            kk = torch.from_numpy(Kc[b][h // G].astype(np.float64)).view(1, L, D)
            vv = torch.from_numpy(Vc[b][h // G].astype(np.float64)).view(1, L, D)
            want = torch.nn.functional.scaled_dot_product_attention(
                qq, kk, vv, scale=scale).view(D).numpy()
            np.testing.assert_allclose(got[b, h], want, rtol=0, atol=ATOL)


# ---------------------------------------------------------------------------
# closed forms

def _tiny(seed=0, lens=(1, 7, 16, 33), H=4, Hkv=4, D=64, bs=16, pool=16, dtype="f32"):
    cfg = DecodeConfig("t", len(lens), H, Hkv, D, bs, dtype, ("fixed", tuple(lens)),
                       pool=("fixed", pool))
    return make_decode_inputs(cfg, seed)


def test_identity_tables_are_contiguous_runs():
    """--tables identity: each sequence's pages are one contiguous run of the
    pool, in logical order, sequences one after another; the shuffled pool
    holds the same block counts as a permutation of those ids."""
    cfg = DecodeConfig("t", 5, 4, 4, 64, 16, "f32", ("fixed", (1, 7, 16, 33, 48)),
                       pool=("fixed", 24))
    ident = make_decode_inputs(cfg, 3, shuffle=False)
    shuf = make_decode_inputs(cfg, 3)
    nb = [(L + 15) // 16 for L in (1, 7, 16, 33, 48)]
    start = 0
    for b, n in enumerate(nb):
        assert ident.block_tables[b, :n].tolist() == list(range(start, start + n))
        assert (ident.block_tables[b, n:] == -1).all()
        assert ((shuf.block_tables[b, :n] >= 0).all() and (shuf.block_tables[b, n:] == -1).all())
        start += n
    used = shuf.block_tables[shuf.block_tables >= 0]
    assert len(set(used.tolist())) == sum(nb)


def test_single_token_returns_v_exactly():
    inp = _tiny(lens=(1, 1, 1))
    out = oracle.paged_decode_inputs(inp)
    for b in range(3):
        phys = inp.block_tables[b, 0]
        for h in range(4):
            assert np.array_equal(out[b, h], inp.v_cache[phys, h, 0].astype(np.float64))


def test_identical_keys_give_mean_of_v():
    inp = _tiny(lens=(5, 16, 33))
    inp.k_cache[:] = inp.k_cache[0, 0, 0]       # every key the same vector
    out = oracle.paged_decode_inputs(inp)
    for b in range(3):
        L = int(inp.context_lens[b])
        for h in range(4):
            vs = [inp.v_cache[inp.block_tables[b, t // 16], h, t % 16] for t in range(L)]
            np.testing.assert_allclose(out[b, h], np.mean(np.array(vs, np.float64), 0),
                                       rtol=0, atol=1e-13)


def test_zero_scale_gives_mean_of_v():
    inp = _tiny(lens=(3, 20))
    out = oracle.paged_decode(inp.q, inp.k_cache, inp.v_cache, inp.block_tables,
                              inp.context_lens, scale=0.0, dtype="f32")
    for b in range(2):
        L = int(inp.context_lens[b])
        for h in range(4):
            vs = [inp.v_cache[inp.block_tables[b, t // 16], h, t % 16] for t in range(L)]
            np.testing.assert_allclose(out[b, h], np.mean(np.array(vs, np.float64), 0),
                                       rtol=0, atol=1e-13)


def test_two_tokens_logistic_closed_form():
    # two tokens: the weight of token 0 is the logistic function of s0 - s1
    inp = _tiny(lens=(2,), D=16)
    out = oracle.paged_decode_inputs(inp)
    phys = inp.block_tables[0, 0]
    sc = inp.cfg.scale
    for h in range(4):
        q = inp.q[0, h].astype(np.float64)
        k0, k1 = (inp.k_cache[phys, h, i].astype(np.float64) for i in (0, 1))
        v0, v1 = (inp.v_cache[phys, h, i].astype(np.float64) for i in (0, 1))
        w0 = 1.0 / (1.0 + math.exp(sc * (float(q @ k1) - float(q @ k0))))
        np.testing.assert_allclose(out[0, h], w0 * v0 + (1 - w0) * v1, rtol=0, atol=1e-13)


def test_dominant_key_returns_its_value():
    inp = _tiny(lens=(33,), D=16)
    phys0 = inp.block_tables[0, 0]
    for h in range(4):
        q = inp.q[0, h].astype(np.float64)
        # make token 0's logit exceed every other by > 60
        inp.k_cache[phys0, h, 0] = (q / np.dot(q, q) * 200.0 / inp.cfg.scale).astype(np.float32)
    out = oracle.paged_decode_inputs(inp)
    for h in range(4):
        np.testing.assert_allclose(out[0, h], inp.v_cache[phys0, h, 0], rtol=0, atol=1e-12)


def test_key_shift_invariance():
    # adding one vector u to every key adds the same constant to every logit
    g = np.random.default_rng(5)
    inp = _tiny(lens=(9, 40), D=16)
    # dyadic values, so k + u is exact in float32
    inp.k_cache[:] = g.integers(-32, 33, size=inp.k_cache.shape) / 8.0
    inp.q[:] = g.integers(-32, 33, size=inp.q.shape) / 8.0
    base = oracle.paged_decode_inputs(inp)
    u = (g.integers(-32, 33, size=16) / 8.0).astype(np.float32)
    inp.k_cache += u
    shifted = oracle.paged_decode_inputs(inp)
    np.testing.assert_allclose(shifted, base, rtol=0, atol=1e-12)


def test_gqa_head_grouping():
    # every value of KV head g is the constant c_g, so query head h must return
    # c_{h // G}: a wrong head map (e.g. h % Hkv) fails
    inp = _tiny(lens=(7, 30), H=8, Hkv=2, D=16)
    inp.v_cache[:, 0] = 3.0
    inp.v_cache[:, 1] = -5.0
    out = oracle.paged_decode_inputs(inp)
    for h in range(8):
        want = 3.0 if h // 4 == 0 else -5.0
        np.testing.assert_allclose(out[:, h], want, rtol=0, atol=1e-13)


def test_zero_length_row_is_zero():
    inp = _tiny(lens=(0, 5, 0))
    out = oracle.paged_decode_inputs(inp)
    assert np.all(out[0] == 0) and np.all(out[2] == 0)
    assert np.all(np.isfinite(out))


# ---------------------------------------------------------------------------
# invariants of the paging itself

def test_physical_permutation_invariance_exact():
    inp = _tiny(seed=3, lens=(1, 7, 16, 33, 48), pool=24)
    base = oracle.paged_decode_inputs(inp)
    perm = np.random.default_rng(9).permutation(inp.num_blocks)   # old -> new
    K2 = np.empty_like(inp.k_cache); V2 = np.empty_like(inp.v_cache)
    K2[perm] = inp.k_cache
    V2[perm] = inp.v_cache
    T2 = inp.block_tables.copy()
    m = T2 >= 0
    T2[m] = perm[T2[m]]
    out = oracle.paged_decode(inp.q, K2, V2, T2, inp.context_lens, scale=inp.cfg.scale,
                              dtype="f32")
    assert np.array_equal(out, base)


@pytest.mark.parametrize("kind", ["nan", "inf"])
def test_unused_slots_never_read(kind):
    clean = _tiny(seed=4, lens=(1, 7, 16, 33))
    cfg = clean.cfg
    poisoned = make_decode_inputs(cfg, 4, poison=kind)
    assert np.array_equal(clean.block_tables, poisoned.block_tables)
    a = oracle.paged_decode_inputs(clean)
    b = oracle.paged_decode_inputs(poisoned)
    assert np.all(np.isfinite(b))
    assert np.array_equal(a, b)


def test_shared_prefix_blocks_equal_private_copies():
    # two sequences whose tables share their first blocks give exactly the
    # output they give when each has private copies of those blocks
    inp = _tiny(seed=6, lens=(40, 40), pool=16)
    shared = inp.block_tables.copy()
    shared[1, :2] = shared[0, :2]                    # seq 1 shares 2 blocks of seq 0
    a = oracle.paged_decode(inp.q, inp.k_cache, inp.v_cache, shared, inp.context_lens,
                            scale=inp.cfg.scale, dtype="f32")
    K2, V2 = inp.k_cache.copy(), inp.v_cache.copy()
    private = shared.copy()
    free = [i for i in range(16) if i not in set(shared.ravel().tolist())]
    for j in range(2):
        K2[free[j]] = K2[shared[0, j]]
        V2[free[j]] = V2[shared[0, j]]
        private[1, j] = free[j]
    b = oracle.paged_decode(inp.q, K2, V2, private, inp.context_lens,
                            scale=inp.cfg.scale, dtype="f32")
    assert np.array_equal(a, b)


@pytest.mark.parametrize("seed", range(4))
def test_brute_force_tiny(seed):
    g = np.random.default_rng(seed)
    B = int(g.integers(1, 4))
    Hkv = int(g.integers(1, 3))
    G = int(g.integers(1, 3))
    D = int(g.integers(1, 9))
    bs = int(g.choice([1, 3, 4]))
    lens = tuple(int(x) for x in g.integers(0, 41, size=B))
    nb = sum((L + bs - 1) // bs for L in lens)
    cfg = DecodeConfig("b", B, Hkv * G, Hkv, D, bs, "f32", ("fixed", lens),
                       pool=("fixed", nb + 3))
    inp = make_decode_inputs(cfg, seed)
    got = oracle.paged_decode_inputs(inp)
    want = brute.paged_decode(inp.q.astype(np.float64), inp.k_cache.astype(np.float64),
                              inp.v_cache.astype(np.float64), inp.block_tables,
                              inp.context_lens, cfg.scale)
    np.testing.assert_allclose(got, np.array(want).reshape(got.shape), rtol=0, atol=ATOL)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_half_storage_matches_brute_on_decoded_values(dtype):
    inp = _tiny(seed=7, lens=(5, 17), H=4, Hkv=2, D=8, dtype=dtype)
    got = oracle.paged_decode_inputs(inp)
    if dtype == "f16":
        dec = lambda a: a.astype(np.float64)
    else:
        dec = _bf16_bits_to_f64_torch
    want = brute.paged_decode(dec(inp.q), dec(inp.k_cache), dec(inp.v_cache),
                              inp.block_tables, inp.context_lens, inp.cfg.scale)
    np.testing.assert_allclose(got, np.array(want).reshape(got.shape), rtol=0, atol=ATOL)


def test_sampled_rows_match_full():
    inp = _tiny(seed=8, lens=(3, 17, 33, 1), H=8, Hkv=4)
    full = oracle.paged_decode_inputs(inp)
    rows = np.array([[0, 7], [2, 3], [3, 0], [1, 5]], dtype=np.int32)
    part = oracle.paged_decode_inputs(inp, rows=rows)
    for i, (b, h) in enumerate(rows):
        assert np.array_equal(part[i], full[b, h])


def test_bad_table_entry_rejected():
    inp = _tiny(lens=(20,))
    inp.block_tables[0, 1] = 999
    with pytest.raises(ValueError):
        oracle.paged_decode_inputs(inp)


# ---------------------------------------------------------------------------
# sliding window

def test_window_at_least_the_length_is_full_attention():
    inp = _tiny(seed=20, lens=(1, 7, 16, 33))
    full = oracle.paged_decode_inputs(inp)
    assert np.array_equal(oracle.paged_decode_inputs(inp, window=33), full)
    assert np.array_equal(oracle.paged_decode_inputs(inp, window=1000), full)


def test_window_of_one_returns_the_last_value():
    inp = _tiny(seed=21, lens=(1, 7, 16, 33))
    out = oracle.paged_decode_inputs(inp, window=1)
    for b, L in enumerate(inp.context_lens):
        t = int(L) - 1
        phys = inp.block_tables[b, t // 16]
        for h in range(4):
            assert np.array_equal(out[b, h], inp.v_cache[phys, h, t % 16].astype(np.float64))


@pytest.mark.parametrize("W", [2, 15, 16, 17, 40])
def test_window_equals_sdpa_on_the_last_tokens(W):
    g = np.random.default_rng(300 + W)
    B, Hkv, G, D, bs = 3, 2, 2, 16, 4
    lens = np.array([50, 9, 23])
    Kc = [[g.standard_normal((int(lens[b]), D)).astype(np.float32) for _ in range(Hkv)]
          for b in range(B)]
    Vc = [[g.standard_normal((int(lens[b]), D)).astype(np.float32) for _ in range(Hkv)]
          for b in range(B)]
    nblocks = int(((lens + bs - 1) // bs).sum()) + 3
    K, V, tables, lens32 = _scatter_contiguous(Kc, Vc, bs, nblocks, W)
    q = g.standard_normal((B, Hkv * G, D)).astype(np.float32)
    got = oracle.paged_decode(q, K, V, tables, lens32, scale=0.3, dtype="f32", window=W)
    for b in range(B):
        L = int(lens[b])
        lo = max(0, L - W)
        for h in range(Hkv * G):
            kk = torch.from_numpy(Kc[b][h // G][lo:].astype(np.float64)).view(1, L - lo, D)
            vv = torch.from_numpy(Vc[b][h // G][lo:].astype(np.float64)).view(1, L - lo, D)
            qq = torch.from_numpy(q[b, h].astype(np.float64)).view(1, 1, D)
            want = torch.nn.functional.scaled_dot_product_attention(
                qq, kk, vv, scale=0.3).view(D).numpy()
            np.testing.assert_allclose(got[b, h], want, rtol=0, atol=ATOL)


def test_window_never_reads_released_entries():
    inp = _tiny(seed=22, lens=(40, 33))
    a = oracle.paged_decode_inputs(inp, window=10)
    inp.block_tables[0, :1] = -1                      # tokens 0..15 lie before 30
    inp.block_tables[1, :1] = -1                      # tokens 0..15 lie before 23
    b = oracle.paged_decode_inputs(inp, window=10)
    assert np.array_equal(a, b)


def test_window_brute_force():
    inp = _tiny(seed=23, lens=(5, 17, 33), H=4, Hkv=2, D=8)
    for W in (1, 4, 16, 20):
        got = oracle.paged_decode_inputs(inp, window=W)
        want = brute.paged_decode(inp.q.astype(np.float64), inp.k_cache.astype(np.float64),
                                  inp.v_cache.astype(np.float64), inp.block_tables,
                                  inp.context_lens, inp.cfg.scale, window=W)
        np.testing.assert_allclose(got, np.array(want).reshape(got.shape), rtol=0, atol=ATOL)
