"""GPU parity of paged decode attention against the float64 oracle.

Small cases compare every output element; the full-size workloads compare a
seeded sample of (sequence, head) rows (the oracle computes rows one by one)
and check properties of the whole output.  Tolerances: |d| <= 1e-5 for fp32,
|d| <= 2e-3 + 1e-2 |ref| for fp16 / bf16 caches.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_346_b200 as pkv
from tests.gpu_util import DeviceInputs, assert_close, sample_rows, to_f64
from workloads import CONFIGS, DecodeConfig, make_decode_inputs

pytestmark = pytest.mark.gpu

def _cfg(dtype, Hq, Hkv, D, bs, lens, pool_extra=7):
    nb = sum((L + bs - 1) // bs for L in lens)
    return DecodeConfig("case", len(lens), Hq, Hkv, D, bs, dtype, ("fixed", tuple(lens)),
                        pool=("fixed", nb + pool_extra))


def _kernels_for(dtype, G):
    ks = [pkv.PKV_KERNEL_SIMT]
    if dtype != "f32" and G <= 16 and pkv.pkv_decode_has_kernel(pkv.PKV_KERNEL_MMA):
        ks.append(pkv.PKV_KERNEL_MMA)
    return ks


def test_tiny_fp32_config_all_rows():
    inp = make_decode_inputs(CONFIGS["tiny_fp32"], seed=1)
    ref = oracle.paged_decode_inputs(inp)
    got = to_f64(DeviceInputs(inp).decode())
    assert_close(got, ref, "f32", "tiny fp32")


RAGGED = (1, 15, 16, 17, 63, 64, 65, 200, 513, 1100)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("partition", [0, 64, 512])
def test_ragged_multi_tile(dtype, G, partition):
    cfg = _cfg(dtype, 2 * G, 2, 128, 16, RAGGED)
    inp = make_decode_inputs(cfg, seed=10 + G)
    ref = oracle.paged_decode_inputs(inp)
    dev = DeviceInputs(inp)
    for kern in _kernels_for(dtype, G):
        got = to_f64(dev.decode(partition_size=partition, kernel=kern, fill_out=7.0))
        assert_close(got, ref, dtype, f"{dtype} G={G} P={partition} kernel={kern}")


@pytest.mark.parametrize("dtype,D", [("f32", 64), ("f16", 64), ("bf16", 64), ("f16", 256),
                                     ("bf16", 256)])
@pytest.mark.parametrize("bs", [16, 32, 64])
def test_head_dims_and_block_sizes(dtype, D, bs):
    G = 4
    cfg = _cfg(dtype, 2 * G, 2, D, bs, (1, 31, 32, 33, 130, 700))
    inp = make_decode_inputs(cfg, seed=3 + bs)
    ref = oracle.paged_decode_inputs(inp)
    dev = DeviceInputs(inp)
    for kern in _kernels_for(dtype, G):
        for P in (0, 128):
            got = to_f64(dev.decode(partition_size=P, kernel=kern))
            assert_close(got, ref, dtype, f"{dtype} D={D} bs={bs} P={P} kernel={kern}")


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("G", [3, 5, 6, 7, 9, 12, 16])
def test_uneven_groups(dtype, G):
    """Groups that fill an 8-head tile (3-7) or a 16-head tile (9, 12) only in
    part: the heads past the group are zero q rows of the tile and are never
    stored; split and unsplit."""
    cfg = _cfg(dtype, 2 * G, 2, 128, 16, (5, 77, 600))
    inp = make_decode_inputs(cfg, seed=20 + G)
    ref = oracle.paged_decode_inputs(inp)
    dev = DeviceInputs(inp)
    for kern in _kernels_for(dtype, G):
        for P in (0, 64):
            got = to_f64(dev.decode(partition_size=P, kernel=kern))
            assert_close(got, ref, dtype, f"{dtype} G={G} P={P} kernel={kern}")


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_single_token_returns_v_bits(dtype):
    cfg = _cfg(dtype, 8, 2, 128, 16, (1, 1, 1))
    inp = make_decode_inputs(cfg, seed=4)
    dev = DeviceInputs(inp)
    for kern in _kernels_for(dtype, 4):
        out = dev.decode(kernel=kern).cpu()
        for b in range(3):
            phys = int(inp.block_tables[b, 0])
            for h in range(8):
                assert torch.equal(out[b, h], dev.v[phys, h // 4, 0].cpu()), (kern, b, h)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_zero_length_rows_are_zero(dtype):
    cfg = _cfg(dtype, 8, 2, 128, 16, (0, 40, 0, 700))
    inp = make_decode_inputs(cfg, seed=6)
    ref = oracle.paged_decode_inputs(inp)
    dev = DeviceInputs(inp)
    for kern in _kernels_for(dtype, 4):
        got = to_f64(dev.decode(kernel=kern, fill_out=float("nan")))
        assert np.all(got[0] == 0) and np.all(got[2] == 0)
        assert_close(got, ref, dtype, f"kernel={kern}")


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("kind", ["nan", "inf"])
def test_poisoned_unused_slots_bit_identical(dtype, kind):
    cfg = _cfg(dtype, 8, 2, 128, 16, RAGGED)
    clean = DeviceInputs(make_decode_inputs(cfg, seed=8))
    dirty = DeviceInputs(make_decode_inputs(cfg, seed=8, poison=kind))
    for kern in _kernels_for(dtype, 4):
        for P in (0, 64):
            a = clean.decode(partition_size=P, kernel=kern).clone()
            b = dirty.decode(partition_size=P, kernel=kern).clone()
            assert torch.equal(a, b), (kern, P)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_physical_placement_bit_identical(dtype):
    """Contiguous (identity) placement and a shuffled pool give bit-identical
    results: the table changes where pages live, not the arithmetic."""
    cfg = _cfg(dtype, 16, 4, 128, 16, RAGGED, pool_extra=0)
    a_in = make_decode_inputs(cfg, seed=9, shuffle=False)
    b_in = make_decode_inputs(cfg, seed=9, shuffle=True)
    # move a's pages to b's physical positions
    perm = np.empty(a_in.num_blocks, dtype=np.int64)
    for bb in range(cfg.num_seqs):
        for j in range((int(a_in.context_lens[bb]) + 15) // 16):
            perm[a_in.block_tables[bb, j]] = b_in.block_tables[bb, j]
    b_in.k_cache[perm] = a_in.k_cache
    b_in.v_cache[perm] = a_in.v_cache
    b_in.q[:] = a_in.q
    A, Bd = DeviceInputs(a_in), DeviceInputs(b_in)
    for kern in _kernels_for(dtype, 4):
        assert torch.equal(A.decode(kernel=kern).clone(), Bd.decode(kernel=kern).clone())


def test_repeat_runs_bit_identical():
    cfg = _cfg("f16", 40, 40, 128, 16, RAGGED)
    dev = DeviceInputs(make_decode_inputs(cfg, seed=12))
    first = dev.decode().clone()
    for _ in range(3):
        assert torch.equal(dev.decode(), first)


def test_max_context_len_bound_larger_than_needed():
    # the host bound may exceed every length: more (empty) partitions, same result
    cfg = _cfg("bf16", 8, 2, 128, 16, (5, 300, 1000))
    inp = make_decode_inputs(cfg, seed=13)
    ref = oracle.paged_decode_inputs(inp)
    dev = DeviceInputs(inp)
    got = to_f64(dev.decode(max_context_len=inp.max_blocks_per_seq * 16, partition_size=128))
    assert_close(got, ref, "bf16", "loose bound")


def test_bad_table_entry_is_flagged_not_read():
    cfg = _cfg("f16", 4, 4, 128, 16, (40, 40))
    inp = make_decode_inputs(cfg, seed=14)
    inp.block_tables[1, 1] = 10 ** 6          # outside the pool
    dev = DeviceInputs(inp)
    pkv.pkv_device_status(clear=True)
    dev.decode()
    assert pkv.pkv_device_status(clear=True) & pkv.PKV_DEV_BAD_BLOCK
    # row 0 does not touch the bad entry and stays exact
    ref = oracle.paged_decode(inp.q[:1], inp.k_cache, inp.v_cache, inp.block_tables[:1],
                              inp.context_lens[:1], scale=cfg.scale, dtype="f16")
    assert_close(to_f64(dev.out[:1]), ref, "f16", "row 0")


def test_bad_length_is_flagged():
    cfg = _cfg("f16", 4, 4, 128, 16, (40, 40))
    inp = make_decode_inputs(cfg, seed=15)
    inp.context_lens[0] = -3
    dev = DeviceInputs(inp)
    pkv.pkv_device_status(clear=True)
    out = dev.decode()
    assert pkv.pkv_device_status(clear=True) & pkv.PKV_DEV_BAD_LEN
    assert torch.all(out[0] == 0)


# ---------------------------------------------------------------------------
# full-size workloads: sampled rows + whole-output properties

FULL = ["llama2_13b_layer", "gqa_bs16", "gqa_bs32", "long_context"]


@pytest.fixture(scope="module")
def full_inputs():
    cache = {}

    def get(name):
        if name not in cache:
            cache.clear()
            torch.cuda.empty_cache()
            inp = make_decode_inputs(CONFIGS[name], seed=2)
            cache[name] = (inp, DeviceInputs(inp))
        return cache[name]
    return get


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled_rows(name, full_inputs):
    inp, dev = full_inputs(name)
    c = inp.cfg
    n = 24 if name == "long_context" else 96
    rows = sample_rows(c.num_seqs, c.num_q_heads, n, seed=sum(name.encode()))
    # always include the longest and the shortest sequence
    lb, sb = int(np.argmax(inp.context_lens)), int(np.argmin(inp.context_lens))
    rows = np.unique(np.concatenate([rows, [[lb, 0], [sb, c.num_q_heads - 1]]]).astype(np.int32),
                     axis=0)
    ref = oracle.paged_decode_inputs(inp, rows=rows)
    for kern in _kernels_for(c.dtype, c.group):
        out = dev.decode(partition_size=c.partition_size, kernel=kern)
        got = to_f64(out[torch.from_numpy(rows[:, 0]).long().cuda(),
                         torch.from_numpy(rows[:, 1]).long().cuda()])
        assert_close(got, ref, c.dtype, f"{name} kernel={kern}")
        full = to_f64(out)
        assert np.all(np.isfinite(full))
        # every output is a convex combination of the sequence's values: within
        # the N(0,1) value range, never beyond the largest |v| in the pool
        vmax = float(torch.max(torch.abs(dev.v.float())))
        assert np.all(np.abs(full) <= vmax * 1.01 + 1e-3)


@pytest.mark.parametrize("dtype,G", [("f16", 1), ("bf16", 8), ("f32", 2)])
def test_schedule_order_changes_no_bit(dtype, G):
    """Scheduling the longest sequences first only changes timing: outputs
    are bit-identical to the natural order."""
    cfg = _cfg(dtype, 2 * G, 2, 128 if dtype != "f32" else 64, 16, RAGGED)
    inp = make_decode_inputs(cfg, seed=40 + G)
    dev = DeviceInputs(inp)
    order = torch.from_numpy(pkv.pkv_decode_schedule_order(inp.context_lens)).cuda()
    for kern in _kernels_for(dtype, G):
        for P in (0, 64):
            a = dev.decode(partition_size=P, kernel=kern).clone()
            b = dev.decode(partition_size=P, kernel=kern, seq_order=order, fill_out=3.0).clone()
            assert torch.equal(a, b), (kern, P)


def test_bad_schedule_order_entry_is_flagged():
    cfg = _cfg("f16", 4, 4, 128, 16, (40, 40))
    dev = DeviceInputs(make_decode_inputs(cfg, seed=16))
    pkv.pkv_device_status(clear=True)
    dev.decode(seq_order=torch.tensor([1, 7], dtype=torch.int32, device="cuda"))
    assert pkv.pkv_device_status(clear=True) & pkv.PKV_DEV_BAD_ORDER



# ---------------------------------------------------------------------------
# sliding window

@pytest.mark.parametrize("dtype,G", [("f16", 1), ("bf16", 8), ("f32", 1), ("bf16", 4)])
@pytest.mark.parametrize("W", [1, 15, 16, 17, 100, 600, 5000])
def test_sliding_window(dtype, G, W):
    D = 128 if dtype != "f32" else 64
    cfg = _cfg(dtype, 2 * G, 2, D, 16, RAGGED)
    inp = make_decode_inputs(cfg, seed=50 + G)
    ref = oracle.paged_decode_inputs(inp, window=W)
    dev = DeviceInputs(inp)
    for kern in _kernels_for(dtype, G):
        for P in (0, 64):
            got = to_f64(dev.decode(partition_size=P, kernel=kern, sliding_window=W,
                                    fill_out=7.0))
            assert_close(got, ref, dtype, f"{dtype} G={G} W={W} P={P} kernel={kern}")


@pytest.mark.parametrize("dtype,G", [("f16", 1), ("bf16", 8)])
def test_sliding_window_released_blocks_are_never_read(dtype, G):
    """Blocks wholly before the window may be released (entry -1) and reused:
    poisoning them and clearing their table entries changes no bit."""
    W = 100
    cfg = _cfg(dtype, 2 * G, 2, 128, 16, RAGGED)
    inp = make_decode_inputs(cfg, seed=60)
    a = DeviceInputs(inp).decode(sliding_window=W).clone()
    from workloads import poison_value
    pv = poison_value(dtype, "nan")
    for bb, L in enumerate(inp.context_lens):
        for j in range(max(0, (int(L) - W)) // 16):
            phys = inp.block_tables[bb, j]
            inp.k_cache[phys] = pv
            inp.v_cache[phys] = pv
            inp.block_tables[bb, j] = -1
    pkv.pkv_device_status(clear=True)
    b = DeviceInputs(inp).decode(sliding_window=W).clone()
    assert pkv.pkv_device_status(clear=True) == 0
    assert torch.equal(a, b)


# ---------------------------------------------------------------------------
# a grid of several waves, every element

@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("partition,W", [(64, 0), (0, 0), (64, 100), (512, 0)])
def test_many_waves_all_rows(dtype, partition, W):
    """160 ragged sequences x 8 KV heads x 4-head groups (a grid of several
    waves of CTAs per SM): every output element against the oracle, and the
    longest-first order changes no bit."""
    g = np.random.default_rng(33)
    lens = tuple(int(x) for x in g.integers(1, 700, size=160))
    cfg = _cfg(dtype, 32, 8, 128, 16, lens)
    inp = make_decode_inputs(cfg, seed=33)
    ref = oracle.paged_decode_inputs(inp, window=W)
    dev = DeviceInputs(inp)
    got = to_f64(dev.decode(partition_size=partition, fill_out=5.0, sliding_window=W))
    assert_close(got, ref, dtype, f"{dtype} P={partition} W={W}")
    order = torch.from_numpy(pkv.pkv_decode_schedule_order(inp.context_lens)).cuda()
    again = to_f64(dev.decode(partition_size=partition, seq_order=order, fill_out=-5.0,
                              sliding_window=W))
    assert np.array_equal(got, again)
