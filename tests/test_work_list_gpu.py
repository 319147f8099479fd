"""GPU decode over a work list (pkv_paged_attention_decode_items and its
E4M3 form): the same partitions as the grid decode, scheduled as a list of
(sequence, partition) pairs, longest first.  Outputs must equal the grid
decode's with the same partition size bit for bit, and the oracle's within
the stated tolerance; empty sequences give zero rows; bad items are flagged
and skipped.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_346_b200 as pkv
from tests.gpu_util import assert_close, to_device, to_f64
from workloads import DecodeConfig, make_decode_inputs, make_e4m3_pages

pytestmark = pytest.mark.gpu

RAGGED = (0, 1, 15, 16, 17, 63, 64, 65, 200, 513, 1100, 2600)


def _cfg(dtype, Hq, Hkv, D, bs, lens, pool_extra=7):
    nb = sum((L + bs - 1) // bs for L in lens)
    return DecodeConfig("items", len(lens), Hq, Hkv, D, bs, dtype, ("fixed", tuple(lens)),
                        pool=("fixed", nb + pool_extra))


def _ws(c, span, P):
    n = pkv.pkv_decode_workspace_size(c.num_seqs, c.num_q_heads, c.num_kv_heads, c.head_dim,
                                      span, P)
    return torch.empty(max(16, n), dtype=torch.uint8, device="cuda")


def _decode(inp, dtype, P, W=0, items=None, order=None, kernel=pkv.PKV_KERNEL_AUTO):
    c = inp.cfg
    mcl = inp.max_context_len
    span = min(mcl, W + c.block_size - 1) if W else mcl
    q = to_device(inp.q, dtype)
    out = torch.full_like(q, float("nan"))
    pkv.pkv_paged_attention_decode(
        out, q, to_device(inp.k_cache, dtype), to_device(inp.v_cache, dtype),
        to_device(inp.block_tables), to_device(inp.context_lens), c.scale, c.block_size, mcl,
        partition_size=P, workspace=_ws(c, span, P), seq_order=order, items=items,
        sliding_window=W, kernel=kernel)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("dtype,Hq,Hkv,D,kernel", [
    ("f16", 4, 4, 128, pkv.PKV_KERNEL_SIMT),     # MHA on the CUDA cores
    ("bf16", 16, 2, 128, pkv.PKV_KERNEL_MMA),    # GQA on the tensor cores
    ("f16", 32, 2, 64, pkv.PKV_KERNEL_MMA),      # 16-head tiles
    ("f32", 4, 2, 64, pkv.PKV_KERNEL_SIMT),
])
@pytest.mark.parametrize("P,W", [(64, 0), (512, 0), (1024, 0), (256, 300)])
def test_items_equal_the_grid_decode_and_the_oracle(dtype, Hq, Hkv, D, kernel, P, W):
    inp = make_decode_inputs(_cfg(dtype, Hq, Hkv, D, 16, RAGGED), seed=51)
    items = torch.from_numpy(
        pkv.pkv_decode_schedule_items(inp.context_lens, 16, P, sliding_window=W)).cuda()
    order = torch.from_numpy(pkv.pkv_decode_schedule_order(inp.context_lens)).cuda()
    grid = _decode(inp, dtype, P, W, order=order, kernel=kernel)
    listed = _decode(inp, dtype, P, W, items=items, kernel=kernel)
    assert torch.equal(grid, listed)
    ref = oracle.paged_decode_inputs(inp, window=W)
    got = to_f64(listed)
    assert (got[0] == 0).all()  # the empty sequence
    assert_close(got, ref, dtype, f"{dtype} G {Hq // Hkv} P {P} W {W}")
    assert pkv.pkv_device_status(clear=True) == 0


@pytest.mark.parametrize("per_page", [False, True])
@pytest.mark.parametrize("G,P,W", [(1, 512, 0), (8, 512, 0), (8, 1024, 0), (8, 1024, 700),
                                   (8, 64, 0)])
def test_e4m3_items_equal_the_grid_decode_and_the_oracle(per_page, G, P, W):
    """2- and 4-warp CTAs (partitions up to 512 tokens, and over), with and
    without a window, both scale modes."""
    inp = make_decode_inputs(_cfg("bf16", 2 * G, 2, 128, 16, RAGGED), seed=52 + G)
    pages = make_e4m3_pages(inp, 5, per_page=per_page)
    c = inp.cfg

    def codes(a):
        return torch.from_numpy(np.ascontiguousarray(a)).cuda().view(torch.float8_e4m3fn)

    k, v = codes(pages.k_cache), codes(pages.v_cache)
    ks, vs = torch.from_numpy(pages.k_scale).cuda(), torch.from_numpy(pages.v_scale).cuda()
    q, bt, cl = to_device(inp.q, "bf16"), to_device(inp.block_tables), to_device(inp.context_lens)
    items = torch.from_numpy(
        pkv.pkv_decode_schedule_items(inp.context_lens, 16, P, sliding_window=W)).cuda()
    mcl = inp.max_context_len
    span = min(mcl, W + 15) if W else mcl
    outs = []
    for kw in ({"items": items}, {"seq_order": None}):
        out = torch.full_like(q, float("nan"))
        pkv.pkv_paged_attention_decode_e4m3(out, q, k, v, ks, vs, bt, cl, c.scale, 16, mcl,
                                            partition_size=P, workspace=_ws(c, span, P),
                                            sliding_window=W, **kw)
        torch.cuda.synchronize()
        outs.append(out)
    assert torch.equal(outs[0], outs[1])
    ref = oracle.paged_decode(inp.q, pages.k_cache, pages.v_cache, inp.block_tables,
                              inp.context_lens, scale=c.scale, dtype="bf16", kv_dtype="e4m3",
                              k_scale=pages.k_scale, v_scale=pages.v_scale, window=W)
    assert_close(to_f64(outs[0]), ref, "bf16", f"E4M3 G {G} P {P} W {W} per_page {per_page}")
    assert pkv.pkv_device_status(clear=True) == 0


@pytest.mark.parametrize("per_page", [False, True])
def test_e4m3_gqa_batch_shape_items(per_page):
    """The GQA batch's shape with E4M3 pages at a reduced batch, 4096-token
    partitions: every row against the oracle, and equal to the grid decode
    bit for bit."""
    g = np.random.default_rng(56)
    lens = np.exp(g.normal(np.log(512), 1.0, size=200)).astype(np.int32).clip(32, 8192)
    lens[:3] = (8192, 6000, 4097)
    lens[7] = 0
    inp = make_decode_inputs(_cfg("bf16", 64, 8, 128, 16, tuple(int(x) for x in lens)), seed=57)
    pages = make_e4m3_pages(inp, 6, per_page=per_page)
    c = inp.cfg

    def codes(a):
        return torch.from_numpy(np.ascontiguousarray(a)).cuda().view(torch.float8_e4m3fn)

    k, v = codes(pages.k_cache), codes(pages.v_cache)
    ks, vs = torch.from_numpy(pages.k_scale).cuda(), torch.from_numpy(pages.v_scale).cuda()
    q, bt, cl = to_device(inp.q, "bf16"), to_device(inp.block_tables), to_device(inp.context_lens)
    items = torch.from_numpy(pkv.pkv_decode_schedule_items(inp.context_lens, 16, 4096)).cuda()
    order = torch.from_numpy(pkv.pkv_decode_schedule_order(inp.context_lens)).cuda()
    outs = []
    for kw in ({"items": items}, {"seq_order": order}):
        out = torch.full_like(q, float("nan"))
        pkv.pkv_paged_attention_decode_e4m3(out, q, k, v, ks, vs, bt, cl, c.scale, 16,
                                            inp.max_context_len, partition_size=4096,
                                            workspace=_ws(c, inp.max_context_len, 4096), **kw)
        torch.cuda.synchronize()
        outs.append(out)
    assert torch.equal(outs[0], outs[1])
    ref = oracle.paged_decode(inp.q, pages.k_cache, pages.v_cache, inp.block_tables,
                              inp.context_lens, scale=c.scale, dtype="bf16", kv_dtype="e4m3",
                              k_scale=pages.k_scale, v_scale=pages.v_scale)
    got = to_f64(outs[0])
    assert (got[7] == 0).all()
    assert_close(got, ref, "bf16", f"E4M3 GQA shape per_page {per_page}")
    assert pkv.pkv_device_status(clear=True) == 0


def test_bad_items_are_flagged_and_skipped():
    inp = make_decode_inputs(_cfg("f16", 4, 4, 128, 16, (40, 40)), seed=53)
    good = pkv.pkv_decode_schedule_items(inp.context_lens, 16, 64)
    # a sequence outside the batch, a negative partition, a partition past
    # the sequence's (skipped, not flagged); the listed rows are still right
    bad = np.concatenate([good, [[7, 0], [1, -2], [0, 5]]]).astype(np.int32)
    pkv.pkv_device_status(clear=True)
    out = _decode(inp, "f16", 64, items=torch.from_numpy(bad).cuda())
    assert pkv.pkv_device_status(clear=True) & pkv.PKV_DEV_BAD_ORDER
    assert_close(to_f64(out), oracle.paged_decode_inputs(inp), "f16", "bad items")


def test_gqa_batch_shape_items():
    """The GQA batch's shape and lengths (lognormal, 4096-token partitions,
    a few sequences split in two) at a reduced batch: items against the
    oracle on every row."""
    g = np.random.default_rng(54)
    lens = np.exp(g.normal(np.log(512), 1.0, size=48)).astype(np.int32).clip(32, 8192)
    lens[:3] = (8192, 6000, 4097)
    inp = make_decode_inputs(_cfg("bf16", 64, 8, 128, 16, tuple(int(x) for x in lens)), seed=55)
    items = torch.from_numpy(pkv.pkv_decode_schedule_items(inp.context_lens, 16, 4096)).cuda()
    out = _decode(inp, "bf16", 4096, items=items)
    assert_close(to_f64(out), oracle.paged_decode_inputs(inp), "bf16", "GQA shape, items")
    assert pkv.pkv_device_status(clear=True) == 0


@pytest.mark.parametrize("kernel", [pkv.PKV_KERNEL_MMA, pkv.PKV_KERNEL_SIMT])
def test_reduce_several_sequences_per_cta(kernel):
    """300 sequences, 64 query heads: the reduce's small form gives each CTA 8
    heads of S = 9 consecutive sequences (34 CTAs in y, the last with 3),
    with split sequences scattered among them (every 7th long, some CTAs with
    two or none) and an empty one.  Every row against the oracle, for the
    work list and the partition grid, which must agree bit for bit."""
    g = np.random.default_rng(61)
    lens = g.integers(16, 600, size=300).astype(np.int32)
    lens[::7] = g.integers(1100, 4000, size=lens[::7].size)
    lens[100] = 0
    lens[101] = 1024  # exactly one 1024-token partition: direct
    cfg = _cfg("bf16", 64, 8, 128, 16, tuple(int(x) for x in lens), pool_extra=3)
    inp = make_decode_inputs(cfg, seed=62)
    P = 1024
    items = torch.from_numpy(pkv.pkv_decode_schedule_items(inp.context_lens, 16, P)).cuda()
    order = torch.from_numpy(pkv.pkv_decode_schedule_order(inp.context_lens)).cuda()
    listed = _decode(inp, "bf16", P, items=items, kernel=kernel)
    grid = _decode(inp, "bf16", P, order=order, kernel=kernel)
    assert torch.equal(listed, grid)
    got = to_f64(listed)
    assert (got[100] == 0).all()
    assert_close(got, oracle.paged_decode_inputs(inp), "bf16", f"reduce S>1 kernel={kernel}")
    assert pkv.pkv_device_status(clear=True) == 0
