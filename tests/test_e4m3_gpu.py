"""GPU parity of the FP8 E4M3 page path against the oracle.

Quantising append: bit-exact codes (both sides divide in float32 and round to
the nearest E4M3 value, ties to even, saturating at 448).  Decode over E4M3
pages: |d| <= 2e-3 + 1e-2 |ref| against the float64 oracle over the
dequantised values, the tolerance of the 16-bit decode (the codes widen
exactly; what differs is float32 accumulation and the output rounding).
Block copies and swaps of E4M3 pools: bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_346_b200 as pkv
from oracle.cache_ops import copy_blocks, kv_cache_append_e4m3
from tests.gpu_util import TORCH_DTYPE, assert_close, sample_rows, to_device, to_f64
from workloads import CONFIGS, DecodeConfig, make_decode_inputs, make_e4m3_pages, normal_fill

pytestmark = pytest.mark.gpu

RAGGED = (1, 15, 16, 17, 63, 64, 65, 200, 513, 1100)


def _codes(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda().view(torch.float8_e4m3fn)


class E4M3Inputs:
    """Device copies of a decode batch whose pages are E4M3 codes."""

    def __init__(self, inp, seed, per_page=False, v_scale_range=None):
        c = inp.cfg
        self.inp = inp
        self.pages = make_e4m3_pages(inp, seed, per_page=per_page)
        if v_scale_range is not None:  # widen the V scales
            g = np.random.default_rng(seed + 77)
            lo, hi = v_scale_range
            shape = self.pages.v_scale.shape
            if len(shape) == 1:  # one per KV head: both ends of the range
                self.pages.v_scale = np.geomspace(lo, hi, shape[0]).astype(np.float32)
            else:
                self.pages.v_scale = np.exp(g.uniform(np.log(lo), np.log(hi),
                                                      size=shape)).astype(np.float32)
        self.q = to_device(inp.q, c.dtype)
        self.k = _codes(self.pages.k_cache)
        self.v = _codes(self.pages.v_cache)
        self.ks = torch.from_numpy(self.pages.k_scale).cuda()
        self.vs = torch.from_numpy(self.pages.v_scale).cuda()
        self.bt = to_device(inp.block_tables)
        self.cl = to_device(inp.context_lens)
        self.out = torch.empty_like(self.q)

    def decode(self, partition_size=0, sliding_window=0, seq_order=None, fill_out=None,
               kernel=pkv.PKV_KERNEL_AUTO):
        c = self.inp.cfg
        mcl = self.inp.max_context_len
        span = min(mcl, sliding_window + c.block_size - 1) if sliding_window > 0 else mcl
        ws_bytes = pkv.pkv_decode_workspace_size(c.num_seqs, c.num_q_heads, c.num_kv_heads,
                                                 c.head_dim, span, partition_size)
        ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
        if fill_out is not None:
            self.out.fill_(fill_out)
        pkv.pkv_paged_attention_decode_e4m3(self.out, self.q, self.k, self.v, self.ks, self.vs,
                                            self.bt, self.cl, c.scale, c.block_size, mcl,
                                            partition_size=partition_size, workspace=ws,
                                            sliding_window=sliding_window, seq_order=seq_order,
                                            kernel=kernel)
        torch.cuda.synchronize()
        return self.out

    def oracle(self, rows=None, window=0):
        c = self.inp.cfg
        return oracle.paged_decode(self.inp.q, self.pages.k_cache, self.pages.v_cache,
                                   self.inp.block_tables, self.inp.context_lens, scale=c.scale,
                                   dtype=c.dtype, kv_dtype="e4m3", k_scale=self.pages.k_scale,
                                   v_scale=self.pages.v_scale, rows=rows, window=window)


KERNELS = (pkv.PKV_KERNEL_SIMT, pkv.PKV_KERNEL_MMA)


def _cfg(dtype, Hq, Hkv, D, bs, lens, pool_extra=7):
    nb = sum((L + bs - 1) // bs for L in lens)
    return DecodeConfig("case", len(lens), Hq, Hkv, D, bs, dtype, ("fixed", tuple(lens)),
                        pool=("fixed", nb + pool_extra))


# ---------------------------------------------------------------------------
# quantising append

@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("H,D,bs", [(40, 128, 16), (8, 128, 32), (2, 256, 64), (3, 16, 16)])
def test_append_e4m3_bit_exact(dtype, H, D, bs):
    N, T = 40, 260
    g = np.random.default_rng(H * 7 + D + bs)
    K = np.zeros((N, H, bs, D), np.uint8)
    V = np.zeros_like(K)
    # a wide spread: scales make some quotients saturate and some subnormal
    k = normal_fill((T, H, D), dtype, 11)
    v = normal_fill((T, H, D), dtype, 12)
    ks = g.uniform(1e-3, 0.05, size=H).astype(np.float32)
    vs = g.uniform(1e-3, 0.05, size=H).astype(np.float32)
    ks[0] = 2e-3        # |k| / ks beyond 448 for |k| > 0.9: saturation
    vs[-1] = 40.0       # quotients in the subnormal range
    slots = g.choice(N * bs, size=T, replace=False).astype(np.int64)
    slots[g.random(T) < 0.1] = -1
    dK, dV = _codes(K), _codes(V)
    pkv.pkv_kv_cache_append_e4m3(dK, dV, to_device(k, dtype), to_device(v, dtype),
                                 torch.from_numpy(ks).cuda(), torch.from_numpy(vs).cuda(),
                                 torch.from_numpy(slots).cuda())
    kv_cache_append_e4m3(K, V, k, v, slots, ks, vs, dtype)
    torch.cuda.synchronize()
    gotk = dK.view(torch.uint8).cpu().numpy()
    gotv = dV.view(torch.uint8).cpu().numpy()
    assert np.array_equal(gotk, K), int((gotk != K).sum())
    assert np.array_equal(gotv, V), int((gotv != V).sum())
    # the spread really reached both ends
    assert ((K & 0x7F) == 0x7E).any() and ((V & 0x78) == 0).any()


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_append_e4m3_bit_exact_at_rounding_boundaries(dtype):
    """Values whose quotient lies on, or within an ulp of, the midpoint
    between two E4M3 codes (ties go to the even code): the append's fast
    multiply-by-reciprocal path must hand these to the division and still
    match the float32 quotient's rounding bit for bit."""
    from workloads import round_to_dtype
    H, D, bs, N = 4, 128, 16, 8
    codes = np.arange(126, dtype=np.uint8)
    vals = oracle.decode_bits(codes, "e4m3")
    mids = (vals[:-1] + vals[1:]) / 2.0                       # 125 midpoints
    scales = np.array([1.0, 3.0, 0.1, 2.0 ** -7], np.float32)  # one per KV head
    T = 4
    k = np.zeros((T, H, D), np.float64)
    for h in range(H):
        x = np.concatenate([mids, -mids, mids * (1 + 2 ** -9), mids * (1 - 2 ** -9)])
        x = np.resize(x * scales[h], T * D).reshape(T, D)
        k[:, h, :] = x
    k = round_to_dtype(k, dtype)
    v = k[::-1].copy()
    slots = np.arange(T, dtype=np.int64) * bs + 3
    K = np.zeros((N, H, bs, D), np.uint8)
    V = np.zeros_like(K)
    dK, dV = _codes(K), _codes(V)
    sc = torch.from_numpy(scales).cuda()
    pkv.pkv_kv_cache_append_e4m3(dK, dV, to_device(k, dtype), to_device(v, dtype), sc, sc,
                                 torch.from_numpy(slots).cuda())
    kv_cache_append_e4m3(K, V, k, v, slots, scales, scales, dtype)
    torch.cuda.synchronize()
    assert np.array_equal(dK.view(torch.uint8).cpu().numpy(), K)
    assert np.array_equal(dV.view(torch.uint8).cpu().numpy(), V)
    # the first head's first 125 quotients are exact ties: each went to the
    # neighbour with the even code
    assert np.all(K[3 // bs, 0, 3, :125] % 2 == 0)


def test_append_e4m3_bad_slot_flagged():
    N, H, bs, D = 4, 2, 16, 128
    dK = _codes(np.zeros((N, H, bs, D), np.uint8))
    dV = _codes(np.zeros((N, H, bs, D), np.uint8))
    k = torch.ones(2, H, D, dtype=torch.float16, device="cuda")
    s = torch.ones(H, dtype=torch.float32, device="cuda")
    pkv.pkv_device_status(clear=True)
    pkv.pkv_kv_cache_append_e4m3(dK, dV, k, k, s, s,
                                 torch.tensor([3, N * bs], dtype=torch.int64, device="cuda"))
    assert pkv.pkv_device_status(clear=True) & pkv.PKV_DEV_BAD_SLOT
    got = dK.view(torch.uint8).cpu().numpy()
    assert (got[0, :, 3] == 0x38).all() and got.sum() == 0x38 * H * D


# ---------------------------------------------------------------------------
# decode over E4M3 pages

@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("G", [1, 2, 4, 8, 3])
@pytest.mark.parametrize("partition", [0, 64, 512])
def test_decode_e4m3_ragged(dtype, G, partition):
    cfg = _cfg(dtype, 2 * G, 2, 128, 16, RAGGED)
    inp = make_decode_inputs(cfg, seed=70 + G)
    dev = E4M3Inputs(inp, seed=70 + G)
    ref = dev.oracle()
    for kern in KERNELS:
        got = to_f64(dev.decode(partition_size=partition, fill_out=7.0, kernel=kern))
        assert_close(got, ref, dtype, f"e4m3 {dtype} G={G} P={partition} kernel={kern}")


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("D", [128, 256])
@pytest.mark.parametrize("bs", [16, 32, 64])
def test_decode_e4m3_head_dims_block_sizes(dtype, D, bs):
    cfg = _cfg(dtype, 4, 2, D, bs, (1, 31, 32, 33, 130, 700))
    inp = make_decode_inputs(cfg, seed=80 + bs)
    dev = E4M3Inputs(inp, seed=80 + bs)
    ref = dev.oracle()
    for kern in KERNELS:
        for P in (0, 64):
            got = to_f64(dev.decode(partition_size=P, fill_out=-3.0, kernel=kern))
            assert_close(got, ref, dtype, f"e4m3 {dtype} D={D} bs={bs} P={P} kernel={kern}")


@pytest.mark.parametrize("W", [1, 17, 600])
def test_decode_e4m3_window_and_order(W):
    cfg = _cfg("bf16", 8, 2, 128, 16, RAGGED)
    inp = make_decode_inputs(cfg, seed=90)
    dev = E4M3Inputs(inp, seed=90)
    ref = dev.oracle(window=W)
    order = torch.from_numpy(pkv.pkv_decode_schedule_order(inp.context_lens)).cuda()
    for kern in KERNELS:
        a = to_f64(dev.decode(partition_size=64, sliding_window=W, kernel=kern))
        assert_close(a, ref, "bf16", f"e4m3 W={W} kernel={kern}")
        b = to_f64(dev.decode(partition_size=64, sliding_window=W, seq_order=order,
                              fill_out=1.0, kernel=kern))
        assert np.array_equal(a, b)


def test_decode_e4m3_zero_length_and_unsupported():
    cfg = _cfg("f16", 2, 2, 128, 16, (0, 5))
    inp = make_decode_inputs(cfg, seed=91)
    dev = E4M3Inputs(inp, seed=91)
    for kern in KERNELS:
        out = to_f64(dev.decode(fill_out=9.0, kernel=kern))
        assert np.all(out[0] == 0.0)
        assert_close(out, dev.oracle(), "f16", f"e4m3 zero length kernel={kern}")
    # head_dim 64 rows are 64 bytes: not built
    cfg64 = _cfg("f16", 2, 2, 64, 16, (5, 5))
    dev64 = E4M3Inputs(make_decode_inputs(cfg64, seed=92), seed=92)
    with pytest.raises(pkv.PagedKVError) as e:
        dev64.decode()
    assert e.value.status == -7


def test_decode_e4m3_full_size_sampled_rows():
    """The Llama-2-13B layer shape with E4M3 pages, in the launch configuration
    the benchmark times (default partition, longest-first order)."""
    inp = make_decode_inputs(CONFIGS["llama2_13b_layer"], seed=2)
    dev = E4M3Inputs(inp, seed=2)
    c = inp.cfg
    rows = sample_rows(c.num_seqs, c.num_q_heads, 96, seed=13)
    lb, sb = int(np.argmax(inp.context_lens)), int(np.argmin(inp.context_lens))
    rows = np.unique(np.concatenate([rows, [[lb, 0], [sb, c.num_q_heads - 1]]]).astype(np.int32),
                     axis=0)
    ref = dev.oracle(rows=rows)
    order = torch.from_numpy(pkv.pkv_decode_schedule_order(inp.context_lens)).cuda()
    vmax = float(np.max(np.abs(dev.v.float().cpu().numpy()))) * float(dev.vs.max())
    for kern in (pkv.PKV_KERNEL_AUTO, pkv.PKV_KERNEL_SIMT):
        out = dev.decode(seq_order=order, kernel=kern)
        got = to_f64(out[torch.from_numpy(rows[:, 0]).long().cuda(),
                         torch.from_numpy(rows[:, 1]).long().cuda()])
        assert_close(got, ref, c.dtype, f"llama2_13b_layer e4m3 kernel={kern}")
        full = to_f64(out)
        assert np.all(np.isfinite(full))
        # convex combinations of the values: never beyond the largest |value|
        assert np.all(np.abs(full) <= vmax * 1.01 + 1e-3)


@pytest.mark.parametrize("G", [1, 8])
def test_decode_e4m3_poisoned_slots_and_extreme_q(G):
    """NaN codes in slots no sequence uses change no bit; q far outside the
    fp16 range (bf16 q of 1e30 and 1e-30 magnitudes) still gives the
    oracle's result on the tensor-core kernel (q enters it rescaled by a
    power of two)."""
    cfg = _cfg("bf16", 2 * G, 2, 128, 16, RAGGED)
    inp = make_decode_inputs(cfg, seed=95)
    dev = E4M3Inputs(inp, seed=95)
    a = dev.decode(partition_size=64).clone()
    live = np.zeros((inp.num_blocks, 16), dtype=bool)
    for bb, L in enumerate(inp.context_lens):
        for j in range((int(L) + 15) // 16):
            live[inp.block_tables[bb, j], :min(16, int(L) - 16 * j)] = True
    kc = dev.pages.k_cache.copy()
    vc = dev.pages.v_cache.copy()
    kc.transpose(0, 2, 1, 3)[~live] = 0x7F
    vc.transpose(0, 2, 1, 3)[~live] = 0xFF
    dev.k.copy_(_codes(kc))
    dev.v.copy_(_codes(vc))
    b = dev.decode(partition_size=64, fill_out=5.0).clone()
    assert torch.equal(a, b)
    dev.k.copy_(_codes(dev.pages.k_cache))
    dev.v.copy_(_codes(dev.pages.v_cache))
    for mag in (1e30, 1e-30):
        from workloads import round_to_dtype
        qx = round_to_dtype(inp.q.view(np.uint16).astype(np.uint32).__lshift__(16)
                            .view(np.float32) * np.float32(mag), "bf16")
        dev.inp = type(inp)(inp.cfg, qx, inp.k_cache, inp.v_cache, inp.block_tables,
                            inp.context_lens, inp.num_blocks)
        dev.q.copy_(to_device(qx, "bf16"))
        ref = dev.oracle()
        for kern in KERNELS:
            got = to_f64(dev.decode(kernel=kern, fill_out=2.0))
            assert_close(got, ref, "bf16", f"e4m3 q x {mag} kernel={kern}")
    dev.inp = inp


# ---------------------------------------------------------------------------
# E4M3 pools through the byte-moving operations

def test_copy_blocks_e4m3_bit_exact():
    N, H, bs, D = 120, 8, 16, 128
    g = np.random.default_rng(17)
    K = g.integers(0, 256, size=(N, H, bs, D), dtype=np.uint8)
    V = g.integers(0, 256, size=(N, H, bs, D), dtype=np.uint8)
    ids = g.permutation(N)
    pairs = np.stack([ids[:40], ids[40:80]], axis=1).astype(np.int32)
    dK, dV = _codes(K), _codes(V)
    pkv.pkv_copy_blocks(dK, dV, torch.from_numpy(pairs).cuda())
    copy_blocks(K, V, pairs.tolist())
    torch.cuda.synchronize()
    assert np.array_equal(dK.view(torch.uint8).cpu().numpy(), K)
    assert np.array_equal(dV.view(torch.uint8).cpu().numpy(), V)


def test_swap_e4m3_round_trip():
    N, M, H, bs, D = 30, 20, 4, 32, 128
    g = np.random.default_rng(18)
    K = g.integers(0, 256, size=(N, H, bs, D), dtype=np.uint8)
    V = g.integers(0, 256, size=(N, H, bs, D), dtype=np.uint8)
    dK, dV = _codes(K), _codes(V)
    hK = torch.zeros((M, H, bs, D), dtype=torch.uint8).pin_memory().view(torch.float8_e4m3fn)
    hV = torch.zeros((M, H, bs, D), dtype=torch.uint8).pin_memory().view(torch.float8_e4m3fn)
    out_pairs = np.stack([np.arange(10), np.arange(10) + 5], axis=1).astype(np.int32)
    pkv.pkv_swap_blocks(hK, hV, dK, dV, torch.from_numpy(out_pairs).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(hK.view(torch.uint8).numpy()[5:15], K[:10])
    back = np.stack([np.arange(10) + 5, np.arange(20, 30)], axis=1).astype(np.int32)
    pkv.pkv_swap_blocks(dK, dV, hK, hV, torch.from_numpy(back).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(dK.view(torch.uint8).cpu().numpy()[20:30], K[:10])
    assert np.array_equal(dV.view(torch.uint8).cpu().numpy()[20:30], V[:10])


# ---------------------------------------------------------------------------
# a scale per page ([num_blocks, Hkv])

@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_append_e4m3_per_page_bit_exact(dtype):
    N, H, bs, D, T = 30, 4, 16, 128, 200
    g = np.random.default_rng(55)
    K = np.zeros((N, H, bs, D), np.uint8)
    V = np.zeros_like(K)
    k = normal_fill((T, H, D), dtype, 31)
    v = normal_fill((T, H, D), dtype, 32)
    ks = np.exp(g.uniform(np.log(1e-3), np.log(0.5), size=(N, H))).astype(np.float32)
    vs = np.exp(g.uniform(np.log(1e-3), np.log(50.0), size=(N, H))).astype(np.float32)
    slots = g.choice(N * bs, size=T, replace=False).astype(np.int64)
    slots[g.random(T) < 0.1] = -1
    dK, dV = _codes(K), _codes(V)
    pkv.pkv_kv_cache_append_e4m3(dK, dV, to_device(k, dtype), to_device(v, dtype),
                                 torch.from_numpy(ks).cuda(), torch.from_numpy(vs).cuda(),
                                 torch.from_numpy(slots).cuda())
    kv_cache_append_e4m3(K, V, k, v, slots, ks, vs, dtype)
    torch.cuda.synchronize()
    assert np.array_equal(dK.view(torch.uint8).cpu().numpy(), K)
    assert np.array_equal(dV.view(torch.uint8).cpu().numpy(), V)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("G", [5, 7, 9, 12])
@pytest.mark.parametrize("per_page", [False, True])
def test_decode_e4m3_partial_head_tiles(dtype, G, per_page):
    """Groups that fill an 8-head tile (5, 7) or a 16-head tile (9, 12) only in
    part: the heads past the group are zero q columns (rows) of the tile and
    are never stored; split and unsplit, per-head and per-page scales."""
    cfg = _cfg(dtype, 2 * G, 2, 128, 16, RAGGED)
    inp = make_decode_inputs(cfg, seed=140 + G)
    dev = E4M3Inputs(inp, seed=140 + G, per_page=per_page)
    ref = dev.oracle()
    for kern in KERNELS:
        for P in (0, 64):
            got = to_f64(dev.decode(partition_size=P, fill_out=5.0, kernel=kern))
            assert_close(got, ref, dtype,
                         f"e4m3 {dtype} G={G} per_page={per_page} P={P} kernel={kern}")


@pytest.mark.parametrize("G", [1, 4, 8])
@pytest.mark.parametrize("partition", [0, 64])
def test_decode_e4m3_per_page_scales(G, partition):
    """Per-page scales from the workload generator (uniform in [1/64, 1/16])."""
    cfg = _cfg("bf16", 2 * G, 2, 128, 16, RAGGED)
    inp = make_decode_inputs(cfg, seed=120 + G)
    dev = E4M3Inputs(inp, seed=120 + G, per_page=True)
    ref = dev.oracle()
    for kern in KERNELS:
        got = to_f64(dev.decode(partition_size=partition, kernel=kern, fill_out=6.0))
        assert_close(got, ref, "bf16", f"per-page G={G} P={partition} kernel={kern}")


@pytest.mark.parametrize("G", [1, 8, 16])
@pytest.mark.parametrize("per_page", [False, True])
def test_decode_e4m3_scales_five_decades(G, per_page):
    """V scales spread over five decades (5e-3 .. 500, one per page or one per
    KV head), so outputs are small weighted means of values up to ~2e5, where
    the absolute part of the tolerance is tiny against the values.  Both
    kernels meet the usual fp16 / bf16 tolerance: the CUDA-core kernel keeps
    every softmax weight in fp32, the tensor-core kernel feeds each weight to
    the fp16 MMA as two terms, hi = fp16(p) and lo = fp16(p - hi), which
    carry ~22 significant bits."""
    cfg = _cfg("bf16", 2 * G, 2, 128, 16, RAGGED)
    inp = make_decode_inputs(cfg, seed=140 + G)
    dev = E4M3Inputs(inp, seed=140 + G, per_page=per_page, v_scale_range=(5e-3, 500.0))
    ref = dev.oracle()
    vd = torch.from_numpy(dev.pages.v_cache).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    vsc = dev.pages.v_scale[:, :, None, None] if per_page else dev.pages.v_scale[None, :, None, None]
    assert float(np.max(np.abs(vd * vsc))) > 1e4  # the spread really reached large values
    for kern in KERNELS:
        for P in (0, 64):
            got = to_f64(dev.decode(partition_size=P, kernel=kern, fill_out=6.0))
            assert_close(got, ref, "bf16",
                         f"wide V scales per_page={per_page} G={G} P={P} kernel={kern}")


@pytest.mark.parametrize("spread", ["log_uniform_1e-20_40", "alternating_1e-20_40"])
@pytest.mark.parametrize("G,D", [(1, 128), (8, 128), (16, 128), (8, 256)])
def test_decode_e4m3_per_page_v_scales_far_apart(spread, G, D):
    """Per-page V scales far apart: log-uniform over 1e-20 .. 40, or pages
    alternating between 1e-20 and 40 by physical block, through the 8-head
    tiles at head_dim 128 and 256 and the 16-head tiles.  The tensor-core
    kernel's per-warp reference V scale moves on most pages, up or down by up
    to ~2^71; outputs (weighted means dominated by the large-scale pages)
    must meet the bf16 tolerance on both kernels.  The largest scale keeps
    values (up to 448 * 40) where float32 sums of them still resolve the
    absolute tolerance after cancellation."""
    cfg = _cfg("bf16", 2 * G, 2, D, 16, RAGGED)
    inp = make_decode_inputs(cfg, seed=150 + G + D)
    dev = E4M3Inputs(inp, seed=150 + G + D, per_page=True)
    n = dev.pages.v_scale.shape[0]
    if spread.startswith("alternating"):
        vs = np.where(np.arange(n) % 2 == 0, 1e-20, 40.0)[:, None]
        vs = np.broadcast_to(vs, dev.pages.v_scale.shape)
    else:
        g = np.random.default_rng(160 + G + D)
        vs = np.exp(g.uniform(np.log(1e-20), np.log(40.0), size=dev.pages.v_scale.shape))
    dev.pages.v_scale = np.ascontiguousarray(vs, dtype=np.float32)
    dev.vs = torch.from_numpy(dev.pages.v_scale).cuda()
    ref = dev.oracle()
    assert np.isfinite(ref).all() and np.abs(ref).max() > 10
    for kern in KERNELS:
        for P in (0, 64):
            got = to_f64(dev.decode(partition_size=P, kernel=kern, fill_out=6.0))
            assert_close(got, ref, "bf16", f"V scales {spread} G={G} P={P} kernel={kern}")


def test_decode_e4m3_per_page_window_and_bs32():
    cfg = _cfg("f16", 8, 2, 128, 32, RAGGED)
    inp = make_decode_inputs(cfg, seed=130)
    dev = E4M3Inputs(inp, seed=130, per_page=True)
    for W in (0, 40):
        ref = dev.oracle(window=W)
        for kern in KERNELS:
            got = to_f64(dev.decode(partition_size=64, sliding_window=W, kernel=kern))
            assert_close(got, ref, "f16", f"per-page bs32 W={W} kernel={kern}")
