"""Decode at the limits of the C ABI: the largest partition (8192 tokens) with
sequences several partitions long, many thousands of sequences in one grid,
head_dim 256 with 16-head groups and 64-token blocks, on both kernels and
with E4M3 pages.  Every output element against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_346_b200 as pkv
from tests.gpu_util import DeviceInputs, assert_close, to_f64
from tests.test_e4m3_gpu import E4M3Inputs
from workloads import DecodeConfig, make_decode_inputs

pytestmark = pytest.mark.gpu


def _cfg(dtype, Hq, Hkv, D, bs, lens, pool_extra=5):
    nb = sum((L + bs - 1) // bs for L in lens)
    return DecodeConfig("limits", len(lens), Hq, Hkv, D, bs, dtype, ("fixed", tuple(lens)),
                        pool=("fixed", nb + pool_extra))


def _kernels(dtype, G):
    ks = [pkv.PKV_KERNEL_SIMT]
    if dtype != "f32" and G <= 16:
        ks.append(pkv.PKV_KERNEL_MMA)
    return ks


@pytest.mark.parametrize("dtype,G", [("f16", 1), ("bf16", 8)])
def test_largest_partition_split_k(dtype, G):
    """8192-token partitions; sequences of 1, 8191, 8192, 8193 and 20000
    tokens (up to three partitions merged by the log-sum-exp reduce)."""
    cfg = _cfg(dtype, 2 * G, 2, 128, 16, (1, 8191, 8192, 8193, 20000))
    inp = make_decode_inputs(cfg, seed=101)
    ref = oracle.paged_decode_inputs(inp)
    dev = DeviceInputs(inp)
    for kern in _kernels(dtype, G):
        got = to_f64(dev.decode(partition_size=8192, kernel=kern, fill_out=4.0))
        assert_close(got, ref, dtype, f"P=8192 G={G} kernel={kern}")


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_many_sequences_one_grid(dtype):
    """6000 short sequences (grid.z = 6000), 8 KV heads, groups of 4: outputs
    are means of a few values, where the rounding of the softmax weights
    shows most."""
    g = np.random.default_rng(102)
    lens = tuple(int(x) for x in g.integers(0, 40, size=6000))
    cfg = _cfg(dtype, 32, 8, 128, 16, lens)
    inp = make_decode_inputs(cfg, seed=102)
    ref = oracle.paged_decode_inputs(inp)
    dev = DeviceInputs(inp)
    order = torch.from_numpy(pkv.pkv_decode_schedule_order(inp.context_lens)).cuda()
    for kern in _kernels(dtype, 4):
        got = to_f64(dev.decode(kernel=kern, seq_order=order, fill_out=-2.0))
        assert_close(got, ref, dtype, f"6000 sequences {dtype} kernel={kern}")


@pytest.mark.parametrize("G", [1, 4])
def test_many_short_sequences_e4m3(G):
    """The same stress for E4M3 pages (fp16 weights in the tensor-core kernel)."""
    g = np.random.default_rng(105)
    lens = tuple(int(x) for x in g.integers(0, 40, size=3000))
    cfg = _cfg("f16", 4 * G, 4, 128, 16, lens)
    inp = make_decode_inputs(cfg, seed=105)
    dev = E4M3Inputs(inp, seed=105)
    ref = dev.oracle()
    for kern in (pkv.PKV_KERNEL_SIMT, pkv.PKV_KERNEL_MMA):
        got = to_f64(dev.decode(kernel=kern, fill_out=-2.0))
        assert_close(got, ref, "f16", f"3000 sequences e4m3 G={G} kernel={kern}")


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("bs", [16, 64])
def test_head_dim_256_group_16(dtype, bs):
    """head_dim 256 with 16 query heads per KV head (16-row tensor-core tiles)."""
    cfg = _cfg(dtype, 32, 2, 256, bs, (3, 64, 65, 700, 2100))
    inp = make_decode_inputs(cfg, seed=103)
    ref = oracle.paged_decode_inputs(inp)
    dev = DeviceInputs(inp)
    for kern in _kernels(dtype, 16):
        for P in (0, 64):
            got = to_f64(dev.decode(partition_size=P, kernel=kern, fill_out=1.0))
            assert_close(got, ref, dtype, f"D=256 G=16 bs={bs} P={P} kernel={kern}")


@pytest.mark.parametrize("D,G,bs", [(256, 16, 64), (128, 16, 32), (256, 1, 16)])
def test_e4m3_limits(D, G, bs):
    """E4M3 pages at head_dim 256, 16-head groups and 64-token blocks."""
    cfg = _cfg("bf16", 2 * G, 2, D, bs, (1, 63, 64, 65, 1500, 5000))
    inp = make_decode_inputs(cfg, seed=104)
    dev = E4M3Inputs(inp, seed=104)
    ref = dev.oracle()
    kerns = [pkv.PKV_KERNEL_SIMT, pkv.PKV_KERNEL_MMA] if G <= 16 else [pkv.PKV_KERNEL_SIMT]
    for kern in kerns:
        for P in (0, 512, 8192):
            got = to_f64(dev.decode(partition_size=P, kernel=kern, fill_out=3.0))
            assert_close(got, ref, "bf16", f"e4m3 D={D} G={G} bs={bs} P={P} kernel={kern}")
