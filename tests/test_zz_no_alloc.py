"""The decode entry point that allocates nothing.

pkv_paged_attention_decode_static_ws serves callers that cannot allocate
device memory (a plugin whose host application owns all device memory, a
serving loop that must not take cudaMalloc's device synchronisation): it takes
the partition scratch from a fixed array inside the library instead of a
caller workspace.  These tests call it through the C ABI and compare it with
the regular entry point on the same inputs, for two calls in a row (the array
keeps the previous call's contents, which must not matter).

This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import paged_kv_cache_346_b200 as pkv
from paged_kv_cache_346_b200 import _binding as b
from tests.gpu_util import DeviceInputs, assert_close, to_f64
from workloads import DecodeConfig, make_decode_inputs


def _static_ws_call(dev: DeviceInputs, out: torch.Tensor, partition_size: int) -> int:
    inp, c = dev.inp, dev.inp.cfg
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return b.lib.pkv_paged_attention_decode_static_ws(
        p(out), p(dev.q), p(dev.k), p(dev.v), p(dev.bt), p(dev.cl), None, c.num_seqs,
        c.num_q_heads, c.num_kv_heads, c.head_dim, c.block_size, inp.max_blocks_per_seq,
        inp.num_blocks, inp.max_context_len, c.scale, 0, pkv.torch_dtype_code(dev.q.dtype),
        partition_size, pkv.PKV_KERNEL_AUTO,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,Hq,Hkv,bs", [("bf16", 16, 2, 16), ("f16", 8, 8, 32),
                                             ("f32", 4, 4, 16)])
def test_static_workspace_matches_caller_workspace(dtype, Hq, Hkv, bs):
    lens = (5, 300, 1200, 3000, 1)
    nb = sum((L + bs - 1) // bs for L in lens)
    cfg = DecodeConfig("no_alloc", len(lens), Hq, Hkv, 128 if dtype != "f32" else 64, bs, dtype,
                       ("fixed", lens), pool=("fixed", nb + 5))
    P = 256                                  # several partitions: the scratch is used
    for seed in (31, 32):                    # two calls in a row, different inputs
        dev = DeviceInputs(make_decode_inputs(cfg, seed=seed))
        want = to_f64(dev.decode(partition_size=P))
        out = torch.full_like(dev.q, float("nan"))
        assert _static_ws_call(dev, out, P) == b.PKV_OK
        torch.cuda.synchronize()
        assert_close(to_f64(out), want, dtype, f"static workspace, seed {seed}")


def test_static_workspace_rejects_shapes_beyond_its_size():
    # the size check happens before anything touches a device
    need = pkv.pkv_decode_workspace_size(4096, 64, 8, 128, 131072, 512)
    assert need > b.PKV_STATIC_WORKSPACE_BYTES
    rc = b.lib.pkv_paged_attention_decode_static_ws(
        None, None, None, None, None, None, None, 4096, 64, 8, 128, 16, 8192, 1 << 20, 131072,
        0.1, 0, b.PKV_BF16, 512, 0, None)
    assert rc == b.PKV_EBOUNDS
