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

import oracle
import paged_kv_cache_346_b200 as pkv
from paged_kv_cache_346_b200 import _binding as b
from tests.gpu_util import DeviceInputs, assert_close, to_f64
from workloads import DecodeConfig, make_decode_inputs


def _static_ws_call(dev: DeviceInputs, out: torch.Tensor, partition_size: int,
                    sliding_window: int = 0) -> int:
    inp, c = dev.inp, dev.inp.cfg
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return b.lib.pkv_paged_attention_decode_static_ws(
        p(out), p(dev.q), p(dev.k), p(dev.v), p(dev.bt), p(dev.cl), None, c.num_seqs,
        c.num_q_heads, c.num_kv_heads, c.head_dim, c.block_size, inp.max_blocks_per_seq,
        inp.num_blocks, inp.max_context_len, c.scale, sliding_window,
        pkv.torch_dtype_code(dev.q.dtype), partition_size, pkv.PKV_KERNEL_AUTO,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,Hq,Hkv,bs", [("bf16", 16, 2, 16), ("f16", 8, 8, 32),
                                             ("f32", 4, 4, 16)])
@pytest.mark.parametrize("window", [0, 700])
def test_static_workspace_matches_caller_workspace(dtype, Hq, Hkv, bs, window):
    """Same kernels, same partitioning: the output equals the caller-workspace
    call's bit for bit, and both are within tolerance of the oracle."""
    lens = (5, 300, 1200, 3000, 1)
    nb = sum((L + bs - 1) // bs for L in lens)
    cfg = DecodeConfig("no_alloc", len(lens), Hq, Hkv, 128 if dtype != "f32" else 64, bs, dtype,
                       ("fixed", lens), pool=("fixed", nb + 5))
    P = 256                                  # several partitions: the scratch is used
    for seed in (31, 32):                    # two calls in a row, different inputs
        inp = make_decode_inputs(cfg, seed=seed)
        dev = DeviceInputs(inp)
        want = dev.decode(partition_size=P, sliding_window=window).clone()
        out = torch.full_like(dev.q, float("nan"))
        assert _static_ws_call(dev, out, P, window) == b.PKV_OK
        torch.cuda.synchronize()
        assert torch.equal(out, want), f"static workspace differs, seed {seed} window {window}"
        ref = oracle.paged_decode_inputs(inp, window=window)
        assert_close(to_f64(out), ref, dtype, f"static workspace vs oracle, seed {seed}")
    assert pkv.pkv_device_status(clear=True) == 0


_FAKE = ctypes.c_void_p(1 << 20)   # aligned, never dereferenced: every check fails first


def _static_ws_host(**over):
    a = dict(B=4096, Hq=64, Hkv=8, D=128, bs=16, mb=8192, N=1 << 20, maxlen=131072, win=0, P=512)
    a.update(over)
    return b.lib.pkv_paged_attention_decode_static_ws(
        _FAKE, _FAKE, _FAKE, _FAKE, _FAKE, _FAKE, None, a["B"], a["Hq"], a["Hkv"], a["D"], a["bs"],
        a["mb"], a["N"], a["maxlen"], 0.1, a["win"], b.PKV_BF16, a["P"], 0, None)


def test_static_workspace_rejects_shapes_beyond_its_size():
    # the size check happens before anything touches a device
    need = pkv.pkv_decode_workspace_size(4096, 64, 8, 128, 131072, 512)
    assert need > b.PKV_STATIC_WORKSPACE_BYTES
    assert _static_ws_host() == b.PKV_EBOUNDS
    # sized on the attended span: a 4096-token window still needs too much here
    need_w = pkv.pkv_decode_workspace_size(4096, 64, 8, 128, 4096 + 15, 512)
    assert need_w > b.PKV_STATIC_WORKSPACE_BYTES
    assert _static_ws_host(win=4096) == b.PKV_EBOUNDS


@pytest.mark.parametrize("over,code", [
    (dict(P=100), b.PKV_EINVAL),        # not a multiple of 64: as the regular entry point
    (dict(D=96), b.PKV_EUNSUPPORTED),
    (dict(Hq=6, Hkv=4), b.PKV_EINVAL),
    (dict(B=0), b.PKV_OK),              # an empty batch, whatever the context bound
])
def test_static_workspace_argument_checks_come_first(over, code):
    """Bad arguments get the regular entry point's status, not PKV_EBOUNDS,
    even where the shape would also be too large for the array."""
    assert _static_ws_host(**over) == code
