"""Swapping pages between the device pool and a page-locked host pool: the
native allocator decides the moves, pkv_swap_blocks moves the bytes; the
pools must match the oracle's copies bit for bit and a decode after swap-in
must match the oracle on the original data."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_346_b200 as pkv
from oracle.cache_ops import copy_blocks
from paged_kv_cache_346_b200 import _binding as b
from tests.gpu_util import assert_close, to_device, to_f64
from workloads import normal_fill

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.cpu().view(torch.int16).numpy()


def _move(dst, src, pairs):
    """Oracle of a page move between two pools."""
    for s, d in pairs:
        dst[d] = src[s]


def test_swap_out_and_in_round_trip():
    H, bs, D, N, NH = 8, 16, 128, 80, 48
    K = normal_fill((N, H, bs, D), "f16", 1)
    V = normal_fill((N, H, bs, D), "f16", 2)
    dK, dV = to_device(K), to_device(V)
    hK = torch.zeros((NH, H, bs, D), dtype=torch.float16).pin_memory()
    hV = torch.zeros((NH, H, bs, D), dtype=torch.float16).pin_memory()
    HK, HV = np.zeros((NH, H, bs, D), np.float16), np.zeros((NH, H, bs, D), np.float16)
    alloc = pkv.BlockAllocator(N, bs, num_host_blocks=NH)
    lens = [300, 77, 500]
    for i, L in enumerate(lens):
        assert alloc.add_seq(i, L) == 0
    # swap out sequence 1 and 2
    moved = []
    for sid in (1, 2):
        st, pairs = alloc.swap_out(sid)
        assert st == 0
        pkv.pkv_swap_blocks(hK, hV, dK, dV, torch.tensor(pairs, dtype=torch.int32).cuda())
        _move(HK, K, pairs)
        _move(HV, V, pairs)
        moved += pairs
    torch.cuda.synchronize()
    assert np.array_equal(hK.view(torch.int16).numpy(), HK.view(np.int16))
    assert np.array_equal(hV.view(torch.int16).numpy(), HV.view(np.int16))
    # another sequence reuses the freed device blocks and overwrites them
    assert alloc.add_seq(7, 16 * 20) == 0
    reused = alloc.block_table(7)
    junk = torch.full((len(reused), H, bs, D), 9.0, dtype=torch.float16, device="cuda")
    dK[torch.tensor(reused).cuda()] = junk
    K[reused] = np.float16(9.0)
    # swap sequence 2 back in (to fresh blocks) and decode it with sequence 0
    st, pairs = alloc.swap_in(2)
    assert st == 0
    pkv.pkv_swap_blocks(dK, dV, hK, hV, torch.tensor(pairs, dtype=torch.int32).cuda())
    _move(K, HK, pairs)
    _move(V, HV, pairs)
    tables, cl = alloc.build_block_tables([0, 2], max_blocks=40)
    q = normal_fill((2, H, D), "f16", 3)
    out = torch.empty((2, H, D), dtype=torch.float16, device="cuda")
    ws = torch.empty(pkv.pkv_decode_workspace_size(2, H, H, D, 500) + 16, dtype=torch.uint8,
                     device="cuda")
    pkv.pkv_paged_attention_decode(out, to_device(q), dK, dV, to_device(tables), to_device(cl),
                                   1 / np.sqrt(D), bs, 500, workspace=ws)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(dK), K.view(np.int16))
    assert np.array_equal(_bits(dV), V.view(np.int16))
    ref = oracle.paged_decode(q, K, V, tables, cl, scale=1 / np.sqrt(D), dtype="f16")
    assert_close(to_f64(out), ref, "f16", "after swap-in")
    assert pkv.pkv_device_status(clear=True) == 0


def test_swap_refuses_pageable_host_memory():
    H, bs, D = 2, 16, 64
    dK = torch.zeros((4, H, bs, D), dtype=torch.float16, device="cuda")
    pageable = np.zeros((4, H, bs, D), np.float16)          # not page-locked
    pairs = torch.tensor([[0, 1]], dtype=torch.int32, device="cuda")
    p = ctypes.c_void_p(pageable.ctypes.data)
    d = ctypes.c_void_p(dK.data_ptr())
    rc = b.lib.pkv_swap_blocks(p, p, d, d, ctypes.c_void_p(pairs.data_ptr()), 1, 4, 4, H, D, bs,
                               b.PKV_F16, None)
    assert rc == b.PKV_EINVAL


def test_swap_flags_out_of_range_pairs():
    H, bs, D = 2, 16, 64
    dK = torch.zeros((4, H, bs, D), dtype=torch.float16, device="cuda")
    hK = torch.zeros((2, H, bs, D), dtype=torch.float16).pin_memory()
    pkv.pkv_device_status(clear=True)
    pkv.pkv_swap_blocks(hK, hK, dK, dK, torch.tensor([[0, 5]], dtype=torch.int32, device="cuda"))
    assert pkv.pkv_device_status(clear=True) & pkv.PKV_DEV_BAD_BLOCK
