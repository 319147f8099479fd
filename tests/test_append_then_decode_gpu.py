"""The decode launched directly behind the KV append on one stream.

The decode starts as a programmatic dependent of the append: it may become
resident while the append runs and reads the schedule order, lengths and
table before waiting for it, but no page.  Here the append writes each
sequence's newest token (the last of its context) after ~40K padding tokens
into unused blocks, so it runs long and the decode's first wave is resident
while the real tokens are still being written; the caches hold other values
in those slots before.  The decode must see the appended tokens: its output
is compared with the oracle's decode over the oracle's appended caches, every
row, under the stated tolerance.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_346_b200 as pkv
from oracle.cache_ops import kv_cache_append, kv_cache_append_e4m3
from tests.gpu_util import assert_close, to_device, to_f64
from workloads import DecodeConfig, make_decode_inputs, make_e4m3_pages, normal_fill

pytestmark = pytest.mark.gpu

PAD_BLOCKS = 2560      # unused blocks the padding tokens go to
PAD_TOKENS = 40000


def _lens(B: int, seed: int) -> np.ndarray:
    # mostly one- or two-slice sequences (their newest token sits in the
    # first pages a CTA reads), a few long ones, one empty sequence
    g = np.random.default_rng(seed)
    lens = g.integers(1, 40, size=B).astype(np.int32)
    lens[::9] = g.integers(300, 1300, size=lens[::9].size)
    lens[5] = 0
    return lens


def _append_inputs(inp, seed: int, dtype: str):
    """Slots and values: padding tokens into blocks no table holds, then the
    newest token of every non-empty sequence (position L - 1)."""
    c = inp.cfg
    bs, Hkv, D = c.block_size, c.num_kv_heads, c.head_dim
    used = set(int(x) for x in inp.block_tables[inp.block_tables >= 0].ravel())
    free = np.array([b for b in range(inp.num_blocks) if b not in used], dtype=np.int64)
    g = np.random.default_rng(seed + 11)
    pad = g.choice(free.size * bs, size=PAD_TOKENS, replace=False)
    pad_slots = free[pad // bs] * bs + pad % bs
    real = []
    for b, L in enumerate(inp.context_lens.tolist()):
        if L > 0:
            real.append(int(inp.block_tables[b, (L - 1) // bs]) * bs + (L - 1) % bs)
    slots = np.concatenate([pad_slots, np.array(real, dtype=np.int64)])
    T = slots.size
    k = normal_fill((T, Hkv, D), dtype, seed * 100 + 7)
    v = normal_fill((T, Hkv, D), dtype, seed * 100 + 8)
    return slots, k, v


def _inputs(Hq, Hkv, dtype, seed):
    B = 64
    lens = _lens(B, seed)
    used = int(sum(-(-int(L) // 16) for L in lens))
    cfg = DecodeConfig("append_then_decode", B, Hq, Hkv, 128, 16, dtype, ("fixed", ()),
                       pool=("fixed", used + PAD_BLOCKS))
    return make_decode_inputs(cfg, seed, lens=lens)


@pytest.mark.parametrize("Hq,Hkv,dtype,kernel", [
    (8, 8, "f16", pkv.PKV_KERNEL_SIMT),
    (32, 8, "bf16", pkv.PKV_KERNEL_MMA),
    (32, 8, "f16", pkv.PKV_KERNEL_SIMT),
])
@pytest.mark.parametrize("window", [0, 24])
def test_decode_sees_the_append_before_it(Hq, Hkv, dtype, kernel, window):
    inp = _inputs(Hq, Hkv, dtype, seed=3)
    c = inp.cfg
    slots, k, v = _append_inputs(inp, 3, dtype)
    dK, dV = to_device(inp.k_cache, dtype), to_device(inp.v_cache, dtype)
    dq, dbt, dcl = to_device(inp.q, dtype), to_device(inp.block_tables), to_device(inp.context_lens)
    dk, dv, ds = to_device(k, dtype), to_device(v, dtype), torch.from_numpy(slots).cuda()
    order = torch.from_numpy(pkv.pkv_decode_schedule_order(inp.context_lens)).cuda()
    mcl = inp.max_context_len
    span = min(mcl, window + c.block_size - 1) if window else mcl
    ws = torch.empty(max(16, pkv.pkv_decode_workspace_size(c.num_seqs, Hq, Hkv, 128, span, 0)),
                     dtype=torch.uint8, device="cuda")
    out = torch.full_like(dq, float("nan"))
    torch.cuda.synchronize()
    # nothing between the two launches
    pkv.pkv_kv_cache_append(dK, dV, dk, dv, ds)
    pkv.pkv_paged_attention_decode(out, dq, dK, dV, dbt, dcl, c.scale, c.block_size, mcl,
                                   workspace=ws, seq_order=order, sliding_window=window,
                                   kernel=kernel)
    torch.cuda.synchronize()
    K, V = inp.k_cache.copy(), inp.v_cache.copy()
    kv_cache_append(K, V, k, v, slots)
    ref = oracle.paged_decode(inp.q, K, V, inp.block_tables, inp.context_lens, scale=c.scale,
                              dtype=dtype, window=window)
    got = to_f64(out)
    assert (got[5] == 0).all()                    # the empty sequence: zero rows
    assert_close(got, ref, dtype, f"G {Hq // Hkv} window {window}")
    assert pkv.pkv_device_status(clear=True) == 0


@pytest.mark.parametrize("window", [0, 24])
def test_e4m3_decode_sees_the_quantising_append_before_it(window):
    inp = _inputs(32, 8, "bf16", seed=4)
    c = inp.cfg
    pages = make_e4m3_pages(inp, 4)
    slots, k, v = _append_inputs(inp, 4, "bf16")

    def codes(a):
        return torch.from_numpy(np.ascontiguousarray(a)).cuda().view(torch.float8_e4m3fn)

    dK, dV = codes(pages.k_cache), codes(pages.v_cache)
    ks, vs = torch.from_numpy(pages.k_scale).cuda(), torch.from_numpy(pages.v_scale).cuda()
    dq, dbt, dcl = to_device(inp.q, "bf16"), to_device(inp.block_tables), to_device(inp.context_lens)
    dk, dv, ds = to_device(k, "bf16"), to_device(v, "bf16"), torch.from_numpy(slots).cuda()
    order = torch.from_numpy(pkv.pkv_decode_schedule_order(inp.context_lens)).cuda()
    mcl = inp.max_context_len
    span = min(mcl, window + c.block_size - 1) if window else mcl
    ws = torch.empty(max(16, pkv.pkv_decode_workspace_size(c.num_seqs, 32, 8, 128, span, 0)),
                     dtype=torch.uint8, device="cuda")
    out = torch.full_like(dq, float("nan"))
    torch.cuda.synchronize()
    pkv.pkv_kv_cache_append_e4m3(dK, dV, dk, dv, ks, vs, ds)
    pkv.pkv_paged_attention_decode_e4m3(out, dq, dK, dV, ks, vs, dbt, dcl, c.scale,
                                        c.block_size, mcl, workspace=ws, seq_order=order,
                                        sliding_window=window)
    torch.cuda.synchronize()
    K, V = pages.k_cache.copy(), pages.v_cache.copy()
    kv_cache_append_e4m3(K, V, k, v, slots, pages.k_scale, pages.v_scale, "bf16")
    ref = oracle.paged_decode(inp.q, K, V, inp.block_tables, inp.context_lens, scale=c.scale,
                              dtype="bf16", kv_dtype="e4m3", k_scale=pages.k_scale,
                              v_scale=pages.v_scale, window=window)
    got = to_f64(out)
    assert (got[5] == 0).all()
    assert_close(got, ref, "bf16", f"E4M3 window {window}")
    assert pkv.pkv_device_status(clear=True) == 0
