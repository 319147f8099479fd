"""Parallel sampling with copy-on-write prefix sharing, end to end on the GPU.

Prompts share a prefix whose last block is partly filled; every sample is a
fork of its prompt.  The native allocator hands out the slots and the block
copies; the GPU runs copy_blocks, kv_cache_append and the decode.  The oracle
side replays the same operations with the allocator model and the oracle's
cache operations, and runs the float64 decode: allocator results and caches
must be bit-identical, attention within tolerance.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_346_b200 as pkv
from oracle import block_manager as bm
from oracle.cache_ops import copy_blocks, kv_cache_append
from tests.gpu_util import assert_close, to_device, to_f64
from workloads import draw_cow_recipe, normal_fill

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.cpu().view(torch.int16).numpy()


def _run(num_prompts, samples, prefix, tail_hi, H=8, D=128, bs=16, steps=3, seed=5):
    rec = draw_cow_recipe(seed=seed, num_prompts=num_prompts, samples=samples, prefix=prefix,
                          tail_hi=tail_hi)
    N = sum(-(-int(L) // bs) for L in rec.shared_lens) + num_prompts * samples * (
        3 + -(-tail_hi // bs))
    nat, mod = pkv.BlockAllocator(N, bs), bm.BlockManagerModel(N, bs)
    B = num_prompts * samples
    for x in (nat, mod):
        for p in range(num_prompts):
            assert x.add_seq(10_000 + p, int(rec.shared_lens[p])) == 0
            for s in range(samples):
                assert x.fork(10_000 + p, p * samples + s) == 0
            assert x.free_seq(10_000 + p) == 0
    K = normal_fill((N, H, bs, D), "f16", seed * 10 + 1)
    V = normal_fill((N, H, bs, D), "f16", seed * 10 + 2)
    dK, dV = to_device(K), to_device(V)
    seqs = np.arange(B)
    maxb = N
    q_all = normal_fill((steps, B, H, D), "f16", seed * 10 + 3)
    knew = normal_fill((steps, B, H, D), "f16", seed * 10 + 4)
    vnew = normal_fill((steps, B, H, D), "f16", seed * 10 + 5)
    total_pairs = 0
    for step in range(steps):
        # host: one new token per sample
        st, slots, pairs, done = nat.append_slots(seqs)
        assert st == 0 and done == B
        want = [mod.append_slot(int(s)) for s in seqs]
        assert slots.tolist() == [w[1] for w in want]
        assert [tuple(p) for p in pairs.tolist()] == [(w[2], w[3]) for w in want if w[2] >= 0]
        total_pairs += len(pairs)
        tables, lens = nat.build_block_tables(seqs, maxb)
        for i, s in enumerate(seqs):
            t = mod.block_table(int(s))
            assert tables[i, :len(t)].tolist() == t and lens[i] == mod.seq_len(int(s))
        # device: copies, append, decode
        if len(pairs):
            pkv.pkv_copy_blocks(dK, dV, to_device(pairs))
        pkv.pkv_kv_cache_append(dK, dV, to_device(knew[step]), to_device(vnew[step]),
                                to_device(slots))
        q = to_device(q_all[step])
        out = torch.empty_like(q)
        L = int(lens.max())
        ws = torch.empty(max(16, pkv.pkv_decode_workspace_size(B, H, H, D, L)),
                         dtype=torch.uint8, device="cuda")
        pkv.pkv_paged_attention_decode(out, q, dK, dV, to_device(tables), to_device(lens),
                                       1.0 / np.sqrt(D), bs, L, workspace=ws)
        # oracle side
        if len(pairs):
            copy_blocks(K, V, pairs.tolist())
        kv_cache_append(K, V, knew[step], vnew[step], slots)
        torch.cuda.synchronize()
        assert np.array_equal(_bits(dK), K.view(np.int16))
        assert np.array_equal(_bits(dV), V.view(np.int16))
        ref = oracle.paged_decode(q_all[step], K, V, tables, lens, scale=1.0 / np.sqrt(D),
                                  dtype="f16")
        assert_close(to_f64(out), ref, "f16", f"step {step}")
    assert pkv.pkv_device_status(clear=True) == 0
    return total_pairs, nat


def test_fork_step_copies_each_shared_partial_block():
    pairs, nat = _run(num_prompts=4, samples=8, prefix=64, tail_hi=40, steps=1)
    # per prompt: every sample but the last holder copies the shared partial block
    assert pairs == 4 * 7


def test_steps_after_the_fork_copy_nothing():
    pairs, nat = _run(num_prompts=3, samples=4, prefix=32, tail_hi=40, steps=4)
    assert pairs == 3 * 3


def test_cow_sampling_shape_sampled():
    # the full 40-head shape with a shorter prefix (the full-size workload runs
    # in the benchmark)
    _run(num_prompts=2, samples=8, prefix=1024, tail_hi=64, H=40, steps=2)
