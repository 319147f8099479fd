"""The shared-prefix decode against the oracle.

Sequences that hold the same physical blocks at the start of their tables
(parallel samples forked from one prompt, "pagedattention vllm" §Copy-on-Write
Sharing) attend to the same keys and values there; the shared-prefix decode
reads those pages once per group (group pass, tensor cores) and the rest of
each sequence with the regular kernels, then merges.  Its result is the
attention over each sequence's whole context: compared with the float64
oracle over the same tables within the fp16 / bf16 tolerance.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_346_b200 as pkv
from tests.gpu_util import assert_close, to_device, to_f64
from workloads import draw_cow_recipe, normal_fill

pytestmark = pytest.mark.gpu


def _sampling_batch(num_prompts, samples, prefix, tail_hi, Hkv, D, bs, dtype, seed):
    """Prompts of prefix + r tokens forked into samples with private tails
    (the native allocator's tables); pools of N(0, 1) values."""
    rec = draw_cow_recipe(seed=seed, num_prompts=num_prompts, samples=samples, prefix=prefix,
                          tail_hi=tail_hi)
    B = num_prompts * samples
    N = sum(-(-int(L) // bs) for L in rec.shared_lens) + B * (3 + -(-tail_hi // bs))
    al = pkv.BlockAllocator(N, bs)
    for p in range(num_prompts):
        assert al.add_seq(10_000 + p, int(rec.shared_lens[p])) == 0
        for s in range(samples):
            assert al.fork(10_000 + p, p * samples + s) == 0
        assert al.free_seq(10_000 + p) == 0
    for i in range(B):
        for _ in range(int(rec.tail_lens[i])):
            assert al.append_slot(i)[0] == 0
    tables, lens = al.build_block_tables(np.arange(B), N)
    maxb = int(max(-(-int(x) // bs) for x in lens))
    tables = np.ascontiguousarray(tables[:, :maxb])
    K = normal_fill((N, Hkv, bs, D), dtype, seed * 10 + 1)
    V = normal_fill((N, Hkv, bs, D), dtype, seed * 10 + 2)
    return tables, lens.astype(np.int32), K, V


def _decode_groups(q, K, V, tables, lens, spl, members, dtype, bs, P=0, order=None,
                   kernel=pkv.PKV_KERNEL_AUTO):
    B, Hq, D = q.shape
    Hkv = K.shape[1]
    mcl = int(lens.max())
    mpl = int(spl.max()) if spl.size else 0
    dq = to_device(q, dtype)
    out = torch.full_like(dq, 7.0)
    ws = torch.empty(max(16, pkv.pkv_decode_prefix_groups_workspace_size(B, Hq, Hkv, D, mcl,
                                                                         mpl, P)),
                     dtype=torch.uint8, device="cuda")
    gm = torch.from_numpy(members if members.size else np.full((0, 1), -1, np.int32)).cuda()
    pkv.pkv_paged_attention_decode_prefix_groups(
        out, dq, to_device(K, dtype), to_device(V, dtype), to_device(tables), to_device(lens),
        to_device(spl), gm, 1.0 / np.sqrt(D), bs, mcl, mpl, partition_size=P, workspace=ws,
        seq_order=None if order is None else to_device(order), kernel=kernel)
    torch.cuda.synchronize()
    return to_f64(out)


@pytest.mark.parametrize("dtype,Hq,Hkv", [("f16", 8, 8), ("bf16", 8, 8), ("bf16", 16, 2),
                                          ("f16", 32, 4)])
@pytest.mark.parametrize("P", [0, 64, 256])
def test_sampling_groups_match_oracle(dtype, Hq, Hkv, P):
    """8 samples per prompt share a 200 + r token prompt (whole blocks shared,
    the partial one copied on write); MHA puts 8 members x 1 head in one tile,
    GQA 8 members x G heads in tiles of 16 rows.  P 64 splits the prefix over
    several partitions."""
    D, bs = 128, 16
    tables, lens, K, V = _sampling_batch(3, 8, 200, 90, Hkv, D, bs, dtype, seed=11)
    spl, members = pkv.pkv_decode_prefix_groups(tables, lens, bs)
    assert len(members) == 3 and (spl >= 192).all() and (spl % bs == 0).all()
    q = normal_fill((len(lens), Hq, D), dtype, 12)
    got = _decode_groups(q, K, V, tables, lens, spl, members, dtype, bs, P)
    ref = oracle.paged_decode(q, K, V, tables, lens, scale=1.0 / np.sqrt(D), dtype=dtype)
    assert_close(got, ref, dtype, f"prefix groups {dtype} Hq={Hq} Hkv={Hkv} P={P}")
    assert pkv.pkv_device_status(clear=True) == 0


@pytest.mark.parametrize("kernel", [pkv.PKV_KERNEL_SIMT, pkv.PKV_KERNEL_MMA])
def test_groups_with_order_odd_members_and_no_tail(kernel):
    """Groups of 2, 3 and 5 members, one member whose whole context is the
    shared prefix (no token of its own), sequences in no group, a longest
    first schedule, and either kernel for the rest."""
    D, bs, H = 128, 16, 4
    dtype = "bf16"
    g = np.random.default_rng(5)
    N = 200
    perm = g.permutation(N).astype(np.int32)
    nxt = iter(perm.tolist())
    specs = [(2, 7), (3, 4), (5, 10)]   # (members, shared full blocks)
    tables, lens = [], []
    for members, nshared in specs:
        shared = [next(nxt) for _ in range(nshared)]
        for m in range(members):
            tail = 0 if (members == 3 and m == 1) else int(g.integers(1, 60))
            own = [next(nxt) for _ in range(-(-tail // bs))]
            tables.append(shared + own)
            lens.append(nshared * bs + tail)
    for L in (5, 300):                  # in no group
        tables.append([next(nxt) for _ in range(-(-L // bs))])
        lens.append(L)
    maxb = max(len(t) for t in tables)
    bt = np.full((len(tables), maxb), -1, np.int32)
    for i, t in enumerate(tables):
        bt[i, :len(t)] = t
    lens = np.array(lens, np.int32)
    spl, members = pkv.pkv_decode_prefix_groups(bt, lens, bs, max_group_size=8)
    assert len(members) == 3
    assert spl[-1] == 0 and spl[-2] == 0
    K = normal_fill((N, H, bs, D), dtype, 21)
    V = normal_fill((N, H, bs, D), dtype, 22)
    q = normal_fill((len(lens), 4 * H, D), dtype, 23)
    order = pkv.pkv_decode_schedule_order(lens)
    ref = oracle.paged_decode(q, K, V, bt, lens, scale=1.0 / np.sqrt(D), dtype=dtype)
    for P in (0, 64):
        got = _decode_groups(q, K, V, bt, lens, spl, members, dtype, bs, P, order=order,
                             kernel=kernel)
        assert_close(got, ref, dtype, f"odd groups P={P} kernel={kernel}")
    assert pkv.pkv_device_status(clear=True) == 0


def test_no_groups_is_the_regular_decode_bit_for_bit():
    D, bs = 128, 16
    tables, lens, K, V = _sampling_batch(2, 4, 100, 50, 8, D, bs, "f16", seed=3)
    q = normal_fill((len(lens), 8, D), "f16", 4)
    spl = np.zeros(len(lens), np.int32)
    got = _decode_groups(q, K, V, tables, lens, spl, np.zeros((0, 4), np.int32), "f16", bs, 64)
    dq = to_device(q, "f16")
    out = torch.empty_like(dq)
    ws = torch.empty(max(16, pkv.pkv_decode_workspace_size(len(lens), 8, 8, D, int(lens.max()),
                                                           64)), dtype=torch.uint8,
                     device="cuda")
    pkv.pkv_paged_attention_decode(out, dq, to_device(K, "f16"), to_device(V, "f16"),
                                   to_device(tables), to_device(lens), 1.0 / np.sqrt(D), bs,
                                   int(lens.max()), partition_size=64, workspace=ws)
    torch.cuda.synchronize()
    assert np.array_equal(got, to_f64(out))


def test_member_with_other_blocks_is_flagged():
    """A group whose second member holds a different block inside the prefix
    breaks the contract: flagged PKV_DEV_BAD_GROUP."""
    D, bs = 128, 16
    tables, lens, K, V = _sampling_batch(1, 4, 64, 20, 8, D, bs, "f16", seed=9)
    spl, members = pkv.pkv_decode_prefix_groups(tables, lens, bs)
    assert len(members) == 1 and spl[0] == 64
    bad = tables.copy()
    bad[1, 2] = int(tables[:, :].max()) + 1      # another (valid) block of the pool
    q = normal_fill((len(lens), 8, D), "f16", 10)
    pkv.pkv_device_status(clear=True)
    _decode_groups(q, K, V, bad, lens, spl, members, "f16", bs)
    assert pkv.pkv_device_status(clear=True) & pkv.PKV_DEV_BAD_GROUP
