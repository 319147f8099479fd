"""GPU kv_cache_append and copy_blocks against the oracle's definitions:
the whole caches must be bit-identical afterwards."""
import numpy as np
import pytest
import torch

import paged_kv_cache_346_b200 as pkv
from oracle.cache_ops import copy_blocks, kv_cache_append
from tests.gpu_util import to_device
from workloads import normal_fill

pytestmark = pytest.mark.gpu


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.cpu().view(torch.int16 if t.element_size() == 2 else torch.int32).numpy()


def _npbits(a: np.ndarray) -> np.ndarray:
    return a.view(np.int16 if a.itemsize == 2 else np.int32)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("H,D,bs", [(40, 128, 16), (8, 128, 32), (4, 64, 16), (2, 256, 64)])
def test_append_bit_exact(dtype, H, D, bs):
    N, T = 50, 300
    g = np.random.default_rng(H + D + bs)
    K = normal_fill((N, H, bs, D), dtype, 1)
    V = normal_fill((N, H, bs, D), dtype, 2)
    k = normal_fill((T, H, D), dtype, 3)
    v = normal_fill((T, H, D), dtype, 4)
    slots = g.choice(N * bs, size=T, replace=False).astype(np.int64)   # distinct slots
    slots[g.random(T) < 0.1] = -1                                      # padding tokens
    dK, dV = to_device(K, dtype), to_device(V, dtype)
    pkv.pkv_kv_cache_append(dK, dV, to_device(k, dtype), to_device(v, dtype),
                            torch.from_numpy(slots).cuda())
    kv_cache_append(K, V, k, v, slots)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(dK), _npbits(K))
    assert np.array_equal(_bits(dV), _npbits(V))


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
def test_copy_blocks_bit_exact(dtype):
    N, H, bs, D = 300, 40, 16, 128
    g = np.random.default_rng(7)
    K = normal_fill((N, H, bs, D), dtype, 5)
    V = normal_fill((N, H, bs, D), dtype, 6)
    ids = g.permutation(N)
    pairs = np.stack([ids[:100], ids[100:200]], axis=1).astype(np.int32)  # dsts distinct, not srcs
    dK, dV = to_device(K, dtype), to_device(V, dtype)
    pkv.pkv_copy_blocks(dK, dV, torch.from_numpy(pairs).cuda())
    copy_blocks(K, V, pairs.tolist())
    torch.cuda.synchronize()
    assert np.array_equal(_bits(dK), _npbits(K))
    assert np.array_equal(_bits(dV), _npbits(V))


def test_bad_slot_and_pair_are_flagged_and_skipped():
    N, H, bs, D = 8, 2, 16, 64
    K = normal_fill((N, H, bs, D), "f16", 8)
    V = normal_fill((N, H, bs, D), "f16", 9)
    dK, dV = to_device(K, "f16"), to_device(V, "f16")
    k = to_device(normal_fill((2, H, D), "f16", 10), "f16")
    pkv.pkv_device_status(clear=True)
    pkv.pkv_kv_cache_append(dK, dV, k, k, torch.tensor([N * bs, -5], dtype=torch.int64,
                                                        device="cuda"))
    assert pkv.pkv_device_status(clear=True) & pkv.PKV_DEV_BAD_SLOT
    pkv.pkv_copy_blocks(dK, dV, torch.tensor([[0, N], [-1, 2]], dtype=torch.int32, device="cuda"))
    assert pkv.pkv_device_status(clear=True) & pkv.PKV_DEV_BAD_BLOCK
    assert np.array_equal(_bits(dK), _npbits(K)) and np.array_equal(_bits(dV), _npbits(V))
