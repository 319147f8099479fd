"""Cache write and copy operations as their plain definitions.

TEST INFRASTRUCTURE ONLY (tests and the smoke check).

kv_cache_append: a new token's key and value go into the slot the block
manager handed out for it; blocks are filled as a sequence grows ("What is
PagedAttention ..." §How it works).  A flat slot s names physical block
s // block_size, offset s % block_size; a negative slot is a padding token and
writes nothing.

copy_blocks: before a sequence writes into a block it shares, the block is
copied to a fresh one ("pagedattention vllm" §Copy-on-Write Sharing); a copy
covers the whole block, every KV head, for K and for V.

Both work on numpy arrays in place and move bits only.
"""
from __future__ import annotations

import numpy as np


def kv_cache_append(k_cache: np.ndarray, v_cache: np.ndarray, k: np.ndarray,
                    v: np.ndarray, slot_mapping: np.ndarray) -> None:
    """k_cache/v_cache [N, Hkv, bs, D]; k/v [T, Hkv, D]; slot_mapping int [T]."""
    bs = k_cache.shape[2]
    for t in range(len(slot_mapping)):
        s = int(slot_mapping[t])
        if s < 0:
            continue
        blk, off = divmod(s, bs)
        for h in range(k_cache.shape[1]):
            k_cache[blk, h, off, :] = k[t, h, :]
            v_cache[blk, h, off, :] = v[t, h, :]


def copy_blocks(k_cache: np.ndarray, v_cache: np.ndarray, pairs) -> None:
    """pairs: sequence of (src, dst) physical block ids, applied in order."""
    for src, dst in pairs:
        k_cache[int(dst)] = k_cache[int(src)]
        v_cache[int(dst)] = v_cache[int(src)]
