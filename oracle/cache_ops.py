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


# ---------------------------------------------------------------------------
# quantised pages: FP8 E4M3 codes with one float32 scale per KV head
# ("pagedattention vllm" §Comparison with Alternatives: paging combines with
# quantisation).  The code of a value x is E4M3(x / scale): the division is
# a float32 division (the precision the kernel decides in), the rounding is
# to nearest, ties to even, and values beyond the largest finite code (448)
# saturate to it; NaN stays NaN.

E4M3_MAX = 448.0


def e4m3_encode(y32: np.ndarray) -> np.ndarray:
    """float32 values -> E4M3 codes (uint8), round to nearest even, saturating."""
    y = np.asarray(y32, dtype=np.float32).astype(np.float64)
    sign = np.signbit(y).astype(np.uint8)
    a = np.abs(y)
    code = np.zeros(a.shape, dtype=np.int64)
    nan = np.isnan(a)
    big = ~nan & (a >= E4M3_MAX)
    sub = ~nan & ~big & (a < 2.0 ** -6)
    nrm = ~nan & ~big & ~sub
    # subnormals: multiples of 2^-9
    code[sub] = np.rint(a[sub] * 2.0 ** 9).astype(np.int64)   # rint: ties to even
    # normals: 2^e * (1 + m/8)
    e = np.floor(np.log2(np.where(nrm, a, 1.0))).astype(np.int64)
    # guard log2 rounding at exact powers of two
    e = np.where(nrm & (2.0 ** e > a), e - 1, e)
    e = np.where(nrm & (2.0 ** (e + 1) <= a), e + 1, e)
    m = np.rint((np.where(nrm, a, 1.0) / 2.0 ** e - 1.0) * 8.0).astype(np.int64)
    carry = m == 8
    e = np.where(carry, e + 1, e)
    m = np.where(carry, 0, m)
    code = np.where(nrm, ((e + 7) << 3) | m, code)
    code = np.where(big, 0x7E, code)
    code = np.where(nan, 0x7F, code)
    return (code.astype(np.uint8) | (sign << 7)).astype(np.uint8)


def to_f32(x: np.ndarray, dtype: str) -> np.ndarray:
    """Storage values (bf16 as uint16 bits) -> float32, exactly."""
    if dtype == "bf16":
        return (np.asarray(x, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)
    return np.asarray(x).astype(np.float32)


def kv_cache_append_e4m3(k_cache: np.ndarray, v_cache: np.ndarray, k: np.ndarray, v: np.ndarray,
                         slot_mapping: np.ndarray, k_scale: np.ndarray, v_scale: np.ndarray,
                         in_dtype: str) -> None:
    """Append with quantisation: k_cache/v_cache uint8 codes [N, Hkv, bs, D];
    k/v [T, Hkv, D] in in_dtype; scales float32 [Hkv] (per KV head) or
    [N, Hkv] (per page: the scale of the block the slot lies in)."""
    ks = np.asarray(k_scale, dtype=np.float32)
    vs = np.asarray(v_scale, dtype=np.float32)
    bs = k_cache.shape[2]
    slots = np.asarray(slot_mapping, dtype=np.int64)
    if ks.ndim == 1:
        ksel = np.broadcast_to(ks, (len(slots), ks.size))
        vsel = np.broadcast_to(vs, (len(slots), vs.size))
    else:  # per page; padding slots (< 0) are never written, any row will do
        blk = np.where(slots >= 0, slots // bs, 0)
        ksel, vsel = ks[blk], vs[blk]
    kq = e4m3_encode(to_f32(k, in_dtype) / ksel[:, :, None])
    vq = e4m3_encode(to_f32(v, in_dtype) / vsel[:, :, None])
    kv_cache_append(k_cache, v_cache, kq, vq, slots)
