"""CPU oracle for paged decode attention and its cache and allocator operations.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg are the only callers.  The library never imports this
package, and this package never imports the library; they share only the
seeded input generators in ``workloads``.

Parts:
  paged_decode      float64 C oracle of softmax(q K^T scale) V read through the
                    block table (paged_decode_oracle.c)
  brute             pure-Python version of the same for tiny cases
  cache_ops         kv_cache_append / copy_blocks as their plain definitions
  block_manager     the block allocator as a Python model (free list, reference
                    counts, fork, copy-on-write)
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

from workloads import DTYPE_CODE, DecodeInputs

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "paged_decode_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (float64, OpenMP).  No CUDA involved."""
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            L.pkvo_decode_f16.restype = ctypes.c_double
            L.pkvo_decode_f16.argtypes = [ctypes.c_uint16]
            L.pkvo_decode_bf16.restype = ctypes.c_double
            L.pkvo_decode_bf16.argtypes = [ctypes.c_uint16]
            L.pkvo_decode_f32.restype = ctypes.c_double
            L.pkvo_decode_f32.argtypes = [ctypes.c_uint32]
            L.pkvo_decode_e4m3.restype = ctypes.c_double
            L.pkvo_decode_e4m3.argtypes = [ctypes.c_uint8]
            L.pkvo_decode_array.restype = None
            L.pkvo_decode_array.argtypes = [ctypes.c_int, ctypes.c_void_p,
                                            ctypes.c_void_p, ctypes.c_int64]
            L.pkvo_paged_decode.restype = ctypes.c_int
            L.pkvo_paged_decode.argtypes = [
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_int64, ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int64,
                ctypes.c_int]
            L.pkvo_max_threads.restype = ctypes.c_int
            _lib = L
    return _lib


def max_threads() -> int:
    return int(lib().pkvo_max_threads())


def decode_bits(arr: np.ndarray, dtype: str) -> np.ndarray:
    """Decode a storage array (float32, float16, or bf16 bits as uint16) to
    float64 with the oracle's own bit decoders."""
    a = np.ascontiguousarray(arr)
    out = np.empty(a.shape, dtype=np.float64)
    lib().pkvo_decode_array(DTYPE_CODE[dtype], a.ctypes.data, out.ctypes.data, a.size)
    return out


def paged_decode(q, k_cache, v_cache, block_tables, context_lens, *, scale: float,
                 dtype: str, num_kv_heads: int | None = None, rows=None,
                 threads: int = 0, window: int = 0, kv_dtype: str | None = None,
                 k_scale=None, v_scale=None) -> np.ndarray:
    """float64 paged decode attention (window > 0: over each sequence's last
    `window` tokens only).  dtype is q's storage type; kv_dtype the caches'
    (default: the same; "e4m3" for FP8 codes, with float32 k_scale / v_scale
    per KV head [Hkv], or per page [N, Hkv]).

    q [B, Hq, D]; k_cache, v_cache [N, Hkv, bs, D] in the storage dtype
    (bf16 as uint16 bits); block_tables int32 [B, max_blocks];
    context_lens int32 [B].  rows: optional int array [R, 2] of (b, h) pairs;
    then the result is [R, D], else [B, Hq, D].
    """
    q = np.ascontiguousarray(q)
    k_cache = np.ascontiguousarray(k_cache)
    v_cache = np.ascontiguousarray(v_cache)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    B, Hq, D = q.shape
    N, Hkv, bs, D2 = k_cache.shape
    assert D2 == D and v_cache.shape == k_cache.shape
    assert num_kv_heads in (None, Hkv)
    if rows is not None:
        r = np.ascontiguousarray(rows, dtype=np.int32).reshape(-1, 2)
        out = np.empty((r.shape[0], D), dtype=np.float64)
        rp, nr = r.ctypes.data, r.shape[0]
    else:
        out = np.empty((B, Hq, D), dtype=np.float64)
        rp, nr = None, 0
    kvd = DTYPE_CODE[kv_dtype or dtype]
    ks = None if k_scale is None else np.ascontiguousarray(k_scale, dtype=np.float32)
    vs = None if v_scale is None else np.ascontiguousarray(v_scale, dtype=np.float32)
    per_block = 0
    for sc in (ks, vs):
        if sc is not None:
            if sc.shape == (N, Hkv):
                per_block = 1
            elif sc.shape != (Hkv,):
                raise ValueError("scales must be [Hkv] or [num_blocks, Hkv]")
    if ks is not None and vs is not None and ks.shape != vs.shape:
        raise ValueError("k_scale and v_scale must have the same shape")
    rc = lib().pkvo_paged_decode(out.ctypes.data, q.ctypes.data, k_cache.ctypes.data,
                                 v_cache.ctypes.data, bt.ctypes.data, cl.ctypes.data,
                                 B, Hq, Hkv, D, bs, bt.shape[1], N, float(scale),
                                 int(window), DTYPE_CODE[dtype], kvd,
                                 None if ks is None else ks.ctypes.data,
                                 None if vs is None else vs.ctypes.data, per_block, rp, nr,
                                 int(threads))
    if rc != 0:
        raise ValueError(f"oracle rejected the inputs (code {rc})")
    return out


def paged_decode_inputs(inp: DecodeInputs, rows=None, threads: int = 0,
                        window: int = 0) -> np.ndarray:
    c = inp.cfg
    return paged_decode(inp.q, inp.k_cache, inp.v_cache, inp.block_tables,
                        inp.context_lens, scale=c.scale, dtype=c.dtype, rows=rows,
                        threads=threads, window=window)
