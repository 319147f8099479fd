"""ctypes binding of libpagedkv.so (include/pagedkv.h).

Argument marshalling only: torch tensors are passed as their device pointers
and shapes, the current CUDA stream as a handle; every step of the computation
runs in the library's kernels.  There is no fallback: if the library is not
built, importing this module fails.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libpagedkv.so")

PKV_OK, PKV_EINVAL, PKV_ENOMEM, PKV_ENOSEQ, PKV_EEXIST, PKV_EBOUNDS, PKV_ECUDA, \
    PKV_EUNSUPPORTED = 0, -1, -2, -3, -4, -5, -6, -7
PKV_F32, PKV_F16, PKV_BF16, PKV_E4M3 = 0, 1, 2, 3
PKV_KERNEL_AUTO, PKV_KERNEL_SIMT, PKV_KERNEL_MMA = 0, 1, 2
PKV_DEV_BAD_BLOCK, PKV_DEV_BAD_LEN, PKV_DEV_BAD_SLOT, PKV_DEV_TIMEOUT, PKV_DEV_BAD_ORDER, \
    PKV_DEV_DRAIN_TIMEOUT, PKV_DEV_BAD_GROUP = 1, 2, 4, 8, 16, 32, 64
PKV_STATIC_WORKSPACE_BYTES = 64 * 1024 * 1024
PKV_MAX_PREFIX_GROUP = 64

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python paged_kv_cache_346_b200/build.py`")

_c = ctypes
_vp, _i32, _i64, _sz, _f32 = _c.c_void_p, _c.c_int, _c.c_int64, _c.c_size_t, _c.c_float

lib = _c.CDLL(LIB_PATH)

# name -> (restype, argtypes); one line per declaration in pagedkv.h
SIGNATURES = {
    "pkv_status_string": (_c.c_char_p, [_i32]),
    "pkv_version": (_i32, []),
    "pkv_decode_has_kernel": (_i32, [_i32]),
    "pkv_decode_default_partition": (_i32, [_i32, _i32, _i32]),
    "pkv_decode_workspace_size": (_sz, [_i32, _i32, _i32, _i32, _i32, _i32]),
    "pkv_paged_attention_decode": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32,
                                          _i32, _i32, _i32, _i32, _i32, _f32, _i32, _i32, _i32,
                                          _vp, _sz, _i32, _vp]),
    "pkv_paged_attention_decode_static_ws": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32,
                                                    _i32, _i32, _i32, _i32, _i32, _i32, _i32,
                                                    _f32, _i32, _i32, _i32, _i32, _vp]),
    "pkv_paged_attention_decode_e4m3": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp,
                                               _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32,
                                               _i32, _f32, _i32, _i32, _i32, _vp, _sz, _i32,
                                               _vp]),
    "pkv_decode_schedule_order": (_i32, [_vp, _i32, _vp]),
    "pkv_decode_schedule_items": (_i32, [_vp, _i32, _i32, _i32, _i32, _vp, _i32, _vp]),
    "pkv_paged_attention_decode_items": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32,
                                                _i32, _i32, _i32, _i32, _i32, _i32, _i32, _f32,
                                                _i32, _i32, _i32, _vp, _sz, _i32, _vp]),
    "pkv_paged_attention_decode_e4m3_items": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp,
                                                     _vp, _vp, _i32, _i32, _i32, _i32, _i32,
                                                     _i32, _i32, _i32, _i32, _f32, _i32, _i32,
                                                     _i32, _vp, _sz, _i32, _vp]),
    "pkv_paged_attention_decode_prefix_groups": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                                        _vp, _i32, _i32, _i32, _i32, _i32, _i32,
                                                        _i32, _i32, _i32, _i32, _i32, _f32, _i32,
                                                        _i32, _vp, _sz, _i32, _vp]),
    "pkv_decode_prefix_groups_workspace_size": (_sz, [_i32, _i32, _i32, _i32, _i32, _i32, _i32]),
    "pkv_decode_prefix_groups": (_i32, [_vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _i32,
                                        _vp]),
    "pkv_kv_cache_append": (_i32, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32,
                                   _vp]),
    "pkv_kv_cache_append_e4m3": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32,
                                        _i32, _i32, _i32, _i32, _vp]),
    "pkv_copy_blocks": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp]),
    "pkv_swap_blocks": (_i32, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32,
                               _i32, _vp]),
    "pkv_device_status": (_i32, [_c.POINTER(_c.c_uint), _i32]),
    "pkv_debug_wait_timeout": (_i32, [_c.c_longlong, _vp]),
    "pkv_alloc_create": (_i32, [_i32, _i32, _c.POINTER(_vp)]),
    "pkv_alloc_create_swap": (_i32, [_i32, _i32, _i32, _c.POINTER(_vp)]),
    "pkv_alloc_swap_out": (_i32, [_vp, _i64, _vp, _i32, _c.POINTER(_i32)]),
    "pkv_alloc_swap_in": (_i32, [_vp, _i64, _vp, _i32, _c.POINTER(_i32)]),
    "pkv_alloc_is_swapped": (_i32, [_vp, _i64, _c.POINTER(_i32)]),
    "pkv_alloc_slide_window": (_i32, [_vp, _i64, _i32, _c.POINTER(_i32)]),
    "pkv_alloc_add_seq_prefix": (_i32, [_vp, _i64, _vp, _i32, _c.POINTER(_i32)]),
    "pkv_alloc_cache_stats": (_i32, [_vp, _c.POINTER(_c.c_int32), _c.POINTER(_c.c_int32)]),
    "pkv_alloc_evictable_list": (_i32, [_vp, _vp, _i32, _c.POINTER(_i32)]),
    "pkv_alloc_destroy": (None, [_vp]),
    "pkv_alloc_add_seq": (_i32, [_vp, _i64, _i32]),
    "pkv_alloc_fork": (_i32, [_vp, _i64, _i64]),
    "pkv_alloc_append_slot": (_i32, [_vp, _i64, _c.POINTER(_i64), _c.POINTER(_c.c_int32),
                                     _c.POINTER(_c.c_int32)]),
    "pkv_alloc_append_slots": (_i32, [_vp, _vp, _i32, _vp, _vp, _c.POINTER(_i32),
                                      _c.POINTER(_i32)]),
    "pkv_alloc_free_seq": (_i32, [_vp, _i64]),
    "pkv_alloc_seq_len": (_i32, [_vp, _i64, _c.POINTER(_i32)]),
    "pkv_alloc_block_table": (_i32, [_vp, _i64, _vp, _i32, _c.POINTER(_i32)]),
    "pkv_alloc_build_block_tables": (_i32, [_vp, _vp, _i32, _vp, _i32, _c.c_int32, _vp]),
    "pkv_alloc_refcount": (_i32, [_vp, _c.c_int32, _c.POINTER(_i32)]),
    "pkv_alloc_stats": (_i32, [_vp, _vp]),
    "pkv_alloc_free_list": (_i32, [_vp, _vp, _i32, _c.POINTER(_i32)]),
}

for _name, (_res, _args) in SIGNATURES.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class PagedKVError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = lib.pkv_status_string(status).decode()
        super().__init__(f"{what}: {msg} ({status})" if what else f"{msg} ({status})")


def check(status: int, what: str = "") -> int:
    if status != PKV_OK:
        raise PagedKVError(status, what)
    return status


class AllocStats(_c.Structure):
    _fields_ = [("num_blocks", _c.c_int32), ("block_size", _c.c_int32),
                ("free_blocks", _c.c_int32), ("used_blocks", _c.c_int32),
                ("shared_blocks", _c.c_int32), ("num_seqs", _c.c_int32),
                ("refcount_sum", _c.c_int64), ("logical_tokens", _c.c_int64),
                ("num_host_blocks", _c.c_int32), ("free_host_blocks", _c.c_int32),
                ("swapped_seqs", _c.c_int32), ("reserved", _c.c_int32)]

    def as_dict(self) -> dict:
        return {f: getattr(self, f) for f, _ in self._fields_}
