"""pagedkv: PagedAttention decode for NVIDIA B200 (sm_100a).

Python face of the C library (include/pagedkv.h).  The functions carry the C
names and take torch tensors; they pass pointers, sizes and the current CUDA
stream through and raise PagedKVError on a non-zero status.  All computation
happens in libpagedkv.so.

    pkv_paged_attention_decode   paged decode attention (+ log-sum-exp reduce)
    pkv_kv_cache_append          new tokens' K/V -> their slots
    pkv_paged_attention_decode_e4m3 / pkv_kv_cache_append_e4m3
                                 the same over FP8 E4M3 pages with per-head scales
    pkv_copy_blocks              copy-on-write block copies
    BlockAllocator               host block manager (free list, refcounts, CoW)
"""
from __future__ import annotations

import ctypes

import torch

from . import _binding as _b
from ._binding import (PKV_BF16, PKV_E4M3, PKV_DEV_BAD_BLOCK, PKV_DEV_BAD_LEN, PKV_DEV_BAD_ORDER,
                       PKV_DEV_BAD_GROUP, PKV_DEV_BAD_SLOT, PKV_DEV_DRAIN_TIMEOUT, PKV_DEV_TIMEOUT,
                       PKV_F16, PKV_F32,
                       PKV_KERNEL_AUTO, PKV_KERNEL_MMA, PKV_KERNEL_SIMT, PagedKVError, check, lib)

__all__ = [
    "pkv_paged_attention_decode", "pkv_decode_workspace_size", "pkv_decode_has_kernel",
    "pkv_paged_attention_decode_static_ws", "pkv_swap_blocks", "pkv_decode_default_partition",
    "pkv_kv_cache_append", "pkv_copy_blocks", "pkv_device_status", "BlockAllocator",
    "PagedKVError", "lib", "PKV_F32", "PKV_F16", "PKV_BF16", "PKV_KERNEL_AUTO",
    "PKV_KERNEL_SIMT", "PKV_KERNEL_MMA", "PKV_DEV_BAD_BLOCK", "PKV_DEV_BAD_LEN",
    "PKV_DEV_BAD_SLOT", "PKV_DEV_TIMEOUT", "PKV_DEV_BAD_ORDER", "PKV_DEV_DRAIN_TIMEOUT",
    "torch_dtype_code",
    "pkv_decode_schedule_order", "pkv_decode_schedule_items", "pkv_paged_attention_decode_e4m3",
    "pkv_kv_cache_append_e4m3",
    "pkv_paged_attention_decode_prefix_groups", "pkv_decode_prefix_groups",
    "pkv_decode_prefix_groups_workspace_size", "PKV_DEV_BAD_GROUP",
    "PKV_E4M3", "pkv_debug_wait_timeout",
]

_DTYPE = {torch.float32: PKV_F32, torch.float16: PKV_F16, torch.bfloat16: PKV_BF16,
          torch.float8_e4m3fn: PKV_E4M3}


def torch_dtype_code(dt: torch.dtype) -> int:
    try:
        return _DTYPE[dt]
    except KeyError:
        raise PagedKVError(_b.PKV_EINVAL, f"dtype {dt}") from None


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dev(t: torch.Tensor, name: str) -> torch.Tensor:
    if not t.is_cuda:
        raise PagedKVError(_b.PKV_EINVAL, f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise PagedKVError(_b.PKV_EINVAL, f"{name} must be contiguous")
    return t


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def pkv_decode_has_kernel(kernel: int) -> bool:
    return bool(lib.pkv_decode_has_kernel(int(kernel)))


def pkv_decode_default_partition(num_seqs: int, num_kv_heads: int, max_context_len: int) -> int:
    return int(lib.pkv_decode_default_partition(num_seqs, num_kv_heads, max_context_len))


def pkv_decode_workspace_size(num_seqs: int, num_q_heads: int, num_kv_heads: int,
                              head_dim: int, max_context_len: int,
                              partition_size: int = 0) -> int:
    return int(lib.pkv_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                             max_context_len, partition_size))


def _check_order(seq_order, items, num_seqs: int, partition_size: int) -> None:
    if seq_order is not None and items is not None:
        raise PagedKVError(_b.PKV_EINVAL, "give seq_order or items, not both")
    if seq_order is not None:
        _dev(seq_order, "seq_order")
        if seq_order.dtype != torch.int32 or seq_order.numel() != num_seqs:
            raise PagedKVError(_b.PKV_EINVAL, "seq_order must be int32 [num_seqs]")
    if items is not None:
        _dev(items, "items")
        if items.dtype != torch.int32 or items.dim() != 2 or items.shape[1] != 2 or \
                not items.is_contiguous():
            raise PagedKVError(_b.PKV_EINVAL, "items must be a contiguous int32 [n, 2] tensor")
        if partition_size <= 0:
            raise PagedKVError(_b.PKV_EINVAL, "a work list needs its partition_size")


def pkv_paged_attention_decode(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
                               v_cache: torch.Tensor, block_tables: torch.Tensor,
                               context_lens: torch.Tensor, scale: float, block_size: int,
                               max_context_len: int, *, partition_size: int = 0,
                               workspace: torch.Tensor | None = None,
                               seq_order: torch.Tensor | None = None,
                               items: torch.Tensor | None = None,
                               sliding_window: int = 0,
                               kernel: int = PKV_KERNEL_AUTO, stream=None) -> torch.Tensor:
    """out [B, Hq, D] <- paged decode attention (see pkv_paged_attention_decode
    in pagedkv.h).  k_cache/v_cache [N, Hkv, block_size, D]; block_tables
    int32 [B, max_blocks]; context_lens int32 [B]; max_context_len is a host
    bound of context_lens.  workspace: a CUDA tensor of at least
    pkv_decode_workspace_size(...) bytes when sequences span partitions.
    seq_order: optional int32 [B] schedule order (pkv_decode_schedule_order);
    or items: an int32 [n, 2] work list (pkv_decode_schedule_items, cut with
    this partition_size, which must then be given) for
    pkv_paged_attention_decode_items.
    sliding_window: 0, or attend only to each sequence's last W tokens."""
    for t, n in ((out, "out"), (q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache"),
                 (block_tables, "block_tables"), (context_lens, "context_lens")):
        _dev(t, n)
    _check_order(seq_order, items, q.shape[0], partition_size)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise PagedKVError(_b.PKV_EINVAL, "block_tables / context_lens must be int32")
    if not (q.dtype == out.dtype == k_cache.dtype == v_cache.dtype):
        raise PagedKVError(_b.PKV_EINVAL, "q, out, k_cache, v_cache must share a dtype")
    B, Hq, D = q.shape
    N, Hkv, bs, D2 = k_cache.shape
    if (D2 != D or bs != block_size or tuple(out.shape) != (B, Hq, D) or
            tuple(v_cache.shape) != tuple(k_cache.shape) or block_tables.shape[0] != B or
            context_lens.shape[0] != B):
        raise PagedKVError(_b.PKV_EINVAL, "shape mismatch")
    ws_bytes = 0
    if workspace is not None:
        _dev(workspace, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    if items is not None:
        check(lib.pkv_paged_attention_decode_items(
            _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
            _ptr(context_lens), _ptr(items), items.shape[0], B, Hq, Hkv, D, bs,
            block_tables.shape[1], N, int(max_context_len), float(scale), int(sliding_window),
            torch_dtype_code(q.dtype), int(partition_size), _ptr(workspace), ws_bytes,
            int(kernel), _stream(stream)),
            "pkv_paged_attention_decode_items")
        return out
    check(lib.pkv_paged_attention_decode(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        _ptr(context_lens), _ptr(seq_order), B, Hq, Hkv, D, bs, block_tables.shape[1], N,
        int(max_context_len), float(scale), int(sliding_window), torch_dtype_code(q.dtype),
        int(partition_size), _ptr(workspace), ws_bytes, int(kernel), _stream(stream)),
        "pkv_paged_attention_decode")
    return out


def pkv_paged_attention_decode_e4m3(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
                                    v_cache: torch.Tensor, k_scale: torch.Tensor,
                                    v_scale: torch.Tensor, block_tables: torch.Tensor,
                                    context_lens: torch.Tensor, scale: float, block_size: int,
                                    max_context_len: int, *, partition_size: int = 0,
                                    workspace: torch.Tensor | None = None,
                                    seq_order: torch.Tensor | None = None,
                                    items: torch.Tensor | None = None,
                                    sliding_window: int = 0, kernel: int = PKV_KERNEL_AUTO,
                                    stream=None) -> torch.Tensor:
    """Paged decode over FP8 E4M3 pages (pkv_paged_attention_decode_e4m3 in
    pagedkv.h): k_cache/v_cache torch.float8_e4m3fn [N, Hkv, block_size, D];
    k_scale/v_scale float32 [Hkv], or [N, Hkv] for a scale per page; q and
    out fp16 or bf16.  items: a work list as for pkv_paged_attention_decode
    (pkv_paged_attention_decode_e4m3_items)."""
    for t, n in ((out, "out"), (q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache"),
                 (k_scale, "k_scale"), (v_scale, "v_scale"), (block_tables, "block_tables"),
                 (context_lens, "context_lens")):
        _dev(t, n)
    _check_order(seq_order, items, q.shape[0], partition_size)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise PagedKVError(_b.PKV_EINVAL, "block_tables / context_lens must be int32")
    if k_cache.dtype != torch.float8_e4m3fn or v_cache.dtype != torch.float8_e4m3fn:
        raise PagedKVError(_b.PKV_EINVAL, "k_cache / v_cache must be float8_e4m3fn")
    if q.dtype != out.dtype or k_scale.dtype != torch.float32 or v_scale.dtype != torch.float32:
        raise PagedKVError(_b.PKV_EINVAL, "q/out dtypes differ or scales are not float32")
    B, Hq, D = q.shape
    N, Hkv, bs, D2 = k_cache.shape
    if (D2 != D or bs != block_size or tuple(out.shape) != (B, Hq, D) or
            tuple(v_cache.shape) != tuple(k_cache.shape) or block_tables.shape[0] != B or
            context_lens.shape[0] != B or tuple(k_scale.shape) != tuple(v_scale.shape) or
            tuple(k_scale.shape) not in ((Hkv,), (N, Hkv))):
        raise PagedKVError(_b.PKV_EINVAL, "shape mismatch")
    per_block = 1 if k_scale.dim() == 2 else 0
    ws_bytes = 0
    if workspace is not None:
        _dev(workspace, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    if items is not None:
        check(lib.pkv_paged_attention_decode_e4m3_items(
            _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale),
            per_block, _ptr(block_tables), _ptr(context_lens), _ptr(items), items.shape[0], B,
            Hq, Hkv, D, bs, block_tables.shape[1], N, int(max_context_len), float(scale),
            int(sliding_window), torch_dtype_code(q.dtype), int(partition_size),
            _ptr(workspace), ws_bytes, int(kernel), _stream(stream)),
            "pkv_paged_attention_decode_e4m3_items")
        return out
    check(lib.pkv_paged_attention_decode_e4m3(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale),
        per_block, _ptr(block_tables), _ptr(context_lens), _ptr(seq_order), B, Hq, Hkv, D, bs,
        block_tables.shape[1], N, int(max_context_len), float(scale), int(sliding_window),
        torch_dtype_code(q.dtype), int(partition_size), _ptr(workspace), ws_bytes, int(kernel),
        _stream(stream)),
        "pkv_paged_attention_decode_e4m3")
    return out


def pkv_paged_attention_decode_static_ws(out: torch.Tensor, q: torch.Tensor,
                                         k_cache: torch.Tensor, v_cache: torch.Tensor,
                                         block_tables: torch.Tensor, context_lens: torch.Tensor,
                                         scale: float, block_size: int, max_context_len: int, *,
                                         partition_size: int = 0,
                                         seq_order: torch.Tensor | None = None,
                                         sliding_window: int = 0,
                                         kernel: int = PKV_KERNEL_AUTO,
                                         stream=None) -> torch.Tensor:
    """pkv_paged_attention_decode without a caller workspace, for callers that
    cannot allocate device memory: the partition scratch is a fixed
    PKV_STATIC_WORKSPACE_BYTES array inside the library (shared by all calls
    on a device; calls that overlap on the GPU race on it).  Shapes needing
    more scratch than that raise PagedKVError (PKV_EBOUNDS)."""
    for t, n in ((out, "out"), (q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache"),
                 (block_tables, "block_tables"), (context_lens, "context_lens")):
        _dev(t, n)
    B, Hq, D = q.shape
    N, Hkv, bs, _ = k_cache.shape
    check(lib.pkv_paged_attention_decode_static_ws(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        _ptr(context_lens), _ptr(seq_order), B, Hq, Hkv, D, bs, block_tables.shape[1], N,
        int(max_context_len), float(scale), int(sliding_window), torch_dtype_code(q.dtype),
        int(partition_size), int(kernel), _stream(stream)),
        f"pkv_paged_attention_decode_static_ws (scratch limit "
        f"{_b.PKV_STATIC_WORKSPACE_BYTES} bytes)")
    return out


def pkv_decode_prefix_groups(block_tables, context_lens, block_size: int,
                             max_group_size: int = 16, min_prefix_blocks: int = 1):
    """Host arrays: the shared-prefix groups of a batch (pkv_decode_prefix_groups
    in pagedkv.h).  -> (seq_prefix_len int32 [B], group_members int32
    [num_groups, largest group], -1 padded).  The member rows are cut to the
    largest group found, so the group pass's tile holds no empty rows beyond
    it (8 samples of an MHA model fill an 8-row tile)."""
    import numpy as np
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    B = lens.size
    if bt.ndim != 2 or bt.shape[0] != B:
        raise PagedKVError(_b.PKV_EINVAL, "block_tables must be [num_seqs, max_blocks]")
    spl = np.zeros(B, dtype=np.int32)
    cap = max(B // 2, 1)
    members = np.full((cap, max_group_size), -1, dtype=np.int32)
    ng = ctypes.c_int(0)
    check(lib.pkv_decode_prefix_groups(bt.ctypes.data if B else None,
                                       lens.ctypes.data if B else None, B, bt.shape[1],
                                       block_size, max_group_size, min_prefix_blocks,
                                       spl.ctypes.data, members.ctypes.data, cap,
                                       ctypes.byref(ng)), "pkv_decode_prefix_groups")
    members = members[:ng.value]
    width = int((members >= 0).sum(axis=1).max()) if ng.value else 1
    return spl, np.ascontiguousarray(members[:, :width])


def pkv_decode_prefix_groups_workspace_size(num_seqs: int, num_q_heads: int, num_kv_heads: int,
                                            head_dim: int, max_context_len: int,
                                            max_prefix_len: int, partition_size: int = 0) -> int:
    return int(lib.pkv_decode_prefix_groups_workspace_size(
        num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len, max_prefix_len,
        partition_size))


def pkv_paged_attention_decode_prefix_groups(
        out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
        block_tables: torch.Tensor, context_lens: torch.Tensor, seq_prefix_len: torch.Tensor,
        group_members: torch.Tensor, scale: float, block_size: int, max_context_len: int,
        max_prefix_len: int, *, partition_size: int = 0,
        workspace: torch.Tensor | None = None, seq_order: torch.Tensor | None = None,
        kernel: int = PKV_KERNEL_AUTO, stream=None) -> torch.Tensor:
    """out [B, Hq, D] <- paged decode attention with shared prefixes read once
    per group (pkv_paged_attention_decode_prefix_groups in pagedkv.h).
    seq_prefix_len int32 [B] and group_members int32 [num_groups, max_group_size]
    on the device (pkv_decode_prefix_groups builds them on the host);
    workspace: pkv_decode_prefix_groups_workspace_size(...) bytes."""
    for t, n in ((out, "out"), (q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache"),
                 (block_tables, "block_tables"), (context_lens, "context_lens"),
                 (seq_prefix_len, "seq_prefix_len"), (group_members, "group_members")):
        _dev(t, n)
    if seq_order is not None:
        _dev(seq_order, "seq_order")
    if (block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32 or
            seq_prefix_len.dtype != torch.int32 or group_members.dtype != torch.int32):
        raise PagedKVError(_b.PKV_EINVAL, "tables, lengths and groups must be int32")
    if not (q.dtype == out.dtype == k_cache.dtype == v_cache.dtype):
        raise PagedKVError(_b.PKV_EINVAL, "q, out, k_cache, v_cache must share a dtype")
    B, Hq, D = q.shape
    N, Hkv, bs, D2 = k_cache.shape
    if (D2 != D or bs != block_size or tuple(out.shape) != (B, Hq, D) or
            tuple(v_cache.shape) != tuple(k_cache.shape) or block_tables.shape[0] != B or
            context_lens.shape[0] != B or seq_prefix_len.shape[0] != B or
            group_members.dim() != 2):
        raise PagedKVError(_b.PKV_EINVAL, "shape mismatch")
    ng, mgs = group_members.shape
    ws_bytes = 0
    if workspace is not None:
        _dev(workspace, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    check(lib.pkv_paged_attention_decode_prefix_groups(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        _ptr(context_lens), _ptr(seq_order), _ptr(seq_prefix_len),
        _ptr(group_members) if ng else None, ng, max(mgs, 1), B, Hq, Hkv, D, bs,
        block_tables.shape[1], N, int(max_context_len), int(max_prefix_len), float(scale),
        torch_dtype_code(q.dtype), int(partition_size), _ptr(workspace), ws_bytes, int(kernel),
        _stream(stream)), "pkv_paged_attention_decode_prefix_groups")
    return out


def pkv_decode_schedule_items(context_lens, block_size: int, partition_size: int,
                              sliding_window: int = 0):
    """Host int32 array [n, 2] of (sequence, partition) pairs, longest
    partition first, for the decode's items argument (pkv_decode_schedule_items
    in pagedkv.h)."""
    import numpy as np
    lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    n = _b._c.c_int(0)
    cap = int(np.maximum(lens, 0).sum() // max(1, int(partition_size))) + 2 * lens.size + 1
    while True:
        items = np.empty((cap, 2), dtype=np.int32)
        rc = lib.pkv_decode_schedule_items(lens.ctypes.data, lens.size, int(block_size),
                                           int(partition_size), int(sliding_window),
                                           items.ctypes.data, cap, _b._c.byref(n))
        if rc != _b.PKV_EBOUNDS or n.value <= cap:
            break
        cap = n.value
    check(rc, "pkv_decode_schedule_items")
    return items[:n.value].copy()


def pkv_decode_schedule_order(context_lens):
    """Host int32 array [B]: sequence indices by decreasing length (ties by
    index), for the decode's seq_order argument."""
    import numpy as np
    lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    order = np.empty(lens.size, dtype=np.int32)
    check(lib.pkv_decode_schedule_order(lens.ctypes.data, lens.size, order.ctypes.data),
          "pkv_decode_schedule_order")
    return order


def pkv_kv_cache_append(k_cache: torch.Tensor, v_cache: torch.Tensor, k: torch.Tensor,
                        v: torch.Tensor, slot_mapping: torch.Tensor, *, stream=None) -> None:
    """k/v [T, Hkv, D] -> cache slots slot_mapping (int64 [T], < 0 = skip)."""
    for t, n in ((k_cache, "k_cache"), (v_cache, "v_cache"), (k, "k"), (v, "v"),
                 (slot_mapping, "slot_mapping")):
        _dev(t, n)
    if slot_mapping.dtype != torch.int64:
        raise PagedKVError(_b.PKV_EINVAL, "slot_mapping must be int64")
    if not (k.dtype == v.dtype == k_cache.dtype == v_cache.dtype):
        raise PagedKVError(_b.PKV_EINVAL, "dtype mismatch")
    N, Hkv, bs, D = k_cache.shape
    T = k.shape[0]
    if (tuple(k.shape) != (T, Hkv, D) or tuple(v.shape) != (T, Hkv, D) or
            slot_mapping.shape[0] != T or tuple(v_cache.shape) != tuple(k_cache.shape)):
        raise PagedKVError(_b.PKV_EINVAL, "shape mismatch")
    check(lib.pkv_kv_cache_append(_ptr(k_cache), _ptr(v_cache), _ptr(k), _ptr(v),
                                  _ptr(slot_mapping), T, Hkv, D, bs, N,
                                  torch_dtype_code(k.dtype), _stream(stream)),
          "pkv_kv_cache_append")


def pkv_kv_cache_append_e4m3(k_cache: torch.Tensor, v_cache: torch.Tensor, k: torch.Tensor,
                             v: torch.Tensor, k_scale: torch.Tensor, v_scale: torch.Tensor,
                             slot_mapping: torch.Tensor, *, stream=None) -> None:
    """fp16/bf16 k/v [T, Hkv, D] -> E4M3 codes of k / k_scale[h] (and v) in
    the float8_e4m3fn caches' slots; k_scale/v_scale [Hkv], or [N, Hkv] for
    the scale of the page each slot lies in."""
    for t, n in ((k_cache, "k_cache"), (v_cache, "v_cache"), (k, "k"), (v, "v"),
                 (k_scale, "k_scale"), (v_scale, "v_scale"), (slot_mapping, "slot_mapping")):
        _dev(t, n)
    if slot_mapping.dtype != torch.int64:
        raise PagedKVError(_b.PKV_EINVAL, "slot_mapping must be int64")
    if k_cache.dtype != torch.float8_e4m3fn or v_cache.dtype != torch.float8_e4m3fn or \
            k.dtype != v.dtype or k_scale.dtype != torch.float32 or \
            v_scale.dtype != torch.float32:
        raise PagedKVError(_b.PKV_EINVAL, "dtype mismatch")
    N, Hkv, bs, D = k_cache.shape
    T = k.shape[0]
    if (tuple(k.shape) != (T, Hkv, D) or tuple(v.shape) != (T, Hkv, D) or
            slot_mapping.shape[0] != T or tuple(v_cache.shape) != tuple(k_cache.shape) or
            tuple(k_scale.shape) != tuple(v_scale.shape) or
            tuple(k_scale.shape) not in ((Hkv,), (N, Hkv))):
        raise PagedKVError(_b.PKV_EINVAL, "shape mismatch")
    check(lib.pkv_kv_cache_append_e4m3(_ptr(k_cache), _ptr(v_cache), _ptr(k), _ptr(v),
                                       _ptr(k_scale), _ptr(v_scale),
                                       1 if k_scale.dim() == 2 else 0, _ptr(slot_mapping), T,
                                       Hkv, D, bs, N, torch_dtype_code(k.dtype), _stream(stream)),
          "pkv_kv_cache_append_e4m3")


def pkv_copy_blocks(k_cache: torch.Tensor, v_cache: torch.Tensor, block_pairs: torch.Tensor,
                    *, stream=None) -> None:
    """block_pairs int32 [n, 2] of (src, dst): whole-block copies of K and V."""
    for t, n in ((k_cache, "k_cache"), (v_cache, "v_cache"), (block_pairs, "block_pairs")):
        _dev(t, n)
    if block_pairs.dtype != torch.int32 or (block_pairs.numel() and block_pairs.shape[-1] != 2):
        raise PagedKVError(_b.PKV_EINVAL, "block_pairs must be int32 [n, 2]")
    N, Hkv, bs, D = k_cache.shape
    check(lib.pkv_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(block_pairs),
                              block_pairs.numel() // 2, Hkv, D, bs, N,
                              torch_dtype_code(k_cache.dtype), _stream(stream)),
          "pkv_copy_blocks")


def pkv_swap_blocks(dst_k: torch.Tensor, dst_v: torch.Tensor, src_k: torch.Tensor,
                    src_v: torch.Tensor, block_pairs: torch.Tensor, *, stream=None) -> None:
    """Whole-block copies (src block of the src pools -> dst block of the dst
    pools); either side may be a page-locked host tensor (pin_memory)."""
    for t, n in ((dst_k, "dst_k"), (dst_v, "dst_v"), (src_k, "src_k"), (src_v, "src_v"),
                 (block_pairs, "block_pairs")):
        if not t.is_contiguous():
            raise PagedKVError(_b.PKV_EINVAL, f"{n} must be contiguous")
        if not t.is_cuda and not t.is_pinned():
            raise PagedKVError(_b.PKV_EINVAL, f"{n} must be on the GPU or page-locked")
    if block_pairs.dtype != torch.int32 or (block_pairs.numel() and block_pairs.shape[-1] != 2):
        raise PagedKVError(_b.PKV_EINVAL, "block_pairs must be int32 [n, 2]")
    if not (dst_k.dtype == dst_v.dtype == src_k.dtype == src_v.dtype):
        raise PagedKVError(_b.PKV_EINVAL, "dtype mismatch")
    Ns, Hkv, bs, D = src_k.shape
    Nd = dst_k.shape[0]
    if tuple(dst_k.shape[1:]) != (Hkv, bs, D):
        raise PagedKVError(_b.PKV_EINVAL, "shape mismatch")
    check(lib.pkv_swap_blocks(_ptr(dst_k), _ptr(dst_v), _ptr(src_k), _ptr(src_v),
                              _ptr(block_pairs), block_pairs.numel() // 2, Ns, Nd, Hkv, D, bs,
                              torch_dtype_code(src_k.dtype), _stream(stream)),
          "pkv_swap_blocks")


def pkv_debug_wait_timeout(limit_cycles: int, *, stream=None) -> None:
    """Run the bounded-wait self-test: one kernel gives up waiting after
    limit_cycles clock cycles and flags PKV_DEV_TIMEOUT."""
    check(lib.pkv_debug_wait_timeout(int(limit_cycles), _stream(stream)),
          "pkv_debug_wait_timeout")


def pkv_device_status(clear: bool = False) -> int:
    """OR of PKV_DEV_* bits set on the current device (synchronises)."""
    flags = ctypes.c_uint(0)
    check(lib.pkv_device_status(ctypes.byref(flags), int(bool(clear))), "pkv_device_status")
    return int(flags.value)


class BlockAllocator:
    """Host block manager (pkv_alloc_*): free list, reference counts, fork and
    copy-on-write.  Not thread-safe."""

    def __init__(self, num_blocks: int, block_size: int, num_host_blocks: int = 0):
        h = ctypes.c_void_p()
        check(lib.pkv_alloc_create_swap(num_blocks, num_host_blocks, block_size,
                                        ctypes.byref(h)), "pkv_alloc_create_swap")
        self._h = h
        self._destroy = lib.pkv_alloc_destroy   # kept: module globals may be gone at exit
        self.num_blocks = num_blocks
        self.num_host_blocks = num_host_blocks
        self.block_size = block_size

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            self._destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    # operations: return the status code (callers compare against the model)
    def add_seq(self, seq_id: int, num_tokens: int) -> int:
        return lib.pkv_alloc_add_seq(self._h, seq_id, num_tokens)

    def fork(self, parent: int, child: int) -> int:
        return lib.pkv_alloc_fork(self._h, parent, child)

    def append_slot(self, seq_id: int):
        """-> (status, slot, cow_src, cow_dst)"""
        slot = ctypes.c_int64(-1)
        src = ctypes.c_int32(-1)
        dst = ctypes.c_int32(-1)
        st = lib.pkv_alloc_append_slot(self._h, seq_id, ctypes.byref(slot), ctypes.byref(src),
                                       ctypes.byref(dst))
        if st != 0:
            return st, -1, -1, -1
        return st, slot.value, src.value, dst.value

    def append_slots(self, seq_ids):
        """-> (status, slots int64 [n], cow_pairs int32 [n_cow, 2], num_done)"""
        import numpy as np
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = ids.size
        slots = np.full(n, -1, dtype=np.int64)
        pairs = np.full((max(n, 1), 2), -1, dtype=np.int32)
        ncow = ctypes.c_int(0)
        done = ctypes.c_int(0)
        st = lib.pkv_alloc_append_slots(self._h, ids.ctypes.data, n, slots.ctypes.data,
                                        pairs.ctypes.data, ctypes.byref(ncow),
                                        ctypes.byref(done))
        return st, slots, pairs[:ncow.value].copy(), done.value

    def free_seq(self, seq_id: int) -> int:
        return lib.pkv_alloc_free_seq(self._h, seq_id)

    def _swap(self, fn, seq_id: int):
        # size the pair buffer from the table length (a query that changes nothing)
        n = ctypes.c_int(0)
        st = lib.pkv_alloc_block_table(self._h, seq_id, None, 0, ctypes.byref(n))
        if st not in (0, _b.PKV_EBOUNDS):
            return st, []
        buf = (ctypes.c_int32 * max(2 * n.value, 2))()
        st = fn(self._h, seq_id, buf, n.value, ctypes.byref(n))
        if st != 0:
            return st, []
        return st, [(buf[2 * i], buf[2 * i + 1]) for i in range(n.value)]

    def swap_out(self, seq_id: int):
        """-> (status, [(device block, host block), ...])"""
        return self._swap(lib.pkv_alloc_swap_out, seq_id)

    def swap_in(self, seq_id: int):
        """-> (status, [(host block, device block), ...])"""
        return self._swap(lib.pkv_alloc_swap_in, seq_id)

    def slide_window(self, seq_id: int, window: int):
        """-> (status, entries released)"""
        n = ctypes.c_int(0)
        st = lib.pkv_alloc_slide_window(self._h, seq_id, window, ctypes.byref(n))
        return st, (n.value if st == 0 else 0)

    def add_seq_prefix(self, seq_id: int, tokens):
        """New sequence for a prompt of token ids, reusing cached full blocks of
        an identical prefix.  -> (status, prompt tokens found in the cache)"""
        import numpy as np
        tk = np.ascontiguousarray(tokens, dtype=np.int32)
        n = ctypes.c_int(0)
        st = lib.pkv_alloc_add_seq_prefix(self._h, seq_id, tk.ctypes.data if tk.size else None,
                                          tk.size, ctypes.byref(n))
        return st, (n.value if st == 0 else 0)

    def cache_stats(self) -> tuple[int, int]:
        """(registered prefix blocks, evictable blocks)"""
        c, e = ctypes.c_int32(0), ctypes.c_int32(0)
        check(lib.pkv_alloc_cache_stats(self._h, ctypes.byref(c), ctypes.byref(e)),
              "pkv_alloc_cache_stats")
        return c.value, e.value

    def evictable_list(self) -> list[int]:
        n = ctypes.c_int(0)
        buf = (ctypes.c_int32 * max(self.num_blocks, 1))()
        check(lib.pkv_alloc_evictable_list(self._h, buf, self.num_blocks, ctypes.byref(n)),
              "pkv_alloc_evictable_list")
        return list(buf[:n.value])

    def is_swapped(self, seq_id: int) -> bool:
        v = ctypes.c_int(0)
        check(lib.pkv_alloc_is_swapped(self._h, seq_id, ctypes.byref(v)), "pkv_alloc_is_swapped")
        return bool(v.value)

    def apply(self, op):
        kind = op[0]
        if kind == "swap_out":
            return self.swap_out(op[1])
        if kind == "swap_in":
            return self.swap_in(op[1])
        if kind == "slide":
            return self.slide_window(op[1], op[2])
        if kind == "add":
            return self.add_seq(op[1], op[2])
        if kind == "fork":
            return self.fork(op[1], op[2])
        if kind == "append":
            return self.append_slot(op[1])
        if kind == "free":
            return self.free_seq(op[1])
        if kind == "prefix":
            return self.add_seq_prefix(op[1], op[2])
        raise ValueError(kind)

    # queries
    def seq_len(self, seq_id: int) -> int:
        n = ctypes.c_int(0)
        check(lib.pkv_alloc_seq_len(self._h, seq_id, ctypes.byref(n)), "pkv_alloc_seq_len")
        return n.value

    def block_table(self, seq_id: int) -> list[int]:
        n = ctypes.c_int(0)
        st = lib.pkv_alloc_block_table(self._h, seq_id, None, 0, ctypes.byref(n))
        if st not in (0, _b.PKV_EBOUNDS):
            check(st, "pkv_alloc_block_table")
        buf = (ctypes.c_int32 * max(n.value, 1))()
        check(lib.pkv_alloc_block_table(self._h, seq_id, buf, n.value, ctypes.byref(n)),
              "pkv_alloc_block_table")
        return list(buf[:n.value])

    def build_block_tables(self, seq_ids, max_blocks: int, fill: int = -1):
        """-> (tables int32 [n, max_blocks], context_lens int32 [n]) numpy arrays"""
        import numpy as np
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        tables = np.empty((ids.size, max_blocks), dtype=np.int32)
        lens = np.empty(ids.size, dtype=np.int32)
        check(lib.pkv_alloc_build_block_tables(self._h, ids.ctypes.data, ids.size,
                                               tables.ctypes.data, max_blocks, fill,
                                               lens.ctypes.data),
              "pkv_alloc_build_block_tables")
        return tables, lens

    def refcount(self, block: int) -> int:
        n = ctypes.c_int(0)
        check(lib.pkv_alloc_refcount(self._h, block, ctypes.byref(n)), "pkv_alloc_refcount")
        return n.value

    def stats(self) -> dict:
        s = _b.AllocStats()
        check(lib.pkv_alloc_stats(self._h, ctypes.byref(s)), "pkv_alloc_stats")
        return s.as_dict()

    def free_list(self) -> list[int]:
        n = ctypes.c_int(0)
        buf = (ctypes.c_int32 * max(self.num_blocks, 1))()
        check(lib.pkv_alloc_free_list(self._h, buf, self.num_blocks, ctypes.byref(n)),
              "pkv_alloc_free_list")
        return list(buf[:n.value])
