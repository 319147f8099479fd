"""The C-ABI library loads, exports every function include/*.h declares, and
rejects bad arguments on the host before touching a device."""
import ctypes
import glob
import os
import re

import pytest

from paged_kv_cache_346_b200 import _binding as b

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names |= set(re.findall(r"^PKV_API\s+[\w\s\*]+?\b(pkv_\w+)\s*\(", text, flags=re.M))
    return names


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 20
    for n in sorted(names):
        assert hasattr(b.lib, n), n
    # and the binding declares a signature for each
    assert names == set(b.SIGNATURES), names ^ set(b.SIGNATURES)


def test_header_constants_match_the_binding():
    """Every #define PKV_* number in include/*.h has the binding's value."""
    found = {}
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        for name, val in re.findall(r"^#define\s+(PKV_\w+)\s+\(?(0x[0-9A-Fa-f]+|\d+)u?",
                                    open(h).read(), flags=re.M):
            found[name] = int(val, 0)
    assert {"PKV_DEV_BAD_BLOCK", "PKV_DEV_TIMEOUT", "PKV_DEV_DRAIN_TIMEOUT"} <= set(found)
    for name, val in found.items():
        if name == "PKV_STATIC_WORKSPACE_BYTES":
            continue   # an expression, checked below
        assert getattr(b, name) == val, name
    assert b.PKV_STATIC_WORKSPACE_BYTES == 64 * 1024 * 1024


def test_status_strings_and_version():
    assert b.lib.pkv_status_string(0) == b"ok"
    assert b.lib.pkv_status_string(-2) == b"no free block"
    assert b.lib.pkv_version() >= 10000


def _decode(**over):
    a = dict(out=None, q=None, k=None, v=None, bt=None, cl=None, order=None, B=4, Hq=8, Hkv=2, D=128,
             bs=16, mb=8, N=64, maxlen=100, scale=0.1, win=0, dt=b.PKV_F16, P=0, ws=None, wsb=0,
             kern=0, stream=None)
    a.update(over)
    return b.lib.pkv_paged_attention_decode(
        a["out"], a["q"], a["k"], a["v"], a["bt"], a["cl"], a["order"], a["B"], a["Hq"], a["Hkv"], a["D"],
        a["bs"], a["mb"], a["N"], a["maxlen"], a["scale"], a["win"], a["dt"], a["P"], a["ws"], a["wsb"],
        a["kern"], a["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(Hq=6, Hkv=4), b.PKV_EINVAL),                 # heads do not divide
    (dict(B=-1), b.PKV_EINVAL),
    (dict(maxlen=8 * 16 + 1), b.PKV_EINVAL),            # longer than the table allows
    (dict(P=100), b.PKV_EINVAL),                        # not a multiple of 64
    (dict(P=16384), b.PKV_EINVAL),
    (dict(scale=float("nan")), b.PKV_EINVAL),
    (dict(win=-1), b.PKV_EINVAL),
    (dict(dt=7), b.PKV_EINVAL),
    (dict(kern=9), b.PKV_EINVAL),
    (dict(spb=2, out=ctypes.c_void_p(1 << 20), q=ctypes.c_void_p(1 << 20),
          k=ctypes.c_void_p(1 << 20), v=ctypes.c_void_p(1 << 20), ks=ctypes.c_void_p(1 << 20),
          vs=ctypes.c_void_p(1 << 20), bt=ctypes.c_void_p(1 << 20),
          cl=ctypes.c_void_p(1 << 20)), b.PKV_EINVAL),     # scale mode 0 or 1
    (dict(D=96), b.PKV_EUNSUPPORTED),
    (dict(bs=8, maxlen=50), b.PKV_EUNSUPPORTED),
    (dict(dt=b.PKV_F32, D=256), b.PKV_EUNSUPPORTED),
    (dict(), b.PKV_EINVAL),                             # null pointers
])
def test_decode_host_checks(over, code):
    assert _decode(**over) == code


def test_decode_empty_batch_is_a_no_op():
    assert _decode(B=0) == b.PKV_OK


def test_decode_needs_workspace_for_long_contexts():
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: the check fails first
    assert _decode(out=fake, q=fake, k=fake, v=fake, bt=fake, cl=fake, maxlen=1000,
                   P=512) == b.PKV_EINVAL


def test_workspace_size_formula():
    f = b.lib.pkv_decode_workspace_size
    assert f(8, 32, 8, 128, 512, 512) == 0                    # one partition
    assert f(8, 32, 8, 128, 513, 512) == 8 * 32 * 2 * 130 * 4
    assert f(8, 32, 8, 128, 131072, 512) == 8 * 32 * 256 * 130 * 4
    p = b.lib.pkv_decode_default_partition(8, 8, 131072)
    assert f(8, 32, 8, 128, 131072, 0) == f(8, 32, 8, 128, 131072, p)


def test_default_partition_rule():
    d = b.lib.pkv_decode_default_partition
    assert d(64, 40, 2048) == 4096      # many units: 4096 (one partition here)
    assert d(256, 8, 8192) == 4096
    assert d(8, 8, 131072) == 2048      # few long sequences: 2048
    assert d(1, 1, 4096) == 64          # tiny batches split finer
    p = d(4, 4, 512)
    assert 64 <= p <= 512 and p % 64 == 0
    # a few sequences behind a 4096-token window (span 4096 + 15): one wave of
    # at most 3 CTAs per SM, as long as that allows
    p = d(8, 8, 4111)
    assert p == 704 and 64 * -(-4111 // p) <= 3 * 148 < 64 * -(-4111 // (p - 64))
    assert d(8, 8, 16384) == 1024       # 512 CTAs at 2048: the many-CTA rule


def test_append_and_copy_host_checks():
    f = b.lib.pkv_kv_cache_append
    assert f(None, None, None, None, None, 0, 4, 128, 16, 10, b.PKV_F16, None) == b.PKV_OK
    assert f(None, None, None, None, None, 3, 4, 128, 16, 10, b.PKV_F16, None) == b.PKV_EINVAL
    assert f(None, None, None, None, None, 3, 4, 7, 16, 10, b.PKV_F16, None) == b.PKV_EINVAL
    g = b.lib.pkv_copy_blocks
    assert g(None, None, None, 0, 4, 128, 16, 10, b.PKV_F16, None) == b.PKV_OK
    assert g(None, None, None, 2, 4, 128, 16, 10, b.PKV_F16, None) == b.PKV_EINVAL
    assert g(None, None, None, -1, 4, 128, 16, 10, b.PKV_F16, None) == b.PKV_EINVAL


def _decode_e4m3(**over):
    a = dict(out=None, q=None, k=None, v=None, ks=None, vs=None, spb=0, bt=None, cl=None,
             order=None, B=4, Hq=8, Hkv=2, D=128, bs=16, mb=8, N=64, maxlen=100, scale=0.1, win=0,
             dt=b.PKV_F16, P=0, ws=None, wsb=0, kern=0, stream=None)
    a.update(over)
    return b.lib.pkv_paged_attention_decode_e4m3(
        a["out"], a["q"], a["k"], a["v"], a["ks"], a["vs"], a["spb"], a["bt"], a["cl"], a["order"],
        a["B"],
        a["Hq"], a["Hkv"], a["D"], a["bs"], a["mb"], a["N"], a["maxlen"], a["scale"], a["win"],
        a["dt"], a["P"], a["ws"], a["wsb"], a["kern"], a["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(dt=b.PKV_F32), b.PKV_EINVAL),                 # q / out must be 16-bit
    (dict(dt=b.PKV_E4M3), b.PKV_EINVAL),
    (dict(D=64), b.PKV_EUNSUPPORTED),                   # 64-byte rows
    (dict(kern=9), b.PKV_EINVAL),
    (dict(spb=2, out=ctypes.c_void_p(1 << 20), q=ctypes.c_void_p(1 << 20),
          k=ctypes.c_void_p(1 << 20), v=ctypes.c_void_p(1 << 20), ks=ctypes.c_void_p(1 << 20),
          vs=ctypes.c_void_p(1 << 20), bt=ctypes.c_void_p(1 << 20),
          cl=ctypes.c_void_p(1 << 20)), b.PKV_EINVAL),     # scale mode 0 or 1
    (dict(Hq=6, Hkv=4), b.PKV_EINVAL),
    (dict(), b.PKV_EINVAL),                             # null pointers
    (dict(B=0), b.PKV_OK),
])
def test_decode_e4m3_host_checks(over, code):
    assert _decode_e4m3(**over) == code


def test_decode_e4m3_mma_group_limit():
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: the kernel check fails first
    assert _decode_e4m3(out=fake, q=fake, k=fake, v=fake, ks=fake, vs=fake, bt=fake, cl=fake,
                        Hq=34, Hkv=2, maxlen=50, kern=b.PKV_KERNEL_MMA) == b.PKV_EUNSUPPORTED


def test_e4m3_pages_need_their_own_entry():
    # the 16-bit decode refuses E4M3 pages (they need scales)
    assert _decode(dt=b.PKV_E4M3) == b.PKV_EINVAL
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: the scale check fails first
    assert _decode_e4m3(out=fake, q=fake, k=fake, v=fake, bt=fake, cl=fake) == b.PKV_EINVAL


def test_append_e4m3_host_checks():
    f = b.lib.pkv_kv_cache_append_e4m3
    args = [None] * 6 + [0, None]   # pointers, scale_per_block = 0, slot_mapping
    assert f(*args, 0, 4, 128, 16, 10, b.PKV_F16, None) == b.PKV_OK
    assert f(*args, 3, 4, 128, 16, 10, b.PKV_F16, None) == b.PKV_EINVAL   # null pointers
    assert f(*args, 0, 4, 120, 16, 10, b.PKV_F16, None) == b.PKV_EINVAL   # head_dim % 16
    assert f(*args, 0, 4, 128, 16, 10, b.PKV_F32, None) == b.PKV_EINVAL   # input type
    assert f(*args, 0, 4, 128, 16, 10, b.PKV_E4M3, None) == b.PKV_EINVAL
    # E4M3 pools move as bytes through the plain cache operations
    g = b.lib.pkv_copy_blocks
    assert g(None, None, None, 0, 4, 128, 16, 10, b.PKV_E4M3, None) == b.PKV_OK
    assert g(None, None, None, 0, 1, 8, 1, 10, b.PKV_E4M3, None) == b.PKV_EINVAL  # 8-byte blocks


def test_schedule_order_longest_first():
    import numpy as np
    import paged_kv_cache_346_b200 as pkv
    lens = np.array([5, 100, 7, 100, 0, 64], dtype=np.int32)
    assert pkv.pkv_decode_schedule_order(lens).tolist() == [1, 3, 5, 2, 0, 4]
    assert pkv.pkv_decode_schedule_order(np.zeros(0, np.int32)).tolist() == []


def test_wait_timeout_selftest_host_checks():
    f = b.lib.pkv_debug_wait_timeout
    assert f(0, None) == b.PKV_EINVAL
    assert f(-5, None) == b.PKV_EINVAL
    assert f(5_000_000_000, None) == b.PKV_EINVAL


def test_append_e4m3_scale_mode_checked():
    f = b.lib.pkv_kv_cache_append_e4m3
    assert f(*([None] * 6), 2, None, 0, 4, 128, 16, 10, b.PKV_F16, None) == b.PKV_EINVAL
    assert f(*([None] * 6), 1, None, 0, 4, 128, 16, 10, b.PKV_F16, None) == b.PKV_OK
