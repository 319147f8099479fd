"""Failure detection on the GPU without a fault: a bounded wait that runs out.

Every wait in the decode kernels (for a page copy to land) gives up after a
cycle limit, flags PKV_DEV_TIMEOUT and leaves.  pkv_debug_wait_timeout runs
the same bounded wait on a barrier that nothing completes, with a short limit;
the host then reads the flag, and the context keeps working."""
import time

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_346_b200 as pkv
from tests.gpu_util import DeviceInputs, assert_close, to_f64
from workloads import DecodeConfig, make_decode_inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_flags():
    pkv.pkv_device_status(clear=True)
    t0 = time.time()
    pkv.pkv_debug_wait_timeout(2_000_000)      # ~1 ms at B200 clocks
    torch.cuda.synchronize()
    assert time.time() - t0 < 10
    assert pkv.pkv_device_status(clear=True) & pkv.PKV_DEV_TIMEOUT
    assert pkv.pkv_device_status(clear=True) == 0   # cleared


def test_device_usable_after_a_timeout():
    pkv.pkv_debug_wait_timeout(1_000_000)
    torch.cuda.synchronize()
    pkv.pkv_device_status(clear=True)
    cfg = DecodeConfig("after_timeout", 3, 8, 2, 128, 16, "bf16", ("fixed", (5, 300, 70)),
                       pool=("fixed", 40))
    inp = make_decode_inputs(cfg, seed=8)
    got = to_f64(DeviceInputs(inp).decode(partition_size=64))
    assert_close(got, oracle.paged_decode_inputs(inp), "bf16", "after timeout")
    assert pkv.pkv_device_status(clear=True) == 0
