"""Helpers for the GPU parity tests: move seeded inputs to the device, run the
library's decode, compare with the oracle under the stated tolerances."""
import numpy as np
import torch

import paged_kv_cache_346_b200 as pkv

TORCH_DTYPE = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def to_device(a: np.ndarray, dtype: str | None = None) -> torch.Tensor:
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy()


class DeviceInputs:
    def __init__(self, inp):
        c = inp.cfg
        self.inp = inp
        self.q = to_device(inp.q, c.dtype)
        self.k = to_device(inp.k_cache, c.dtype)
        self.v = to_device(inp.v_cache, c.dtype)
        self.bt = to_device(inp.block_tables)
        self.cl = to_device(inp.context_lens)
        self.out = torch.empty_like(self.q)

    def decode(self, partition_size=0, kernel=pkv.PKV_KERNEL_AUTO, max_context_len=None,
               fill_out=None, seq_order=None, sliding_window=0):
        c = self.inp.cfg
        mcl = self.inp.max_context_len if max_context_len is None else max_context_len
        span = min(mcl, sliding_window + c.block_size - 1) if sliding_window > 0 else mcl
        ws_bytes = pkv.pkv_decode_workspace_size(c.num_seqs, c.num_q_heads, c.num_kv_heads,
                                                 c.head_dim, span, partition_size)
        ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
        if fill_out is not None:
            self.out.fill_(fill_out)
        pkv.pkv_paged_attention_decode(self.out, self.q, self.k, self.v, self.bt, self.cl,
                                       c.scale, c.block_size, mcl,
                                       partition_size=partition_size, workspace=ws,
                                       seq_order=seq_order, sliding_window=sliding_window,
                                       kernel=kernel)
        torch.cuda.synchronize()
        return self.out


def tolerance(dtype: str, ref: np.ndarray) -> np.ndarray:
    # fp32: |d| <= 1e-5; fp16 / bf16 caches with fp32 accumulation:
    # |d| <= 2e-3 + 1e-2 |ref|
    if dtype == "f32":
        return np.full(ref.shape, 1e-5)
    return 2e-3 + 1e-2 * np.abs(ref)


def assert_close(got: np.ndarray, ref: np.ndarray, dtype: str, what: str = ""):
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    tol = tolerance(dtype, ref)
    bad = err > tol
    if bad.any():
        i = np.unravel_index(np.argmax(err - tol), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside tolerance; worst at "
                             f"{i}: got {got[i]!r} ref {ref[i]!r} err {err[i]:.3g} tol {tol[i]:.3g}")
    return float(err.max())


def sample_rows(B: int, Hq: int, n: int, seed: int) -> np.ndarray:
    g = np.random.default_rng(seed)
    b = g.integers(0, B, size=n)
    h = g.integers(0, Hq, size=n)
    rows = np.stack([b, h], axis=1).astype(np.int32)
    return np.unique(rows, axis=0)
