"""Seeded synthetic inputs for paged decode attention.

This module only draws inputs: context lengths, the scattering of logical
blocks over a physical pool, block tables and the q/K/V values, rounded to the
storage dtype.  It holds none of the attention arithmetic, so both the CPU
oracle and the CUDA path can take their inputs from here without sharing any
of the method's code.

Shapes (one decode step of one layer):
  q, out        [num_seqs, num_q_heads, head_dim]
  k/v cache     [num_blocks, num_kv_heads, block_size, head_dim]
  block_tables  int32 [num_seqs, max_blocks_per_seq]   (-1 past the used entries)
  context_lens  int32 [num_seqs]

The pages fix the block idea (fixed-size blocks of e.g. 16 tokens scattered
through a pool, one table per sequence mapping logical to physical blocks:
"What is PagedAttention ..." §How it works; "pagedattention vllm"
§PagedAttention Design) but no layout; the layout above is this library's.
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace

import numpy as np

DTYPES = ("f32", "f16", "bf16")
DTYPE_CODE = {"f32": 0, "f16": 1, "bf16": 2, "e4m3": 3}
ELEM_BYTES = {"f32": 4, "f16": 2, "bf16": 2, "e4m3": 1}

# numbers drawn per generator chunk; fixed so results do not depend on the
# number of threads used to draw them
_CHUNK = 1 << 22


@dataclass(frozen=True)
class DecodeConfig:
    """One paged-decode workload.

    lens: ("fixed", (l0, l1, ...)) | ("uniform", lo, hi) (inclusive integers)
          | ("lognormal", median, sigma, lo, hi)
    pool: ("fixed", n_blocks) | ("factor", f)  -- pool = ceil(f * blocks used)
    """
    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str
    lens: tuple
    pool: tuple = ("factor", 1.2)
    partition_size: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    def with_(self, **kw) -> "DecodeConfig":
        return replace(self, **kw)


# The five workloads: a tiny fp32 case, a Llama-2-13B-shaped layer (40 heads
# MHA, head_dim 128, fp16), a GQA batch (64/8 heads, bf16, block 16 or 32), a
# long-context batch split into 512-token partitions, and parallel sampling with
# copy-on-write prefix sharing.
CONFIGS = {
    "tiny_fp32": DecodeConfig(
        "tiny_fp32", 4, 4, 4, 64, 16, "f32", ("fixed", (1, 7, 16, 33)),
        pool=("fixed", 16)),
    "llama2_13b_layer": DecodeConfig(
        "llama2_13b_layer", 64, 40, 40, 128, 16, "f16", ("uniform", 128, 2048)),
    "gqa_bs16": DecodeConfig(
        "gqa_bs16", 256, 64, 8, 128, 16, "bf16", ("lognormal", 512, 1.0, 32, 8192)),
    "gqa_bs32": DecodeConfig(
        "gqa_bs32", 256, 64, 8, 128, 32, "bf16", ("lognormal", 512, 1.0, 32, 8192)),
    "long_context": DecodeConfig(
        "long_context", 8, 32, 8, 128, 16, "bf16", ("uniform", 32768, 131072),
        partition_size=512),
}

# copy-on-write sampling workload: 32 prompts x 8 samples share a 1024-token
# prefix (+ r tokens, r in [1, 15], so the last shared block is partly filled),
# private tails of 1..512 tokens; 40 heads MHA, head_dim 128, fp16, block 16.
COW_SAMPLING = dict(num_prompts=32, samples=8, prefix=1024, r_lo=1, r_hi=15,
                    tail_lo=1, tail_hi=512, num_q_heads=40, num_kv_heads=40,
                    head_dim=128, block_size=16, dtype="f16")


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def draw_context_lens(cfg: DecodeConfig, seed: int) -> np.ndarray:
    kind = cfg.lens[0]
    g = rng(seed * 1000 + 1)
    if kind == "fixed":
        lens = np.asarray(cfg.lens[1], dtype=np.int64)
        assert lens.size == cfg.num_seqs
    elif kind == "uniform":
        lo, hi = cfg.lens[1], cfg.lens[2]
        lens = g.integers(lo, hi + 1, size=cfg.num_seqs)
    elif kind == "lognormal":
        med, sigma, lo, hi = cfg.lens[1:5]
        x = np.exp(math.log(med) + sigma * g.standard_normal(cfg.num_seqs))
        lens = np.clip(np.rint(x), lo, hi).astype(np.int64)
    else:
        raise ValueError(kind)
    return lens.astype(np.int32)


def blocks_needed(lens: np.ndarray, block_size: int) -> np.ndarray:
    return (lens.astype(np.int64) + block_size - 1) // block_size


def round_to_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32/float64 values to the storage dtype (round to nearest even).

    Returns float32 / float16 arrays, or uint16 bit patterns for bf16.
    """
    if dtype == "f32":
        return x.astype(np.float32)
    if dtype == "f16":
        return x.astype(np.float16)
    if dtype == "bf16":
        b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
        lsb = (b >> np.uint32(16)) & np.uint32(1)
        return ((b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)
    raise ValueError(dtype)


def storage_np_dtype(dtype: str):
    return {"f32": np.float32, "f16": np.float16, "bf16": np.uint16}[dtype]


def normal_fill(shape, dtype: str, seed: int, threads: int = 8) -> np.ndarray:
    """N(0,1) values rounded to `dtype`, drawn chunk by chunk from seeded PCG64
    streams (one per chunk), so the result is fixed by `seed` alone."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=storage_np_dtype(dtype))
    nchunks = (n + _CHUNK - 1) // _CHUNK
    seeds = np.random.SeedSequence(seed).spawn(nchunks)

    def work(i):
        lo = i * _CHUNK
        hi = min(n, lo + _CHUNK)
        g = np.random.Generator(np.random.PCG64(seeds[i]))
        out[lo:hi] = round_to_dtype(g.standard_normal(hi - lo, dtype=np.float32), dtype)

    if nchunks <= 1:
        for i in range(nchunks):
            work(i)
    else:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(work, range(nchunks)))
    return out.reshape(shape)


def poison_value(dtype: str, kind: str = "nan"):
    """Bit pattern / value used to poison cache slots that must never be read."""
    if dtype == "f32":
        return np.float32(np.nan if kind == "nan" else np.inf)
    if dtype == "f16":
        return np.float16(np.nan if kind == "nan" else np.inf)
    return np.uint16(0x7FC0 if kind == "nan" else 0x7F80)


@dataclass
class DecodeInputs:
    cfg: DecodeConfig
    q: np.ndarray              # [B, Hq, D] storage dtype
    k_cache: np.ndarray        # [N, Hkv, bs, D]
    v_cache: np.ndarray
    block_tables: np.ndarray   # int32 [B, max_blocks]
    context_lens: np.ndarray   # int32 [B]
    num_blocks: int

    @property
    def max_blocks_per_seq(self) -> int:
        return self.block_tables.shape[1]

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.context_lens.size else 0


def assign_blocks(lens: np.ndarray, block_size: int, num_blocks: int, seed: int,
                  max_blocks: int | None = None, shuffle: bool = True,
                  fill: int = -1) -> np.ndarray:
    """Scatter each sequence's logical blocks over the pool: the pool ids are a
    seeded random permutation (or the identity, for a contiguous layout) and
    sequences take consecutive runs of it."""
    nb = blocks_needed(lens, block_size)
    total = int(nb.sum())
    if total > num_blocks:
        raise ValueError("pool too small")
    mb = int(nb.max()) if max_blocks is None and nb.size else (max_blocks or 1)
    mb = max(mb, 1)
    perm = rng(seed * 1000 + 2).permutation(num_blocks) if shuffle else np.arange(num_blocks)
    tables = np.full((lens.size, mb), fill, dtype=np.int32)
    pos = 0
    for b in range(lens.size):
        n = int(nb[b])
        tables[b, :n] = perm[pos:pos + n]
        pos += n
    return tables


def make_decode_inputs(cfg: DecodeConfig, seed: int = 0, *, shuffle: bool = True,
                       poison: str | None = None, lens: np.ndarray | None = None,
                       table_fill: int = -1, threads: int = 8) -> DecodeInputs:
    """Build one seeded decode batch.

    poison: None, "nan" or "inf" -- write that value into every cache slot that
    no sequence uses (the tail of each last block and the unused pool blocks).
    """
    if lens is None:
        lens = draw_context_lens(cfg, seed)
    lens = np.asarray(lens, dtype=np.int32)
    nb = blocks_needed(lens, cfg.block_size)
    used = int(nb.sum())
    if cfg.pool[0] == "fixed":
        num_blocks = int(cfg.pool[1])
    else:
        num_blocks = max(1, int(math.ceil(cfg.pool[1] * used)))
    tables = assign_blocks(lens, cfg.block_size, num_blocks, seed, shuffle=shuffle,
                           fill=table_fill)
    H, bs, D = cfg.num_kv_heads, cfg.block_size, cfg.head_dim
    q = normal_fill((cfg.num_seqs, cfg.num_q_heads, D), cfg.dtype, seed * 1000 + 3, threads)
    k = normal_fill((num_blocks, H, bs, D), cfg.dtype, seed * 1000 + 4, threads)
    v = normal_fill((num_blocks, H, bs, D), cfg.dtype, seed * 1000 + 5, threads)
    if poison is not None:
        pv = poison_value(cfg.dtype, poison)
        live = np.zeros((num_blocks, bs), dtype=bool)
        for b in range(lens.size):
            L = int(lens[b])
            for j in range(int(nb[b])):
                n_in = min(bs, L - j * bs)
                live[tables[b, j], :n_in] = True
        dead = ~live
        k.transpose(0, 2, 1, 3)[dead] = pv
        v.transpose(0, 2, 1, 3)[dead] = pv
    return DecodeInputs(cfg, q, k, v, tables, lens, num_blocks)


def kv_bytes_per_token(cfg: DecodeConfig, kv_dtype: str | None = None) -> int:
    return 2 * cfg.num_kv_heads * cfg.head_dim * ELEM_BYTES[kv_dtype or cfg.dtype]


def algorithmic_bytes(cfg: DecodeConfig, lens: np.ndarray, window: int = 0,
                      kv_dtype: str | None = None, per_page_scales: bool = False) -> int:
    """Bytes a decode step must move at least once: K and V of every attended
    token (the last `window` of each sequence when window > 0), q in and out,
    the block-table entries used and the lengths (and the scales of quantised
    pages, kv_dtype "e4m3": one K and one V float32 per KV head, or per
    attended (block, KV head) page with per_page_scales)."""
    e = ELEM_BYTES[cfg.dtype]
    lens = np.asarray(lens, dtype=np.int64)
    if window > 0:
        lo = np.maximum(lens - window, 0)
        att = lens - lo
        nblk = (lens + cfg.block_size - 1) // cfg.block_size - lo // cfg.block_size
    else:
        att = lens
        nblk = blocks_needed(lens, cfg.block_size)
    kv = int(att.sum()) * kv_bytes_per_token(cfg, kv_dtype)
    qo = 2 * lens.size * cfg.num_q_heads * cfg.head_dim * e
    tab = int(nblk.sum()) * 4
    scales = 0
    if kv_dtype == "e4m3":
        scales = 8 * cfg.num_kv_heads * (int(nblk.sum()) if per_page_scales else 1)
    return kv + qo + tab + 4 * lens.size + scales


# ---------------------------------------------------------------------------
# quantised (FP8 E4M3) pages

# Codes: sign uniform, the other 7 bits uniform over [0, E4M3_TOP] (exponent
# field <= 12, magnitudes below 64; no NaN), drawn from seeded PCG64 chunks
# like normal_fill.  Scales: one per KV head for K and for V, uniform in
# [1/64, 1/16], so the stored values span about +-4.
E4M3_TOP = 0x67


def e4m3_codes(shape, seed: int, threads: int = 8) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint8)
    nchunks = (n + _CHUNK - 1) // _CHUNK
    seeds = np.random.SeedSequence(seed).spawn(max(nchunks, 1))

    def work(i):
        lo = i * _CHUNK
        hi = min(n, lo + _CHUNK)
        g = np.random.Generator(np.random.PCG64(seeds[i]))
        mag = g.integers(0, E4M3_TOP + 1, size=hi - lo, dtype=np.uint8)
        sign = g.integers(0, 2, size=hi - lo, dtype=np.uint8) << np.uint8(7)
        out[lo:hi] = mag | sign

    if nchunks <= 1:
        for i in range(nchunks):
            work(i)
    else:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(work, range(nchunks)))
    return out.reshape(shape)


def e4m3_scales(num_kv_heads: int, seed: int) -> tuple[np.ndarray, np.ndarray]:
    g = rng(seed * 1000 + 11)
    ks = g.uniform(1 / 64, 1 / 16, size=num_kv_heads).astype(np.float32)
    vs = g.uniform(1 / 64, 1 / 16, size=num_kv_heads).astype(np.float32)
    return ks, vs


def e4m3_page_scales(num_blocks: int, num_kv_heads: int, seed: int):
    """Per-page scales ([num_blocks, Hkv] for K and for V), uniform in
    [1/64, 1/16] like the per-head ones."""
    g = rng(seed * 1000 + 12)
    ks = g.uniform(1 / 64, 1 / 16, size=(num_blocks, num_kv_heads)).astype(np.float32)
    vs = g.uniform(1 / 64, 1 / 16, size=(num_blocks, num_kv_heads)).astype(np.float32)
    return ks, vs


@dataclass
class QuantisedPages:
    k_cache: np.ndarray   # uint8 E4M3 codes [N, Hkv, bs, D]
    v_cache: np.ndarray
    k_scale: np.ndarray   # float32 [Hkv]
    v_scale: np.ndarray


def make_e4m3_pages(inp: "DecodeInputs", seed: int = 0, threads: int = 8,
                    per_page: bool = False) -> QuantisedPages:
    """E4M3 pages of the same shape as inp's caches (same tables and lengths;
    inp.q stays the query), with per-head scales, or per-page ones."""
    shape = inp.k_cache.shape
    k = e4m3_codes(shape, seed * 1000 + 14, threads)
    v = e4m3_codes(shape, seed * 1000 + 15, threads)
    if per_page:
        ks, vs = e4m3_page_scales(shape[0], shape[1], seed)
    else:
        ks, vs = e4m3_scales(shape[1], seed)
    return QuantisedPages(k, v, ks, vs)


# ---------------------------------------------------------------------------
# copy-on-write sampling recipe (the allocator builds the tables)

@dataclass
class CowRecipe:
    num_prompts: int
    samples: int
    shared_lens: np.ndarray    # [num_prompts]  1024 + r
    tail_lens: np.ndarray      # [num_prompts * samples]


def draw_cow_recipe(seed: int = 5, **over) -> CowRecipe:
    c = dict(COW_SAMPLING)
    c.update(over)
    g = rng(seed * 1000 + 7)
    r = g.integers(c["r_lo"], c["r_hi"] + 1, size=c["num_prompts"])
    tails = g.integers(c["tail_lo"], c["tail_hi"] + 1, size=c["num_prompts"] * c["samples"])
    return CowRecipe(c["num_prompts"], c["samples"], (c["prefix"] + r).astype(np.int64),
                     tails.astype(np.int64))


def random_alloc_ops(seed: int, n_ops: int, max_seqs: int = 24, max_len: int = 200,
                     swap: bool = False, slide: bool = False, prefix: bool = False):
    """A seeded random script of allocator operations (add / fork / append /
    free, swap_out / swap_in when `swap`, sliding-window releases when
    `slide`, prompts through the prefix cache when `prefix`) for differential
    tests of the block manager.  Prefix prompts start with one of four fixed
    token sequences (synthetic token ids) cut at a random length, and some
    continue with random tokens, so prompts share prefixes of varied lengths."""
    g = rng(seed * 1000 + 9)
    ops = []
    next_id = 0
    live = []
    if prefix:
        gp = rng(seed * 1000 + 10)
        templates = [gp.integers(0, 50, size=max_len) for _ in range(4)]
    for _ in range(n_ops):
        r = g.random()
        if slide and live and g.random() < 0.1:
            ops.append(("slide", live[int(g.integers(len(live)))], int(g.integers(1, 40))))
            continue
        if swap and live and g.random() < 0.15:
            ops.append(("swap_out" if g.random() < 0.5 else "swap_in",
                        live[int(g.integers(len(live)))]))
            continue
        if not live or (r < 0.25 and len(live) < max_seqs):
            n = int(g.integers(0, max_len + 1))
            if prefix and gp.random() < 0.7:
                t = templates[int(gp.integers(4))][:n].copy()
                cut = int(gp.integers(0, n + 1)) if gp.random() < 0.5 else n
                t[cut:] = gp.integers(0, 50, size=n - cut)
                ops.append(("prefix", next_id, tuple(int(x) for x in t)))
            else:
                ops.append(("add", next_id, n))
            live.append(next_id)
            next_id += 1
        elif r < 0.45 and len(live) < max_seqs:
            parent = live[int(g.integers(len(live)))]
            ops.append(("fork", parent, next_id))
            live.append(next_id)
            next_id += 1
        elif r < 0.85:
            ops.append(("append", live[int(g.integers(len(live)))]))
        else:
            sid = live.pop(int(g.integers(len(live))))
            ops.append(("free", sid))
    return ops
