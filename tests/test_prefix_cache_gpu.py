"""Prefix caching end to end on the GPU.

Requests whose prompts begin the same way share the cached K/V blocks of that
beginning instead of computing and storing them again ("pagedattention vllm"
§vLLM Integration and §Advanced Features: automatic prefix caching;
"PagedAttention" glossary entry: prompt caching).  Here the native block
manager admits prompts with pkv_alloc_add_seq_prefix, the caller appends only
the tokens the cache did not hold (pkv_kv_cache_append at the slots of the
sequence's table) and the batch is decoded on the GPU.

The K/V of a prompt token is a deterministic function of the prompt up to and
including it (as in a model, where a token's keys and values depend on every
earlier token), so a block served from the cache holds exactly what a fresh
computation would write.  Checked at every phase, on the allocator model
(oracle/block_manager.py) and the oracle:
  * allocator: cached-token counts, tables, lengths, evictable list and stats
    bit-exact between the native allocator and the model;
  * caches: the device pools bit-exact against a host replay of the same
    appends;
  * attention: the decode over the shared pool within tolerance of the float64
    oracle over each request's freshly computed, privately stored K/V (an
    identity-table pool), so a wrong cache hit or a wrong block shows up.
Phases: prompts from a few shared stems (hits on blocks in use); free some
requests and admit new ones that take blocks back from the evictable list;
fill the pool until blocks are evicted, then admit a prompt whose cached
prefix was evicted (fewer hits, recomputed).
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_346_b200 as pkv
from oracle import block_manager as bm
from oracle.cache_ops import kv_cache_append
from tests.gpu_util import assert_close, to_device, to_f64
from workloads import normal_fill, round_to_dtype

pytestmark = pytest.mark.gpu

BS = 16


def _prompt_kv(tokens, H, D, dtype):
    """K and V [len, H, D] of a prompt: token t's rows are drawn from a
    generator seeded by a hash chained over tokens[0..t]."""
    L = len(tokens)
    k = np.empty((L, H, D), np.float32)
    v = np.empty((L, H, D), np.float32)
    h = 0x9E3779B97F4A7C15
    for t, tok in enumerate(tokens):
        h = (h * 0x100000001B3 ^ (int(tok) + 1)) & 0xFFFFFFFFFFFFFFFF
        x = np.random.default_rng(h).standard_normal((2, H, D), dtype=np.float32)
        k[t], v[t] = x[0], x[1]
    return round_to_dtype(k, dtype), round_to_dtype(v, dtype)


class Harness:
    def __init__(self, N, Hq, Hkv, D, dtype, seed):
        self.N, self.Hq, self.Hkv, self.D, self.dtype = N, Hq, Hkv, D, dtype
        self.nat = pkv.BlockAllocator(N, BS)
        self.mod = bm.BlockManagerModel(N, BS)
        # the pools start as garbage; both sides hold the same garbage
        self.K = normal_fill((N, Hkv, BS, D), dtype, seed * 10 + 1)
        self.V = normal_fill((N, Hkv, BS, D), dtype, seed * 10 + 2)
        self.dK, self.dV = to_device(self.K, dtype), to_device(self.V, dtype)
        self.prompts = {}
        self.rng = np.random.default_rng(seed)

    def admit(self, sid, tokens):
        """add_seq_prefix on both allocators; append the uncached tokens.
        -> cached token count"""
        st, cached = self.nat.add_seq_prefix(sid, tokens)
        assert (st, cached) == self.mod.add_seq_prefix(sid, tokens), sid
        assert st == 0, st
        assert self.nat.block_table(sid) == self.mod.block_table(sid)
        self.prompts[sid] = list(tokens)
        table = np.array(self.mod.block_table(sid), np.int64)
        t = np.arange(cached, len(tokens))
        if t.size:
            slots = table[t // BS] * BS + t % BS
            k, v = _prompt_kv(tokens, self.Hkv, self.D, self.dtype)
            pkv.pkv_kv_cache_append(self.dK, self.dV, to_device(k[cached:], self.dtype),
                                    to_device(v[cached:], self.dtype), to_device(slots))
            kv_cache_append(self.K, self.V, k[cached:], v[cached:], slots)
        return cached

    def free(self, sid):
        assert self.nat.free_seq(sid) == 0 and self.mod.free_seq(sid) == 0
        del self.prompts[sid]

    def check(self, seed):
        nat, mod = self.nat, self.mod
        assert nat.evictable_list() == mod.evictable_list()
        assert nat.free_list() == mod.free_list()
        assert nat.cache_stats() == mod.cache_stats()
        torch.cuda.synchronize()
        view = np.int16 if self.K.dtype.itemsize == 2 else np.int32
        got_k = self.dK.cpu().view(torch.int16 if view is np.int16 else torch.int32).numpy()
        got_v = self.dV.cpu().view(torch.int16 if view is np.int16 else torch.int32).numpy()
        assert np.array_equal(got_k, self.K.view(view))
        assert np.array_equal(got_v, self.V.view(view))
        # decode every resident request over the shared pool
        sids = sorted(self.prompts)
        B = len(sids)
        maxb = max(-(-len(self.prompts[s]) // BS) for s in sids)
        tables, lens = nat.build_block_tables(sids, maxb)
        for i, s in enumerate(sids):
            assert tables[i, :len(mod.block_table(s))].tolist() == mod.block_table(s)
            assert lens[i] == mod.seq_len(s) == len(self.prompts[s])
        q = normal_fill((B, self.Hq, self.D), self.dtype, seed)
        scale = 1.0 / np.sqrt(self.D)
        dq = to_device(q, self.dtype)
        out = torch.empty_like(dq)
        L = int(lens.max())
        for P in (0, 64):
            ws = torch.empty(max(16, pkv.pkv_decode_workspace_size(B, self.Hq, self.Hkv, self.D,
                                                                   L, P)),
                             dtype=torch.uint8, device="cuda")
            pkv.pkv_paged_attention_decode(out, dq, self.dK, self.dV, to_device(tables),
                                           to_device(lens), scale, BS, L, partition_size=P,
                                           workspace=ws)
            torch.cuda.synchronize()
            got = to_f64(out)
            # the oracle over each request's own freshly computed K/V, stored
            # privately (identity tables)
            nb = [-(-len(self.prompts[s]) // BS) for s in sids]
            Kf = np.zeros((sum(nb), self.Hkv, BS, self.D), self.K.dtype)
            Vf = np.zeros_like(Kf)
            ft = np.zeros((B, maxb), np.int32)
            base = 0
            for i, s in enumerate(sids):
                k, v = _prompt_kv(self.prompts[s], self.Hkv, self.D, self.dtype)
                n = len(self.prompts[s])
                for t in range(n):
                    Kf[base + t // BS, :, t % BS] = k[t]
                    Vf[base + t // BS, :, t % BS] = v[t]
                ft[i, :nb[i]] = np.arange(base, base + nb[i])
                base += nb[i]
            ref = oracle.paged_decode(q, Kf, Vf, ft, lens, scale=scale, dtype=self.dtype)
            assert_close(got, ref, self.dtype, f"prefix-cached decode P={P}")
        assert pkv.pkv_device_status(clear=True) == 0


@pytest.mark.parametrize("dtype,Hq,Hkv", [("f16", 8, 8), ("bf16", 32, 4)])
def test_prefix_cache_decode_matches_fresh_prompts(dtype, Hq, Hkv):
    D, N = 128, 60
    hz = Harness(N, Hq, Hkv, D, dtype, seed=7 if dtype == "f16" else 8)
    g = hz.rng
    stems = [g.integers(0, 500, size=n).tolist() for n in (70, 121, 40)]

    def prompt(stem, cut, extra):
        return stems[stem][:cut] + g.integers(500, 1000, size=extra).tolist()

    # phase 1: requests from shared stems; later ones hit blocks in use
    hits = []
    plan = [(0, 70, 9), (0, 70, 0), (1, 121, 5), (0, 48, 20), (1, 100, 0), (2, 40, 3)]
    for sid, (stem, cut, extra) in enumerate(plan):
        hits.append(hz.admit(sid, prompt(stem, cut, extra)))
    assert hits[0] == 0 and hits[1] == 64 and hits[3] == 48 and hits[4] == 96
    hz.check(seed=100)

    # phase 2: free three requests; their registered blocks become evictable
    # and are taken back by new requests with the same beginnings
    for sid in (0, 1, 2):
        hz.free(sid)
    assert hz.nat.cache_stats()[1] > 0
    back = hz.admit(10, prompt(0, 70, 30))
    assert back == 64
    assert hz.admit(11, prompt(1, 121, 0)) == 112
    hz.check(seed=101)

    # phase 3: the last request of stem 2 leaves, so stem 2's registered
    # blocks are the evictable list; a long fresh prompt needs two blocks more
    # than the free stack holds and evicts them
    hz.free(5)
    assert len(hz.nat.evictable_list()) == 2
    free_now = len(hz.nat.free_list())
    hz.admit(20, g.integers(1000, 2000, size=(free_now + 2) * BS - 3).tolist())
    assert hz.nat.cache_stats()[1] == 0 and len(hz.nat.free_list()) == 0
    hz.check(seed=102)

    # phase 4: a prompt that begins like stem 2 finds nothing cached any more
    # and is computed and appended in full
    hz.free(20)
    assert hz.admit(21, prompt(2, 40, 8)) == 0
    hz.check(seed=103)
