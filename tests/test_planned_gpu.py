"""The planned decode (host plan, persistent CTAs) over E4M3 pages against
the oracle: the same attention over each sequence's context, whatever the
plan's CTA count and piece size, with a sliding window and with scales per
head or per page."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_346_b200 as pkv
from tests.gpu_util import assert_close, to_device, to_f64
from workloads import DecodeConfig, make_decode_inputs, make_e4m3_pages

pytestmark = pytest.mark.gpu

RAGGED = (1, 15, 16, 17, 63, 64, 65, 200, 513, 1100, 0, 2047)


def _codes(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda().view(torch.float8_e4m3fn)


class Planned:
    def __init__(self, dtype, Hq, Hkv, bs, lens, seed, per_page=False):
        nb = sum((L + bs - 1) // bs for L in lens)
        cfg = DecodeConfig("planned", len(lens), Hq, Hkv, 128, bs, dtype, ("fixed", tuple(lens)),
                           pool=("fixed", nb + 9))
        self.inp = inp = make_decode_inputs(cfg, seed=seed)
        self.pages = make_e4m3_pages(inp, seed, per_page=per_page)
        self.cfg = cfg
        self.q = to_device(inp.q, dtype)
        self.k, self.v = _codes(self.pages.k_cache), _codes(self.pages.v_cache)
        self.ks = torch.from_numpy(self.pages.k_scale).cuda()
        self.vs = torch.from_numpy(self.pages.v_scale).cuda()
        self.bt, self.cl = to_device(inp.block_tables), to_device(inp.context_lens)

    def plan(self, num_ctas, piece_tokens=0, window=0, order=None):
        c = self.cfg
        return pkv.pkv_decode_plan(self.inp.context_lens, c.num_q_heads, c.num_kv_heads,
                                   c.head_dim, c.block_size, num_ctas=num_ctas,
                                   sliding_window=window, seq_order=order,
                                   piece_tokens=piece_tokens)

    def decode(self, plan, fill=5.0, ws=None, calls=1):
        c = self.cfg
        out = torch.full_like(self.q, fill)
        if ws is None:
            ws = pkv.planned_workspace(plan, c.head_dim)
        for _ in range(calls):
            pkv.pkv_paged_attention_decode_planned(out, self.q, self.k, self.v, self.ks, self.vs,
                                                   self.bt, self.cl, plan,
                                                   torch.from_numpy(plan).cuda(), c.scale,
                                                   c.block_size, workspace=ws)
        torch.cuda.synchronize()
        return to_f64(out)

    def oracle(self, window=0):
        c = self.cfg
        return oracle.paged_decode(self.inp.q, self.pages.k_cache, self.pages.v_cache,
                                   self.inp.block_tables, self.inp.context_lens, scale=c.scale,
                                   dtype=c.dtype, kv_dtype="e4m3", k_scale=self.pages.k_scale,
                                   v_scale=self.pages.v_scale, window=window)


@pytest.mark.parametrize("dtype,Hq,Hkv,bs", [("bf16", 16, 2, 16), ("f16", 4, 4, 32),
                                             ("bf16", 24, 2, 64), ("f16", 40, 8, 16)])
@pytest.mark.parametrize("per_page", [False, True])
def test_planned_matches_oracle(dtype, Hq, Hkv, bs, per_page):
    pl = Planned(dtype, Hq, Hkv, bs, RAGGED, seed=Hq + bs, per_page=per_page)
    ref = pl.oracle()
    auto = pkv.pkv_decode_planned_ctas(Hq, Hkv, 128, bs)
    assert auto >= 148
    for C, pt in ((1, 0), (3, 64), (7, 256), (auto, 0), (50, 128)):
        plan = pl.plan(C, pt)
        # two calls on one workspace: the unit counters come back to zero
        got = pl.decode(plan, calls=2)
        assert_close(got, ref, dtype, f"planned C={C} pt={pt} per_page={per_page}")
    assert pkv.pkv_device_status(clear=True) == 0


@pytest.mark.parametrize("W", [1, 40, 500])
def test_planned_sliding_window(W):
    pl = Planned("bf16", 16, 2, 16, RAGGED, seed=3 + W)
    ref = pl.oracle(window=W)
    order = pkv.pkv_decode_schedule_order(pl.inp.context_lens)
    for C, pt in ((5, 64), (200, 0)):
        got = pl.decode(pl.plan(C, pt, window=W, order=order))
        assert_close(got, ref, "bf16", f"planned window {W} C={C}")
    assert pkv.pkv_device_status(clear=True) == 0


def test_planned_matches_regular_decode():
    """Same kernel arithmetic per piece as the regular tensor-core decode: the
    results agree to rounding (the split points differ)."""
    pl = Planned("bf16", 16, 2, 16, RAGGED, seed=99)
    c = pl.cfg
    out = torch.empty_like(pl.q)
    mcl = pl.inp.max_context_len
    ws = torch.empty(max(16, pkv.pkv_decode_workspace_size(c.num_seqs, 16, 2, 128, mcl)),
                     dtype=torch.uint8, device="cuda")
    pkv.pkv_paged_attention_decode_e4m3(out, pl.q, pl.k, pl.v, pl.ks, pl.vs, pl.bt, pl.cl,
                                        c.scale, c.block_size, mcl, workspace=ws)
    torch.cuda.synchronize()
    got = pl.decode(pl.plan(pkv.pkv_decode_planned_ctas(16, 2, 128, 16)))
    assert_close(got, to_f64(out), "bf16", "planned vs regular")


def test_planned_empty_and_tiny_batches():
    """Sequences of length 0 get zero rows; more CTAs than pieces leave CTAs
    with nothing to do."""
    pl = Planned("f16", 8, 8, 16, (0, 3, 0, 16), seed=5)
    ref = pl.oracle()
    for C in (1, 64):
        got = pl.decode(pl.plan(C, 0))
        assert_close(got, ref, "f16", f"tiny planned C={C}")
    assert pkv.pkv_device_status(clear=True) == 0


def test_plan_outside_its_batch_is_flagged():
    """A piece that runs past its sequence (a plan made for other lengths) is
    skipped and flagged, not read."""
    pl = Planned("bf16", 16, 2, 16, RAGGED, seed=7)
    plan = pl.plan(4, 64)
    h = pkv.plan_header(plan)
    IW = 16
    items = plan[16 + h["num_ctas"] + 1:].reshape(-1, IW)
    i = int(np.argmax(items[:, 3]))          # the longest sequence's last piece
    bad = plan.copy()
    base = 16 + h["num_ctas"] + 1 + i * IW
    bad[base + 3] = items[i, 2] + 4096       # longer than any piece may be
    pkv.pkv_device_status(clear=True)
    pl.decode(bad)
    assert pkv.pkv_device_status(clear=True) & pkv.PKV_DEV_BAD_PLAN
