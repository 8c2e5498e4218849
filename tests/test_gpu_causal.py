"""GPU parity of the causal-window variant (the autoregressive extension)
against the fp64 oracle, through the C ABI.

Bars: the inputs are first repaired per chunk (tests/_gap.py) until every
query block's top-k boundary gap, against the key means of its visible
prefix, is at least 1e-4 relative; then the block map equals the oracle's on
every query block and is bit-equal between the fused forward and the
standalone selector; the sparse branch (also run on the oracle's own map),
the low-rank branch and the fused output on every row within max-abs 2e-2
and relative L2 1e-2; the prefix states within relative L2 1e-4. And the
variant's defining property on the device: rewriting the tokens of later
chunks leaves every result of the earlier chunks bit-identical.
"""
import numpy as np
import pytest
import torch

import oracle.sda_oracle as O
from sparse_rank_attention_block_b200 import sda, synthetic as S

from _gap import repair_gaps_causal
from _gpu import TOL_C_REL_L2, assert_close, ensure_lib, to_dev
from _util import f32

pytestmark = pytest.mark.gpu

GAP = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()


def run_causal(w, inp, map_for_attn=None, host=True):
    """Every entry point on `inp`; returns host numpy results (device tensors with host=False)."""
    p = sda.params_of(w)
    d = to_dev(inp)
    ws = sda.Workspace(p)
    keep = sda.sda_keep_count(p)
    nq = sda.sda_query_blocks(p)
    assert nq == w.n_qblk
    nc = w.L // w.chunk_tokens
    idx = torch.full((w.B, w.H, nq, keep), -7, dtype=torch.int32, device="cuda")
    o = torch.empty_like(d["q"])
    sda.sda_forward(p, d["q"], d["k"], d["v"], d["p_q"], d["p_k"], d["g"], o, idx, ws.ptr, ws.nbytes)
    idx2 = torch.full_like(idx, -7)
    sda.sda_block_select(p, d["q"], d["k"], idx2, ws.ptr, ws.nbytes)
    o_lr = torch.empty_like(d["q"])
    c = torch.empty((w.B, w.H, nc, w.rank, w.d), dtype=torch.float32, device="cuda")
    sda.sda_lowrank_fwd(p, d["q"], d["k"], d["v"], d["p_q"], d["p_k"], o_lr, c, ws.ptr, ws.nbytes)
    out = {}
    if map_for_attn is not None:
        o_s = torch.empty_like(d["q"])
        m = torch.from_numpy(np.ascontiguousarray(map_for_attn, dtype=np.int32)).cuda()
        sda.sda_sparse_attn_fwd(p, d["q"], d["k"], d["v"], m, o_s, ws.ptr, ws.nbytes)
        out["o_s"] = o_s
    ws.check()
    torch.cuda.synchronize()
    out.update(o=o, map_fused=idx, map=idx2, o_lr=o_lr, C=c)
    if not host:
        return out
    return {k: (f32(v) if v.dtype == torch.bfloat16 else v.cpu().numpy()) for k, v in out.items()}


def oracle(w, inp, rows=None, heads=None):
    hs = slice(None) if heads is None else heads
    t = [inp.q, inp.k, inp.v]
    q, k, v = (x[:, :, hs].float().numpy() for x in t)
    g = inp.g.float().numpy()
    if g.ndim == 3:
        g = g[:, :, hs]
    return O.causal_forward(q, k, v, f32(inp.p_q), f32(inp.p_k), g, grid=(w.grid_t, w.grid_h, w.grid_w),
                            block_q=w.block_q, block_k=w.block_k, sparsity=w.sparsity,
                            pairs=(w.pairs_t, w.pairs_h, w.pairs_w), causal_frames=w.causal_frames,
                            rope_base=w.rope_base, rms_eps=w.rms_eps, rows=rows)


def _pairs(r):
    return {16: (2, 3, 3), 32: (4, 6, 6), 64: (8, 12, 12)}[r]


def _case(name, seed, d=64, bq=64, r=16, **kw):
    pt, ph, pw = _pairs(r)
    return S.TINY.replace(name=name, d=d, block_q=bq, rank=r, pairs_t=pt, pairs_h=ph, pairs_w=pw, seed=seed, **kw)


CASES = [
    # 65-token chunks: every chunk end inside a key block, one partial query block per chunk
    _case("causal-d64-bq64-F1", 51, grid_t=4, grid_h=5, grid_w=13, sparsity=0.6, causal_frames=1),
    _case("causal-d64-bq64-F2", 52, grid_t=6, grid_h=7, grid_w=11, sparsity=0.75, causal_frames=2),
    # tcgen05 attention with the fused readout (one C per chunk), 3 query blocks per chunk
    _case("causal-d128-bq128-r32-F1", 53, d=128, bq=128, r=32, grid_t=3, grid_h=9, grid_w=30, sparsity=0.8,
          causal_frames=1),
    _case("causal-d128-bq128-r16-B2-gph-F2", 54, d=128, bq=128, r=16, B=2, H=3, grid_t=4, grid_h=5, grid_w=13,
          sparsity=0.7, causal_frames=2, gate_per_head=1),
    # chunks of exactly 128 tokens (no edge block), r = 64
    _case("causal-d64-bq128-r64-F1", 55, bq=128, r=64, grid_t=4, grid_h=8, grid_w=16, sparsity=0.5,
          causal_frames=1),
    _case("causal-d128-bq64-r32-F3", 56, d=128, r=32, grid_t=6, grid_h=6, grid_w=10, sparsity=0.9, causal_frames=3),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_causal_matches_oracle(w):
    inp = S.make_inputs(w)
    repair_gaps_causal(inp, w)
    ref = oracle(w, inp)
    assert float(ref["gap"].min()) >= GAP
    got = run_causal(w, inp, map_for_attn=ref["map"])
    assert np.array_equal(got["map_fused"], got["map"]), "forward and selector maps differ"
    assert np.array_equal(got["map"], ref["map"]), "block map differs from the oracle"
    assert_close(got["C"], ref["C"], "prefix states", max_abs=np.inf, rel_l2=TOL_C_REL_L2)
    assert_close(got["o_s"], ref["o_s"], "o_s on the oracle's map")
    assert_close(got["o_lr"], ref["o_lr"], "o_lr")
    assert_close(got["o"], ref["o"], "o")


@pytest.mark.parametrize("w", [CASES[0], CASES[2], CASES[3]], ids=lambda w: w.name)
def test_later_chunks_change_nothing_on_device(w):
    inp = S.make_inputs(w)
    a = run_causal(w, inp)
    other = S.make_inputs(w, seed=w.seed + 1000)
    hi = w.chunk_tokens  # rewrite everything after the first chunk
    for n in ("q", "k", "v"):
        getattr(inp, n)[:, hi:] = getattr(other, n)[:, hi:]
    b = run_causal(w, inp)
    nq0 = -(-w.chunk_tokens // w.block_q)
    assert np.array_equal(a["map"][:, :, :nq0], b["map"][:, :, :nq0])
    assert np.array_equal(a["C"][:, :, 0], b["C"][:, :, 0])
    for key in ("o", "o_lr"):
        assert np.array_equal(a[key][:, :hi], b[key][:, :hi]), key
        assert not np.array_equal(a[key][:, hi:], b[key][:, hi:]), key


def test_one_chunk_equals_bidirectional_bitwise():
    """causal_frames = T on the warp-MMA paths: the same launches' arithmetic as no window."""
    w = CASES[1].replace(name="causal-one-chunk", causal_frames=6)
    inp = S.make_inputs(w)
    a = run_causal(w, inp)
    b = run_causal(w.replace(causal_frames=0), inp)
    for key in ("map", "map_fused", "o", "o_lr"):
        assert np.array_equal(a[key], b[key]), key
    assert np.array_equal(a["C"][:, :, 0], b["C"][:, :, 0])


@pytest.mark.slow
def test_causal_720p_full_size_sampled():
    """The 14B-720P-like layer with 3-frame chunks (7 chunks of 10,800 tokens), as the
    benchmark times it: oracle on two heads, sampled rows of every chunk."""
    w = S.WAN14B_720P.replace(causal_frames=3)
    inp = S.make_inputs(w)
    heads = [0, w.H - 1]
    repair_gaps_causal(inp, w, heads=heads)
    dev = run_causal(w, inp, host=False)
    got = {k: dev[k].cpu().numpy() for k in ("map", "map_fused", "C")}
    rng = np.random.default_rng(7)
    n = 96
    rows = np.stack([np.zeros(n, dtype=np.int64), rng.integers(0, w.L, n), rng.integers(0, 2, n)], axis=1)
    ends = np.array([[0, c * w.chunk_tokens + e, hh] for c in range(7) for e in (-1, 0) for hh in (0, 1)
                     if 0 <= c * w.chunk_tokens + e < w.L])
    rows = np.concatenate([rows, ends])
    ref = oracle(w, inp, rows=rows, heads=heads)
    gmap = got["map"][:, heads]
    assert float(ref["gap"].min()) >= GAP
    assert np.array_equal(gmap, ref["map"]), "block map differs from the oracle"
    assert np.array_equal(got["map_fused"], got["map"])
    assert_close(got["C"][:, heads], ref["C"], "prefix states", max_abs=np.inf, rel_l2=TOL_C_REL_L2)
    sel = (rows[:, 0], rows[:, 1], np.array(heads)[rows[:, 2]])
    for key in ("o", "o_lr"):
        got[key] = f32(dev[key][tuple(torch.from_numpy(np.asarray(i)).cuda() for i in sel)])
    assert_close(got["o_lr"], ref["o_lr"], "sampled o_lr")
    assert_close(got["o"], ref["o"], "sampled o")
