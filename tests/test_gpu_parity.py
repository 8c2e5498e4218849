"""GPU parity: every C-ABI call against the fp64 oracle on the same seeded inputs.

Bar: block map bit-exact (inputs repaired so that no top-k boundary gap is
below 1e-4 relative); outputs within max-abs 2e-2 and relative-L2 1e-2; the
state C within relative-L2 1e-4.
"""
import numpy as np
import pytest
import torch

import oracle.sda_oracle as O
from sparse_rank_attention_block_b200 import sda, synthetic as S

from _gap import repair_gaps
from _gpu import TOL_C_REL_L2, assert_close, ensure_lib, run_all, to_dev
from _util import bf16_round, f32

pytestmark = pytest.mark.gpu


def oracle_full(w, inp):
    return O.forward(f32(inp.q), f32(inp.k), f32(inp.v), f32(inp.p_q), f32(inp.p_k), f32(inp.g),
                     grid=(w.grid_t, w.grid_h, w.grid_w), block_q=w.block_q, block_k=w.block_k,
                     sparsity=w.sparsity, pairs=(w.pairs_t, w.pairs_h, w.pairs_w), rope_base=w.rope_base,
                     rms_eps=w.rms_eps)


def check_all(w, inp, ref, got):
    assert got["keep"] == ref["keep"]
    assert np.array_equal(got["map"], ref["map"]), "block map differs from the oracle"
    assert np.array_equal(got["map_fused"], ref["map"]), "fused-call block map differs from the oracle"
    assert_close(got["o_s"], ref["o_s"], "o_s")
    assert_close(got["C"], ref["C"], "C", max_abs=np.inf, rel_l2=TOL_C_REL_L2)
    assert_close(got["o_lr"], ref["o_lr"], "o_lr")
    assert_close(got["o"], ref["o"], "o (fused)")
    # the standalone gate is checked on the same bf16 O_s / O_lr it was given
    g = f32(inp.g).astype(np.float64)
    gg = g if g.ndim == 3 else g[:, :, None]
    assert_close(got["o_gate"], O.gate_fuse(got["o_s"], got["o_lr"], gg), "gate")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()


def test_tiny_named_layer():
    w = S.TINY
    inp = S.make_inputs(w)
    repair_gaps(inp, w)
    check_all(w, inp, oracle_full(w, inp), run_all(w, inp))


ODD = [
    # ragged tails: L not a multiple of 64 / 128
    S.TINY.replace(name="odd-3x7x11-d64", grid_t=3, grid_h=7, grid_w=11, sparsity=0.5, seed=11),
    S.TINY.replace(name="odd-3x7x11-d128-bq128-r32", grid_t=3, grid_h=7, grid_w=11, d=128, block_q=128,
                   rank=32, pairs_t=4, pairs_h=6, pairs_w=6, sparsity=0.6, seed=12),
    # k = 1 and k = N_kblk
    S.TINY.replace(name="keep-one", grid_t=2, grid_h=9, grid_w=30, sparsity=0.999, seed=13),
    S.TINY.replace(name="keep-all", grid_t=2, grid_h=9, grid_w=30, sparsity=0.0, seed=14),
    # batch > 1, several heads, r = 64, per-head gate
    S.TINY.replace(name="B2-H3-r64-gate-per-head", B=2, H=3, d=128, block_q=128, grid_t=4, grid_h=10,
                   grid_w=13, rank=64, pairs_t=8, pairs_h=12, pairs_w=12, sparsity=0.8, gate_per_head=1, seed=15),
    # single partial block
    S.TINY.replace(name="single-block", grid_t=1, grid_h=1, grid_w=37, sparsity=0.0, seed=16),
    # d = 128, r = 16, ragged: the state pass pools K with its smallest TMEM budget
    S.TINY.replace(name="d128-r16-ragged", d=128, block_q=128, rank=16, pairs_t=2, pairs_h=3, pairs_w=3,
                   grid_t=3, grid_h=9, grid_w=21, sparsity=0.7, seed=18),
    # d = 128 with block_q = 64: the unfused forward (standalone tcgen05 readout), ragged
    S.TINY.replace(name="d128-bq64-r32-ragged", d=128, block_q=64, rank=32, pairs_t=4, pairs_h=6, pairs_w=6,
                   grid_t=3, grid_h=7, grid_w=19, sparsity=0.8, seed=19),
    # d = 64 with block_q = 128, r = 32
    S.TINY.replace(name="d64-bq128-r32", block_q=128, rank=32, pairs_t=4, pairs_h=6, pairs_w=6, grid_t=3,
                   grid_h=12, grid_w=20, sparsity=0.9, seed=17),
    # d = 64 with an odd head count and B = 2: the state pass pairs heads, the last pair of each
    # batch has one head (the second reads zeros and writes nothing)
    S.TINY.replace(name="d64-B2-H3-r32-ragged", B=2, H=3, rank=32, pairs_t=4, pairs_h=6, pairs_w=6, grid_t=3,
                   grid_h=7, grid_w=23, sparsity=0.7, seed=20),
]


@pytest.mark.parametrize("w", ODD, ids=lambda w: w.name)
def test_odd_shapes(w):
    inp = S.make_inputs(w)
    repair_gaps(inp, w)
    check_all(w, inp, oracle_full(w, inp), run_all(w, inp))


def test_zero_gate_is_sparse_branch():
    """g = 0: the fused output is exactly the sparse branch (same fp32 row, one bf16 rounding)."""
    w = S.TINY
    inp = S.make_inputs(w)
    repair_gaps(inp, w)
    inp.g.zero_()
    got = run_all(w, inp)
    assert np.array_equal(got["o"], got["o_s"])
    assert np.array_equal(got["o_gate"], got["o_s"])


def test_deterministic():
    w = S.TINY.replace(name="det", grid_t=3, grid_h=16, grid_w=24, seed=21)
    inp = S.make_inputs(w)
    a = run_all(w, inp)
    b = run_all(w, inp)
    for key in ("map", "o_s", "o_lr", "C", "o", "o_gate"):
        assert np.array_equal(a[key], b[key]), key


@pytest.mark.parametrize("w", [S.TINY, S.TINY.replace(name="bq128", d=128, block_q=128, rank=32, pairs_t=4,
                                                      pairs_h=6, pairs_w=6)], ids=lambda w: w.name)
def test_bad_block_index_reported(w):
    p = sda.params_of(w)
    inp = S.make_inputs(w)
    d = to_dev(inp)
    ws = sda.Workspace(p)
    keep = sda.sda_keep_count(p)
    idx = torch.zeros((w.B, w.H, w.n_qblk, keep), dtype=torch.int32, device="cuda")
    idx[0, 0, 3, 2] = w.n_kblk + 5
    idx[0, 1, 0, 0] = -1
    o = torch.empty_like(d["q"])
    sda.sda_sparse_attn_fwd(p, d["q"], d["k"], d["v"], idx, o, ws.ptr, ws.nbytes)
    with pytest.raises(sda.SdaError):
        ws.check()
    ws.check()  # the status word is cleared by the read


def test_forward_host_matches_device():
    w = S.TINY.replace(name="host", grid_t=3, grid_h=10, grid_w=16, seed=22)
    inp = S.make_inputs(w)
    p = sda.params_of(w)
    got = run_all(w, inp, fused_only=True)
    n = sda.sda_forward_host_buffer_size(p)
    buf = torch.empty(n + 256, dtype=torch.uint8, device="cuda")
    ptr = buf.data_ptr() + (-buf.data_ptr()) % 256
    sda.sda_workspace_init(ptr, n)
    pins = {k: getattr(inp, k).pin_memory() for k in ("q", "k", "v", "p_q", "p_k", "g")}
    o_host = torch.empty_like(inp.q).pin_memory()
    sda.sda_forward_host(p, pins["q"], pins["k"], pins["v"], pins["p_q"], pins["p_k"], pins["g"], o_host, ptr, n)
    assert np.array_equal(f32(o_host), got["o"])


# ---------------------------------------------------------------------------
# full-size named layers, in the launch configuration the benchmark times
# ---------------------------------------------------------------------------

def _sample_rows(w, n, seed):
    rng = np.random.default_rng(seed)
    rows = np.stack([rng.integers(0, w.B, n), rng.integers(0, w.L, n), rng.integers(0, w.H, n)], axis=1)
    tail = np.array([[0, l, h] for h in (0, w.H - 1) for l in range(w.L - 3, w.L)])  # ragged last block
    head = np.array([[0, l, w.H // 2] for l in range(0, 3)])
    return np.concatenate([rows, tail, head])


@pytest.mark.slow
@pytest.mark.parametrize("w", [S.WAN13B_480P, S.WAN14B_480P, S.WAN14B_720P], ids=lambda w: w.name)
def test_named_layer_full_size(w):
    inp = S.make_inputs(w)
    repair_gaps(inp, w)
    got = run_all(w, inp)
    q, k, v = f32(inp.q), f32(inp.k), f32(inp.v)
    rows = _sample_rows(w, 384, seed=w.seed)
    ref = O.forward(q, k, v, f32(inp.p_q), f32(inp.p_k), f32(inp.g), grid=(w.grid_t, w.grid_h, w.grid_w),
                    block_q=w.block_q, block_k=w.block_k, sparsity=w.sparsity,
                    pairs=(w.pairs_t, w.pairs_h, w.pairs_w), rope_base=w.rope_base, rms_eps=w.rms_eps, rows=rows)
    assert np.array_equal(got["map"], ref["map"]), "block map differs from the oracle"
    assert np.array_equal(got["map_fused"], ref["map"]), "fused-call block map differs from the oracle"
    assert_close(got["C"], ref["C"], f"{w.name}: C", max_abs=np.inf, rel_l2=TOL_C_REL_L2)
    sel = (rows[:, 0], rows[:, 1], rows[:, 2])
    assert_close(got["o_s"][sel], ref["o_s"], f"{w.name}: sampled o_s")
    assert_close(got["o_lr"][sel], ref["o_lr"], f"{w.name}: sampled o_lr")
    assert_close(got["o"][sel], ref["o"], f"{w.name}: sampled o")


_SWEEP_PARITY = ("sweep-B2-L8192-s0.97-r64", "sweep-B1-L131072-s0.90-r16", "sweep-B1-L131072-s0.97-r32",
                 "sweep-B1-L65536-s0.97-r32", "sweep-B1-L65536-s0.90-r32")


@pytest.mark.parametrize("w", [w for w in S.sweep_points() if w.name in _SWEEP_PARITY], ids=lambda w: w.name)
def test_sweep_corner_full_size(w):
    """Sweep points at full size (B=2 with r=64; the 128k-token layer with r=16 and with r=32 at
    s=0.97; the 64k-token layer at s=0.97 and 0.90), sampled rows."""
    test_named_layer_full_size(w)


@pytest.mark.parametrize("n_kblk,sparsity", [(32, 0.9), (32, 0.5), (300, 0.9), (1000, 0.9), (1500, 0.9),
                                             (1500, 0.5), (2048, 0.9), (1000, 0.97), (1182, 0.97), (2048, 0.97),
                                             (2048, 0.96875)])
def test_selector_exact_ties(n_kblk, sparsity):
    """Closed form with exact score ties, over every selection width of the selector (the
    candidate path up to k = 64, including the widest rows it takes, and the full-row path above).

    Q is one constant vector q0 and every key block is constant, equal to base
    or to base + q0 (blocks b = 1 mod 3), so every pooled score of a row is
    exactly one of two values. The top-k rule (score descending, index
    ascending) keeps the lowest-index high blocks first, then the lowest-index
    low blocks; every query block gets the same map.
    """
    d, bk = 64, 64
    w = S.TINY.replace(name=f"ties-{n_kblk}", H=1, d=d, grid_t=1, grid_h=1, grid_w=n_kblk * bk, sparsity=sparsity)
    p = sda.params_of(w)
    keep = sda.sda_keep_count(p)
    g = torch.Generator().manual_seed(n_kblk)
    q0 = torch.rand(d, generator=g) + 0.5                   # positive entries: q0 . q0 > 0
    base = torch.randn(d, generator=g)
    high = (torch.arange(n_kblk) % 3) == 1
    kb = base[None, :] + high[:, None].float() * q0[None, :]  # [n_kblk, d]
    q = q0.to(torch.bfloat16).expand(1, w.L, 1, d).contiguous()
    k = kb.repeat_interleave(bk, dim=0).to(torch.bfloat16).reshape(1, w.L, 1, d).contiguous()
    hi_idx = torch.nonzero(high).flatten()
    lo_idx = torch.nonzero(~high).flatten()
    want = torch.sort(torch.cat([hi_idx, lo_idx])[:keep]).values.numpy()
    ws = sda.Workspace(p)
    idx = torch.full((1, 1, w.n_qblk, keep), -1, dtype=torch.int32, device="cuda")
    sda.sda_block_select(p, q.cuda(), k.cuda(), idx, ws.ptr, ws.nbytes)
    ws.check()
    got = idx.cpu().numpy()
    assert np.array_equal(got, np.broadcast_to(want, got.shape)), f"first row {got[0, 0, 0]} want {want}"
