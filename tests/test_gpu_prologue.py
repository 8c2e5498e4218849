"""GPU parity of the prologue (backbone Q/K RMSNorm + full-d 3D RoPE) and of
the chain it feeds, against the fp64 oracle.

Prologue bar: every bf16 output within its own rounding of the oracle's
value (|got - want| <= 2^-8 |want| + 1e-5: half an ulp of bf16 is 2^-9
relative; the rest covers the fp32 arithmetic). Chain bar: the north-star
output tolerances (max-abs 2e-2, relative L2 1e-2) on O, and the block map
equal to the oracle's on every row whose boundary gap is at least 1e-4 (the
selector decides on the bf16 rotated q/k on both sides).
"""
import numpy as np
import pytest
import torch

import oracle.sda_oracle as O
from sparse_rank_attention_block_b200 import sda, synthetic as S

from _gpu import TOL_MAX_ABS, TOL_REL_L2, assert_close, ensure_lib
from _util import f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()


def raw_inputs(w, seed):
    """Un-normalised q, k (the generator's V recipe scaled per token and head) and norm weights."""
    g = torch.Generator().manual_seed(seed)
    a = S.make_inputs(w, seed=seed)
    b = S.make_inputs(w, seed=seed + 1)
    scale = lambda: torch.exp(torch.randn((w.B, w.L, w.H, 1), generator=g))  # noqa: E731
    q_raw = (a.v.float() * scale()).to(torch.bfloat16)
    k_raw = (b.v.float() * scale()).to(torch.bfloat16)
    q_raw[0, 0, 0] = 0.0                      # a zero row
    w_q = (0.5 + torch.rand((w.H, w.d), generator=g)).to(torch.bfloat16)
    w_k = (0.5 + torch.rand((w.H, w.d), generator=g)).to(torch.bfloat16)
    return q_raw, k_raw, w_q, w_k, a


def run_prologue(w, q_raw, k_raw, w_q, w_k):
    p = sda.params_of(w)
    dev = [x.cuda() for x in (q_raw, k_raw, w_q, w_k)]
    outs = [torch.empty_like(dev[0]) for _ in range(4)]
    sda.sda_qk_prologue(p, *dev, *outs)
    torch.cuda.synchronize()
    return outs  # q_norm, k_norm, q_rot, k_rot (device)


def oracle_prologue(w, q_raw, k_raw, w_q, w_k):
    pos = O.grid_positions(w.grid_t, w.grid_h, w.grid_w)
    qn, qr = O.qk_prologue(f32(q_raw), f32(w_q), w.rms_eps, pos, w.rope_base)
    kn, kr = O.qk_prologue(f32(k_raw), f32(w_k), w.rms_eps, pos, w.rope_base)
    return qn, kn, qr, kr


SHAPES = [
    S.TINY.replace(name="pro-d64-ragged", grid_t=3, grid_h=5, grid_w=7, seed=41),
    S.TINY.replace(name="pro-d128-B2", B=2, H=3, d=128, block_q=128, rank=32, pairs_t=4, pairs_h=6, pairs_w=6,
                   grid_t=2, grid_h=9, grid_w=13, seed=42),
    S.TINY.replace(name="pro-d128-H40", H=40, d=128, block_q=128, rank=32, pairs_t=4, pairs_h=6, pairs_w=6,
                   grid_t=3, grid_h=4, grid_w=11, seed=43),
]


@pytest.mark.parametrize("w", SHAPES, ids=lambda w: w.name)
def test_prologue_matches_oracle(w):
    q_raw, k_raw, w_q, w_k, _ = raw_inputs(w, w.seed)
    got = [f32(x) for x in run_prologue(w, q_raw, k_raw, w_q, w_k)]
    want = oracle_prologue(w, q_raw, k_raw, w_q, w_k)
    for name, g_, w_ in zip(("q_norm", "k_norm", "q_rot", "k_rot"), got, want):
        err = np.abs(g_ - w_)
        bound = 2.0 ** -8 * np.abs(w_) + 1e-5
        assert np.all(err <= bound), f"{name}: worst excess {np.max(err - bound):.3g}"
    assert not got[0][0, 0, 0].any()         # the zero row stays zero


@pytest.mark.parametrize("w", SHAPES[1:], ids=lambda w: w.name)
def test_prologue_then_path(w):
    """Rotated q/k into the selector and the sparse branch, normalised q/k into the low-rank branch."""
    q_raw, k_raw, w_q, w_k, a = raw_inputs(w, w.seed + 100)
    p = sda.params_of(w)
    qn, kn, qr, kr = run_prologue(w, q_raw, k_raw, w_q, w_k)
    v, p_q, p_k, g = (x.cuda() for x in (a.v, a.p_q, a.p_k, a.g))
    ws = sda.Workspace(p)
    keep = sda.sda_keep_count(p)
    idx = torch.full((w.B, w.H, w.n_qblk, keep), -1, dtype=torch.int32, device="cuda")
    o_s, o_lr, o = (torch.empty_like(v) for _ in range(3))
    sda.sda_block_select(p, qr, kr, idx, ws.ptr, ws.nbytes)
    sda.sda_sparse_attn_fwd(p, qr, kr, v, idx, o_s, ws.ptr, ws.nbytes)
    sda.sda_lowrank_fwd(p, qn, kn, v, p_q, p_k, o_lr, None, ws.ptr, ws.nbytes)
    sda.sda_gate_fuse(p, o_s, o_lr, g, o)
    ws.check()
    torch.cuda.synchronize()

    # oracle chain; the prologue's outputs are bf16 at the interface, so the oracle rounds them too
    bf = lambda x: torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).float().numpy()  # noqa: E731
    qn_o, kn_o, qr_o, kr_o = (bf(x) for x in oracle_prologue(w, q_raw, k_raw, w_q, w_k))
    vv, pq, pk, gg = f32(a.v), f32(a.p_q), f32(a.p_k), f32(a.g)
    bmap, gap, _ = O.block_map(qr_o, kr_o, w.block_q, w.block_k, w.sparsity)
    axis, freq = O.rope_frequencies(w.pairs_t, w.pairs_h, w.pairs_w, w.rope_base)
    ang = O.rope_angles(O.grid_positions(w.grid_t, w.grid_h, w.grid_w), axis, freq)
    C = O.lowrank_state(kn_o, vv, pk, ang)
    o_s_o = O.sparse_attention(qr_o, kr_o, vv, bmap, w.block_q, w.block_k)
    o_lr_o = O.lowrank_readout(O.lowrank_features(qn_o, pq, ang[None, :, None, :]), C[:, None], w.rms_eps)
    o_o = O.gate_fuse(o_s_o, o_lr_o, gg[:, :, None])

    got_map = idx.cpu().numpy()
    clear = gap >= 1e-4
    assert clear.mean() > 0.9
    assert np.array_equal(got_map[clear], bmap[clear])
    assert_close(f32(o_lr), o_lr_o, "o_lr (normalised q/k)")
    if clear.all():
        assert_close(f32(o), o_o, "o (prologue chain)")
    else:
        rows = np.broadcast_to(clear[:, :, :, None], clear.shape + (w.block_q,))
        rows = rows.transpose(0, 2, 3, 1).reshape(w.B, -1, w.H)[:, : w.L]       # [B, L, H] rows of clear blocks
        assert_close(f32(o)[rows], o_o[rows], "o (prologue chain, clear rows)")
