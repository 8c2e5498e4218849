"""Input recipe: determinism, shapes and the gap repair (CPU)."""
import numpy as np
import torch

from sparse_rank_attention_block_b200 import synthetic as S

from _gap import min_gap, repair_gaps


def test_named_shapes():
    assert S.TINY.L == 2048 and S.TINY.n_kblk == 32
    assert S.WAN13B_480P.L == 32760 and S.WAN13B_480P.n_qblk == 256 and S.WAN13B_480P.n_kblk == 512
    assert S.WAN14B_720P.L == 75600 and S.WAN14B_720P.n_qblk == 591 and S.WAN14B_720P.n_kblk == 1182
    assert len(S.sweep_points()) == 90


def test_deterministic_and_normalised():
    w = S.TINY.replace(grid_t=1, grid_h=8, grid_w=16)
    a = S.make_inputs(w)
    b = S.make_inputs(w)
    for x, y in zip((a.q, a.k, a.v, a.p_q, a.p_k, a.g), (b.q, b.k, b.v, b.p_q, b.p_k, b.g)):
        assert torch.equal(x, y)
    assert a.q.dtype == torch.bfloat16 and a.q.shape == (1, 128, 2, 64)
    rms = a.q.float().pow(2).mean(-1).sqrt()
    assert torch.allclose(rms, torch.ones_like(rms), atol=1e-2)
    assert float(a.g.abs().max()) <= 0.1


def test_gap_repair_tiny():
    w = S.TINY
    inp = S.make_inputs(w)
    repair_gaps(inp, w)
    assert min_gap(inp, w) >= 1e-4
