"""GPU parity of the per-token FP8 E4M3 quantisation against its oracle.

Bar: byte-exact codes and bit-exact fp32 scales (the kernel and the oracle
take every rounding decision in IEEE float32 and E4M3 round-to-nearest-even).
Inputs are seeded synthetic bf16 tensors of the forward's [B, L, H, d] shape,
with zero tokens, signed zeros and per-token magnitudes from 2^-30 to 2^30.
"""
import numpy as np
import pytest
import torch

from oracle.fp8_quant import quant_fp8_per_token
from sparse_rank_attention_block_b200 import sda, synthetic as S

from _gpu import ensure_lib

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()


def make_x(w, seed):
    """bf16 [B, L, H, d]: the generator's V tensor with per-token magnitudes and edge rows."""
    x = S.make_inputs(w, seed=seed).v.float()
    g = torch.Generator().manual_seed(seed)
    mag = torch.pow(2.0, torch.randint(-30, 31, (w.B, w.L, 1, 1), generator=g).float())
    x = x * mag
    x[0, 0] = 0.0                     # a zero token
    if w.L > 2:
        x[0, 1, :, ::3] = -0.0        # signed zeros inside a live token
        x[0, 2] = 0.0
        x[0, 2, 0, 0] = -1e-30        # a token whose only nonzero entry is tiny
    return x.to(torch.bfloat16)


def run(w, x):
    p = sda.params_of(w)
    xd = x.cuda()
    xq = torch.empty(x.shape, dtype=torch.uint8, device="cuda")
    sc = torch.empty((w.B, w.L), dtype=torch.float32, device="cuda")
    sda.sda_quant_fp8(p, xd, xq, sc)
    torch.cuda.synchronize()
    return xq.cpu().numpy(), sc.cpu().numpy()


SHAPES = [
    S.TINY,                                                            # H*d = 128: one chunk per lane
    S.TINY.replace(name="h12-d128", B=2, H=12, d=128, grid_t=2, grid_h=5, grid_w=7),      # 1536
    S.TINY.replace(name="h40-d128", H=40, d=128, grid_t=3, grid_h=7, grid_w=11),          # 5120 (14B layer)
    S.TINY.replace(name="h128-d128", H=128, d=128, grid_t=1, grid_h=3, grid_w=5),         # 16384: the limit
    S.TINY.replace(name="h3-d64", H=3, d=64, grid_t=1, grid_h=1, grid_w=9),               # 192: ragged lanes
]


@pytest.mark.parametrize("w", SHAPES, ids=lambda w: w.name)
def test_quant_fp8_exact(w):
    x = make_x(w, seed=31)
    got_q, got_s = run(w, x)
    want_q, want_s = quant_fp8_per_token(x.float().numpy())
    assert np.array_equal(got_s.view(np.uint32), want_s.view(np.uint32)), "scales differ"
    bad = np.argwhere(got_q != want_q)
    assert bad.size == 0, f"{len(bad)} codes differ, first at {bad[:3].tolist()}"


def test_quant_fp8_full_size_sampled():
    """The 14B-720P layer's output shape ([1, 75600, 40, 128]); the oracle checks 2,000 sampled tokens."""
    w = S.WAN14B_720P
    x = make_x(w, seed=32)
    got_q, got_s = run(w, x)
    rng = np.random.default_rng(3)
    li = np.sort(np.concatenate([[0, 1, 2, w.L - 1], rng.choice(w.L, 2000, replace=False)]))
    xs = x[:, li].float().numpy()
    want_q, want_s = quant_fp8_per_token(xs)
    assert np.array_equal(got_s[:, li].view(np.uint32), want_s.view(np.uint32))
    assert np.array_equal(got_q[:, li], want_q)
