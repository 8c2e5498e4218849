"""Pins of the prologue oracle (backbone Q/K RMSNorm + full-d 3D RoPE), CPU only."""
import numpy as np

import oracle.sda_oracle as O


def _case(seed=0, B=2, L=30, H=3, d=64, grid=(2, 3, 5)):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, L, H, d)) * rng.uniform(0.1, 10.0, (B, L, H, 1))
    w = rng.uniform(0.5, 1.5, (H, d))
    pos = O.grid_positions(*grid)
    return x, w, pos


def test_pair_split():
    assert O.full_rope_pairs(64) == (8, 12, 12)
    assert O.full_rope_pairs(128) == (16, 24, 24)


def test_norm_closed_form_and_weight_after_norm():
    x, w, pos = _case()
    eps = 1e-3
    xn, _ = O.qk_prologue(x, w, eps, pos, 10000.0)
    ms = np.mean(x * x, axis=-1)
    # dividing the weight back out leaves mean square ms / (ms + eps) exactly
    got = np.mean((xn / w) ** 2, axis=-1)
    assert np.allclose(got, ms / (ms + eps), rtol=1e-12, atol=0)
    # scale invariance of the normalisation without eps
    xn0, _ = O.qk_prologue(x, w, 0.0, pos, 10000.0)
    xn1, _ = O.qk_prologue(7.5 * x, w, 0.0, pos, 10000.0)
    assert np.allclose(xn0, xn1, rtol=1e-12, atol=1e-14)


def test_rotation_as_complex_multiplication():
    """Pair m of a token is multiplied by exp(i * angle), angle = coordinate * base^(-mu/n) of its axis."""
    x, w, pos = _case(seed=1, d=64)
    xn, xr = O.qk_prologue(x, w, 1e-6, pos, 10000.0)
    d = x.shape[-1]
    counts = O.full_rope_pairs(d)
    ang = np.zeros((pos.shape[0], d // 2))
    m = 0
    for ax, n in enumerate(counts):
        for mu in range(n):
            ang[:, m] = pos[:, ax] * 10000.0 ** (-mu / n)
            m += 1
    z = xn[..., 0::2] + 1j * xn[..., 1::2]
    zr = z * np.exp(1j * ang)[None, :, None, :]
    assert np.allclose(xr[..., 0::2], zr.real, atol=1e-12)
    assert np.allclose(xr[..., 1::2], zr.imag, atol=1e-12)


def test_rotation_invariants():
    x, w, pos = _case(seed=2, d=128, grid=(3, 4, 5), L=60)
    xn, xr = O.qk_prologue(x, w, 1e-6, pos, 10000.0)
    # every pair keeps its length; the origin token is not rotated
    assert np.allclose(np.hypot(xr[..., 0::2], xr[..., 1::2]), np.hypot(xn[..., 0::2], xn[..., 1::2]), atol=1e-12)
    assert np.allclose(xr[:, 0], xn[:, 0], atol=0)
    # dot products depend only on relative positions: shift every position by one constant
    shifted = pos + np.array([2, 1, 3])
    _, xs = O.qk_prologue(x, w, 1e-6, shifted, 10000.0)
    a = np.einsum("blhd,bmhd->bhlm", xr, xr)
    b = np.einsum("blhd,bmhd->bhlm", xs, xs)
    assert np.allclose(a, b, rtol=1e-10, atol=1e-9)
