"""Pins of the FP8 (E4M3) per-token quantisation oracle (CPU only).

The encoder is checked against torch's float8_e4m3fn cast (a library routine
with round-to-nearest-even) on every value the cast handles without overflow,
against codes decoded by hand from the format definition, and the per-token
quantisation against its round-trip bound and its invariants.
"""
import numpy as np
import pytest
import torch

from oracle.fp8_quant import E4M3_MAX, e4m3_decode, e4m3_encode, quant_fp8_per_token


def torch_e4m3(y: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(y, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_every_code_round_trips():
    codes = np.arange(256, dtype=np.uint8)
    vals = e4m3_decode(codes)
    finite = ~np.isnan(vals)
    assert finite.sum() == 254                            # 0x7F and 0xFF are NaN
    assert np.array_equal(e4m3_encode(vals[finite]), codes[finite])
    assert e4m3_decode(np.uint8(0x7E)) == 448.0 and e4m3_decode(np.uint8(0x01)) == 2.0 ** -9


@pytest.mark.parametrize("table", [
    # value, code: hand-decoded from 1 sign / 4 exponent (bias 7) / 3 mantissa bits
    [(448.0, 0x7E), (-448.0, 0xFE), (1.0, 0x38), (0.5, 0x30), (1.75, 0x3E), (2.0 ** -6, 0x08),
     (2.0 ** -9, 0x01), (7 * 2.0 ** -9, 0x07), (0.0, 0x00), (-0.0, 0x80), (240.0, 0x77), (-3.5, 0xC6)],
])
def test_hand_decoded_codes(table):
    vals = np.array([v for v, _ in table], dtype=np.float32)
    want = np.array([c for _, c in table], dtype=np.uint8)
    assert np.array_equal(e4m3_encode(vals), want)


def test_ties_go_to_even_and_saturation():
    # 1 + 1/16 lies halfway between 1 (M=0) and 1.125 (M=1): even -> 1
    # 1 + 3/16 lies halfway between 1.125 (M=1) and 1.25 (M=2): even -> 1.25
    # 2^-10 lies halfway between 0 and 2^-9: even -> 0; 3 * 2^-10 -> 2^-8 (M=2)
    ties = np.array([1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10, 440.0, -440.0], dtype=np.float32)
    assert np.array_equal(e4m3_encode(ties), np.array([0x38, 0x3A, 0x00, 0x02, 0x7E, 0xFE], dtype=np.uint8))
    big = np.array([448.5, 463.9, 464.0, 1e6, 3e38, -1e6], dtype=np.float32)
    assert np.array_equal(e4m3_encode(big), np.array([0x7E] * 5 + [0xFE], dtype=np.uint8))


def test_matches_torch_cast_in_range():
    rng = np.random.default_rng(5)
    # every float32 midpoint and neighbour of every finite code, plus random values over all scales
    vals = e4m3_decode(np.arange(0x7F, dtype=np.uint8))                    # 0 .. 448
    mids = (vals[:-1] + vals[1:]) / 2
    eps = np.float32(2.0 ** -20)
    grid = np.concatenate([vals, mids, mids * (1 + eps), mids * (1 - eps)]).astype(np.float32)
    rand = (rng.standard_normal(200_000) * np.exp2(rng.uniform(-14, 8, 200_000))).astype(np.float32)
    y = np.concatenate([grid, -grid, rand])
    y = y[np.abs(y) <= E4M3_MAX]
    assert np.array_equal(e4m3_encode(y), torch_e4m3(y))


def test_per_token_round_trip_and_invariants():
    rng = np.random.default_rng(7)
    B, L, H, d = 2, 37, 3, 64
    x = (rng.standard_normal((B, L, H, d)) * np.exp2(rng.integers(-6, 6, (B, L, 1, 1)))).astype(np.float32)
    x = torch.from_numpy(x).to(torch.bfloat16).float().numpy()             # bf16 values
    x[0, 5] = 0.0                                                          # a zero token
    x[1, 3, 0, :4] = -0.0
    codes, scale = quant_fp8_per_token(x)
    assert codes.shape == x.shape and codes.dtype == np.uint8 and scale.shape == (B, L)
    rows = x.reshape(B, L, -1)
    amax = np.abs(rows).max(-1)
    nz = amax > 0
    assert np.array_equal(scale[nz], (amax[nz] / np.float32(448.0)).astype(np.float32))
    assert scale[0, 5] == 1.0 and not codes[0, 5].any()
    # the largest magnitude of every row maps to +-448
    c = codes.reshape(B, L, -1)
    top = np.take_along_axis(c, np.abs(rows).argmax(-1)[..., None], -1)[..., 0]
    assert np.all((top[nz] & 0x7F) == 0x7E)
    # round trip: half a quantum of E4M3 (2^-4 relative for normals, 2^-10 * scale below 2^-6 * scale)
    back = e4m3_decode(c) * scale[..., None]
    err = np.abs(back - rows)
    bound = np.maximum(np.abs(rows) * 2.0 ** -4, 2.0 ** -10 * scale[..., None]) * (1 + 1e-6)
    assert np.all(err <= bound)
    # sign of zero kept
    assert np.all(codes[1, 3, 0, :4] == 0x80)
