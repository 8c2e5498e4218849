"""CPU oracle of the per-token FP8 (E4M3) activation quantisation.

TEST INFRASTRUCTURE ONLY: the plain definition the CUDA quantisation kernel is
checked against. Only the tests, the smoke check of the package entry file and
the CPU-baseline leg of the benchmark may import it; the library never does.

What is computed (SparkDiffusion summary on robotworld.top, section 2.3,
"FP8 quantisation and fused kernels"): activations feeding the linear
projections are quantised to FP8 E4M3 with a scale chosen per token at run
time, scale and cast done in one pass over memory. The pages fix neither the
scale formula nor the rounding; the readings used here (the plainest ones
that the section's per-token dynamic E4M3 scheme supports):

* a token's row is its H*d channels of the [B, L, H, d] tensor (the input of
  the output projection is [B*L, H*d]);
* amax = max_c |x_c|; the codes are E4M3(x_c * (448 / amax)) and the stored
  scale is amax / 448 (x_c ~ code_c * scale), both quotients and the product
  taken in float32 with round-to-nearest-even, so 448 (the largest finite
  E4M3 value) is the image of the row's largest magnitude;
* E4M3 rounding is to nearest, ties to even mantissa, saturating at +-448
  (no infinities; the all-ones pattern is NaN and is never produced); the
  sign of zero is kept;
* a row of zeros gets scale 1 and zero codes.

E4M3 (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits): exponent
field E in 1..15 gives (1 + M/8) * 2^(E-7), E = 0 gives (M/8) * 2^-6; the
largest finite value is 1.75 * 2^8 = 448 (E = 15, M = 6).

Parity pins (tests/test_fp8_pins.py): the encoder against torch's
float8_e4m3fn cast for every in-range value on a dense grid and at random,
hand-decoded table values and ties, saturation, and the per-token round trip.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def e4m3_encode(y) -> np.ndarray:
    """Round float32 values to E4M3 codes (uint8): nearest, ties to even, saturating."""
    y = np.asarray(y, dtype=np.float32).astype(np.float64)
    sign = np.signbit(y)
    a = np.abs(y)
    code = np.zeros(a.shape, dtype=np.uint8)
    sat = a >= E4M3_MAX                     # [448, 464) rounds to 448 anyway; beyond saturates
    small = a < 2.0 ** -6                   # subnormal range: quantum 2^-9
    normal = ~sat & ~small & (a > 0)
    # subnormals (and values that round up into the smallest normal): m in 0..8
    m_sub = np.rint(a[small] / 2.0 ** -9)   # exact quotient, rint = ties to even
    # normals: a in [2^e, 2^(e+1)), quantum 2^(e-3)
    _, ex = np.frexp(a[normal])             # a = f * 2^ex, f in [0.5, 1)
    e = ex - 1
    m = np.rint(a[normal] / np.ldexp(1.0, e - 3))   # 8..16
    up = m >= 16                            # rounded into the next binade
    e = np.where(up, e + 1, e)
    m = np.where(up, 8, m)
    c_norm = ((e + 7).astype(np.int64) << 3) | (m.astype(np.int64) - 8)
    c_norm = np.minimum(c_norm, 0x7E)       # 448 at most (e = 8, m = 14)
    c_sub = np.where(m_sub >= 8, 1 << 3, m_sub.astype(np.int64))  # 8 * 2^-9 = 2^-6: E = 1, M = 0
    code[normal] = c_norm.astype(np.uint8)
    code[small] = c_sub.astype(np.uint8)
    code[sat] = 0x7E
    code = np.where(sign, code | 0x80, code).astype(np.uint8)
    return code


def e4m3_decode(code) -> np.ndarray:
    """E4M3 codes (uint8) to float64 values (the NaN pattern decodes to NaN)."""
    c = np.asarray(code, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    E = (c >> 3) & 0xF
    M = c & 0x7
    v = np.where(E == 0, M / 8.0 * 2.0 ** -6, (1.0 + M / 8.0) * np.ldexp(1.0, E - 7))
    v = np.where((E == 15) & (M == 7), np.nan, v)
    return s * v


def quant_fp8_per_token(x):
    """Per-token E4M3 quantisation of x [..., L, H, d] (bf16 values).

    Returns (codes uint8 [..., L, H, d], scale float32 [..., L]).
    """
    x = np.asarray(x, dtype=np.float32)
    lead = x.shape[:-2]
    rows = x.reshape(lead + (-1,))                                   # [..., H*d]
    amax = np.max(np.abs(rows), axis=-1).astype(np.float32)          # exact: max of float32 values
    zero = amax == 0
    safe = np.where(zero, np.float32(1.0), amax).astype(np.float32)
    inv = np.where(zero, np.float32(0.0), np.float32(E4M3_MAX) / safe).astype(np.float32)   # float32 quotient
    scale = np.where(zero, np.float32(1.0), safe / np.float32(E4M3_MAX)).astype(np.float32)
    y = (rows * inv[..., None]).astype(np.float32)                   # float32 product
    codes = e4m3_encode(y).reshape(x.shape)
    return codes, scale
