"""Pins of the causal-window oracle (the autoregressive extension), CPU only.

Each test checks the oracle against something other than itself: the
bidirectional oracle (one chunk), dense masked attention from torch and a
masked linear-attention sum written as a matrix product (keep-all window),
the causality invariant (tokens of later chunks change nothing), and the
keep / padding rule.
"""
import math
import types

import numpy as np
import pytest
import torch

import oracle.sda_oracle as O

GRID = (4, 3, 11)      # T, Hg, Wg: 33 tokens per frame, L = 132
PAIRS = (1, 2, 1)      # r = 8


def _inputs(seed, B=2, H=2, d=16, r=8, grid=GRID):
    rng = np.random.default_rng(seed)
    L = grid[0] * grid[1] * grid[2]
    q = rng.standard_normal((B, L, H, d))
    k = rng.standard_normal((B, L, H, d))
    v = rng.standard_normal((B, L, H, d))
    p_q = rng.standard_normal((r, d)) / math.sqrt(d)
    p_k = rng.standard_normal((r, d)) / math.sqrt(d)
    g = rng.uniform(-0.5, 0.5, (B, L))
    return q, k, v, p_q, p_k, g


def _run(x, F, s=0.6, bq=8, bk=8, o=O):
    q, k, v, p_q, p_k, g = x
    return o.causal_forward(q, k, v, p_q, p_k, g, grid=GRID, block_q=bq, block_k=bk, sparsity=s,
                            pairs=PAIRS, causal_frames=F, rms_eps=1e-6)


def pin_one_chunk_is_the_bidirectional_method(o):
    x = _inputs(0)
    q, k, v, p_q, p_k, g = x
    got = _run(x, F=GRID[0], o=o)
    want = o.forward(q, k, v, p_q, p_k, g, grid=GRID, block_q=8, block_k=8, sparsity=0.6, pairs=PAIRS,
                     rms_eps=1e-6)
    assert np.array_equal(got["map"], want["map"])
    assert np.array_equal(got["gap"], want["gap"])
    assert np.allclose(got["C"][:, :, 0], want["C"], rtol=0, atol=1e-12)
    for key in ("o_s", "o_lr", "o"):
        assert np.allclose(got[key], want[key], rtol=0, atol=1e-12), key


def pin_keep_all_window_is_dense_masked_attention(o):
    """s = 0 keeps every candidate block: the sparse branch is softmax over
    keys of chunks <= the query's chunk (torch sdpa with a boolean mask), and
    the low-rank readout is RMSNorm of sum_j [chunk(j) <= chunk(i)] (q~_i . k~_j) v_j."""
    x = _inputs(1)
    q, k, v, p_q, p_k, g = x
    F = 1
    out = _run(x, F=F, s=0.0, o=o)
    B, L, H, d = q.shape
    Tc = F * GRID[1] * GRID[2]
    chunk = np.arange(L) // Tc
    mask = chunk[None, :] <= chunk[:, None]                                 # [L_q, L_k]
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(k).permute(0, 2, 1, 3)
    vt = torch.from_numpy(v).permute(0, 2, 1, 3)
    dense = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.from_numpy(mask))
    assert np.allclose(out["o_s"], dense.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-10)

    pos = o.grid_positions(*GRID)
    axis, freq = o.rope_frequencies(*PAIRS, 10000.0)
    ang = o.rope_angles(pos, axis, freq)
    qf = o.lowrank_features(q, p_q, ang[None, :, None, :])                  # [B, L, H, r]
    kf = o.lowrank_features(k, p_k, ang[None, :, None, :])
    a = np.einsum("blhr,bmhr->bhlm", qf, kf) * mask                         # masked (q~ . k~) matrix
    xs = np.einsum("bhlm,bmhd->blhd", a, v)
    o_lr = xs / np.sqrt(np.mean(xs * xs, axis=-1, keepdims=True) + 1e-6)
    assert np.allclose(out["o_lr"], o_lr, rtol=0, atol=1e-10)


def pin_later_chunks_change_nothing_before_them(o):
    """Rewriting every token of chunks > c leaves the map rows, gaps and outputs
    of chunks <= c bit-identical (the key block straddling hi_c is pooled over
    its visible tokens only), and does change chunk c + 1."""
    F = 1
    Tc = F * GRID[1] * GRID[2]
    base = _inputs(2)
    ref = _run(base, F=F, o=o)
    qb = o.causal_query_blocks(base[0].shape[1], Tc, 8)
    for c in range(GRID[0] // F - 1):
        hi = (c + 1) * Tc
        rng = np.random.default_rng(100 + c)
        x = [t.copy() for t in base]
        for t in x[:3]:
            t[:, hi:] = rng.standard_normal(t[:, hi:].shape)
        got = _run(x, F=F, o=o)
        rows = np.array([blk[2] <= c for blk in qb])
        assert np.array_equal(got["map"][:, :, rows], ref["map"][:, :, rows])
        assert np.array_equal(got["gap"][:, :, rows], ref["gap"][:, :, rows])
        assert np.array_equal(got["C"][:, :, :c + 1], ref["C"][:, :, :c + 1])
        for key in ("o_s", "o_lr", "o"):
            assert np.array_equal(got[key][:, :hi], ref[key][:, :hi]), (c, key)
            assert not np.allclose(got[key][:, hi:hi + Tc], ref[key][:, hi:hi + Tc]), (c, key)


def pin_keep_rule_and_padding(o):
    x = _inputs(3)
    out = _run(x, F=1, s=0.7, o=o)
    L = x[0].shape[1]
    Tc = GRID[1] * GRID[2]
    qb = o.causal_query_blocks(L, Tc, 8)
    assert len(qb) == 4 * math.ceil(Tc / 8)
    keep_max = o.keep_count(math.ceil(L / 8), 0.7)
    assert out["map"].shape[-1] == keep_max
    for a, (s0, s1, c) in enumerate(qb):
        assert s1 <= (c + 1) * Tc and s0 >= c * Tc
        n = math.ceil((c + 1) * Tc / 8)
        assert out["cand"][a] == n
        assert out["keep"][a] == o.keep_count(n, 0.7)
        rows = out["map"][:, :, a].reshape(-1, keep_max)
        kc = out["keep"][a]
        assert np.all(rows[:, kc:] == -1)
        assert np.all(np.diff(rows[:, :kc], axis=1) > 0)
        assert np.all((rows[:, :kc] >= 0) & (rows[:, :kc] < n))


def pin_rows_mode_matches_full(o):
    x = _inputs(4, B=1)
    full = _run(x, F=2, o=o)
    rng = np.random.default_rng(5)
    L = x[0].shape[1]
    rows = np.stack([np.zeros(20, dtype=np.int64), rng.integers(0, L, 20), rng.integers(0, 2, 20)], axis=1)
    q, k, v, p_q, p_k, g = x
    part = o.causal_forward(q, k, v, p_q, p_k, g, grid=GRID, block_q=8, block_k=8, sparsity=0.6, pairs=PAIRS,
                            causal_frames=2, rms_eps=1e-6, rows=rows)
    for key in ("o_s", "o_lr", "o"):
        assert np.allclose(part[key], full[key][rows[:, 0], rows[:, 1], rows[:, 2]], rtol=0, atol=1e-12)


PINS = [pin_one_chunk_is_the_bidirectional_method, pin_keep_all_window_is_dense_masked_attention,
        pin_later_chunks_change_nothing_before_them, pin_keep_rule_and_padding, pin_rows_mode_matches_full]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(O)


# plausible mistakes planted in copies of the oracle: each must fail a pin
MUTATIONS = {
    "edge_block_sees_later_chunk": ("km = block_means(k[:, :hi], block_k)",
                                    "km = block_means(k[:, :min(L, hi + block_k - 1)], block_k)[:, :, :-(-hi // block_k)]"),
    "keys_not_limited_to_window": ("keys = keys[keys < hi]", "keys = keys[keys < L]"),
    "state_one_token_short": ("lowrank_state(k[:, :hi], v[:, :hi], p_k, ang[:hi])",
                              "lowrank_state(k[:, :hi - 1], v[:, :hi - 1], p_k, ang[:hi - 1])"),
    "state_of_whole_sequence": ("lowrank_state(k[:, :hi], v[:, :hi], p_k, ang[:hi])",
                                "lowrank_state(k, v, p_k, ang)"),
    "previous_chunk_state": ("o_lr = lowrank_readout(qt, C[bi, hi, li // Tc], rms_eps)",
                             "o_lr = lowrank_readout(qt, C[bi, hi, np.maximum(li // Tc - 1, 0)], rms_eps)"),
    "query_blocks_from_token_zero": ("out.extend((s, min(c1, s + block_q), c) for s in range(c0, c1, block_q))",
                                     "out.extend((s, min(c1, s + block_q), c) for s in range(c0 - c0 % block_q, c1, block_q))"),
}


def _mutant(old, new):
    src = open(O.__file__).read()
    assert src.count(old) == 1, old
    mod = types.ModuleType("oracle_mutant")
    mod.__file__ = O.__file__
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name):
    mod = _mutant(*MUTATIONS[name])
    failed = 0
    for pin in PINS:
        try:
            pin(mod)
        except Exception:  # an assertion, or the mutant breaking outright
            failed += 1
    assert failed > 0, f"no pin caught {name}"
