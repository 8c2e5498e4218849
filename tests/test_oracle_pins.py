"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each `pin_*` function takes the oracle module, so that the mutation tests at
the bottom can re-run the same pins against copies of the oracle with a
plausible mistake planted in them and check that some pin catches it.
"""
import json
import math
import os
import types

import numpy as np
import pytest
import torch

import oracle.sda_oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))
RNG = np.random.default_rng(1234)


def _rand(*shape, seed=0):
    return np.random.default_rng(seed).standard_normal(shape)


def _sdpa(q, k, v, mask=None):
    """Dense softmax(QK^T/sqrt(d))V from torch (fp64), q/k/v [L, d] or [H, L, d]."""
    tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(x)) for x in (q, k, v))
    m = None if mask is None else torch.from_numpy(mask)
    return torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=m).numpy()


# ---------------------------------------------------------------------------
# pins
# ---------------------------------------------------------------------------

def pin_keep_ratio_golden(o):
    """topk keep ratio <-> sparsity and the 97 %/90 % compute ratio printed on the pages."""
    with open(os.path.join(HERE, "golden", "keep_ratio.json")) as f:
        gold = json.load(f)
    for topk, s in gold["topk_keep_ratio_to_sparsity"]:
        for n in (100, 512, 1182, 4096):
            k = o.keep_count(n, s)
            assert abs(k / n - topk) <= 1.0 / n + 1e-12, (n, s, k)
    n = gold["compute_ratio_check_blocks"]
    ratio = o.keep_count(n, 0.97) / o.keep_count(n, 0.90)
    assert abs(ratio - gold["compute_ratio_97_vs_90"]) < 0.02, ratio


def pin_keep_count_closed_form(o):
    """Exact products: (1-s)*N integral gives exactly that many; clamps at the ends."""
    assert o.keep_count(32, 0.75) == 8
    assert o.keep_count(10, 0.9) == 1
    assert o.keep_count(100, 0.9) == 10
    assert o.keep_count(512, 0.0) == 512
    assert o.keep_count(7, 0.999) == 1
    assert o.keep_count(7, 0.5) == 4          # 3.5 -> 4


def pin_positions_raster(o):
    """l = (t*Hg + h)*Wg + w."""
    pos = o.grid_positions(3, 4, 5)
    assert pos.shape == (60, 3)
    for t in range(3):
        for h in range(4):
            for w in range(5):
                assert tuple(pos[(t * 4 + h) * 5 + w]) == (t, h, w)


def pin_block_means_brute_force(o):
    """Pooled score S[a,b] equals the mean of all token-pair dot products q_i.k_j."""
    B, L, H, d = 1, 150, 2, 8          # blocks of 64: 64, 64, 22 (partial)
    q = _rand(B, L, H, d, seed=1)
    k = _rand(B, L, H, d, seed=2)
    S = o.block_scores(o.block_means(q, 64), o.block_means(k, 32))
    ra, rb = o.block_ranges(L, 64), o.block_ranges(L, 32)
    assert S.shape == (B, H, len(ra), len(rb))
    for h in range(H):
        for a, (a0, a1) in enumerate(ra):
            for b, (b0, b1) in enumerate(rb):
                tot = 0.0
                for i in range(a0, a1):
                    for j in range(b0, b1):
                        tot += float(np.dot(q[0, i, h], k[0, j, h]))
                assert abs(S[0, h, a, b] - tot / ((a1 - a0) * (b1 - b0))) < 1e-12


def pin_topk_by_rank_counting(o):
    """Block b is kept iff fewer than k blocks precede it in (score desc, index asc)."""
    rng = np.random.default_rng(7)
    for trial in range(20):
        n = int(rng.integers(2, 40))
        keep = int(rng.integers(1, n + 1))
        s = np.round(rng.standard_normal(n), 1)       # coarse values -> many exact ties
        m, gap = o.select_blocks(s[None, :], keep)
        expect = [b for b in range(n)
                  if sum(1 for c in range(n) if s[c] > s[b] or (s[c] == s[b] and c < b)) < keep]
        assert list(m[0]) == expect
        assert list(m[0]) == sorted(m[0])


def pin_topk_ties_lower_index(o):
    """Identical key blocks score identically; the lower indices win."""
    B, L, H, d = 1, 256, 1, 4
    q = np.ones((B, L, H, d))
    k = np.ones((B, L, H, d))
    k[:, 64:128] = 2.0                       # block 1 best, blocks 0, 2, 3 tie
    m, gap, keep = o.block_map(q, k, 64, 64, 0.5)
    assert keep == 2
    assert list(m[0, 0, 0]) == [0, 1]
    assert list(m[0, 0, 3]) == [0, 1]


def pin_sparse_equals_dense_at_s0(o):
    """With every block kept the sparse branch is softmax(QK^T/sqrt(d))V."""
    B, L, H, d = 1, 200, 2, 16
    q, k, v = (_rand(B, L, H, d, seed=s) for s in (3, 4, 5))
    m, _, keep = o.block_map(q, k, 64, 32, 0.0)
    assert keep == 7
    os_ = o.sparse_attention(q, k, v, m, 64, 32)
    ref = _sdpa(q[0].transpose(1, 0, 2), k[0].transpose(1, 0, 2), v[0].transpose(1, 0, 2))
    assert np.max(np.abs(os_[0].transpose(1, 0, 2) - ref)) < 1e-12


def pin_sparse_equals_masked_dense(o):
    """A hand-built map equals dense attention with the matching boolean mask."""
    B, L, H, d = 1, 230, 2, 8
    bq, bk = 64, 32
    q, k, v = (_rand(B, L, H, d, seed=s) for s in (6, 7, 8))
    nq, nk = -(-L // bq), -(-L // bk)
    rng = np.random.default_rng(9)
    keep = 3
    m = np.stack([np.stack([np.sort(rng.choice(nk, keep, replace=False)) for _ in range(nq)])
                  for _ in range(H)])[None].astype(np.int32)
    m[0, 0, nq - 1] = [0, 3, nk - 1]           # include the partial last key block
    os_ = o.sparse_attention(q, k, v, m, bq, bk)
    for h in range(H):
        mask = np.zeros((L, L), dtype=bool)
        for i in range(L):
            for b in m[0, h, i // bq]:
                mask[i, b * bk:min(L, (b + 1) * bk)] = True
        ref = _sdpa(q[0, :, h], k[0, :, h], v[0, :, h], mask)
        assert np.max(np.abs(os_[0, :, h] - ref)) < 1e-12
    rows = np.array([[0, 5, 1], [0, 229, 0], [0, 130, 1]])
    sub = o.sparse_attention(q, k, v, m, bq, bk, rows=rows)
    for n, (b, l, h) in enumerate(rows):
        assert np.max(np.abs(sub[n] - os_[b, l, h])) < 1e-13


def pin_single_block_constant_v(o):
    """One kept block whose V rows are all equal returns that row exactly."""
    B, L, H, d = 1, 128, 1, 8
    q, k = _rand(B, L, H, d, seed=10), _rand(B, L, H, d, seed=11)
    v = _rand(B, L, H, d, seed=12)
    row = _rand(d, seed=13)
    v[0, 64:128, 0] = row
    m = np.array([[[[1], [1]]]], dtype=np.int32)
    os_ = o.sparse_attention(q, k, v, m, 64, 64)
    assert np.max(np.abs(os_[0, :, 0] - row)) < 1e-14


def pin_elu_plus_one(o):
    x = np.linspace(-6, 6, 1001)
    ref = torch.nn.functional.elu(torch.from_numpy(x)).numpy() + 1.0
    assert np.max(np.abs(o.elu_plus_one(x) - ref)) < 1e-15


def pin_rope_closed_form(o):
    """Angle = coordinate * base^(-mu/n), axes in t, h, w order, counter-clockwise."""
    axis, freq = o.rope_frequencies(2, 3, 3, 10000.0)
    assert list(axis) == [0, 0, 1, 1, 1, 2, 2, 2]
    # pair 0 (t, mu=0) turns by t rad; pair 1 (t, mu=1 of 2) by t/100;
    # pair 3 (h, mu=1 of 3) by h * 10000^(-1/3); pair 5 (w, mu=0) by w rad.
    pos = np.array([[1, 0, 0], [3, 0, 0], [0, 2, 0], [0, 0, 5]])
    ang = o.rope_angles(pos, axis, freq)
    assert abs(ang[0, 0] - 1.0) < 1e-15
    assert abs(ang[1, 1] - 0.03) < 1e-15
    assert abs(ang[2, 3] - 2 * 10000.0 ** (-1.0 / 3.0)) < 1e-15
    assert abs(ang[3, 5] - 5.0) < 1e-15
    assert np.all(ang[3, :5] == 0) and np.all(ang[0, 2:] == 0)
    e = np.zeros(16)
    e[0] = 1.0                                     # unit x of pair 0
    out = o.rope_rotate(e[None, :], ang[0:1])
    assert np.allclose(out[0, :2], [math.cos(1.0), math.sin(1.0)], atol=1e-15, rtol=0)
    y = np.zeros(16)
    y[11] = 1.0                                    # unit y of pair 5 (components 10, 11)
    out = o.rope_rotate(y[None, :], ang[3:4])      # token at w = 5: pair 5 turns by 5 rad
    assert np.allclose(out[0, 10:12], [-math.sin(5.0), math.cos(5.0)], atol=1e-15, rtol=0)
    assert np.max(np.abs(np.delete(out[0], [10, 11]))) == 0.0


def pin_rope_invariants(o):
    """Rotation keeps norms; feature products depend on relative position only."""
    axis, freq = o.rope_frequencies(4, 6, 6, 10000.0)
    pos = np.random.default_rng(3).integers(0, 50, size=(40, 3))
    x = _rand(40, 32, seed=14)
    ang = o.rope_angles(pos, axis, freq)
    y = o.rope_rotate(x, ang)
    assert np.max(np.abs(np.linalg.norm(y, axis=1) - np.linalg.norm(x, axis=1))) < 1e-13
    shift = np.array([7, -3, 11])
    y2 = o.rope_rotate(x, o.rope_angles(pos + shift, axis, freq))
    assert np.max(np.abs(y @ y.T - y2 @ y2.T)) < 1e-12


def pin_lowrank_associativity(o):
    """q~^T C with C = sum_j k~_j v_j^T equals the O(L^2) sum_j (q~.k~_j) v_j."""
    B, L, H, d, r = 1, 60, 2, 8, 6
    q, k, v = (_rand(B, L, H, d, seed=s) for s in (15, 16, 17))
    pq, pk = _rand(r, d, seed=18) / 3, _rand(r, d, seed=19) / 3
    pos = o.grid_positions(3, 4, 5)
    axis, freq = o.rope_frequencies(1, 1, 1, 10000.0)
    ang = o.rope_angles(pos, axis, freq)
    C = o.lowrank_state(k, v, pk, ang)
    for h in range(H):
        qt = o.lowrank_features(q[0, :, h], pq, ang)
        kt = o.lowrank_features(k[0, :, h], pk, ang)
        for i in range(0, L, 7):
            x = np.zeros(d)
            for j in range(L):
                x += float(np.dot(qt[i], kt[j])) * v[0, j, h]
            ref = x / math.sqrt(np.mean(x * x) + 1e-6)
            got = o.lowrank_readout(qt[i], C[0, h], 1e-6)
            assert np.max(np.abs(got - ref)) < 1e-12


def pin_zero_frequency_is_linear_attention(o):
    """With all RoPE frequencies zero, features are phi(P x) (torch elu) and
    the branch is unrotated linear attention with an RMSNorm readout."""
    B, L, H, d, r = 1, 48, 1, 8, 4
    q, k, v = (_rand(B, L, H, d, seed=s) for s in (20, 21, 22))
    g = np.zeros((B, L))
    pq, pk = _rand(r, d, seed=23) / 2, _rand(r, d, seed=24) / 2
    res = o.forward(q, k, v, pq, pk, g, grid=(2, 4, 6), block_q=16, block_k=16, sparsity=0.5,
                    pairs=(1, 1, 0), freq_override=np.zeros(2))
    tq = torch.from_numpy(q[0, :, 0])
    tk = torch.from_numpy(k[0, :, 0])
    fq = torch.nn.functional.elu(tq @ torch.from_numpy(pq).T) + 1
    fk = torch.nn.functional.elu(tk @ torch.from_numpy(pk).T) + 1
    x = (fq @ fk.T) @ torch.from_numpy(v[0, :, 0])
    ref = x / torch.sqrt((x * x).mean(-1, keepdim=True) + 1e-6)
    assert np.max(np.abs(res["o_lr"][0, :, 0] - ref.numpy())) < 1e-12


def pin_readout_unit_rms(o):
    x = _rand(50, 16, seed=25) * 3
    C = np.eye(16)
    y = o.lowrank_readout(x, C, 1e-6)
    rms = np.sqrt(np.mean(y * y, axis=-1))
    assert np.max(np.abs(rms - 1.0)) < 1e-6


def _small_problem(gate):
    B, L, H, d, r = 1, 96, 2, 8, 6
    q, k, v = (_rand(B, L, H, d, seed=s) for s in (30, 31, 32))
    pq, pk = _rand(r, d, seed=33) / 3, _rand(r, d, seed=34) / 3
    g = gate(B, L)
    kw = dict(grid=(2, 6, 8), block_q=32, block_k=16, sparsity=0.5, pairs=(1, 1, 1))
    return q, k, v, pq, pk, g, kw


def pin_gate_zero(o):
    """g = 0 gives exactly the sparse branch."""
    q, k, v, pq, pk, g, kw = _small_problem(lambda B, L: np.zeros((B, L)))
    res = o.forward(q, k, v, pq, pk, g, **kw)
    assert np.array_equal(res["o"], res["o_s"])


def pin_gate_homogeneous_in_v(o):
    """O(alpha V) = alpha O(V): r scales with V, RMSNorm(q~^T C) does not."""
    q, k, v, pq, pk, g, kw = _small_problem(lambda B, L: np.random.default_rng(5).uniform(-1, 1, (B, L)))
    a = o.forward(q, k, v, pq, pk, g, **kw)["o"]
    b = o.forward(q, k, 2.5 * v, pq, pk, g, **kw)["o"]
    assert np.max(np.abs(b - 2.5 * a)) < 1e-5 * np.max(np.abs(a))
    assert np.max(np.abs(b - a)) > 0.1


def pin_gate_closed_form(o):
    """Constant sparse rows c give r = |c|; O = c + g |c| O_lr."""
    os_ = np.full((3, 8), -0.5)
    olr = _rand(3, 8, seed=35)
    g = np.array([0.1, -0.2, 0.0])
    out = o.gate_fuse(os_, olr, g)
    assert np.max(np.abs(out - (os_ + (g * 0.5)[:, None] * olr))) < 1e-15


def pin_rows_mode_matches_full(o):
    q, k, v, pq, pk, g, kw = _small_problem(lambda B, L: np.random.default_rng(6).uniform(-1, 1, (B, L)))
    full = o.forward(q, k, v, pq, pk, g, **kw)
    rows = np.array([[0, 0, 0], [0, 95, 1], [0, 40, 1], [0, 63, 0]])
    sub = o.forward(q, k, v, pq, pk, g, rows=rows, **kw)
    for n, (b, l, h) in enumerate(rows):
        for key in ("o_s", "o_lr", "o"):
            assert np.max(np.abs(sub[key][n] - full[key][b, l, h])) < 1e-13


PINS = [pin_keep_ratio_golden, pin_keep_count_closed_form, pin_positions_raster,
        pin_block_means_brute_force, pin_topk_by_rank_counting, pin_topk_ties_lower_index,
        pin_sparse_equals_dense_at_s0, pin_sparse_equals_masked_dense, pin_single_block_constant_v,
        pin_elu_plus_one, pin_rope_closed_form, pin_rope_invariants, pin_lowrank_associativity,
        pin_zero_frequency_is_linear_attention, pin_readout_unit_rms, pin_gate_zero,
        pin_gate_homogeneous_in_v, pin_gate_closed_form, pin_rows_mode_matches_full]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(O)


# ---------------------------------------------------------------------------
# mutation checks: plausible mistakes planted in copies of the oracle
# ---------------------------------------------------------------------------

MUTATIONS = {
    "dropped_softmax_scale": ("s = (qi @ kj.T) * scale", "s = (qi @ kj.T)"),
    "mean_over_full_block": ("/ (e - s)", "/ block"),
    "ties_to_higher_index": ("np.lexsort((idx, -s))", "np.lexsort((-idx, -s))"),
    "rotation_sign": ("out[..., 0::2] = xe * c - xo * s", "out[..., 0::2] = xe * c + xo * s"),
    "frequency_exponent": ("freq.append(float(base) ** (-mu / n))", "freq.append(float(base) ** (-2 * mu / n))"),
    "phi_without_one": ("np.where(u > 0, u + 1.0,", "np.where(u > 0, u,"),
    "state_reversed_tokens": ("C[b, h] = kt.T @ np.asarray(v[b, :, h]", "C[b, h] = kt.T @ np.asarray(v[b, ::-1, h]"),
    "rmsnorm_sum_not_mean": ("np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)",
                             "np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)"),
    "gate_without_rms": ("(np.asarray(g, dtype=np.float64) * r)[..., None]",
                         "(np.asarray(g, dtype=np.float64) * 1.0)[..., None]"),
    "axes_h_w_swapped": ("for ax, n in enumerate((pairs_t, pairs_h, pairs_w))",
                         "for ax, n in zip((0, 2, 1), (pairs_t, pairs_h, pairs_w))"),
    "raster_h_w_swapped": ("w = l % grid_w", "w = (l // grid_h) % grid_w"),
    "keep_floor": ("math.ceil((1.0 - float(sparsity)) * n_kblk - 1e-6)",
                   "math.floor((1.0 - float(sparsity)) * n_kblk)"),
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
    old, new = MUTATIONS[name]
    mod = _mutant(old, new)
    caught = []
    for pin in PINS:
        try:
            pin(mod)
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches the planted mistake {name}"
