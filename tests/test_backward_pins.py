"""Pins of the backward oracle (gradients of the compensated sparse attention), CPU only.

The gradients are checked against things other than their own chain rule:
central finite differences of the forward oracle (every input, the map held
fixed by a clear top-k gap), torch autograd through an fp64 torch
transcription of the dense (s = 0) forward, and closed forms of the gate
(g = 0 removes the low-rank branch from every gradient but dg). Planted
mistakes in copies of the oracle must each fail a pin.
"""
import math
import types

import numpy as np
import pytest
import torch

import oracle.sda_backward as BW
import oracle.sda_oracle as O

GRID = (2, 3, 8)       # L = 48
PAIRS = (1, 1, 0)      # r = 4
KW = dict(grid=GRID, block_q=8, block_k=8, sparsity=0.5, pairs=PAIRS, rms_eps=1e-6)


def _draw(seed, B=1, H=2, d=8, r=4, gate_per_head=False):
    rng = np.random.default_rng(seed)
    L = GRID[0] * GRID[1] * GRID[2]
    q, k, v = (rng.standard_normal((B, L, H, d)) for _ in range(3))
    p_q = rng.standard_normal((r, d)) / math.sqrt(d)
    p_k = rng.standard_normal((r, d)) / math.sqrt(d)
    g = rng.uniform(-1.0, 1.0, (B, L, H) if gate_per_head else (B, L))
    dO = rng.standard_normal((B, L, H, d))
    return dict(q=q, k=k, v=v, p_q=p_q, p_k=p_k, g=g), dO


def _clear_inputs(gate_per_head=False):
    """First seed whose every top-k boundary gap is wide, so that the finite
    differences below never move the block map."""
    for seed in range(200):
        x, dO = _draw(seed, gate_per_head=gate_per_head)
        _, gap, _ = O.block_map(x["q"], x["k"], 8, 8, 0.5)
        if gap.min() > 2e-3:
            return x, dO
    raise AssertionError("no clear seed")


def _loss(o, x, dO, **kw):
    f = o.forward(x["q"], x["k"], x["v"], x["p_q"], x["p_k"], x["g"], **kw)
    return float(np.sum(f["o"] * dO)), f["map"]


def pin_finite_differences(bw, gate_per_head=False):
    x, dO = _clear_inputs(gate_per_head)
    got = bw.backward(x["q"], x["k"], x["v"], x["p_q"], x["p_k"], x["g"], dO, **KW)
    base_map = got["fwd"]["map"]
    rng = np.random.default_rng(11)
    names = {"q": "dq", "k": "dk", "v": "dv", "p_q": "dp_q", "p_k": "dp_k", "g": "dg"}
    for name, gname in names.items():
        grad = got[gname]
        flat = rng.choice(x[name].size, size=6, replace=False)
        for f in flat:
            idx = np.unravel_index(f, x[name].shape)
            hstep = 1e-5
            vals = []
            for sgn in (1.0, -1.0):
                xx = {kk: vv.copy() for kk, vv in x.items()}
                xx[name][idx] += sgn * hstep
                l, m = _loss(O, xx, dO, **KW)
                assert np.array_equal(m, base_map)
                vals.append(l)
            fd = (vals[0] - vals[1]) / (2 * hstep)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])


def pin_finite_differences_gate_per_head(bw):
    pin_finite_differences(bw, gate_per_head=True)


def pin_autograd_dense(bw):
    """s = 0 keeps every block: the whole forward as fp64 torch ops (dense SDPA,
    linear attention with the same rotation), differentiated by autograd."""
    x, dO = _draw(3)
    kw = dict(KW, sparsity=0.0)
    got = bw.backward(x["q"], x["k"], x["v"], x["p_q"], x["p_k"], x["g"], dO, **kw)
    t = {n: torch.tensor(a, dtype=torch.float64, requires_grad=True) for n, a in x.items()}
    B, L, H, d = x["q"].shape
    pos = O.grid_positions(*GRID)
    axis, freq = O.rope_frequencies(*PAIRS, 10000.0)
    ang = torch.tensor(O.rope_angles(pos, axis, freq))[None, :, None, :]   # [1, L, 1, r/2]

    def feats(z, P):
        u = z @ P.T
        f = torch.nn.functional.elu(u) + 1.0
        xe, xo = f[..., 0::2], f[..., 1::2]
        c, s = torch.cos(ang), torch.sin(ang)
        return torch.stack([xe * c - xo * s, xe * s + xo * c], dim=-1).flatten(-2)

    o_s = torch.nn.functional.scaled_dot_product_attention(
        t["q"].permute(0, 2, 1, 3), t["k"].permute(0, 2, 1, 3), t["v"].permute(0, 2, 1, 3)).permute(0, 2, 1, 3)
    qt, kt = feats(t["q"], t["p_q"]), feats(t["k"], t["p_k"])
    C = torch.einsum("blhr,blhd->bhrd", kt, t["v"])
    X = torch.einsum("blhr,bhrd->blhd", qt, C)
    o_lr = X / torch.sqrt(X.pow(2).mean(-1, keepdim=True) + 1e-6)
    r = torch.sqrt(o_s.pow(2).mean(-1))
    out = o_s + (t["g"][:, :, None] * r)[..., None] * o_lr
    (out * torch.tensor(dO)).sum().backward()
    for name, gname in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("p_q", "dp_q"), ("p_k", "dp_k"), ("g", "dg")):
        want = t[name].grad.numpy()
        assert np.allclose(got[gname], want, rtol=1e-9, atol=1e-11), name


def pin_closed_gate_removes_low_rank(bw):
    """g = 0: O = O_s, so P_q, P_k get no gradient, dq/dk/dv are the sparse
    branch's alone, and dg = r (dO . O_lr)."""
    x, dO = _draw(4)
    x["g"][:] = 0.0
    got = bw.backward(x["q"], x["k"], x["v"], x["p_q"], x["p_k"], x["g"], dO, **KW)
    assert not got["dp_q"].any() and not got["dp_k"].any()
    f = got["fwd"]
    dq, dk, dv = bw.sparse_attention_backward(x["q"], x["k"], x["v"], f["map"], 8, 8, dO)
    assert np.array_equal(got["dq"], dq) and np.array_equal(got["dk"], dk) and np.array_equal(got["dv"], dv)
    assert np.allclose(got["dg"], np.sum(f["r"][..., None] * dO * f["o_lr"], axis=(2, 3)), rtol=1e-13, atol=0)


CAUSAL_KW = dict(KW, causal_frames=1)   # two chunks of 24 tokens
# 16-token key blocks: block 1 straddles the chunk boundary (chunk 0 sees its
# first 8 keys); keep-all, so that every query block attends to it
CAUSAL_EDGE_KW = dict(KW, causal_frames=1, block_k=16, sparsity=0.0)


def _causal_clear_inputs(kw):
    """First seed whose causal top-k boundary gaps are all wide (any seed when every block is kept)."""
    for seed in range(300):
        x, dO = _draw(100 + seed)
        if kw["sparsity"] == 0.0:
            return x, dO
        _, gap, _, _ = O.causal_block_map(x["q"], x["k"], kw["block_q"], kw["block_k"], kw["sparsity"], 24)
        if gap.min() > 2e-3:
            return x, dO
    raise AssertionError("no clear seed")


def pin_causal_finite_differences(bw, kw=CAUSAL_KW):
    x, dO = _causal_clear_inputs(kw)
    got = bw.causal_backward(x["q"], x["k"], x["v"], x["p_q"], x["p_k"], x["g"], dO, **kw)
    base_map = got["fwd"]["map"]
    rng = np.random.default_rng(12)
    names = {"q": "dq", "k": "dk", "v": "dv", "p_q": "dp_q", "p_k": "dp_k", "g": "dg"}
    for name, gname in names.items():
        grad = got[gname]
        for f in rng.choice(x[name].size, size=6, replace=False):
            idx = np.unravel_index(f, x[name].shape)
            hstep = 1e-5
            vals = []
            for sgn in (1.0, -1.0):
                xx = {kk: vv.copy() for kk, vv in x.items()}
                xx[name][idx] += sgn * hstep
                fw = O.causal_forward(xx["q"], xx["k"], xx["v"], xx["p_q"], xx["p_k"], xx["g"], **kw)
                assert np.array_equal(fw["map"], base_map)
                vals.append(float(np.sum(fw["o"] * dO)))
            fd = (vals[0] - vals[1]) / (2 * hstep)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])


def pin_causal_finite_differences_edge_block(bw):
    pin_causal_finite_differences(bw, CAUSAL_EDGE_KW)


def pin_causal_one_chunk_is_bidirectional(bw):
    """A window of every frame is one chunk: the causal backward is the bidirectional one."""
    x, dO = _draw(5)
    a = bw.causal_backward(x["q"], x["k"], x["v"], x["p_q"], x["p_k"], x["g"], dO, **dict(KW, causal_frames=GRID[0]))
    b = bw.backward(x["q"], x["k"], x["v"], x["p_q"], x["p_k"], x["g"], dO, **KW)
    for name in ("dq", "dk", "dv", "dp_q", "dp_k", "dg"):
        assert np.allclose(a[name], b[name], rtol=1e-11, atol=1e-13), name


def pin_causal_later_chunks_inert(bw):
    """dO on chunk 0 alone: no token of chunk 1 influences chunk 0's outputs, so its
    dq, dk, dv are exactly zero; dO on chunk 1 alone reaches chunk 0's keys."""
    x, dO = _draw(6)
    d0 = dO.copy()
    d0[:, 24:] = 0.0
    got = bw.causal_backward(x["q"], x["k"], x["v"], x["p_q"], x["p_k"], x["g"], d0, **CAUSAL_KW)
    for name in ("dq", "dk", "dv"):
        assert not got[name][:, 24:].any(), name
        assert got[name][:, :24].any(), name
    d1 = dO.copy()
    d1[:, :24] = 0.0
    got = bw.causal_backward(x["q"], x["k"], x["v"], x["p_q"], x["p_k"], x["g"], d1, **CAUSAL_KW)
    assert got["dk"][:, :24].any() and got["dv"][:, :24].any()
    assert not got["dq"][:, :24].any()


PINS = [pin_finite_differences, pin_finite_differences_gate_per_head, pin_autograd_dense,
        pin_closed_gate_removes_low_rank, pin_causal_finite_differences, pin_causal_finite_differences_edge_block,
        pin_causal_one_chunk_is_bidirectional, pin_causal_later_chunks_inert]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(BW)


MUTATIONS = {
    "rotation_not_inverted": ("return O.rope_rotate(x, -ang)", "return O.rope_rotate(x, ang)"),
    "phi_prime_one": ("return np.where(u > 0, 1.0, np.exp(np.minimum(u, 0.0)))", "return np.ones_like(u)"),
    "rmsnorm_without_projection": ("return (dy - y * np.mean(dy * y, axis=-1, keepdims=True)) / rho",
                                   "return dy / rho"),
    "softmax_without_centring": ("ds = p * (dp - np.sum(doi * o, axis=1, keepdims=True))", "ds = p * dp"),
    "gate_ignores_r_path": ("do_s = dO + np.where(r > 0, dr / (d * safe), 0.0)[..., None] * o_s", "do_s = dO"),
    "dk_without_scale": ("return (ds @ kj) * scale, (ds.T @ qi) * scale, p.T @ doi",
                         "return (ds @ kj) * scale, ds.T @ qi, p.T @ doi"),
    "state_grad_to_v_transposed": ('dv_lr = np.einsum("bhrd,blhr->blhd", dC, kt)',
                                   'dv_lr = np.einsum("bhrd,blhr->blhd", dC[:, ::-1], kt)'),
    "causal_prefix_sum_instead_of_suffix": ("G = np.cumsum(dC[:, :, ::-1], axis=2)[:, :, ::-1]",
                                            "G = np.cumsum(dC, axis=2)"),
    "causal_keys_past_the_window": ("keys = keys[keys < hi]", "keys = keys"),
    "causal_state_of_the_wrong_chunk": ("Crow = C[:, :, chunk]                                                  # [B, H, L, r, d]",
                                        "Crow = C[:, :, np.minimum(chunk + 1, C.shape[2] - 1)]"),
}


def _mutant(old, new):
    src = open(BW.__file__).read()
    assert src.count(old) == 1, old
    mod = types.ModuleType("oracle.sda_backward_mutant")
    mod.__file__ = BW.__file__
    mod.__package__ = "oracle"
    exec(compile(src.replace(old, new), "sda_backward_mutant", "exec"), mod.__dict__)
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
