"""fp64 CPU oracle of the backward of the compensated sparse attention forward.

TEST INFRASTRUCTURE ONLY, like `oracle.sda_oracle`: only the tests, the
package's smoke check and the benchmark's CPU legs may import it.

Training with the method backpropagates through both branches: the sparse
warm-up adds the low-rank projections and the gate as new trained parameters
and needs a backward kernel of the sparse attention (H3 portability report,
sections 2.1 and 2.2; SparkDiffusion summary on robotworld.top, section 2.4:
the warm-up starts from a gate near zero). Given the upstream gradient dO of
the forward output (robotworld summary, section 2.1)

    O_i = O_s,i + g_i r_i O_lr,i,   r_i = RMS(O_s,i),   O_lr,i = X_i / rho_i,
    X_i = q~_i^T C,   rho_i = sqrt(mean_c X_i,c^2 + eps),   C = sum_j k~_j v_j^T,
    q~ = R(p) phi(P_q q),   k~ = R(p) phi(P_k k),
    O_s,i = sum_{j kept} softmax_j(q_i . k_j / sqrt(d)) v_j,

this module returns dq, dk, dv, dP_q, dP_k and dg, each step the chain rule of
one forward step taken in reverse order. The block map is piecewise constant
in the inputs and carries no gradient (the selection is held fixed, as in the
forward's own top-k); r_i = 0 rows (an all-zero sparse output) get no gradient
through r. Every step runs in float64.

Pins (tests/test_backward_pins.py): central finite differences of the scalar
loss sum(O * dO) through the forward oracle, for every input, on inputs whose
top-k gaps keep the map fixed; torch autograd through an fp64 torch
transcription of the dense (s = 0) forward; closed forms for the gate. The
causal-window backward (causal_backward) is pinned the same way through
sda_oracle.causal_forward, by its reduction to backward() when the window is
one chunk, and by causality (an upstream gradient on chunk 0 alone leaves every
later token's gradients exactly zero).
"""
from __future__ import annotations

import math

import numpy as np

from . import sda_oracle as O


def _rope_inverse(x: np.ndarray, ang: np.ndarray) -> np.ndarray:
    """R^T x: the transpose of a rotation by ang is the rotation by -ang."""
    return O.rope_rotate(x, -ang)


def _phi_prime(u: np.ndarray) -> np.ndarray:
    """d/du (elu(u) + 1) = 1 for u > 0, exp(u) otherwise."""
    return np.where(u > 0, 1.0, np.exp(np.minimum(u, 0.0)))


def gate_backward(o_s, o_lr, g, dO):
    """Backward of O = O_s + g r O_lr, r = RMS(O_s) over the last axis.

    Returns (d o_s, d o_lr, dg) with dg shaped like g broadcast to o_s[..., 0].
    dr = g (dO . O_lr); dO_s = dO + dr * O_s / (d r); dO_lr = g r dO; dg = r (dO . O_lr).
    """
    d = o_s.shape[-1]
    r = O.sparse_rms(o_s)
    dot = np.sum(dO * o_lr, axis=-1)
    dr = g * dot
    safe = np.where(r > 0, r, 1.0)
    do_s = dO + np.where(r > 0, dr / (d * safe), 0.0)[..., None] * o_s
    do_lr = (g * r)[..., None] * dO
    dg = r * dot
    return do_s, do_lr, dg


def rmsnorm_backward(x, eps: float, dy):
    """Backward of y = x / sqrt(mean(x^2) + eps) over the last axis:
    dx = (dy - y * mean(dy * y)) / rho."""
    rho = np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    y = x / rho
    return (dy - y * np.mean(dy * y, axis=-1, keepdims=True)) / rho


def features_backward(x, P, ang, dxt):
    """Backward of x~ = R(ang) phi(P x) for rows x [..., d] -> (dx [..., d], dP [r, d])."""
    x = np.asarray(x, dtype=np.float64)
    P = np.asarray(P, dtype=np.float64)
    u = x @ P.T
    du = _rope_inverse(dxt, ang) * _phi_prime(u)
    dx = du @ P
    dP = du.reshape(-1, du.shape[-1]).T @ x.reshape(-1, x.shape[-1])   # sum over every row
    return dx, dP


def _block_backward(qi, kj, vj, doi, scale: float):
    """One query block against its kept keys: s = q_i . k_j / sqrt(d), P = softmax_j(s),
    o_i = sum_j P_ij v_j; dP_ij = do_i . v_j, ds_ij = P_ij (dP_ij - do_i . o_i).
    Returns (dq_i = sum_j ds_ij k_j / sqrt(d), the per-key dk_j = sum_i ds_ij q_i / sqrt(d)
    and dv_j = sum_i P_ij do_i)."""
    s = (qi @ kj.T) * scale
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    o = p @ vj
    dp = doi @ vj.T
    ds = p * (dp - np.sum(doi * o, axis=1, keepdims=True))
    return (ds @ kj) * scale, (ds.T @ qi) * scale, p.T @ doi


def sparse_attention_backward(q, k, v, bmap, block_q: int, block_k: int, do_s):
    """Backward of the block-sparse softmax attention with a fixed map: every
    query block's _block_backward, the key-side terms added to the keys of its
    kept blocks.
    """
    B, L, H, d = q.shape
    scale = 1.0 / math.sqrt(d)
    dq = np.zeros((B, L, H, d))
    dk = np.zeros((B, L, H, d))
    dv = np.zeros((B, L, H, d))
    for b in range(B):
        for h in range(H):
            for a, (s0, s1) in enumerate(O.block_ranges(L, block_q)):
                keys = O.kept_keys(bmap[b, h, a], L, block_k)
                qi = np.asarray(q[b, s0:s1, h], dtype=np.float64)
                kj = np.asarray(k[b, keys, h], dtype=np.float64)
                vj = np.asarray(v[b, keys, h], dtype=np.float64)
                doi = np.asarray(do_s[b, s0:s1, h], dtype=np.float64)
                gq, gk, gv = _block_backward(qi, kj, vj, doi, scale)
                dq[b, s0:s1, h] += gq
                np.add.at(dk[b, :, h], keys, gk)
                np.add.at(dv[b, :, h], keys, gv)
    return dq, dk, dv


def causal_sparse_attention_backward(q, k, v, bmap, block_q: int, block_k: int, chunk_tokens: int, do_s):
    """The same for the causal window: query blocks tile each chunk on their
    own, a block of chunk c attends to the keys below hi_c = (c + 1) Tc of its
    kept blocks (-1 entries of the map are padding)."""
    B, L, H, d = q.shape
    scale = 1.0 / math.sqrt(d)
    dq = np.zeros((B, L, H, d))
    dk = np.zeros((B, L, H, d))
    dv = np.zeros((B, L, H, d))
    for b in range(B):
        for h in range(H):
            for a, (s0, s1, c) in enumerate(O.causal_query_blocks(L, chunk_tokens, block_q)):
                hi = min(L, (c + 1) * chunk_tokens)
                row = bmap[b, h, a]
                keys = O.kept_keys(row[row >= 0], L, block_k)
                keys = keys[keys < hi]
                qi = np.asarray(q[b, s0:s1, h], dtype=np.float64)
                kj = np.asarray(k[b, keys, h], dtype=np.float64)
                vj = np.asarray(v[b, keys, h], dtype=np.float64)
                doi = np.asarray(do_s[b, s0:s1, h], dtype=np.float64)
                gq, gk, gv = _block_backward(qi, kj, vj, doi, scale)
                dq[b, s0:s1, h] += gq
                np.add.at(dk[b, :, h], keys, gk)
                np.add.at(dv[b, :, h], keys, gv)
    return dq, dk, dv


def backward(q, k, v, p_q, p_k, g, dO, *, grid, block_q, block_k, sparsity, pairs, rope_base=10000.0,
             rms_eps=1e-6):
    """Gradients of sum(O * dO) with respect to q, k, v, P_q, P_k and g.

    Same keyword arguments as the forward oracle; dO like q. Returns a dict
    with 'dq', 'dk', 'dv' ([B, L, H, d]), 'dp_q', 'dp_k' ([r, d]), 'dg' (like
    g: [B, L] summed over heads, or [B, L, H]) and the forward dict 'fwd'.
    """
    B, L, H, d = q.shape
    fwd = O.forward(q, k, v, p_q, p_k, g, grid=grid, block_q=block_q, block_k=block_k, sparsity=sparsity,
                    pairs=pairs, rope_base=rope_base, rms_eps=rms_eps)
    pos = O.grid_positions(*grid)
    axis, freq = O.rope_frequencies(*pairs, rope_base)
    ang = O.rope_angles(pos, axis, freq)                                   # [L, r/2]
    angb = ang[None, :, None, :]
    g = np.asarray(g, dtype=np.float64)
    gg = g if g.ndim == 3 else np.broadcast_to(g[:, :, None], (B, L, H))
    dO = np.asarray(dO, dtype=np.float64)

    # gate
    do_s, do_lr, dg_full = gate_backward(fwd["o_s"], fwd["o_lr"], gg, dO)
    dg = dg_full if g.ndim == 3 else dg_full.sum(axis=2)

    # low-rank readout: O_lr = RMSNorm(X), X = q~^T C
    C = fwd["C"]                                                           # [B, H, r, d]
    qt = O.lowrank_features(q, p_q, angb)                                  # [B, L, H, r]
    X = np.einsum("blhr,bhrd->blhd", qt, C)
    dX = rmsnorm_backward(X, rms_eps, do_lr)
    dqt = np.einsum("bhrd,blhd->blhr", C, dX)
    dC = np.einsum("blhr,blhd->bhrd", qt, dX)
    dq_lr, dp_q = features_backward(q, p_q, angb, dqt)

    # state: C = sum_j k~_j v_j^T
    kt = O.lowrank_features(k, p_k, angb)
    dv_lr = np.einsum("bhrd,blhr->blhd", dC, kt)
    dkt = np.einsum("bhrd,blhd->blhr", dC, np.asarray(v, dtype=np.float64))
    dk_lr, dp_k = features_backward(k, p_k, angb, dkt)

    # sparse branch
    dq_s, dk_s, dv_s = sparse_attention_backward(q, k, v, fwd["map"], block_q, block_k, do_s)

    return {"dq": dq_s + dq_lr, "dk": dk_s + dk_lr, "dv": dv_s + dv_lr, "dp_q": dp_q, "dp_k": dp_k,
            "dg": dg, "fwd": fwd}


def causal_backward(q, k, v, p_q, p_k, g, dO, *, grid, block_q, block_k, sparsity, pairs, causal_frames,
                    rope_base=10000.0, rms_eps=1e-6):
    """Gradients of sum(O * dO) for the causal-window forward (sda_oracle.causal_forward).

    Row i of chunk c reads the prefix state C_c = sum_{j < hi_c} k~_j v_j^T, so
    dC_c = sum over the rows of chunk c of q~_i dX_i^T, and key j (chunk c_j)
    enters every C_c with c >= c_j: it receives the suffix sum G_{c_j} =
    sum_{c >= c_j} dC_c, i.e. dv_j += G^T k~_j and dk~_j = G v_j. The gate,
    RMSNorm and feature steps are those of backward(); the sparse branch is
    causal_sparse_attention_backward. Same keyword arguments as
    causal_forward; returns the keys of backward() ('fwd' is the causal forward dict).
    """
    B, L, H, d = q.shape
    Tc = O.causal_chunk_tokens(grid, causal_frames)
    fwd = O.causal_forward(q, k, v, p_q, p_k, g, grid=grid, block_q=block_q, block_k=block_k, sparsity=sparsity,
                           pairs=pairs, causal_frames=causal_frames, rope_base=rope_base, rms_eps=rms_eps)
    pos = O.grid_positions(*grid)
    axis, freq = O.rope_frequencies(*pairs, rope_base)
    ang = O.rope_angles(pos, axis, freq)
    angb = ang[None, :, None, :]
    g = np.asarray(g, dtype=np.float64)
    gg = g if g.ndim == 3 else np.broadcast_to(g[:, :, None], (B, L, H))
    dO = np.asarray(dO, dtype=np.float64)
    chunk = np.arange(L) // Tc                                             # chunk of every token

    # gate
    do_s, do_lr, dg_full = gate_backward(fwd["o_s"], fwd["o_lr"], gg, dO)
    dg = dg_full if g.ndim == 3 else dg_full.sum(axis=2)

    # low-rank readout against the row's prefix state
    C = fwd["C"]                                                           # [B, H, NC, r, d]
    Crow = C[:, :, chunk]                                                  # [B, H, L, r, d]
    qt = O.lowrank_features(q, p_q, angb)                                  # [B, L, H, r]
    X = np.einsum("blhr,bhlrd->blhd", qt, Crow)
    dX = rmsnorm_backward(X, rms_eps, do_lr)
    dqt = np.einsum("bhlrd,blhd->blhr", Crow, dX)
    dC = np.stack([np.einsum("blhr,blhd->bhrd", qt[:, chunk == c], dX[:, chunk == c])
                   for c in range(C.shape[2])], axis=2)                    # [B, H, NC, r, d]
    dq_lr, dp_q = features_backward(q, p_q, angb, dqt)

    # prefix states: key j feeds C_c for every c >= chunk(j)
    G = np.cumsum(dC[:, :, ::-1], axis=2)[:, :, ::-1]
    Grow = G[:, :, chunk]                                                  # [B, H, L, r, d]
    kt = O.lowrank_features(k, p_k, angb)
    dv_lr = np.einsum("bhlrd,blhr->blhd", Grow, kt)
    dkt = np.einsum("bhlrd,blhd->blhr", Grow, np.asarray(v, dtype=np.float64))
    dk_lr, dp_k = features_backward(k, p_k, angb, dkt)

    # sparse branch
    dq_s, dk_s, dv_s = causal_sparse_attention_backward(q, k, v, fwd["map"], block_q, block_k, Tc, do_s)

    return {"dq": dq_s + dq_lr, "dk": dk_s + dk_lr, "dv": dv_s + dv_lr, "dp_q": dp_q, "dp_k": dp_k,
            "dg": dg, "fwd": fwd}
