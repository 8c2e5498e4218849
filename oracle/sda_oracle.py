"""fp64 CPU oracle of the compensated sparse attention forward.

TEST INFRASTRUCTURE ONLY. This module is the plain, slow, obviously correct
definition that the CUDA path is checked against. Only the tests, the smoke
check of the package entry file and the CPU-baseline leg of the benchmark may
import it; the library itself never does, and shares no code with it.

What is computed (SparkDiffusion summary on robotworld.top, section 2.1,
"compensated sparse attention"):

    dense attention        A(Q,K,V) = softmax(Q K^T / sqrt(d)) V
    compensated form       A~ = A_M(Q,K,V) + g (.) C_psi(Q,K,V)
    low-rank features      q~_i = R_r(p_i) phi(P_q q_i),  k~_j = R_r(p_j) phi(P_k k_j)
    global state           C = sum_j k~_j v_j^T
    low-rank readout       O_lr,i = RMSNorm(q~_i^T C)
    gate fusion            O_i = O_s,i + g_i r_i O_lr,i,  r_i = RMS(O_s,i)

Readings where the pages leave a step open (each the plainest reading that
the rest of the pages supports):

* block selection (A_M): mean-pool Q per query block and K per key block over
  the valid tokens of the block, score pooled pairs by their dot product, keep
  the k = ceil((1 - s) * N_kblk - 1e-6) best key blocks per query block
  (clamped to [1, N_kblk]), ties to the lower block index, one map per
  (batch, head); kept indices are returned in ascending order;
* the sparse branch is softmax restricted to the union of kept key blocks,
  renormalised over that set, scale 1/sqrt(d);
* phi = elu + 1; P_q, P_k are [r, d] matrices shared by all heads, no bias;
* R_r: r/2 adjacent pairs (2m, 2m+1); the first pairs_t pairs rotate by the
  token's t coordinate, the next pairs_h by h, the rest by w; inside an axis
  with n pairs, pair mu turns by angle pos * base^(-mu / n);
  (x, y) -> (x cos a - y sin a, x sin a + y cos a);
* C sums over every valid token of the (batch, head);
* RMSNorm(x) = x / sqrt(mean_c x_c^2 + eps), no learned weight;
* r_i = sqrt(mean_c O_s,i,c^2), no eps, from the unrounded sparse output;
  g is per token [B, L] (broadcast over heads) or per token and head [B, L, H].
* token positions come from the (T, Hg, Wg) grid in raster order;
* the causal-window variant (robotworld summary, section 4) groups tokens into
  chunks of F whole latent frames; the queries of chunk c see exactly the
  prefix of chunks 0..c, and every step is the bidirectional method on that
  prefix (query blocks tile each chunk, the key block straddling the prefix
  end is pooled over its visible tokens, keep counts follow each chunk's
  candidate count, the state is the prefix sum). The causal functions at the
  end of this module state it in full.

Parity pins: every function here is checked against something other than
itself (dense attention from torch, brute-force sums, closed-form rotations,
invariants) by the CPU tests of the repository; the RoPE frequency schedule
and pairing are a reading the pages do not fix, so beyond internal
consistency that convention is parity unpinned.

Inputs are the bf16 tensors decoded exactly (to float32 or float64); every
step below runs in float64.
"""
from __future__ import annotations

import math

import numpy as np


# ---------------------------------------------------------------------------
# positions and block geometry
# ---------------------------------------------------------------------------

def grid_positions(grid_t: int, grid_h: int, grid_w: int) -> np.ndarray:
    """(L, 3) int64 grid coordinates (t, h, w) of raster-ordered tokens.

    Token l sits at l = (t * grid_h + h) * grid_w + w: the 3D (t, h, w)
    position p_i that the rank-truncated 3D RoPE rotates by (robotworld
    summary, section 2.1, feature equation).
    """
    L = grid_t * grid_h * grid_w
    l = np.arange(L, dtype=np.int64)
    w = l % grid_w
    h = (l // grid_w) % grid_h
    t = l // (grid_w * grid_h)
    return np.stack([t, h, w], axis=1)


def block_ranges(L: int, block: int):
    """[(start, stop)] token ranges of the ceil(L / block) contiguous blocks."""
    return [(s, min(L, s + block)) for s in range(0, L, block)]


def keep_count(n_kblk: int, sparsity: float) -> int:
    """Kept key blocks per query block.

    The sparse branch keeps a 1 - s fraction of query-key blocks (robotworld
    summary, sections 1 and 2.1); the launch scripts' `topk` argument is that
    keep ratio, 0.1 / 0.05 / 0.03 for 90 / 95 / 97 % sparsity (SparkDiffusion
    README, "single-sample inference"). Reading: k = ceil((1 - s) * N - 1e-6)
    clamped to [1, N]; the 1e-6 keeps e.g. (1 - 0.9) * 10 from rounding up to 2.
    """
    k = math.ceil((1.0 - float(sparsity)) * n_kblk - 1e-6)
    return max(1, min(n_kblk, k))


# ---------------------------------------------------------------------------
# block selector (A_M's mask)
# ---------------------------------------------------------------------------

def block_means(x: np.ndarray, block: int) -> np.ndarray:
    """Mean of x over each token block, per (batch, head).

    x: [B, L, H, d] (exact decode of bf16). Returns [B, H, N, d] float64,
    N = ceil(L / block); a partial last block is averaged over its valid
    tokens only. Block-level scoring is one of the selectors the summary lists
    for A_M (robotworld summary, section 2.1).
    """
    B, L, H, d = x.shape
    ranges = block_ranges(L, block)
    out = np.empty((B, H, len(ranges), d), dtype=np.float64)
    for n, (s, e) in enumerate(ranges):
        out[:, :, n, :] = np.asarray(x[:, s:e], dtype=np.float64).sum(axis=1) / (e - s)
    return out


def block_scores(q_mean: np.ndarray, k_mean: np.ndarray) -> np.ndarray:
    """S[b, h, a, c] = dot(Qbar[b, h, a], Kbar[b, h, c]); no scale (ranking only)."""
    return np.matmul(q_mean, np.swapaxes(k_mean, -1, -2))


def select_blocks(scores: np.ndarray, keep: int):
    """Top-`keep` key blocks of every score row, ties to the lower index.

    scores: [..., Nk]. Returns (block_map [..., keep] int32 ascending,
    gap [...] float64), where gap is the relative boundary gap
    (S_(k) - S_(k+1)) / max_c |S[c]| of each row (inf when keep == Nk).
    """
    Nk = scores.shape[-1]
    flat = scores.reshape(-1, Nk)
    maps = np.empty((flat.shape[0], keep), dtype=np.int32)
    gaps = np.full(flat.shape[0], np.inf)
    idx = np.arange(Nk)
    for row in range(flat.shape[0]):
        s = flat[row]
        # order by (score descending, index ascending)
        order = np.lexsort((idx, -s))
        maps[row] = np.sort(order[:keep])
        if keep < Nk:
            scale = np.max(np.abs(s))
            gaps[row] = (s[order[keep - 1]] - s[order[keep]]) / scale if scale > 0 else 0.0
    return maps.reshape(scores.shape[:-1] + (keep,)), gaps.reshape(scores.shape[:-1])


def block_map(q: np.ndarray, k: np.ndarray, block_q: int, block_k: int, sparsity: float):
    """Pool, score and select: returns (map [B,H,Nq,keep], gap [B,H,Nq], keep)."""
    qm = block_means(q, block_q)
    km = block_means(k, block_k)
    keep = keep_count(km.shape[2], sparsity)
    m, gap = select_blocks(block_scores(qm, km), keep)
    return m, gap, keep


# ---------------------------------------------------------------------------
# sparse branch A_M
# ---------------------------------------------------------------------------

def kept_keys(block_row: np.ndarray, L: int, block_k: int) -> np.ndarray:
    """Token indices of the union of the kept key blocks of one query block."""
    return np.concatenate([np.arange(b * block_k, min(L, (b + 1) * block_k)) for b in block_row])


def softmax_attend(qi, kj, vj, scale: float) -> np.ndarray:
    """softmax_j(q_i . k_j * scale) v_j for the query rows qi over the key set (kj, vj)."""
    qi = np.asarray(qi, dtype=np.float64)
    kj = np.asarray(kj, dtype=np.float64)
    vj = np.asarray(vj, dtype=np.float64)
    s = (qi @ kj.T) * scale
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return (p @ vj) / p.sum(axis=1, keepdims=True)


def sparse_attention(q, k, v, bmap, block_q: int, block_k: int, rows=None) -> np.ndarray:
    """O_s = softmax over kept keys of q_i k_j / sqrt(d), times V.

    The dense attention softmax(Q K^T / sqrt(d)) V of the summary (section
    2.1) restricted to the key blocks the map keeps for the query's block,
    renormalised over that set.

    q, k, v: [B, L, H, d]; bmap: [B, H, Nq, keep]. rows: None for all
    (b, l, h), else an int array [n, 3] of (b, l, h) triples; returns
    [B, L, H, d] or [n, d] float64.
    """
    B, L, H, d = q.shape
    scale = 1.0 / math.sqrt(d)

    def one_group(b, h, a, ls):
        keys = kept_keys(bmap[b, h, a], L, block_k)
        return softmax_attend(q[b, ls, h], k[b, keys, h], v[b, keys, h], scale)

    if rows is None:
        out = np.empty((B, L, H, d), dtype=np.float64)
        for b in range(B):
            for h in range(H):
                for a, (s0, s1) in enumerate(block_ranges(L, block_q)):
                    out[b, s0:s1, h] = one_group(b, h, a, np.arange(s0, s1))
        return out
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 3)
    out = np.empty((rows.shape[0], d), dtype=np.float64)
    # rows of the same (b, h, query block) share their key set: one group each
    group = (rows[:, 0] * H + rows[:, 2]) * (L // block_q + 1) + rows[:, 1] // block_q
    for gid in np.unique(group):
        sel = np.nonzero(group == gid)[0]
        b, l, h = rows[sel[0]]
        out[sel] = one_group(b, h, l // block_q, rows[sel, 1])
    return out


# ---------------------------------------------------------------------------
# low-rank branch C_psi
# ---------------------------------------------------------------------------

def elu_plus_one(u: np.ndarray) -> np.ndarray:
    """phi(u) = elu(u) + 1 = u + 1 for u > 0, exp(u) otherwise."""
    return np.where(u > 0, u + 1.0, np.exp(np.minimum(u, 0.0)))


def rope_frequencies(pairs_t: int, pairs_h: int, pairs_w: int, base: float):
    """Per rotation pair m: (axis index 0/1/2 for t/h/w, angular frequency).

    Inside an axis with n pairs, pair mu has frequency base^(-mu / n).
    """
    axis, freq = [], []
    for ax, n in enumerate((pairs_t, pairs_h, pairs_w)):
        for mu in range(n):
            axis.append(ax)
            freq.append(float(base) ** (-mu / n))
    return np.array(axis, dtype=np.int64), np.array(freq, dtype=np.float64)


def rope_angles(pos: np.ndarray, axis: np.ndarray, freq: np.ndarray) -> np.ndarray:
    """Rotation angle of every pair: pos[..., axis[m]] * freq[m]; pos [..., 3] -> [..., r/2]."""
    return np.asarray(pos, dtype=np.float64)[..., axis] * freq


def rope_rotate(x: np.ndarray, ang: np.ndarray) -> np.ndarray:
    """Rank-truncated 3D RoPE R_r(p): rotate pair (2m, 2m+1) of x by ang[..., m].

    (x, y) -> (x cos a - y sin a, x sin a + y cos a). The rotation sits outside
    the non-linearity, which keeps relative space-time geometry (H3
    portability report, section 1, RoLA row; robotworld summary, section 2.1).
    x: [..., r], ang broadcastable to [..., r/2].
    """
    c = np.cos(ang)
    s = np.sin(ang)
    xe = x[..., 0::2]
    xo = x[..., 1::2]
    out = np.empty(x.shape, dtype=np.float64)
    out[..., 0::2] = xe * c - xo * s
    out[..., 1::2] = xe * s + xo * c
    return out


def lowrank_features(x: np.ndarray, P: np.ndarray, ang: np.ndarray) -> np.ndarray:
    """x~ = R_r(p) phi(P x): x [..., d], P [r, d], ang [..., r/2] -> [..., r]."""
    u = np.asarray(x, dtype=np.float64) @ np.asarray(P, dtype=np.float64).T
    return rope_rotate(elu_plus_one(u), ang)


def lowrank_state(k: np.ndarray, v: np.ndarray, p_k: np.ndarray, ang: np.ndarray) -> np.ndarray:
    """C[b, h] = sum_j k~_j v_j^T over all tokens j of (b, h): returns [B, H, r, d].

    k, v: [B, L, H, d]; ang: [L, r/2] angles of the L tokens.
    """
    B, L, H, d = k.shape
    r = p_k.shape[0]
    C = np.empty((B, H, r, d), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            kt = lowrank_features(k[b, :, h], p_k, ang)                  # [L, r]
            C[b, h] = kt.T @ np.asarray(v[b, :, h], dtype=np.float64)  # sum over j
    return C


def rms_norm(x: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) over the last axis, no weight."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def lowrank_readout(q_tilde: np.ndarray, C: np.ndarray, eps: float) -> np.ndarray:
    """O_lr,i = RMSNorm(q~_i^T C) over the d channels.

    q_tilde: [..., r]; C: [..., r, d] broadcast against it (e.g. the state of
    each row's (batch, head)). Returns [..., d].
    """
    x = np.einsum("...r,...rd->...d", q_tilde, C)
    return rms_norm(x, eps)


# ---------------------------------------------------------------------------
# gate fusion
# ---------------------------------------------------------------------------

def sparse_rms(o_s: np.ndarray) -> np.ndarray:
    """r_i = sqrt(mean_c O_s,i,c^2), the RMS of the sparse output, no eps."""
    return np.sqrt(np.mean(o_s * o_s, axis=-1))


def gate_fuse(o_s: np.ndarray, o_lr: np.ndarray, g: np.ndarray) -> np.ndarray:
    """O_i = O_s,i + g_i r_i O_lr,i (robotworld summary, section 2.1, last equation).

    o_s, o_lr: [..., d]; g broadcast against o_s[..., 0].
    """
    r = sparse_rms(o_s)
    return o_s + (np.asarray(g, dtype=np.float64) * r)[..., None] * o_lr


# ---------------------------------------------------------------------------
# prologue (the step before the path): backbone Q/K RMSNorm + full-d 3D RoPE
# ---------------------------------------------------------------------------

def full_rope_pairs(d: int):
    """Split of the d/2 rotation pairs of the full-d 3D RoPE over (t, h, w).

    The same pattern as the rank-truncated rotation (a quarter of the pairs to
    t, three eighths each to h and w): (d/8, 3d/16, 3d/16).
    """
    return d // 8, 3 * d // 16, 3 * d // 16


def qk_prologue(x_raw: np.ndarray, w: np.ndarray, eps: float, pos: np.ndarray, base: float):
    """Backbone RMSNorm and full-d 3D RoPE of a query or key tensor.

    The low-rank branch reuses the backbone's normalised q/k and the sparse
    branch attends with the rotated ones (robotworld summary, section 2.1,
    "reuse the backbone's normalised query/key before attention"; H3
    portability report, section 2.1, fused_qkv_rope). Per (token, head):
    x_norm = x / sqrt(mean_c x_c^2 + eps) * w (w: the backbone's learned
    weight, [H, d]), x_rot = RoPE_d(p) x_norm over all d/2 pairs.
    x_raw: [B, L, H, d]; pos: [L, 3] grid positions. Returns (x_norm, x_rot).
    """
    x = np.asarray(x_raw, dtype=np.float64)
    d = x.shape[-1]
    x_norm = rms_norm(x, eps) * np.asarray(w, dtype=np.float64)
    axis, freq = rope_frequencies(*full_rope_pairs(d), base)
    ang = rope_angles(pos, axis, freq)                                   # [L, d/2]
    x_rot = rope_rotate(x_norm, ang[None, :, None, :])
    return x_norm, x_rot


# ---------------------------------------------------------------------------
# the whole forward
# ---------------------------------------------------------------------------

def forward(q, k, v, p_q, p_k, g, *, grid, block_q, block_k, sparsity, pairs, rope_base=10000.0,
            rms_eps=1e-6, rows=None, freq_override=None):
    """Compensated sparse attention forward.

    Returns a dict with the block map ('map', [B,H,Nq,k] int32), boundary gaps
    ('gap'), keep count ('keep'), state ('C', [B,H,r,d]), sparse output
    ('o_s'), low-rank output ('o_lr'), RMS ('r') and output ('o'). With rows
    ([n, 3] of (b, l, h)) only those outputs are computed, as [n, d]; the
    map and C are always computed in full.
    g: [B, L] (broadcast over heads) or [B, L, H].
    freq_override: replaces the RoPE frequencies (used by a test that turns
    the rotation off).
    """
    B, L, H, d = q.shape
    pos = grid_positions(*grid)
    assert pos.shape[0] == L
    axis, freq = rope_frequencies(*pairs, rope_base)
    if freq_override is not None:
        freq = np.asarray(freq_override, dtype=np.float64)
    ang = rope_angles(pos, axis, freq)                                     # [L, r/2]
    bmap, gap, keep = block_map(q, k, block_q, block_k, sparsity)
    C = lowrank_state(k, v, p_k, ang)
    g = np.asarray(g, dtype=np.float64)
    if rows is None:
        o_s = sparse_attention(q, k, v, bmap, block_q, block_k)
        qt = lowrank_features(q, p_q, ang[None, :, None, :])               # [B, L, H, r]
        o_lr = lowrank_readout(qt, C[:, None, :, :, :], rms_eps)
        gg = g if g.ndim == 3 else np.broadcast_to(g[:, :, None], (B, L, H))
    else:
        rows = np.asarray(rows, dtype=np.int64).reshape(-1, 3)
        bi, li, hi = rows[:, 0], rows[:, 1], rows[:, 2]
        o_s = sparse_attention(q, k, v, bmap, block_q, block_k, rows=rows)
        qt = lowrank_features(q[bi, li, hi], p_q, ang[li])                  # [n, r]
        o_lr = lowrank_readout(qt, C[bi, hi], rms_eps)
        gg = g[bi, li, hi] if g.ndim == 3 else g[bi, li]
    o = gate_fuse(o_s, o_lr, gg)
    return {"map": bmap, "gap": gap, "keep": keep, "C": C, "o_s": o_s, "o_lr": o_lr,
            "r": sparse_rms(o_s), "o": o}


# ---------------------------------------------------------------------------
# causal-window variant (the autoregressive extension)
# ---------------------------------------------------------------------------
#
# The summary proposes restricting the compensated sparse attention to a
# causal window for autoregressive video diffusion, where latent frames are
# generated chunk by chunk (robotworld summary, section 4, last paragraph; no
# experiments are given). Reading: tokens are grouped into chunks of F whole
# latent frames (Tc = F * Hg * Wg tokens, F dividing T); the queries of chunk c
# see exactly the keys of chunks 0..c, i.e. the prefix [0, hi_c) with
# hi_c = (c + 1) * Tc -- what a chunk-by-chunk generator with a key/value
# cache of the earlier chunks attends to. Every step is the bidirectional
# method applied to that prefix:
#   * query blocks tile each chunk separately (the last one of a chunk may be
#     partial); key blocks tile [0, hi_c) from token 0, the last one averaged
#     over its visible tokens only;
#   * chunk c keeps keep_count(n_c, s) of its n_c = ceil(hi_c / block_k)
#     candidate key blocks; rows are stored padded with -1 to the width
#     keep_count(N_kblk, s) of the last chunk;
#   * the sparse branch attends to the kept blocks' keys below hi_c;
#   * the low-rank state of chunk c is the prefix sum C_c = sum_{j < hi_c} k~_j v_j^T.
# So nothing a row of chunk c produces depends on a token of a later chunk.

def causal_chunk_tokens(grid, causal_frames: int) -> int:
    """Tokens per chunk, Tc = F * Hg * Wg; F must divide the frame count T."""
    T, Hg, Wg = grid
    assert causal_frames >= 1 and T % causal_frames == 0
    return causal_frames * Hg * Wg


def causal_query_blocks(L: int, chunk_tokens: int, block_q: int):
    """[(start, stop, chunk)] of the query blocks, each chunk tiled on its own."""
    out = []
    for c, c0 in enumerate(range(0, L, chunk_tokens)):
        c1 = min(L, c0 + chunk_tokens)
        out.extend((s, min(c1, s + block_q), c) for s in range(c0, c1, block_q))
    return out


def causal_block_map(q, k, block_q: int, block_k: int, sparsity: float, chunk_tokens: int):
    """Selector of the causal variant.

    Returns (map [B, H, Nq, keep_max] int32, -1 padded; gap [B, H, Nq];
    keep per query block [Nq]; candidates per query block [Nq]).
    """
    B, L, H, d = q.shape
    qb = causal_query_blocks(L, chunk_tokens, block_q)
    keep_max = keep_count(-(-L // block_k), sparsity)
    bmap = np.full((B, H, len(qb), keep_max), -1, dtype=np.int32)
    gap = np.empty((B, H, len(qb)))
    keeps = np.empty(len(qb), dtype=np.int64)
    cands = np.empty(len(qb), dtype=np.int64)
    a = 0
    for c0 in range(0, L, chunk_tokens):
        hi = min(L, c0 + chunk_tokens)
        qm = block_means(q[:, c0:hi], block_q)      # this chunk's query blocks
        km = block_means(k[:, :hi], block_k)        # key blocks of the visible prefix
        n = km.shape[2]
        kc = keep_count(n, sparsity)
        m, g = select_blocks(block_scores(qm, km), kc)
        na = qm.shape[2]
        bmap[:, :, a:a + na, :kc] = m
        gap[:, :, a:a + na] = g
        keeps[a:a + na] = kc
        cands[a:a + na] = n
        a += na
    return bmap, gap, keeps, cands


def causal_sparse_attention(q, k, v, bmap, block_q: int, block_k: int, chunk_tokens: int, rows=None):
    """Sparse branch of the causal variant: query block (chunk c) attends to the
    keys j < hi_c of its kept key blocks (-1 entries are padding).

    rows: None for all (b, l, h) -> [B, L, H, d]; else [n, 3] of (b, l, h) -> [n, d].
    """
    B, L, H, d = q.shape
    scale = 1.0 / math.sqrt(d)
    qb = causal_query_blocks(L, chunk_tokens, block_q)

    def one_group(b, h, a, ls):
        c = qb[a][2]
        hi = min(L, (c + 1) * chunk_tokens)
        keys = kept_keys(bmap[b, h, a][bmap[b, h, a] >= 0], L, block_k)
        keys = keys[keys < hi]
        return softmax_attend(q[b, ls, h], k[b, keys, h], v[b, keys, h], scale)

    if rows is None:
        out = np.empty((B, L, H, d), dtype=np.float64)
        for b in range(B):
            for h in range(H):
                for a, (s0, s1, _) in enumerate(qb):
                    out[b, s0:s1, h] = one_group(b, h, a, np.arange(s0, s1))
        return out
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 3)
    starts = np.array([s for s, _, _ in qb])
    a_of = np.searchsorted(starts, rows[:, 1], side="right") - 1
    out = np.empty((rows.shape[0], d), dtype=np.float64)
    group = (rows[:, 0] * H + rows[:, 2]) * len(qb) + a_of
    for gid in np.unique(group):
        sel = np.nonzero(group == gid)[0]
        b, _, h = rows[sel[0]]
        out[sel] = one_group(b, h, a_of[sel[0]], rows[sel, 1])
    return out


def causal_lowrank_state(k, v, p_k, ang, chunk_tokens: int) -> np.ndarray:
    """C_c[b, h] = sum over j < hi_c of k~_j v_j^T: returns [B, H, NC, r, d]."""
    B, L, H, d = k.shape
    his = [min(L, c0 + chunk_tokens) for c0 in range(0, L, chunk_tokens)]
    return np.stack([lowrank_state(k[:, :hi], v[:, :hi], p_k, ang[:hi]) for hi in his], axis=2)


def causal_forward(q, k, v, p_q, p_k, g, *, grid, block_q, block_k, sparsity, pairs, causal_frames,
                   rope_base=10000.0, rms_eps=1e-6, rows=None):
    """The causal-window forward; same result keys as forward() ('C' is [B, H, NC, r, d],
    'keep' and 'cand' are per query block)."""
    B, L, H, d = q.shape
    Tc = causal_chunk_tokens(grid, causal_frames)
    pos = grid_positions(*grid)
    axis, freq = rope_frequencies(*pairs, rope_base)
    ang = rope_angles(pos, axis, freq)
    bmap, gap, keeps, cands = causal_block_map(q, k, block_q, block_k, sparsity, Tc)
    C = causal_lowrank_state(k, v, p_k, ang, Tc)
    g = np.asarray(g, dtype=np.float64)
    if rows is None:
        o_s = causal_sparse_attention(q, k, v, bmap, block_q, block_k, Tc)
        qt = lowrank_features(q, p_q, ang[None, :, None, :])                     # [B, L, H, r]
        Crow = np.moveaxis(C[:, :, np.arange(L) // Tc], 1, 2)                  # [B, L, H, r, d]
        o_lr = lowrank_readout(qt, Crow, rms_eps)
        gg = g if g.ndim == 3 else np.broadcast_to(g[:, :, None], (B, L, H))
    else:
        rows = np.asarray(rows, dtype=np.int64).reshape(-1, 3)
        bi, li, hi = rows[:, 0], rows[:, 1], rows[:, 2]
        o_s = causal_sparse_attention(q, k, v, bmap, block_q, block_k, Tc, rows=rows)
        qt = lowrank_features(q[bi, li, hi], p_q, ang[li])
        o_lr = lowrank_readout(qt, C[bi, hi, li // Tc], rms_eps)
        gg = g[bi, li, hi] if g.ndim == 3 else g[bi, li]
    o = gate_fuse(o_s, o_lr, gg)
    return {"map": bmap, "gap": gap, "keep": keeps, "cand": cands, "C": C, "o_s": o_s, "o_lr": o_lr,
            "r": sparse_rms(o_s), "o": o}
