"""Top-k boundary-gap repair of generated inputs (test side, uses the oracle).

The block map is compared bit-exact between the GPU (fp32 scores) and the
oracle (fp64 scores). That comparison is only meaningful where the k-th and
(k+1)-th best scores of a row are further apart than both sides' rounding, so
every generated problem is first repaired until each row's relative boundary
gap (S_(k) - S_(k+1)) / max |S| is at least `min_gap`: the first query token of
an offending block gets a seeded random nudge (re-rounded to bf16), doubling
its size until the row clears the bar.
"""
import numpy as np

import oracle.sda_oracle as O
from sparse_rank_attention_block_b200.synthetic import perturb_token

from _util import f32


def repair_gaps(inp, w, min_gap=1e-4, max_tries=20):
    """Repair `inp` (synthetic.Inputs, modified in place); returns the number of rows touched."""
    k = f32(inp.k)
    km = O.block_means(k, w.block_k)
    del k
    keep = O.keep_count(km.shape[2], w.sparsity)
    if keep >= km.shape[2]:
        return 0
    q = f32(inp.q)
    qm = O.block_means(q, w.block_q)
    _, gap = O.select_blocks(O.block_scores(qm, km), keep)
    bad = np.argwhere(gap < min_gap)
    for n, (b, h, a) in enumerate(bad):
        l0, l1 = a * w.block_q, min(w.L, (a + 1) * w.block_q)
        eps = 1e-2
        for t in range(max_tries):
            perturb_token(inp.q, int(b), int(l0), int(h), eps, seed=int(1_000_003 * n + t))
            row = inp.q[b, l0:l1, h].float().numpy().astype(np.float64).mean(axis=0)
            s = km[b, h] @ row
            _, g = O.select_blocks(s[None, :], keep)
            if g[0] >= min_gap:
                break
            eps *= 2.0
        else:
            raise RuntimeError(f"gap repair failed for block (b={b}, h={h}, a={a})")
    return len(bad)


def min_gap(inp, w):
    """Smallest relative boundary gap over all score rows (oracle, fp64)."""
    m, gap, keep = O.block_map(f32(inp.q), f32(inp.k), w.block_q, w.block_k, w.sparsity)
    return float(np.min(gap))


def repair_gaps_causal(inp, w, heads=None, min_gap=1e-4, max_tries=20):
    """repair_gaps for the causal-window selector: per chunk c the rows of its
    query blocks are scored against the key means of the visible prefix
    [0, hi_c) (the oracle's causal geometry). Only q is nudged, so the key
    means of every chunk stay as they are. heads: the heads to repair (all by
    default). Returns the number of rows touched."""
    hs = list(range(w.H)) if heads is None else list(heads)
    k = inp.k[:, :, hs].float().numpy().astype(np.float64)
    Tc = w.chunk_tokens
    qb = O.causal_query_blocks(w.L, Tc, w.block_q)
    touched = 0
    for c0 in range(0, w.L, Tc):
        hi = min(w.L, c0 + Tc)
        km = O.block_means(k[:, :hi], w.block_k)            # [B, H', n_c, d]
        keep = O.keep_count(km.shape[2], w.sparsity)
        if keep >= km.shape[2]:
            continue
        blocks = [(a, s0, s1) for a, (s0, s1, _) in enumerate(qb) if c0 <= s0 < hi]
        q = inp.q[:, c0:hi][:, :, hs].float().numpy().astype(np.float64)
        qm = O.block_means(q, w.block_q)                    # [B, H', nq_chunk, d]
        _, gap = O.select_blocks(O.block_scores(qm, km), keep)
        for b, hh, ai in np.argwhere(gap < min_gap):
            a, s0, s1 = blocks[ai]
            h = hs[hh]
            eps = 1e-2
            for t in range(max_tries):
                perturb_token(inp.q, int(b), int(s0), int(h), eps, seed=int(1_000_003 * touched + 7919 * a + t))
                row = inp.q[b, s0:s1, h].float().numpy().astype(np.float64).mean(axis=0)
                _, g = O.select_blocks((km[b, hh] @ row)[None, :], keep)
                if g[0] >= min_gap:
                    break
                eps *= 2.0
            else:
                raise RuntimeError(f"causal gap repair failed for block (b={b}, h={h}, a={a})")
            touched += 1
    return touched
