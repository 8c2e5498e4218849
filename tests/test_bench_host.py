"""Host logic of the benchmark (no GPU): the FLOP and byte counts its roofline
numbers divide by, against brute-force counts over the oracle's own maps."""
import importlib.util
import os

import numpy as np

import oracle.sda_oracle as O
from sparse_rank_attention_block_b200 import synthetic as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
_spec = importlib.util.spec_from_file_location("bench_host", os.path.join(ROOT, "bench.py"))
bench = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(bench)


def _inputs(w):
    inp = S.make_inputs(w)
    return inp.q.float().numpy(), inp.k.float().numpy()


def test_kept_pair_flops_brute_force():
    w = S.TINY.replace(name="flops", grid_t=2, grid_h=7, grid_w=11, sparsity=0.6, H=2, seed=71)
    q, k = _inputs(w)
    bmap, _, _ = O.block_map(q, k, w.block_q, w.block_k, w.sparsity)
    want = 0
    for b in range(w.B):
        for h in range(w.H):
            for a, (s0, s1) in enumerate(O.block_ranges(w.L, w.block_q)):
                keys = O.kept_keys(bmap[b, h, a], w.L, w.block_k)
                want += (s1 - s0) * len(keys)
    assert bench.kept_pair_flops(w, bmap) == 4.0 * w.d * want


def test_causal_pair_flops_brute_force():
    w = S.TINY.replace(name="cflops", grid_t=4, grid_h=5, grid_w=13, sparsity=0.6, H=2, causal_frames=1, seed=72)
    q, k = _inputs(w)
    bmap, _, _, _ = O.causal_block_map(q, k, w.block_q, w.block_k, w.sparsity, w.chunk_tokens)
    want = 0
    for b in range(w.B):
        for h in range(w.H):
            for a, (s0, s1, c) in enumerate(O.causal_query_blocks(w.L, w.chunk_tokens, w.block_q)):
                row = bmap[b, h, a]
                keys = O.kept_keys(row[row >= 0], w.L, w.block_k)
                want += (s1 - s0) * int(np.sum(keys < (c + 1) * w.chunk_tokens))
    assert bench.causal_pair_flops(w, bmap) == 4.0 * w.d * want


def test_stage_bytes_are_whole_tensors():
    w = S.WAN14B_720P
    t = w.B * w.L * w.H * w.d * 2.0
    b = bench.stage_bytes(w)
    assert b == {"select": t, "lowrank_state": 2 * t, "lowrank_readout": 2 * t, "sparse_attn_fused": 4 * t}
    b64 = bench.stage_bytes(w.replace(rank=64))   # the state pass pools K only up to r = 32
    assert b64["select"] == 2 * t


def test_roofline_peak_burst_for_short_full_clock_regions():
    peaks = {"bf16_tflops": 1618.5, "bf16_tflops_sustained": 1371.3, "hbm_gbs": 6531.9}
    full = {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}
    assert bench.roofline_peak(peaks, 0.09, full) == (1618.5, "burst")
    # a long region, a power-capped one, or one well below max clock takes the sustained figure
    assert bench.roofline_peak(peaks, 5.0, full) == (1371.3, "sustained")
    assert bench.roofline_peak(peaks, 0.09, dict(full, reasons=["sw_power_cap"])) == (1371.3, "sustained")
    assert bench.roofline_peak(peaks, 0.09, dict(full, sm_mhz=1300)) == (1371.3, "sustained")


def test_oracle_sample_rate_is_measured_tokens():
    """The CPU baseline's rate is token-head outputs over the seconds spent, in layer tokens."""
    w = S.TINY.replace(name="rate", grid_t=1, grid_h=8, grid_w=32, H=4, seed=72)
    smp = bench.OracleSample(w, heads=2)
    tok, spent, n, est = smp.step(2, seed=0)
    assert n == 2 and spent > 0 and est > 0
    assert tok == 2 * w.block_q * 2 / w.H   # two full query blocks of two of the four heads
