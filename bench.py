#!/usr/bin/env python
"""Benchmark of the compensated sparse attention forward on B200.

One step = one `sda_forward` call (selector, low-rank state and readout,
block-sparse attention with the gate epilogue) over one attention layer of the
14B-720P-like workload (B=1, H=40, d=128, 21x45x80 = 75,600 tokens, s=0.97,
r=32), inputs resident in HBM. Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Under torchrun every rank runs the layer on its own batch (independent
problems, inputs seeded per rank, no collective on the data path: weak
scaling); the timed region is
bracketed by a barrier and a device synchronise, and the slowest rank's time
is reported. `--impl reference` times the fp64 CPU oracle on the host cores
instead (rank 0 only), on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_rank_attention_block_b200 import sda, synthetic as S  # noqa: E402

METRIC = "compensated sparse attn fwd: tokens/s & eff. TFLOPS (frac. of roofline), 1×B200"
STAGES = ["lowrank_state", "select", "lowrank_readout", "sparse_attn_fused"]
# rope table, state, reduce, pool, score, select, attention (readout + gate fused): 128-row query blocks
LAUNCHES_PER_STEP = 7


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": pk["hbm_gbs"], "bf16_tflops": pk["bf16_tflops"],
                "bf16_tflops_sustained": pk.get("bf16_tflops_sustained", pk["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def kept_pair_flops(w, block_map: np.ndarray) -> float:
    """4*d flops per valid (query, key) pair inside the kept blocks (QK^T and PV)."""
    nq_valid = np.minimum(w.block_q, w.L - np.arange(w.n_qblk) * w.block_q).astype(np.float64)   # [Nq]
    nk_valid = np.minimum(w.block_k, w.L - np.arange(w.n_kblk) * w.block_k).astype(np.float64)   # [Nk]
    keys = nk_valid[block_map].sum(axis=-1)                                                        # [B,H,Nq]
    return float((keys * nq_valid[None, None, :]).sum() * 4.0 * w.d)


def causal_pair_flops(w, block_map: np.ndarray) -> float:
    """4*d flops per visible (query, key) pair of the kept blocks of a causal-window map
    (-1 entries are padding; a chunk-c query sees the keys below (c + 1) * Tc)."""
    Tc, nq = w.chunk_tokens, -(-w.chunk_tokens // w.block_q)
    a = np.arange(w.n_qblk)
    c = a // nq
    s0 = c * Tc + (a % nq) * w.block_q
    rows = (np.minimum(s0 + w.block_q, (c + 1) * Tc) - s0).astype(np.float64)                   # [Nq]
    hi = ((c + 1) * Tc)[None, None, :, None]
    kb = block_map.astype(np.int64)
    keys = np.where(kb >= 0, np.clip(hi - kb * w.block_k, 0, w.block_k), 0).sum(axis=-1)        # [B,H,Nq]
    return float((keys * rows[None, None, :]).sum() * 4.0 * w.d)


def roofline_peak(peaks, timed_s: float, clocks: dict):
    """The tensor peak the attention kernel is held against: the burst figure
    (a kernel timed alone, at full clock) unless the timed region is long
    enough for the power cap to bring the clock down, or the clock record
    shows it did (then the sustained figure)."""
    capped = "sw_power_cap" in (clocks.get("reasons") or [])
    mhz, max_mhz = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    slow = bool(mhz and max_mhz and mhz < 0.9 * max_mhz)
    if timed_s < 1.0 and not capped and not slow:
        return peaks["bf16_tflops"], "burst"
    return peaks["bf16_tflops_sustained"], "sustained"


def state_pools_k(w) -> bool:
    """The forward lets the tcgen05 state pass form the key block means at d = 128, r <= 32."""
    return w.d == 128 and w.rank <= 32


def stage_bytes(w) -> dict:
    """Algorithmic HBM bytes per launch of each stage (each tensor read or written once).

    Where the state pass pools K, the selector reads only Q and the state pass
    reads K and V once for both jobs."""
    t = w.B * w.L * w.H * w.d * 2.0
    return {"select": (1 if state_pools_k(w) else 2) * t, "lowrank_state": 2 * t, "lowrank_readout": 2 * t,
            "sparse_attn_fused": 4 * t}   # q, k, v read once and o written


def pre_attn_hbm_frac(w, stage_ms, hbm_gbs) -> float:
    """Selector and state together: their algorithmic bytes over their summed time."""
    b = stage_bytes(w)
    ms = stage_ms["select"] + stage_ms["lowrank_state"]
    return (b["select"] + b["lowrank_state"]) / (ms / 1e3) / 1e9 / hbm_gbs


class Clocks:
    """SM clock, power and clock-event reasons sampled every 10 ms (NVML, read only)
    on a background thread while the timed region runs."""

    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, dev: torch.device):
        self.samples = []
        self.error = None
        self.handle = None
        try:
            import pynvml as nv
            nv.nvmlInit()
            props = torch.cuda.get_device_properties(dev)
            for i in range(nv.nvmlDeviceGetCount()):
                h = nv.nvmlDeviceGetHandleByIndex(i)
                pci = nv.nvmlDeviceGetPciInfo(h)
                if (pci.domain, pci.bus, pci.device) == (props.pci_domain_id, props.pci_bus_id, props.pci_device_id):
                    self.handle = h
            self.nv = nv
            self.bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                         "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                         "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                         "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.handle, nv.NVML_CLOCK_SM) if self.handle else None
        except Exception as e:  # no NVML: report why
            self.error = f"nvml unavailable: {type(e).__name__}"
        if self.handle is None and self.error is None:
            self.error = "nvml: device not found"

    def _run(self):
        nv = self.nv
        while not self.stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append((mhz, rs))
            except Exception:
                pass
            self.stop.wait(0.01)

    def __enter__(self):
        import threading
        if self.handle is not None:
            self.stop = threading.Event()
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        return self

    def __exit__(self, *exc):
        if self.handle is not None:
            self.stop.set()
            self.thread.join(timeout=5)

    def summary(self):
        if self.handle is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "samples": 0, "reasons": [self.error]}
        reasons = sorted({n for _, rs in self.samples for n in self.NAMES if rs & self.bits[n]})
        return {"sm_mhz": statistics.median(m for m, _ in self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples), "reasons": reasons,
                "source": "nvml, 10 ms"}


def dist_setup(n_gpus: int, backend: str = "nccl"):
    """(dist, rank, world, local rank); dist is None for a single process.

    One process per GPU under torchrun (RANK / LOCAL_RANK / WORLD_SIZE /
    MASTER_* from the environment). The process group only brackets the timed
    region and takes the maximum time: no collective touches the layer's data.
    `backend="gloo"` runs the same host logic on CPU processes.
    """
    if n_gpus > 1 or "RANK" in os.environ:
        import datetime
        import torch.distributed as dist
        rank = int(os.environ.get("RANK", 0))
        local = int(os.environ.get("LOCAL_RANK", 0))
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
        return dist, rank, dist.get_world_size(), local
    return None, 0, 1, 0


def time_max_over_ranks(dist, seconds: float, device="cuda") -> float:
    """The slowest rank's time (all-reduce MAX); `seconds` itself for one process."""
    if dist is None:
        return seconds
    t = torch.tensor([seconds], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(w, rank: int) -> int:
    """Seed of the layer that `rank` processes: every rank holds its own batch
    of the global one (rank 0 keeps the workload's seed)."""
    return w.seed + 1000 * rank


def whole_job_tokens_per_s(w, world: int, steps: int, max_s: float) -> float:
    """Tokens of all ranks' layers over the slowest rank's time for `steps` steps."""
    return w.B * w.L * world * steps / max_s


# ---------------------------------------------------------------------------
# CPU oracle (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------

class OracleSample:
    """Time the fp64 oracle on a bounded sample of the workload.

    One pass works on `heads` heads of batch item 0 (every head is an
    independent problem), drawn with the workload's recipe: per head the
    block map and the state C in full, then the outputs (sparse branch,
    low-rank readout, gate) of every token of `n_blocks` seeded random query
    blocks. The reported rate is measured, not extrapolated: the token-head
    outputs produced divided by the seconds spent (map and C included), in
    layer tokens (H token-heads make one token). The full-layer time that
    the per-head costs imply is reported beside it as an estimate.
    """

    def __init__(self, w, heads: int = 1):
        import oracle.sda_oracle as O
        self.O = O
        self.w = w
        self.heads = heads
        inp = S.make_inputs(w.replace(B=1, H=heads))
        f = lambda t: t.float().numpy()  # noqa: E731  exact bf16 decode
        self.q, self.k, self.v = f(inp.q), f(inp.k), f(inp.v)
        self.p_q, self.p_k, self.g = f(inp.p_q), f(inp.p_k), f(inp.g)

    def step(self, n_blocks: int, seed: int = 0):
        """One pass over the sampled heads: (layer tokens produced, seconds spent, blocks per head,
        estimated full-layer seconds)."""
        O, w = self.O, self.w
        axis, freq = O.rope_frequencies(w.pairs_t, w.pairs_h, w.pairs_w, w.rope_base)
        ang = O.rope_angles(O.grid_positions(w.grid_t, w.grid_h, w.grid_w), axis, freq)
        blocks = np.sort(np.random.default_rng(seed).choice(w.n_qblk, size=min(n_blocks, w.n_qblk), replace=False))
        li = np.concatenate([np.arange(a * w.block_q, min(w.L, (a + 1) * w.block_q)) for a in blocks])
        rows = np.stack([np.zeros_like(li), li, np.zeros_like(li)], axis=1)
        per_head, spent = [], 0.0
        for h in range(self.heads):
            q, k, v = (x[:, :, h:h + 1] for x in (self.q, self.k, self.v))
            t0 = time.perf_counter()
            bmap, _, _ = O.block_map(q, k, w.block_q, w.block_k, w.sparsity)
            C = O.lowrank_state(k, v, self.p_k, ang)
            t1 = time.perf_counter()
            o_s = O.sparse_attention(q, k, v, bmap, w.block_q, w.block_k, rows=rows)
            o_lr = O.lowrank_readout(O.lowrank_features(q[0, li, 0], self.p_q, ang[li]), C[0, 0], w.rms_eps)
            O.gate_fuse(o_s, o_lr, self.g[0, li])
            t2 = time.perf_counter()
            per_head.append((t1 - t0) + (t2 - t1) * w.L / len(li))
            spent += t2 - t0
        tokens = len(li) * self.heads / w.H
        return tokens, spent, len(blocks), sum(per_head) / len(per_head) * w.B * w.H

    @staticmethod
    def threads():
        import threadpoolctl
        return max([p.get("num_threads", 1) for p in threadpoolctl.threadpool_info()] + [1])

    def describe(self, n_blocks):
        w = self.w
        return (f"{self.heads} head(s) of {w.name} per step: per head the full block map and state C plus the "
                f"outputs of {n_blocks} of {w.n_qblk} random query blocks; rate = token-head outputs / seconds "
                f"spent (map and C included), in layer tokens of H={w.H} heads")


def run_reference(args, w):
    if int(os.environ.get("RANK", 0)) != 0:
        return 0
    smp = OracleSample(w)
    n_blocks = 64 if args.warmup + args.steps <= 30 else 16
    tokens, secs, ests = 0.0, 0.0, []
    for i in range(args.warmup + args.steps):
        tok, spent, n, est = smp.step(n_blocks, seed=i)
        if i >= args.warmup:
            tokens += tok
            secs += spent
            ests.append(est)
    value = tokens / secs
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w, args.gpus),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": smp.threads(), "kind": "oracle",
                             "cpu_model": cpu_model(), "sample": smp.describe(n_blocks),
                             "layer_seconds_estimate": sum(ests) / len(ests)},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, n_gpus):
    return {"workload": w.name, "B": w.B, "L": w.L, "H": w.H, "d": w.d,
            "grid": [w.grid_t, w.grid_h, w.grid_w], "block_q": w.block_q, "block_k": w.block_k,
            "sparsity": w.sparsity, "rank": w.rank, "rope_pairs": [w.pairs_t, w.pairs_h, w.pairs_w],
            "global_batch": w.B * n_gpus, "seq_len": w.L, "parallelism": f"data-parallel, one independent batch per rank x{n_gpus}",
            "l2": f"inputs larger than L2 (q, k, v {w.B * w.L * w.H * w.d * 2 / 1e6:.0f} MB each)"}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

ATTN_SRCS = [os.path.join(ROOT, "sparse_rank_attention_block_b200", "csrc", f)
             for f in ("sparse_attn_tc.cu", "ex2_fma.cuh", "tc.cuh", "common.cuh")]


def attn_source_sha256() -> str:
    """sha256 over the attention kernel's source files, in a fixed order."""
    import hashlib
    h = hashlib.sha256()
    for f in ATTN_SRCS:
        h.update(open(f, "rb").read())
    return h.hexdigest()


def profiled_traffic(workload: str):
    """DRAM bytes per launch of the attention kernel from the committed ncu summary.

    The summary records the sha256 of the kernel's sources (attn_source_sha256)
    it was taken on; the figure is used only while they are unchanged (else None).
    """
    import re
    path = os.path.join(ROOT, "profiles", f"sparse_attn_tc_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_b = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", text)
    m_h = re.search(r"source_sha256:\s*([0-9a-f]{64})", text)
    if not (m_b and m_h):
        return None
    return int(m_b.group(1)) if attn_source_sha256() == m_h.group(1) else None


def time_calls(fn, stream, iters: int) -> float:
    """Average device milliseconds of fn() over iters calls (after one untimed call)."""
    fn()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(iters):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / iters


def aux_calls(w, p, d, ws, stream, peaks) -> dict:
    """The standalone ABI calls of the HBM-bound steps, timed outside the step.

    Algorithmic bytes: every tensor read or written once (T = one [B,L,H,d]
    bf16 tensor): select reads Q, K (2T); lowrank_fwd reads K, V, Q and
    writes O_lr (4T); gate_fuse reads O_s, O_lr, g and writes O (3T + g);
    quant_fp8 reads one bf16 tensor and writes its E4M3 codes and per-token
    scales (1.5T + 4 B per token); qk_prologue reads raw q, k and writes
    their normalised and rotated forms (6T).
    """
    t = w.B * w.L * w.H * w.d * 2.0
    g_bytes = w.B * w.L * (w.H if w.gate_per_head else 1) * 4.0
    keep = sda.sda_keep_count(p)
    idx = torch.empty((w.B, w.H, w.n_qblk, keep), dtype=torch.int32, device=d["q"].device)
    o_s = torch.empty_like(d["q"])
    o_lr = torch.empty_like(d["q"])
    o = torch.empty_like(d["q"])
    xq = torch.empty(d["q"].shape, dtype=torch.uint8, device=d["q"].device)
    sc = torch.empty((w.B, w.L), dtype=torch.float32, device=d["q"].device)
    wn = torch.ones((w.H, w.d), dtype=torch.bfloat16, device=d["q"].device)
    pro = [torch.empty_like(d["q"]) for _ in range(4)]
    calls = {
        "sda_block_select": (lambda: sda.sda_block_select(p, d["q"], d["k"], idx, ws.ptr, ws.nbytes, stream), 2 * t),
        "sda_lowrank_fwd": (lambda: sda.sda_lowrank_fwd(p, d["q"], d["k"], d["v"], d["p_q"], d["p_k"], o_lr, None,
                                                        ws.ptr, ws.nbytes, stream), 4 * t),
        "sda_gate_fuse": (lambda: sda.sda_gate_fuse(p, o_s, o_lr, d["g"], o, stream), 3 * t + g_bytes),
        "sda_quant_fp8": (lambda: sda.sda_quant_fp8(p, d["v"], xq, sc, stream), 1.5 * t + w.B * w.L * 4.0),
        "sda_qk_prologue": (lambda: sda.sda_qk_prologue(p, d["q"], d["k"], wn, wn, *pro, stream), 6 * t),
    }
    out = {}
    for name, (fn, nbytes) in calls.items():
        ms = time_calls(fn, stream, 5)
        out[name] = {"ms": ms, "hbm_gbs": nbytes / (ms / 1e3) / 1e9,
                     "hbm_frac": nbytes / (ms / 1e3) / 1e9 / peaks["hbm_gbs"]}
    ws.check(stream)
    # the causal-window variant of the whole forward on the same tensors: chunks
    # of 3 latent frames (the frame count must be a multiple of 3)
    if w.grid_t % 3 == 0:
        wc = w.replace(causal_frames=3)
        pc = sda.params_of(wc)
        wsc = sda.Workspace(pc, device=d["q"].device, stream=stream)
        idc = torch.empty((wc.B, wc.H, wc.n_qblk, sda.sda_keep_count(pc)), dtype=torch.int32, device=d["q"].device)
        fc = lambda: sda.sda_forward(pc, d["q"], d["k"], d["v"], d["p_q"], d["p_k"], d["g"], o, idc,  # noqa: E731
                                     wsc.ptr, wsc.nbytes, stream)
        ms = time_calls(fc, stream, 5)
        wsc.check(stream)
        fl = causal_pair_flops(wc, idc.cpu().numpy())
        out["sda_forward_causal_3frame_chunks"] = {
            "ms": ms, "tokens_per_s": wc.B * wc.L / (ms / 1e3), "chunks": wc.L // wc.chunk_tokens,
            "kept_pair_tflops_per_s": fl / (ms / 1e3) / 1e12,
            "note": "whole forward (state, selector, fused attention) in one call; flops over the step time"}
    # the backward on the forward's own map, upstream gradient = the inputs' V
    if not w.causal_frames:
        nb = sda.sda_backward_workspace_size(p)
        wsb = torch.empty(nb + 256, dtype=torch.uint8, device=d["q"].device)
        pb = wsb.data_ptr() + (-wsb.data_ptr()) % 256
        sda.sda_workspace_init(pb, nb, stream)
        idb = torch.empty((w.B, w.H, w.n_qblk, keep), dtype=torch.int32, device=d["q"].device)
        sda.sda_block_select(p, d["q"], d["k"], idb, ws.ptr, ws.nbytes, stream)
        gr = [torch.empty(d["q"].shape, dtype=torch.float32, device=d["q"].device) for _ in range(3)]
        gp = [torch.empty((w.rank, w.d), dtype=torch.float32, device=d["q"].device) for _ in range(2)]
        gg = torch.empty_like(d["g"])
        fb = lambda: sda.sda_backward(p, d["q"], d["k"], d["v"], d["p_q"], d["p_k"], d["g"], idb, d["v"],  # noqa: E731
                                      *gr, *gp, gg, pb, nb, stream)
        ms = time_calls(fb, stream, 3)
        sda.sda_read_status(pb, nb, stream)
        fl = kept_pair_flops(w, idb.cpu().numpy())
        out["sda_backward"] = {
            "ms": ms, "tokens_per_s": w.B * w.L / (ms / 1e3),
            "kept_pair_tflops_per_s": 2.5 * fl / (ms / 1e3) / 1e12,
            "note": "whole backward in one call: forward recompute, gate, low-rank branch (tensor cores), sparse "
                    "branch on the tensor cores (dq kernel per query block, dk/dv kernel per key block); flops = "
                    "2.5x the forward's kept-pair flops (S, dP, dQ, dK, dV: 10 d per pair against 4 d)"}
        del wsb, gr
    return out

def time_config(w, dev, stream, steps: int, peaks) -> dict:
    """One forward configuration timed on its own: inputs drawn on the device with the
    workload's recipe (synthetic.make_inputs_device), 3 warm-up calls, then `steps`
    calls with an event before every stage and after the last (device timing), NVML
    clocks sampled meanwhile. Inputs at these sizes (>= 8k tokens x 40 heads) exceed
    L2 except the tiny and 8k layers, whose figures are therefore L2-warm."""
    p = sda.params_of(w)
    inp = S.make_inputs_device(w, device=dev)
    d = {n: getattr(inp, n) for n in ("q", "k", "v", "p_q", "p_k", "g")}
    ws = sda.Workspace(p, device=dev)
    o = torch.empty_like(d["q"])
    idx = torch.empty((w.B, w.H, w.n_qblk, sda.sda_keep_count(p)), dtype=torch.int32, device=dev)
    for _ in range(3):
        sda.sda_forward(p, d["q"], d["k"], d["v"], d["p_q"], d["p_k"], d["g"], o, idx, ws.ptr, ws.nbytes, stream)
    torch.cuda.synchronize(dev)
    ws.check(stream)
    flops = kept_pair_flops(w, idx.cpu().numpy())
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(STAGES) + 1)] for _ in range(steps)]
    for e in (x for row in ev for x in row):
        e.record(stream)
    torch.cuda.synchronize(dev)
    with Clocks(dev) as clk:
        t0 = time.perf_counter()
        for i in range(steps):
            sda.sda_forward_profiled(p, d["q"], d["k"], d["v"], d["p_q"], d["p_k"], d["g"], o, idx, ws.ptr,
                                     ws.nbytes, [e.cuda_event for e in ev[i]], stream)
        torch.cuda.synchronize(dev)
        wall = time.perf_counter() - t0
    ws.check(stream)
    stage_ms = {s_: sum(e[j].elapsed_time(e[j + 1]) for e in ev) / steps for j, s_ in enumerate(STAGES)}
    total = sum(stage_ms.values())
    clocks = clk.summary()
    peak, kind = roofline_peak(peaks, wall, clocks)
    b = stage_bytes(w)
    attn = stage_ms["sparse_attn_fused"] or stage_ms["lowrank_readout"]
    attn_tf = flops / (attn / 1e3) / 1e12
    out = {"B": w.B, "L": w.L, "H": w.H, "d": w.d, "sparsity": w.sparsity, "rank": w.rank,
           "block_q": w.block_q, "steps": steps, "latency_ms": total, "tokens_per_s": w.B * w.L / (total / 1e3),
           "eff_tflops": flops / (total / 1e3) / 1e12, "kept_block_tflop": flops / 1e12, "stage_ms": stage_ms,
           "attention_tflops": attn_tf, "attention_frac": attn_tf / peak, "attention_peak": f"bf16 {kind}",
           "select_hbm_frac": b["select"] / (stage_ms["select"] / 1e3) / 1e9 / peaks["hbm_gbs"],
           "lowrank_state_hbm_frac": b["lowrank_state"] / (stage_ms["lowrank_state"] / 1e3) / 1e9 / peaks["hbm_gbs"],
           "clocks": clocks, "data": "synthetic, drawn on the device (same recipe)"}
    del d, inp, ws, o, idx
    torch.cuda.empty_cache()
    return out


def other_configs():
    """The other named layers and a bounded sweep subset (s = 0.97, r = 32 at 8k, 32k, 128k tokens)."""
    sweep = [x for x in S.sweep_points() if x.B == 1 and x.sparsity == 0.97 and x.rank == 32
             and x.L in (8192, 32768, 131072)]
    return [S.TINY, S.WAN13B_480P, S.WAN14B_480P] + sweep


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_tiny_full() -> dict:
    """The fp64 oracle on the tiny layer in full (every head, every query block), timed."""
    import oracle.sda_oracle as O
    w = S.TINY
    inp = S.make_inputs(w)
    f = lambda t: t.float().numpy()  # noqa: E731
    t0 = time.perf_counter()
    O.forward(f(inp.q), f(inp.k), f(inp.v), f(inp.p_q), f(inp.p_k), f(inp.g), grid=(w.grid_t, w.grid_h, w.grid_w),
              block_q=w.block_q, block_k=w.block_k, sparsity=w.sparsity, pairs=(w.pairs_t, w.pairs_h, w.pairs_w),
              rope_base=w.rope_base, rms_eps=w.rms_eps)
    sec = time.perf_counter() - t0
    return {"workload": w.name, "seconds": sec, "tokens_per_s": w.B * w.L / sec, "threads": OracleSample.threads(),
            "cpu_model": cpu_model(), "sample": "the whole layer (every head and query block)"}


def run_gpu(args, w):
    dist, rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    sda.lib()
    p = sda.params_of(w)
    inp = S.make_inputs(w, seed=rank_seed(w, rank))
    d = {n: getattr(inp, n).to(dev) for n in ("q", "k", "v", "p_q", "p_k", "g")}
    ws = sda.Workspace(p, device=dev)
    keep = sda.sda_keep_count(p)
    o = torch.empty_like(d["q"])
    idx = torch.empty((w.B, w.H, w.n_qblk, keep), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(events=None):
        if events is not None:
            sda.sda_forward_profiled(p, d["q"], d["k"], d["v"], d["p_q"], d["p_k"], d["g"], o, idx, ws.ptr,
                                     ws.nbytes, [e.cuda_event for e in events], stream)
        else:
            sda.sda_forward(p, d["q"], d["k"], d["v"], d["p_q"], d["p_k"], d["g"], o, idx, ws.ptr, ws.nbytes,
                            stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    ws.check(stream)
    flops = kept_pair_flops(w, idx.cpu().numpy())

    # timed region: K back-to-back steps; every step records an event before
    # each stage and after the last one on the launching stream
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(STAGES) + 1)] for _ in range(args.steps)]
    for e in (x for row in ev for x in row):
        e.record(stream)   # torch creates the underlying cudaEvent on first record
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clk_sampler = Clocks(dev)
    with clk_sampler as clk:
        t0.record(stream)
        for i in range(args.steps):
            step(ev[i])
        t1.record(stream)
        torch.cuda.synchronize(dev)
    total_s = t0.elapsed_time(t1) / 1e3
    stage_ms = {s: sum(e[j].elapsed_time(e[j + 1]) for e in ev) / args.steps for j, s in enumerate(STAGES)}
    ws.check(stream)
    max_s = time_max_over_ranks(dist, total_s)

    # end to end through the host-buffer entry point (copies inside the timed region)
    hb = sda.sda_forward_host_buffer_size(p)
    dbuf = torch.empty(hb + 256, dtype=torch.uint8, device=dev)
    dptr = dbuf.data_ptr() + (-dbuf.data_ptr()) % 256
    sda.sda_workspace_init(dptr, hb, stream)
    pins = {n: getattr(inp, n).pin_memory() for n in ("q", "k", "v", "p_q", "p_k", "g")}
    o_host = torch.empty_like(inp.q).pin_memory()
    e2e_steps = max(1, min(args.steps, 5))
    sda.sda_forward_host(p, pins["q"], pins["k"], pins["v"], pins["p_q"], pins["p_k"], pins["g"], o_host, dptr, hb,
                         stream)
    if dist is not None:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        sda.sda_forward_host(p, pins["q"], pins["k"], pins["v"], pins["p_q"], pins["p_k"], pins["g"], o_host, dptr,
                             hb, stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_s = time_max_over_ranks(dist, e0.elapsed_time(e1) / 1e3)
    h2d = sum(pins[n].numel() * pins[n].element_size() for n in pins)
    d2h = o_host.numel() * o_host.element_size()

    peaks = load_peaks()
    clocks = clk.summary()
    aux = aux_calls(w, p, d, ws, stream, peaks) if not args.no_aux else None
    configs = None
    if world == 1 and not args.no_configs:
        del d, ws, o, idx, dbuf, pins, o_host, inp
        torch.cuda.empty_cache()
        configs = {c.name: time_config(c, dev, stream, 10, peaks) for c in other_configs()}
    traffic = profiled_traffic(w.name)
    if rank == 0:
        ms_step = max_s / args.steps * 1e3
        value = whole_job_tokens_per_s(w, world, args.steps, max_s)
        sparse_ms = stage_ms["sparse_attn_fused"]
        achieved = flops / (sparse_ms / 1e3) / 1e12
        peak, peak_kind = roofline_peak(peaks, max_s, clocks)
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            smp = OracleSample(w, heads=8)
            tok, spent, n, est = smp.step(smp.w.n_qblk)
            cpu = {"value": tok / spent, "unit": "tokens/s", "cores": smp.threads(), "kind": "oracle",
                   "cpu_model": cpu_model(),
                   "sample": smp.describe(n) + f" ({spent:.1f} s of CPU work)",
                   "layer_seconds_estimate": est,
                   "tiny_layer_in_full": oracle_tiny_full()}
        bytes_ = stage_bytes(w)
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, Wan-like token grid)",
            "config": workload_config(w, world),
            "eff_tflops": flops / (ms_step / 1e3) / 1e12,
            "latency_ms": ms_step,
            "stage_ms": stage_ms,
            "stage_hbm_frac": {s: bytes_[s] / (stage_ms[s] / 1e3) / 1e9 / peaks["hbm_gbs"]
                               for s in ("select", "lowrank_state") if stage_ms[s] > 0},
            "pre_attn_hbm_frac": pre_attn_hbm_frac(w, stage_ms, peaks["hbm_gbs"]),
            "kept_block_tflop": flops / 1e12,
            "roofline": {"kernel": "sparse_attn_tc_kernel (fused readout + gate)", "bound": "tensor", "achieved": achieved,
                         "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                         "algorithmic_bytes": bytes_["sparse_attn_fused"],
                         "peak_source": f"{peaks['source']} bf16 {peak_kind}",
                         "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"]},
            "clocks": clocks,
            "e2e": {"value": w.B * w.L * world * e2e_steps / e2e_s, "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": LAUNCHES_PER_STEP * args.steps,
            "aux_calls": aux,
            "configs": configs,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def sweep_subset():
    """Every L and s at B=1, r=32; the r=16 / r=64 and B=2 corners at L=8k and 128k."""
    pts = S.sweep_points()
    keep = []
    for w in pts:
        corner = w.L in (8192, 131072) and w.sparsity == 0.97
        if (w.B == 1 and w.rank == 32) or corner:
            keep.append(w)
    return keep


def run_sweep(args):
    """One JSON line per sweep point: latency split per stage and roofline fractions (device timing)."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    sda.lib()
    peaks = load_peaks()
    stream = torch.cuda.current_stream(dev)
    for w in sweep_subset():
        line = {"sweep_point": w.name}
        line.update(time_config(w, dev, stream, max(args.steps, 1), peaks))
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="sda", choices=["sda", "reference"])
    ap.add_argument("--workload", default=S.WAN14B_720P.name, choices=sorted(S.NAMED))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-aux", action="store_true", help="skip the standalone-call timings")
    ap.add_argument("--no-configs", action="store_true", help="skip the other named layers and sweep subset")
    ap.add_argument("--sweep", action="store_true", help="per-point latency split over the sweep configuration")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    w = S.NAMED[args.workload]
    if args.sweep:
        return run_sweep(args)
    if args.impl == "reference":
        return run_reference(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
