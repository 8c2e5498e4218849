"""Seeded synthetic inputs for the compensated sparse attention forward.

This module only draws inputs. It holds none of the method's arithmetic (no
pooling, scoring, selection, attention, feature map, RoPE, state or gate), so
both the CUDA path and the fp64 oracle may take their inputs from here.

Recipe (shapes follow Wan-style DiT attention layers, whose Q/K/V are laid out
as [B, L, H, d] -- SparkDiffusion H3 portability report, section 3, "model
wall" row):

* token l of a (T, Hg, Wg) latent grid sits at raster position
  l = (t * Hg + h) * Wg + w;
* every channel c of head `head` of Q, K and V is
  z + sin(2*pi*(f_t*t/T + f_h*h/Hg + f_w*w/Wg) + psi), with z ~ N(0, 1) per
  element and, per (tensor, head, channel), integer frequencies
  f_t, f_h, f_w drawn from {1, 2} and a phase psi ~ U(0, 2*pi);
* Q and K are then RMS-normalised per (token, head) over the d channels
  (eps 1e-6, no weight): the branch inputs are the backbone's normalised
  query/key (robotworld summary, section 2.1);
* P_q, P_k ~ N(0, 1/d) of shape [r, d]; g ~ U(-0.1, 0.1) per token [B, L]
  (fp32): the gate starts near zero (robotworld summary, section 2.1);
* Q, K, V, P_q, P_k are rounded to bf16 (round to nearest even).

All random numbers come from numpy's PCG64 with the given seed, drawn in a
fixed order, with z drawn in fixed chunks of tokens.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

_TOKEN_CHUNK = 2048  # z is drawn this many tokens at a time (part of the recipe)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention-layer problem: shapes plus the method's parameters."""

    name: str
    B: int
    H: int
    d: int
    grid_t: int
    grid_h: int
    grid_w: int
    block_q: int
    block_k: int
    sparsity: float
    rank: int
    pairs_t: int
    pairs_h: int
    pairs_w: int
    seed: int
    rope_base: float = 10000.0
    rms_eps: float = 1e-6
    gate_per_head: int = 0
    causal_frames: int = 0   # 0: bidirectional; F: causal window of F-frame chunks

    @property
    def L(self) -> int:
        return self.grid_t * self.grid_h * self.grid_w

    @property
    def chunk_tokens(self) -> int:
        """Tokens per causal chunk (the whole sequence without a window)."""
        return self.causal_frames * self.grid_h * self.grid_w if self.causal_frames else self.L

    @property
    def n_qblk(self) -> int:
        """Query blocks: each causal chunk is tiled on its own."""
        return (self.L // self.chunk_tokens) * -(-self.chunk_tokens // self.block_q)

    @property
    def n_kblk(self) -> int:
        return -(-self.L // self.block_k)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The four named layer shapes plus a generator for the sweep grid.
TINY = Workload("tiny-2x32x32", B=1, H=2, d=64, grid_t=2, grid_h=32, grid_w=32,
                block_q=64, block_k=64, sparsity=0.75, rank=16,
                pairs_t=2, pairs_h=3, pairs_w=3, seed=0)
WAN13B_480P = Workload("wan1.3b-480p-21x30x52", B=1, H=12, d=128, grid_t=21, grid_h=30,
                       grid_w=52, block_q=128, block_k=64, sparsity=0.90, rank=32,
                       pairs_t=4, pairs_h=6, pairs_w=6, seed=1)
WAN14B_480P = Workload("wan14b-480p-21x30x52", B=1, H=40, d=128, grid_t=21, grid_h=30,
                       grid_w=52, block_q=128, block_k=64, sparsity=0.95, rank=32,
                       pairs_t=4, pairs_h=6, pairs_w=6, seed=2)
WAN14B_720P = Workload("wan14b-720p-21x45x80", B=1, H=40, d=128, grid_t=21, grid_h=45,
                       grid_w=80, block_q=128, block_k=64, sparsity=0.97, rank=32,
                       pairs_t=4, pairs_h=6, pairs_w=6, seed=3)

NAMED = {w.name: w for w in (TINY, WAN13B_480P, WAN14B_480P, WAN14B_720P)}

_SWEEP_GRIDS = {8192: (16, 16, 32), 16384: (16, 32, 32), 32768: (32, 32, 32),
                65536: (32, 32, 64), 131072: (32, 64, 64)}
_RANK_SPLITS = {16: (2, 3, 3), 32: (4, 6, 6), 64: (8, 12, 12)}


def sweep_points():
    """The sweep grid: H=40, d=128, B in {1,2}, L in {8k..128k}, s, r."""
    n = 0
    out = []
    for B in (1, 2):
        for L, (t, hh, ww) in _SWEEP_GRIDS.items():
            for s in (0.90, 0.95, 0.97):
                for r in (16, 32, 64):
                    pt, ph, pw = _RANK_SPLITS[r]
                    out.append(Workload(f"sweep-B{B}-L{L}-s{s:.2f}-r{r}", B=B, H=40, d=128,
                                        grid_t=t, grid_h=hh, grid_w=ww, block_q=128,
                                        block_k=64, sparsity=s, rank=r, pairs_t=pt,
                                        pairs_h=ph, pairs_w=pw, seed=100 + n))
                    n += 1
    return out


@dataclasses.dataclass
class Inputs:
    """Host-side inputs. Q/K/V/P are bf16 torch tensors, g is fp32."""

    q: torch.Tensor      # [B, L, H, d] bf16
    k: torch.Tensor      # [B, L, H, d] bf16
    v: torch.Tensor      # [B, L, H, d] bf16
    p_q: torch.Tensor    # [r, d] bf16
    p_k: torch.Tensor    # [r, d] bf16
    g: torch.Tensor      # [B, L] (or [B, L, H]) fp32


def _grid_phase(w: Workload) -> np.ndarray:
    """(L, 3) float64 fractional coordinates t/T, h/Hg, w/Wg in raster order."""
    t = np.arange(w.grid_t, dtype=np.float64) / w.grid_t
    h = np.arange(w.grid_h, dtype=np.float64) / w.grid_h
    x = np.arange(w.grid_w, dtype=np.float64) / w.grid_w
    tt, hh, xx = np.meshgrid(t, h, x, indexing="ij")
    return np.stack([tt.ravel(), hh.ravel(), xx.ravel()], axis=1)


def _draw_tensor(rng: np.random.Generator, w: Workload, normalise: bool) -> torch.Tensor:
    H, d, L, B = w.H, w.d, w.L, w.B
    freqs = torch.from_numpy(rng.integers(1, 3, size=(3, H, d)).astype(np.float32))   # f_t, f_h, f_w
    psi = torch.from_numpy(rng.uniform(0.0, 2.0 * math.pi, size=(H, d)).astype(np.float32))
    frac = torch.from_numpy((2.0 * math.pi * _grid_phase(w)).astype(np.float32))     # (L, 3)
    out = torch.empty((B, L, H, d), dtype=torch.bfloat16)
    for b in range(B):
        for l0 in range(0, L, _TOKEN_CHUNK):
            l1 = min(L, l0 + _TOKEN_CHUNK)
            z = torch.from_numpy(rng.standard_normal(size=(l1 - l0, H, d), dtype=np.float32))
            f = frac[l0:l1]
            phase = (f[:, 0, None, None] * freqs[0] + f[:, 1, None, None] * freqs[1]
                     + f[:, 2, None, None] * freqs[2] + psi)
            x = z + torch.sin(phase)
            if normalise:
                x = x * torch.rsqrt(x.square().mean(-1, keepdim=True) + 1e-6)
            out[b, l0:l1] = x.to(torch.bfloat16)
    return out


def make_inputs(w: Workload, seed: int | None = None) -> Inputs:
    """Draw the inputs of workload `w` (seed defaults to the workload's)."""
    rng = np.random.Generator(np.random.PCG64(w.seed if seed is None else seed))
    q = _draw_tensor(rng, w, normalise=True)
    k = _draw_tensor(rng, w, normalise=True)
    v = _draw_tensor(rng, w, normalise=False)
    sd = 1.0 / math.sqrt(w.d)
    p_q = torch.from_numpy(rng.normal(0.0, sd, size=(w.rank, w.d)).astype(np.float32)).to(torch.bfloat16)
    p_k = torch.from_numpy(rng.normal(0.0, sd, size=(w.rank, w.d)).astype(np.float32)).to(torch.bfloat16)
    gshape = (w.B, w.L, w.H) if w.gate_per_head else (w.B, w.L)
    g = torch.from_numpy(rng.uniform(-0.1, 0.1, size=gshape).astype(np.float32))
    return Inputs(q=q, k=k, v=v, p_q=p_q, p_k=p_k, g=g)


def perturb_token(x: torch.Tensor, b: int, l: int, h: int, eps: float, seed: int) -> None:
    """Add eps * u (u a seeded random unit vector) to x[b, l, h, :], in place, re-rounded to bf16.

    Used by the tests to move a row of block scores away from a near-tie at the
    top-k boundary; it holds no method arithmetic itself.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    u = rng.standard_normal(x.shape[-1])
    u /= np.linalg.norm(u)
    row = x[b, l, h].float().numpy().astype(np.float64) + eps * u
    x[b, l, h] = torch.from_numpy(row.astype(np.float32)).to(torch.bfloat16)


def make_inputs_device(w: Workload, seed: int | None = None, device="cuda") -> Inputs:
    """The same recipe drawn on the device with torch's generator, for timing runs.

    Same shapes, distributions and structure as make_inputs (z ~ N(0, 1) plus
    the per-channel low-frequency sinusoid, Q/K RMS-normalised, P ~ N(0, 1/d),
    g ~ U(-0.1, 0.1), bf16 rounding), but a different random stream: the values
    are not those of make_inputs, so parity tests use make_inputs. Takes
    milliseconds where make_inputs takes seconds per million tokens.
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed if seed is None else seed)
    H, d, L, B = w.H, w.d, w.L, w.B
    frac = torch.from_numpy((2.0 * math.pi * _grid_phase(w)).astype(np.float32)).to(device)   # (L, 3)

    def draw(normalise: bool) -> torch.Tensor:
        freqs = torch.randint(1, 3, (3, H, d), generator=gen, device=device).float()
        psi = torch.rand((H, d), generator=gen, device=device) * (2.0 * math.pi)
        out = torch.empty((B, L, H, d), dtype=torch.bfloat16, device=device)
        for b in range(B):
            for l0 in range(0, L, 8192):
                l1 = min(L, l0 + 8192)
                f = frac[l0:l1]
                phase = (f[:, 0, None, None] * freqs[0] + f[:, 1, None, None] * freqs[1]
                         + f[:, 2, None, None] * freqs[2] + psi)
                x = torch.randn((l1 - l0, H, d), generator=gen, device=device) + torch.sin(phase)
                if normalise:
                    x = x * torch.rsqrt(x.square().mean(-1, keepdim=True) + 1e-6)
                out[b, l0:l1] = x.to(torch.bfloat16)
        return out

    q, k, v = draw(True), draw(True), draw(False)
    sd = 1.0 / math.sqrt(d)
    p_q = (torch.randn((w.rank, d), generator=gen, device=device) * sd).to(torch.bfloat16)
    p_k = (torch.randn((w.rank, d), generator=gen, device=device) * sd).to(torch.bfloat16)
    gshape = (B, L, H) if w.gate_per_head else (B, L)
    g = torch.rand(gshape, generator=gen, device=device) * 0.2 - 0.1
    return Inputs(q=q, k=k, v=v, p_q=p_q, p_k=p_k, g=g)
