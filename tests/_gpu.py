"""Helpers of the GPU parity tests: run every C-ABI call on one problem."""
import numpy as np
import torch

from sparse_rank_attention_block_b200 import build, sda

from _util import f32

# Output tolerances of the floating-point results against the fp64 oracle
# (element-wise max-abs and relative L2 over the compared elements).
TOL_MAX_ABS = 2e-2
TOL_REL_L2 = 1e-2
# State C: fp32 accumulation of features carried to ~16 bits (bf16 head+tail)
# times exact bf16 V; expected relative error ~ 2^-16 per product, averaging
# down over the sum, so a 1e-4 relative-L2 bound leaves a wide margin.
TOL_C_REL_L2 = 1e-4


def ensure_lib():
    if not torch.cuda.is_available():
        raise RuntimeError("GPU tests need a CUDA device")
    build.build()
    return sda.lib()


def to_dev(inp, device="cuda"):
    return {n: getattr(inp, n).to(device).contiguous() for n in ("q", "k", "v", "p_q", "p_k", "g")}


def run_all(w, inp, fused_only=False):
    """Run every entry point on `inp`; returns host numpy results."""
    p = sda.params_of(w)
    d = to_dev(inp)
    ws = sda.Workspace(p)
    keep = sda.sda_keep_count(p)
    out = {"keep": keep}
    dev = d["q"].device
    idx = torch.full((w.B, w.H, w.n_qblk, keep), -1, dtype=torch.int32, device=dev)
    o = torch.empty_like(d["q"])
    sda.sda_forward(p, d["q"], d["k"], d["v"], d["p_q"], d["p_k"], d["g"], o, idx, ws.ptr, ws.nbytes)
    ws.check()
    out["o"] = f32(o)
    out["map_fused"] = idx.cpu().numpy()
    if fused_only:
        return out
    idx2 = torch.full_like(idx, -1)
    sda.sda_block_select(p, d["q"], d["k"], idx2, ws.ptr, ws.nbytes)
    o_s = torch.empty_like(d["q"])
    sda.sda_sparse_attn_fwd(p, d["q"], d["k"], d["v"], idx2, o_s, ws.ptr, ws.nbytes)
    o_lr = torch.empty_like(d["q"])
    c = torch.empty((w.B, w.H, w.rank, w.d), dtype=torch.float32, device=dev)
    sda.sda_lowrank_fwd(p, d["q"], d["k"], d["v"], d["p_q"], d["p_k"], o_lr, c, ws.ptr, ws.nbytes)
    o_g = torch.empty_like(d["q"])
    sda.sda_gate_fuse(p, o_s, o_lr, d["g"], o_g)
    ws.check()
    torch.cuda.synchronize()
    out.update(map=idx2.cpu().numpy(), o_s=f32(o_s), o_lr=f32(o_lr), C=c.cpu().numpy().astype(np.float64),
               o_gate=f32(o_g))
    return out


def assert_close(got, ref, what, max_abs=TOL_MAX_ABS, rel_l2=TOL_REL_L2):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    ma = float(np.max(np.abs(got - ref))) if got.size else 0.0
    rl = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)) if got.size else 0.0
    assert ma <= max_abs and rl <= rel_l2, f"{what}: max-abs {ma:.3e} (tol {max_abs}), rel-L2 {rl:.3e} (tol {rel_l2})"
    return ma, rl
