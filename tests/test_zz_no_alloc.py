"""The workspace-free low-rank entry point (collected last on purpose).

sda_lowrank_fwd_static serves callers that cannot allocate device memory (a
host whose memory planner owns every allocation, or a path where cudaMalloc's
synchronisation is not allowed): it runs the low-rank kernels with their
scratch in the library's static device array. This test calls it through the
C ABI twice in a row and compares it with sda_lowrank_fwd (workspace
version) within the tolerances of the parity tests; it also checks that a
problem too large for the array is refused on the host.
"""
import ctypes

import numpy as np
import pytest
import torch

from sparse_rank_attention_block_b200 import sda, synthetic as S

from _gpu import TOL_C_REL_L2, assert_close, ensure_lib, to_dev
from _util import f32

pytestmark = pytest.mark.gpu


def _run_both(w, seed):
    inp = S.make_inputs(w, seed=seed)
    p = sda.params_of(w)
    d = to_dev(inp)
    ws = sda.Workspace(p)
    ref_o = torch.empty_like(d["q"])
    ref_c = torch.empty((w.B, w.H, w.rank, w.d), dtype=torch.float32, device="cuda")
    sda.sda_lowrank_fwd(p, d["q"], d["k"], d["v"], d["p_q"], d["p_k"], ref_o, ref_c, ws.ptr, ws.nbytes)
    o = torch.empty_like(d["q"])
    c = torch.empty_like(ref_c)
    sda.sda_lowrank_fwd_static(p, d["q"], d["k"], d["v"], d["p_q"], d["p_k"], o, c)
    torch.cuda.synchronize()
    return f32(o), c.cpu().numpy(), f32(ref_o), ref_c.cpu().numpy()


@pytest.mark.parametrize("w", [S.TINY.replace(name="static-a", grid_t=3, grid_h=7, grid_w=11, seed=31),
                               S.TINY.replace(name="static-b", B=2, H=3, d=128, block_q=128, grid_t=4,
                                              grid_h=10, grid_w=13, rank=64, pairs_t=8, pairs_h=12,
                                              pairs_w=12, seed=32)],
                         ids=lambda w: w.name)
def test_static_matches_workspace_version_twice(w):
    ensure_lib()
    for call in range(2):   # two calls in a row share (and reuse) the static array
        o, c, ref_o, ref_c = _run_both(w, seed=w.seed + call)
        assert_close(o, ref_o, f"o_lr, call {call}")
        assert_close(c, ref_c, f"C, call {call}", max_abs=np.inf, rel_l2=TOL_C_REL_L2)


def test_static_rejects_oversized_problem():
    ensure_lib()
    w = S.TINY.replace(name="too-big", B=4, H=96, d=128, block_q=128, grid_t=8, grid_h=32, grid_w=32,
                       rank=64, pairs_t=8, pairs_h=12, pairs_w=12)
    p = sda.params_of(w)
    fake = 256  # never dereferenced: the size check runs on the host first
    # q, k, v, p_q, p_k, o_lr fake; c_out NULL; stream NULL (the signature's 8 arguments after p)
    rc = sda.lib().sda_lowrank_fwd_static(ctypes.byref(p), *([fake] * 6), None, None)
    assert rc == -4
    assert b"32 MiB" in sda.lib().sda_last_error_detail()
