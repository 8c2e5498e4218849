"""Failure detection on the GPU: a bounded in-kernel wait that runs out.

Every wait of the tcgen05 attention kernel on pipeline progress (a TMA tile
landed, an MMA finished, a softmax tile handed over) is bounded. The
diagnostic `sda_set_attention_wait_limit_ns(0)` makes such a wait give up
unless its phase is already complete at the first, non-blocking test, so a
launch reliably takes the failure path with nothing broken: the CTA records a
time-out in the workspace status word, waits (with the normal 2 s limit) for
its own TMA loads and MMAs in flight, frees its tensor memory and exits.

The test checks the whole contract from the host: the call itself returns OK
(the failure is asynchronous), `sda_read_status` reports SDA_ERR_TIMEOUT and
clears the word, and afterwards -- limit restored -- the same problem runs
again on the same device and matches the oracle, which shows that no CTA
left tensor memory allocated (a following CTA would wait forever in its
allocation) and that the context is still usable.
"""
import numpy as np
import pytest
import torch

from sparse_rank_attention_block_b200 import sda, synthetic as S

from _gap import repair_gaps
from _gpu import ensure_lib, run_all, to_dev
from test_gpu_parity import check_all, oracle_full

pytestmark = pytest.mark.gpu

DEFAULT_LIMIT_NS = 2_000_000_000


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()


def _problem():
    # d = 128, 128-row query blocks: the tcgen05 attention kernel (plain and fused forms);
    # several query blocks per head and a ragged tail
    return S.TINY.replace(name="wait-timeout", d=128, block_q=128, rank=32, pairs_t=4, pairs_h=6, pairs_w=6,
                          grid_t=3, grid_h=11, grid_w=21, sparsity=0.7, seed=41)


@pytest.mark.parametrize("call", ["sda_sparse_attn_fwd", "sda_forward"])
def test_attention_wait_timeout_reported_then_recovers(call):
    w = _problem()
    inp = S.make_inputs(w)
    repair_gaps(inp, w)
    p = sda.params_of(w)
    d = to_dev(inp)
    ws = sda.Workspace(p)
    keep = sda.sda_keep_count(p)
    idx = torch.empty((w.B, w.H, w.n_qblk, keep), dtype=torch.int32, device="cuda")
    o = torch.empty_like(d["q"])
    sda.sda_block_select(p, d["q"], d["k"], idx, ws.ptr, ws.nbytes)
    ws.check()  # the selector ran with the normal limits

    prev = sda.sda_set_attention_wait_limit_ns(0)
    try:
        assert prev == DEFAULT_LIMIT_NS
        if call == "sda_sparse_attn_fwd":
            sda.sda_sparse_attn_fwd(p, d["q"], d["k"], d["v"], idx, o, ws.ptr, ws.nbytes)
        else:
            sda.sda_forward(p, d["q"], d["k"], d["v"], d["p_q"], d["p_k"], d["g"], o, idx, ws.ptr, ws.nbytes)
        with pytest.raises(sda.SdaError) as err:
            ws.check()
        assert err.value.code == -7, err.value  # SDA_ERR_TIMEOUT
    finally:
        assert sda.sda_set_attention_wait_limit_ns(prev) == 0
    ws.check()  # the read cleared the word

    # same device, limits restored: the whole forward matches the oracle again
    got = run_all(w, inp)
    check_all(w, inp, oracle_full(w, inp), got)
    # and the workspace that saw the time-out serves a normal call
    sda.sda_forward(p, d["q"], d["k"], d["v"], d["p_q"], d["p_k"], d["g"], o, idx, ws.ptr, ws.nbytes)
    ws.check()
    assert np.array_equal(o.float().cpu().numpy(), got["o"])
