"""Time `sda_backward` on one named synthetic workload (one GPU).

    python -m sparse_rank_attention_block_b200.time_backward wan14b-720p-21x45x80

Inputs come from the workload's device recipe (`synthetic.make_inputs_device`),
the block map from `sda_block_select`, and the upstream gradient of O is the
inputs' V. One untimed call, then five calls between two CUDA events on the
current stream; prints one JSON line with the mean milliseconds per call and
whether the five reruns reproduced the first call's dq, dk and dv bit for bit.
"""
import json
import sys

import torch

from . import sda
from . import synthetic as S


def main(argv=None) -> int:
    argv = sys.argv[1:] if argv is None else argv
    name = argv[0] if argv else S.WAN14B_720P.name
    w = S.NAMED[name]
    dev = torch.device("cuda", 0)
    inp = S.make_inputs_device(w, device=dev)
    d = {n: getattr(inp, n) for n in ("q", "k", "v", "p_q", "p_k", "g")}
    p = sda.params_of(w)
    ws = sda.Workspace(p, device=dev)
    keep = sda.sda_keep_count(p)
    idx = torch.empty((w.B, w.H, w.n_qblk, keep), dtype=torch.int32, device=dev)
    sda.sda_block_select(p, d["q"], d["k"], idx, ws.ptr, ws.nbytes)
    nb = sda.sda_backward_workspace_size(p)
    wsb = torch.empty(nb + 256, dtype=torch.uint8, device=dev)
    pb = wsb.data_ptr() + (-wsb.data_ptr()) % 256
    sda.sda_workspace_init(pb, nb)
    grads = [torch.empty(d["q"].shape, dtype=torch.float32, device=dev) for _ in range(3)]
    gp = [torch.empty((w.rank, w.d), dtype=torch.float32, device=dev) for _ in range(2)]
    gg = torch.empty_like(d["g"])

    def call():
        sda.sda_backward(p, d["q"], d["k"], d["v"], d["p_q"], d["p_k"], d["g"], idx, d["v"],
                         *grads, *gp, gg, pb, nb)

    call()
    torch.cuda.synchronize()
    sda.sda_read_status(pb, nb)
    first = [x.clone() for x in grads]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = 5
    e0.record()
    for _ in range(n):
        call()
    e1.record()
    torch.cuda.synchronize()
    sda.sda_read_status(pb, nb)
    same = all(torch.equal(a, b) for a, b in zip(first, grads))
    print(json.dumps({"workload": name, "ms": e0.elapsed_time(e1) / n, "rerun_bit_identical": same}))
    return 0


if __name__ == "__main__":
    sys.exit(main())
