"""The bench's multi-rank host logic on two CPU processes (gloo, world size 2).

Every (batch, head) of the layer is an independent problem, so several GPUs run
independent batches: each rank draws its own inputs, no collective touches the
data, and the process group only brackets the timed region and takes the
slowest rank's time. These tests run that logic with the gloo backend: the
same collective steps in the same order on both ranks, the maximum over ranks,
per-rank inputs that differ, and the whole-job rate over all ranks' tokens.
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str) -> None:
    sys.path.insert(0, ROOT)
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import bench
    from sparse_rank_attention_block_b200 import synthetic as S

    dist, r, n, local = bench.dist_setup(world, backend="gloo")
    assert (r, n, local) == (rank, world, rank)
    w = S.TINY
    inp = S.make_inputs(w, seed=bench.rank_seed(w, rank))
    # the bench's collective steps, in its order: barrier before the timed
    # region, MAX of the device time, barrier before the end-to-end region,
    # MAX of the end-to-end time, final barrier
    step_s = 0.010 * (rank + 1)           # rank 1 is the slower one
    e2e_s = 0.030 * (world - rank)        # rank 0 is the slower one
    dist.barrier()
    max_s = bench.time_max_over_ranks(dist, step_s, device="cpu")
    dist.barrier()
    max_e2e = bench.time_max_over_ranks(dist, e2e_s, device="cpu")
    # what each rank processed, gathered only to check it here
    sums = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
    dist.all_gather(sums, inp.q.double().sum().reshape(1))
    dist.barrier()
    dist.destroy_process_group()
    value = bench.whole_job_tokens_per_s(w, world, 4, max_s)
    torch.save({"max_s": max_s, "max_e2e": max_e2e, "sums": [float(x) for x in sums], "value": value,
                "shape": tuple(inp.q.shape), "seed": bench.rank_seed(w, rank)},
               os.path.join(out_dir, f"rank{rank}.pt"))


def test_two_gloo_ranks(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [torch.load(tmp_path / f"rank{r}.pt") for r in range(world)]
    for r in res:
        # the slowest rank's time on every rank
        assert r["max_s"] == pytest.approx(0.020)
        assert r["max_e2e"] == pytest.approx(0.060)
        # all ranks' tokens over that time: 2 ranks x B*L tokens x 4 steps / 0.020 s
        assert r["value"] == pytest.approx(2 * 1 * 2048 * 4 / 0.020)
        assert r["shape"] == res[0]["shape"]
    # each rank its own batch: the seeds and the drawn inputs differ, rank 0 keeps the workload's seed
    assert res[0]["seed"] == 0 and res[1]["seed"] != res[0]["seed"]
    assert res[0]["sums"] == res[1]["sums"]
    assert res[0]["sums"][0] != res[0]["sums"][1]


def test_single_process_needs_no_group(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.delenv("RANK", raising=False)
    assert bench.dist_setup(1, backend="gloo") == (None, 0, 1, 0)
    assert bench.time_max_over_ranks(None, 1.25) == 1.25
