"""The multi-GPU plumbing of bench.py (one process per GPU, weak scaling by
replicas, max-over-ranks device time) run as two gloo ranks on CPU: the same
functions bench.py calls under torchrun with NCCL."""
import json
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    from bit_quantized_flashattention_smooth_b200 import workloads as W
    r, wsz, _ = bench.dist_setup(world, backend="gloo")
    res = {"rank": r, "world": wsz}
    # max over ranks of a per-rank device time
    res["allmax"] = bench.allmax(1.0 + r, wsz)
    # whole-job throughput: every rank's units over the slowest rank's time
    res["value"] = bench.weak_scaling_value(10.0, [1.0, 2.0, 4.0, 8.0][r], wsz)
    bench.barrier(wsz)
    # each rank draws its own batch of the workload
    w = W.WORKLOADS["tiny_mha"]
    q, _, _ = W.make_prefill(W.Workload(**{**w.__dict__, "seed": bench.rank_seed(w.seed, r)}))
    sums = [torch.zeros(1, dtype=torch.float64) for _ in range(wsz)]
    dist.all_gather(sums, q.double().sum().reshape(1))
    res["batch_sums"] = [float(t) for t in sums]
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
        json.dump(res, f)


@pytest.mark.parametrize("world", [2])
def test_bench_replicas_over_gloo(world, tmp_path):
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0, f"rank exited with {p.exitcode}"
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["world"] == world
        assert r["allmax"] == float(world)                     # max over ranks, on every rank
        assert r["value"] == pytest.approx(10.0 * world / (2.0 ** (world - 1) * 1e-3))
    sums = res[0]["batch_sums"]
    assert len(set(sums)) == world, "ranks must process different batches"
    assert all(r["batch_sums"] == sums for r in res)
