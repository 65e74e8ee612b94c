"""bench.py's multi-rank plumbing on two CPU processes over gloo.

One process per GPU in the real runs (NCCL); here two host processes stand
in for them: the rendezvous, the max-over-ranks timing, the barrier, the
per-rank workloads (independent sequences: no exchange inside the layer) and
the reference arm, which rank 0 alone runs.
"""
import os
import socket
import sys
import types

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "WORLD_SIZE": str(world), "RANK": str(rank), "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    import bench
    import synth
    args = types.SimpleNamespace(gpus=world, workload="tiny_prefill_2k", steps=1, warmup=0,
                                 ref_step_s=0.05)
    w, r, local, pg = bench.dist_setup(args)
    res = {"world": w, "rank": r, "backend": pg.get_backend()}
    res["max"] = bench.max_over_ranks(float(10 * (rank + 1)), pg)
    bench.barrier(pg)
    sp = bench.rank_workload("tiny_prefill_2k", rank)
    res["seed"] = sp.seed
    q = synth.make_tensor(sp, "q")
    res["q_head"] = q.flatten()[:8].float().tolist()
    line = bench.run_reference(args, w, r, pg)
    res["ref"] = None if line is None else sorted(line)
    bench.barrier(pg)
    pg.destroy_process_group()
    torch.save(res, os.path.join(out_dir, f"rank{rank}.pt"))


def test_two_ranks_over_gloo(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [torch.load(tmp_path / f"rank{r}.pt") for r in range(world)]
    for r, x in enumerate(res):
        assert x["world"] == world and x["rank"] == r and x["backend"] == "gloo"
        assert x["max"] == 10.0 * world            # every rank sees the slowest rank's time
    assert res[0]["seed"] != res[1]["seed"]       # independent sequences per rank
    assert res[0]["q_head"] != res[1]["q_head"]
    assert res[1]["ref"] is None                  # the reference arm runs on rank 0 only
    assert {"impl", "metric", "value", "unit", "cpu_baseline", "e2e"} <= set(res[0]["ref"])
