"""bench.py's multi-rank plumbing on two CPU processes over gloo.

One process per GPU in the real runs (NCCL); here two host processes stand
in for them: the rendezvous, the max-over-ranks timing, the barrier, the
per-rank workloads (independent sequences: no exchange inside the layer),
the group-sharded mode (each rank owns half of one sequence's KV groups; the
oracle run on each shard, gathered over the ranks, must equal the unsharded
layer) and the reference arm, which rank 0 alone runs.
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
    # group sharding: the oracle on this rank's groups, gathered along heads
    import numpy as np
    import oracle as O
    gsp = synth.WorkloadSpec(1, 200, 1000, 800, 16, 4, 64, 32, 128, 4, seed=9)
    pos = np.arange(gsp.q_offset, gsp.q_offset + gsp.seq_q)
    gs, (q, k, v, qi, ki) = bench.group_shard_inputs(gsp, rank, w, "cpu")
    o, _, sel, _ = O.msa_forward(q[0], k[0], v[0], qi[0], ki[0], pos, gsp.block, gsp.topk)
    parts = [torch.empty((gsp.seq_q, gs.shape.n_q_heads, gsp.head_dim), dtype=torch.float64)
             for _ in range(w)]
    pg.all_gather(parts, torch.from_numpy(np.ascontiguousarray(o)))
    sels = [torch.empty(tuple(sel.shape), dtype=torch.int32) for _ in range(w)]
    pg.all_gather(sels, torch.from_numpy(np.ascontiguousarray(sel)))
    res["heads"] = gs.heads
    if rank == 0:
        full = synth.make_inputs(gsp)
        o_f, _, sel_f, _ = O.msa_forward(full.q[0], full.k[0], full.v[0], full.q_idx[0],
                                         full.k_idx[0], pos, gsp.block, gsp.topk)
        res["group_o_equal"] = bool(np.array_equal(torch.cat(parts, 1).numpy(), o_f))
        res["group_sel_equal"] = bool(np.array_equal(torch.cat(sels, 1).numpy(), sel_f))
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
    assert res[0]["heads"] == (0, 8) and res[1]["heads"] == (8, 16)
    assert res[0]["group_o_equal"] and res[0]["group_sel_equal"]
    assert {"impl", "metric", "value", "unit", "cpu_baseline", "e2e"} <= set(res[0]["ref"])
