#!/usr/bin/env python
"""Throughput of the MSA hot path on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl msa|reference]
                    [--workload prefill_128k] [--shard sequence|group]
                    [--skip-long] [--skip-cpu]

Headline step: one MSA forward (index scores -> block top-k -> KV-outer sparse
attention) over one 131072-token sequence per GPU, inputs resident in HBM.
In the same run, and reported in their own objects: batched decode (32
sequences x 128K cache), and the 1M-token context (last 8192-query prefill
chunk, batch-4 decode) beside the in-repo dense causal GQA kernels.  By
default every GPU runs an independent sequence (weak scaling, no collective on
the data path); with --shard group the GPUs split the KV groups of the one
headline sequence instead (strong scaling: each owns G/N groups' K/V, query
heads and index queries plus a replica of the index keys; no exchange inside
the layer).  The time is the max over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time
import types

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "MSA prefill & decode tokens/s at 128K and 1M ctx on 1 B200; % of roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def src_hash(files=None):
    """Hash of the library sources a kernel is built from (all of them by default)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_sparse_gqa_05_b200", "csrc")
    for f in sorted(files or os.listdir(csrc)):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel):
    """DRAM bytes per launch from a committed ncu capture of the current sources."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get("kernels", {}).get(kernel)
    if e is None or e.get("src_sha") != src_hash(e.get("sources")):
        return None   # the kernel changed since the counters were taken
    return e.get("bytes_per_launch_full")


class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            self.path = f"/tmp/msa_clocks_{os.getpid()}.csv"
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "samples": len(sm), "reasons": sorted(reasons)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            raise SystemExit("--gpus N > 1 must be launched with torch.distributed.run")
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        # NCCL between the GPUs; gloo on a host without GPUs (the CPU tests)
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(minutes=10),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(minutes=2))
        pg = dist
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local, pg


def max_over_ranks(x, pg):
    if pg is None:
        return x
    dev = "cuda" if pg.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def rank_workload(name, rank):
    """The named workload with its seed offset by rank: every rank runs an
    independent sequence (weak scaling, no exchange inside the layer)."""
    sp = synth.workload(name)
    return synth.workload(name, seed=sp.seed + 1000 * rank)


def group_shard_inputs(sp, rank, world, device):
    """This rank's group shard of workload ``sp`` (the same sequence on every
    rank): (GroupShard, (q, k, v, q_idx, k_idx)), contiguous, on ``device``."""
    from block_sparse_gqa_05_b200 import shard as S
    from block_sparse_gqa_05_b200.msa import Shape
    gs = S.group_shard(Shape.of(sp), rank, world)
    full = synth.make_inputs(sp, device)
    parts = S.shard_inputs(gs, full.q, full.k, full.v, full.q_idx, full.k_idx)
    del full
    return gs, parts


def barrier(pg):
    if pg is not None:
        pg.barrier()


def timed_loop(fn, steps, warmup, pg, stream):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(pg)
    torch.cuda.synchronize()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(steps):
        fn()
    e.record(stream)
    torch.cuda.synchronize()
    ms = s.elapsed_time(e)
    barrier(pg)
    return max_over_ranks(ms, pg) / steps


# ----------------------------------------------------------- algorithmic work
def positions(sp):
    return np.arange(sp.q_offset, sp.q_offset + sp.seq_q, dtype=np.int64)


def index_flops(sp):
    pos = positions(sp)
    return float(sp.batch * 2 * sp.n_kv_heads * sp.index_dim * (pos + 1).sum())


def selected_attention_flops(sp, sel):
    """4*r*d*128 per selected (token, group, block): the local block as a full block."""
    r = sp.n_q_heads // sp.n_kv_heads
    return float(4 * r * sp.head_dim * 128) * float((sel >= 0).sum().item())


def topk_bytes(sp):
    pos = positions(sp)
    bt = pos // 128
    return float(sp.batch * sp.n_kv_heads * (4 * bt.sum() + 4 * sp.topk * sp.seq_q))


def prefill_step_bound(sp, sel, peaks, ms):
    """The whole prefill step against the sum of its steps' bounds (the
    selection inversion and the combine are implementation steps with no
    algorithmic bound of their own)."""
    tpk = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * 1e12
    bound_ms = 1e3 * (index_flops(sp) / tpk + topk_bytes(sp) / (peaks["hbm_gbs"] * 1e9)
                      + selected_attention_flops(sp, sel) / tpk)
    return {"ms_at_bounds": round(bound_ms, 3), "frac": round(bound_ms / ms, 4),
            "terms": "index FLOP and selected-attention FLOP at sustained bf16, "
                     "top-k bytes at HBM copy bandwidth"}


def dense_flops(sp):
    """Causal GQA attention: 4*H*d FLOP per (query, causal key) pair."""
    pos = positions(sp)
    return float(sp.batch * 4 * sp.n_q_heads * sp.head_dim * (pos + 1).sum())


def dense_roofline(sp, ms, peaks):
    """The dense causal GQA prefill kernel against the sustained bf16 peak."""
    pk = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    a = dense_flops(sp) / (ms / 1e3) / 1e12
    return {"bound": "tensor", "achieved": round(a, 1), "peak": pk, "unit": "TFLOP/s",
            "frac": round(a / pk, 4), "algorithmic_per_launch": dense_flops(sp)}


def combine_bytes(sp, sel):
    """The combine's reads and writes: r partial rows of (2*d + 8) bytes per
    kept (token, group, slot), one bf16 output row per (token, head)."""
    r = sp.n_q_heads // sp.n_kv_heads
    kept = float((sel >= 0).sum().item())
    return kept * r * (2 * sp.head_dim + 8) + float(sp.batch * sp.seq_q * sp.n_q_heads * 2 * sp.head_dim)


def l2_note(sp):
    """How the timed loop relates to the 126 MB L2: its input sizes."""
    q = sp.batch * sp.seq_q * sp.n_q_heads * sp.head_dim * 2
    kv = sp.batch * sp.seq_kv * sp.n_kv_heads * sp.head_dim * 2 * 2
    return f"inputs larger than L2 (Q {q / 2**20:.0f} MiB, K/V {kv / 2**20:.0f} MiB per step)"


def decode_kv_bytes(sp):
    return float(sp.batch * sp.n_kv_heads * sp.topk * 128 * sp.head_dim * 2 * 2)


# --------------------------------------------------------------- msa arm
def run_msa(args, world, rank, pg):
    import block_sparse_gqa_05_b200 as M
    peaks, peak_src = load_peaks()
    stream = torch.cuda.current_stream()
    out = {}
    if args.shard == "group":
        # one sequence, G/world groups per rank: every rank's step covers all
        # of the sequence's tokens for its share of the heads
        sp_full = synth.workload(args.workload)
        gs, parts = group_shard_inputs(sp_full, rank, world, "cuda")
        inp = types.SimpleNamespace(**dict(zip(("q", "k", "v", "q_idx", "k_idx"), parts)))
        sp = dataclasses.replace(sp_full, n_q_heads=gs.shape.n_q_heads,
                                 n_kv_heads=gs.shape.n_kv_heads)
        token_ranks = 1
        torch.cuda.empty_cache()
    else:
        sp = rank_workload(args.workload, rank)
        inp = synth.make_inputs(sp, "cuda")
        token_ranks = world
    sh = M.Shape.of(sp)
    ws = M.alloc_workspace(sh, M.OP_FORWARD)
    o = torch.empty_like(inp.q)
    sel = torch.empty((sp.batch, sp.seq_q, sp.n_kv_heads, sp.topk), dtype=torch.int32,
                      device="cuda")

    def step():
        M.forward(sh, inp.q, inp.k, inp.v, inp.q_idx, inp.k_idx, o=o, lse=None, sel=sel, ws=ws,
                  want_lse=False)

    step()
    torch.cuda.synchronize()
    clk = ClockSampler(torch.cuda.current_device())
    clk.start()
    M.profile_enable(True)
    ms = timed_loop(step, args.steps, args.warmup, pg, stream)
    prof = M.profile_read()
    M.profile_enable(False)
    clocks = clk.stop()
    st = M.device_status()
    if st:
        raise RuntimeError(f"device error word {st}")
    nsteps = args.steps + args.warmup
    kernels = {k: v[0] / v[1] for k, v in prof.items()}   # ms per launch
    launches_per_step = sum(v[1] for v in prof.values()) / nsteps
    tokens = sp.batch * sp.seq_q
    out["value"] = tokens * token_ranks / (ms / 1e3)
    out["ms_per_step"] = ms
    out["gpu_launches"] = int(round(launches_per_step * args.steps))
    out["kernels_ms_per_launch"] = {k: round(v, 4) for k, v in kernels.items()}
    out["clocks"] = clocks
    # roofline of the dominant kernel
    dom = max(kernels, key=lambda k: kernels[k] * prof[k][1])
    work = {
        "kvouter_attn": ("tensor", selected_attention_flops(sp, sel)),
        "index_topk_tc": ("tensor", index_flops(sp)),     # index GEMM with the top-k fused in
        "index_scores_tc": ("tensor", index_flops(sp)),
        "block_topk": ("hbm", topk_bytes(sp)),
        "combine": ("hbm", combine_bytes(sp, sel)),
    }
    bound, amount = work.get(dom, ("tensor", selected_attention_flops(sp, sel)))
    dur_s = kernels[dom] / 1e3
    if bound == "tensor":
        peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
        achieved = amount / dur_s / 1e12
        unit = "TFLOP/s"
    else:
        peak = peaks["hbm_gbs"]
        achieved = amount / dur_s / 1e9
        unit = "GB/s"
    out["roofline"] = {"kernel": dom, "bound": bound, "achieved": round(achieved, 2),
                       "peak": peak, "unit": unit, "frac": round(achieved / peak, 4),
                       "peak_source": f"{peak_src} ({'sustained' if bound == 'tensor' else 'copy'})",
                       "traffic": ncu_traffic(dom),
                       "algorithmic_per_launch": amount}
    traffic = out["roofline"]["traffic"]
    if traffic:
        # the same launch against the time its measured DRAM bytes take at the
        # copy bandwidth (the KV-outer schedule's gather and partial traffic)
        floor_ms = traffic / (peaks["hbm_gbs"] * 1e9) * 1e3
        out["roofline"]["traffic_floor"] = {"ms": round(floor_ms, 3),
                                            "frac": round(floor_ms / kernels[dom], 4)}
    # every stage against its own roof
    stages = {}
    for name, (bnd, amt) in work.items():
        if name in kernels:
            d = kernels[name] / 1e3
            a = amt / d / (1e12 if bnd == "tensor" else 1e9)
            pk = peaks.get("bf16_tflops_sustained") if bnd == "tensor" else peaks["hbm_gbs"]
            stages[name] = {"ms": round(kernels[name], 4), "achieved": round(a, 2),
                            "frac": round(a / pk, 4)}
    out["stages"] = stages
    out["step_roofline"] = prefill_step_bound(sp, sel, peaks, ms)

    # ---- the same layer with the index-alignment KL (msa_forward_alignment:
    # pooled scores kept, the combine's KL variant)
    if args.alignment:
        ka = torch.empty((sp.batch, sp.seq_q, sp.n_kv_heads), dtype=torch.float32, device="cuda")
        wsa = M.alloc_workspace(sh, M.OP_FORWARD_ALIGNMENT)

        def astep():
            M.forward_alignment(sh, inp.q, inp.k, inp.v, inp.q_idx, inp.k_idx, o=o, lse=None,
                                sel=sel, kl=ka, ws=wsa, want_lse=False)
        astep()
        torch.cuda.synchronize()
        M.profile_enable(True)
        ams = timed_loop(astep, 2, 1, pg, stream)
        aprof = M.profile_read()
        M.profile_enable(False)
        out["alignment_forward"] = {
            "ms_per_step": ams,
            "kernels_ms_per_launch": {k: round(v[0] / v[1], 4) for k, v in aprof.items()}}
        del ka, wsa
        torch.cuda.empty_cache()

    # ---- the same workload through the dense causal GQA kernel (the baseline
    # the pages compare MSA against)
    if not args.skip_dense:
        def dstep():
            M.dense_attn_prefill(sh, inp.q, inp.k, inp.v, o=o, lse=None, want_lse=False)
        dms = timed_loop(dstep, 2, 1, pg, stream)
        out["dense_gqa_prefill"] = {"ms_per_step": dms, "value": tokens * token_ranks / (dms / 1e3),
                                    "speedup_msa_vs_dense": round(dms / ms, 2),
                                    "roofline": dense_roofline(sp, dms, peaks)}

    # ---- end to end through the public API with host buffers.  Each step
    # copies its inputs from pinned host memory, runs msa_forward and copies
    # the output back; the copies run on their own streams with two device
    # buffer sets, so step i's upload overlaps step i-1's compute and step
    # i-2's download, as a serving pipeline would run them.  The timed region
    # spans every step's upload, compute and download.
    if not args.skip_e2e:
        names = ("q", "k", "v", "q_idx", "k_idx")
        host = {n: getattr(inp, n).cpu().pin_memory() for n in names}
        o_host = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for _ in range(2)]
        dev = [{n: torch.empty_like(getattr(inp, n)) for n in names} for _ in range(2)]
        o_dev = [torch.empty_like(o) for _ in range(2)]
        s_up, s_cmp, s_down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()
        computed = [None, None]     # compute of the set's last step done
        downloaded = [None, None]   # download of the set's last output done

        def e2e_steps(nsteps):
            for i in range(nsteps):
                b = i % 2
                with torch.cuda.stream(s_up):
                    if computed[b] is not None:
                        s_up.wait_event(computed[b])
                    for n in names:
                        dev[b][n].copy_(host[n], non_blocking=True)
                    up = ev()
                    up.record(s_up)
                with torch.cuda.stream(s_cmp):
                    s_cmp.wait_event(up)
                    if downloaded[b] is not None:
                        s_cmp.wait_event(downloaded[b])
                    M.forward(sh, dev[b]["q"], dev[b]["k"], dev[b]["v"], dev[b]["q_idx"],
                              dev[b]["k_idx"], o=o_dev[b], lse=None, sel=sel, ws=ws,
                              want_lse=False, stream=s_cmp)
                    computed[b] = ev()
                    computed[b].record(s_cmp)
                with torch.cuda.stream(s_down):
                    s_down.wait_event(computed[b])
                    o_host[b].copy_(o_dev[b], non_blocking=True)
                    downloaded[b] = ev()
                    downloaded[b].record(s_down)

        e2e_n = max(4, min(args.steps, 8))
        e2e_steps(2)
        torch.cuda.synchronize()
        barrier(pg)
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(s_up)
        e2e_steps(e2e_n)
        for st_ in (s_cmp, s_down):
            s_up.wait_stream(st_)
        t1.record(s_up)
        torch.cuda.synchronize()
        ems = max_over_ranks(t0.elapsed_time(t1), pg) / e2e_n
        barrier(pg)
        out["e2e"] = {"value": tokens * token_ranks / (ems / 1e3), "unit": "tokens/s",
                      "ms_per_step": ems, "pipelined": "upload / compute / download streams, 2 buffer sets",
                      "h2d_bytes_per_step": int(sum(t.numel() * t.element_size() for t in host.values())),
                      "d2h_bytes_per_step": int(o_host[0].numel() * o_host[0].element_size())}
        del host, o_host, dev, o_dev
    del inp, ws, o, sel
    torch.cuda.empty_cache()

    # ---- isolated top-k over 1024 block scores per (query, group), against torch.topk
    if not args.skip_topk_micro and world == 1:
        out["topk_microbench"] = run_topk_micro(M, args, stream, peaks)
    # ---- decode at 128K, batch 32
    if not args.skip_decode:
        out["decode"] = run_decode(M, rank_workload(args.decode_workload, rank), args, pg, stream,
                                   world, peaks, dense=False)
    # ---- 1M context: prefill chunk + decode, against the dense kernels
    if not args.skip_long:
        out["ctx_1m"] = run_long(M, args, pg, stream, world, rank, peaks)
    return out, sp


def run_topk_micro(M, args, stream, peaks):
    """131072 queries x 8 groups x 1024 pooled block scores (every query at
    position 131071 of a 131072-key context, so all 1024 blocks are
    candidates): msa_block_topk (top-15 + the local block) vs
    torch.topk(pooled, 16, dim=-1) on the same tensor."""
    q, G, nb = 131072, 8, 1024
    sh = M.Shape(batch=q, seq_q=1, seq_kv=nb * 128, q_offset=nb * 128 - 1, n_q_heads=64,
                 n_kv_heads=G, head_dim=128, index_dim=64, block=128, topk=16)
    gen = torch.Generator(device="cuda").manual_seed(33)
    pooled = torch.round(torch.randn((q, 1, G, nb), device="cuda", generator=gen) * 30.0)
    sel = torch.empty((q, 1, G, 16), dtype=torch.int32, device="cuda")
    ms = timed_loop(lambda: M.block_topk(sh, pooled, sel), max(args.steps, 5), 3, None, stream)
    tms = timed_loop(lambda: torch.topk(pooled, 16, dim=-1), max(args.steps, 5), 3, None, stream)
    byts = float(pooled.numel() * 4 + sel.numel() * 4)
    a = byts / (ms / 1e3) / 1e9
    res = {"rows": q * G, "candidates_per_row": nb, "msa_block_topk_ms": round(ms, 4),
           "torch_topk_ms": round(tms, 4), "speedup_vs_torch_topk": round(tms / ms, 2),
           "achieved_gbs": round(a, 1), "frac_of_hbm": round(a / peaks["hbm_gbs"], 4),
           "values": "round(30 * N(0,1)) (integer-valued, many ties)"}
    del pooled, sel
    torch.cuda.empty_cache()
    return res


def graph_ms(fn, reps, steps, warmup, pg, stream):
    """ms per call of fn, replayed from one CUDA graph of ``reps`` calls (a
    decode loop is replayed this way in serving; eager launches would add the
    host's per-launch cost between kernels of a ~0.1 ms step)."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(reps):
            fn()
    torch.cuda.synchronize()
    ms = timed_loop(g.replay, steps, warmup, pg, stream) / reps
    del g
    return ms


def run_decode(M, sp, args, pg, stream, world, peaks, dense):
    inp = synth.make_inputs(sp, "cuda")
    sh = M.Shape.of(sp)
    ws = M.alloc_workspace(sh, M.OP_FORWARD)
    o = torch.empty_like(inp.q)
    sel = torch.empty((sp.batch, 1, sp.n_kv_heads, sp.topk), dtype=torch.int32, device="cuda")

    def step():
        M.forward(sh, inp.q, inp.k, inp.v, inp.q_idx, inp.k_idx, o=o, lse=None, sel=sel, ws=ws,
                  want_lse=False)

    reps, steps = 10, max(args.steps, 5)
    ms = graph_ms(step, reps, steps, args.warmup, pg, stream)
    # the stages one at a time, each replayed from its own graph
    pooled = torch.empty((sp.batch, 1, sp.n_kv_heads, sp.nb), dtype=torch.float32, device="cuda")
    aws = M.alloc_workspace(sh, M.OP_SPARSE_DECODE)
    stages = {
        "index_scores": lambda: M.index_scores(sh, inp.q_idx, inp.k_idx, pooled),
        "block_topk": lambda: M.block_topk(sh, pooled, sel),
        "sparse_attn_decode": lambda: M.sparse_attn_decode(sh, inp.q, inp.k, inp.v, sel, o, None,
                                                           aws, want_lse=False),
    }
    kernels = {k: graph_ms(f, reps, steps, 1, pg, stream) for k, f in stages.items()}
    res = {"workload": f"decode_L{sp.seq_kv}_b{sp.batch}",
           "value": sp.batch * world / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
           "timing": "CUDA graph replay of 10 steps per launch",
           "stages_ms_per_call": {k: round(v, 4) for k, v in kernels.items()}}
    b = decode_kv_bytes(sp)
    a = b / (kernels["sparse_attn_decode"] / 1e3) / 1e9
    res["roofline"] = {"kernel": "decode_attn", "bound": "hbm", "achieved": round(a, 1),
                       "peak": peaks["hbm_gbs"], "unit": "GB/s",
                       "frac": round(a / peaks["hbm_gbs"], 4),
                       "algorithmic_per_launch": b}
    b = float(sp.batch * sp.seq_kv * sp.index_dim * 2)
    a = b / (kernels["index_scores"] / 1e3) / 1e9
    res["index_scan"] = {"achieved_gbs": round(a, 1), "frac": round(a / peaks["hbm_gbs"], 4)}
    step_bytes = b + topk_bytes(sp) + decode_kv_bytes(sp)
    bound_ms = 1e3 * step_bytes / (peaks["hbm_gbs"] * 1e9)
    res["step_roofline"] = {"ms_at_bounds": round(bound_ms, 4), "frac": round(bound_ms / ms, 4),
                            "terms": "k_idx scan + top-k + selected K/V bytes at HBM copy bandwidth"}
    del pooled, aws
    if dense:
        dws = M.alloc_workspace(sh, M.OP_DENSE_DECODE)

        def dstep():
            M.dense_attn_decode(sh, inp.q, inp.k, inp.v, o=o, lse=None, ws=dws, want_lse=False)

        dms = graph_ms(dstep, 2, max(3, args.steps // 2), 1, pg, stream)
        db = float(sp.batch * sp.n_kv_heads * sp.seq_kv * sp.head_dim * 4)
        res["dense_gqa_decode"] = {"ms_per_step": dms, "value": sp.batch * world / (dms / 1e3),
                                   "achieved_gbs": round(db / (dms / 1e3) / 1e9, 1),
                                   "speedup_msa_vs_dense": round(dms / ms, 2)}
    del inp, ws, o, sel
    torch.cuda.empty_cache()
    return res


def run_long(M, args, pg, stream, world, rank, peaks):
    res = {}
    sp = rank_workload("prefill_1m_chunk8k", rank)
    inp = synth.make_inputs(sp, "cuda")
    sh = M.Shape.of(sp)
    ws = M.alloc_workspace(sh, M.OP_FORWARD)
    o = torch.empty_like(inp.q)
    sel = torch.empty((1, sp.seq_q, sp.n_kv_heads, sp.topk), dtype=torch.int32, device="cuda")

    def step():
        M.forward(sh, inp.q, inp.k, inp.v, inp.q_idx, inp.k_idx, o=o, lse=None, sel=sel, ws=ws,
                  want_lse=False)

    M.profile_enable(True)
    ms = timed_loop(step, max(3, args.steps // 2), args.warmup, pg, stream)
    prof = M.profile_read()
    M.profile_enable(False)
    kernels = {k: v[0] / v[1] for k, v in prof.items()}
    pre = {"workload": "prefill_1m_chunk8k", "value": sp.seq_q * world / (ms / 1e3),
           "unit": "tokens/s", "ms_per_step": ms,
           "kernels_ms_per_launch": {k: round(v, 4) for k, v in kernels.items()}}
    if "index_scores_tc" in kernels:
        f = index_flops(sp)
        a = f / (kernels["index_scores_tc"] / 1e3) / 1e12
        pk = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
        pre["roofline"] = {"kernel": "index_scores_tc", "bound": "tensor", "achieved": round(a, 1),
                           "peak": pk, "unit": "TFLOP/s", "frac": round(a / pk, 4),
                           "algorithmic_per_launch": f}
    try:
        def dstep():
            M.dense_attn_prefill(sh, inp.q, inp.k, inp.v, o=o, lse=None, want_lse=False)
        dms = timed_loop(dstep, 2, 1, pg, stream)
        pre["dense_gqa_prefill"] = {"ms_per_step": dms, "value": sp.seq_q * world / (dms / 1e3),
                                    "speedup_msa_vs_dense": round(dms / ms, 2),
                                    "roofline": dense_roofline(sp, dms, peaks)}
    except M.MsaError as e:
        pre["dense_gqa_prefill"] = {"unavailable": str(e)}
    pre["step_roofline"] = prefill_step_bound(sp, sel, peaks, ms)
    res["prefill"] = pre
    del inp, ws, o, sel
    torch.cuda.empty_cache()
    res["decode"] = run_decode(M, rank_workload("decode_1m_b4", rank), args, pg,
                               stream, world, peaks, dense=True)
    return res


# ------------------------------------------------------- oracle (CPU) arm
def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def run_oracle_sample(sp, budget_s, rng_seed=0):
    """Times the oracle on whole query rows of ``sp`` (all groups and heads)
    until ``budget_s`` seconds of oracle work; returns (tokens, seconds, sample).
    Inputs are regenerated on the host from the counter-based generator: the
    full index keys, and only the K/V blocks the sampled rows select (outside
    the timed part)."""
    import oracle as O
    sp = synth.WorkloadSpec(**{**sp.__dict__, "batch": 1})
    lay = synth.plant_layout(sp)
    kidx = synth.make_tensor(sp, "k_idx", lay=lay).double().numpy()[0]
    rng = np.random.default_rng(rng_seed)
    T, N = sp.seq_q, sp.seq_kv
    G, H, d, di = sp.n_kv_heads, sp.n_q_heads, sp.head_dim, sp.index_dim
    cand = [0, 127, 128, T - 1] + rng.integers(0, T, size=2048).tolist()
    K = np.zeros((G, N, d))      # lazily backed: only the filled blocks use memory
    V = np.zeros((G, N, d))
    filled = set()

    def fill(g, b):
        lo, hi = b * sp.block, min((b + 1) * sp.block, N)
        idx = (torch.arange(lo, hi, dtype=torch.int64)[:, None] * d
               + torch.arange(d, dtype=torch.int64)[None, :] + g * N * d).reshape(-1)
        for name, dst in (("k", K), ("v", V)):
            val = synth.values_at(sp, name, idx).float().to(torch.bfloat16).double().numpy()
            dst[g, lo:hi] = val.reshape(hi - lo, d)

    done, secs = 0, 0.0
    for t in cand:
        qi = synth.values_at(sp, "q_idx", torch.arange(t * G * di, (t + 1) * G * di), lay)
        qi = qi.numpy().reshape(1, G, di)
        q = synth.values_at(sp, "q", torch.arange(t * H * d, (t + 1) * H * d))
        q = q.float().to(torch.bfloat16).double().numpy().reshape(1, H, d)
        pos = [sp.q_offset + t]
        t0 = time.perf_counter()
        pooled = O.index_pooled(qi, kidx, pos, sp.block)
        sel = O.block_topk(pooled, pos, sp.block, sp.topk)
        secs += time.perf_counter() - t0
        for g in range(G):
            for b in sel[0, g]:
                if b >= 0 and (g, int(b)) not in filled:
                    fill(g, int(b))
                    filled.add((g, int(b)))
        t0 = time.perf_counter()
        O.sparse_attention(q, K, V, sel, pos, sp.block)
        secs += time.perf_counter() - t0
        done += 1
        if secs >= budget_s:
            break
    return done, secs, (f"{done} query rows (all {G} groups, {H} heads) of the {T}-token "
                        f"prefill over {N} keys; oracle time only, input generation excluded")


def cpu_baseline(sp, budget_s):
    n, s, desc = run_oracle_sample(sp, budget_s)
    return {"value": n / s, "unit": "tokens/s", "cores": oracle_threads(), "kind": "oracle",
            "precision": "fp64 NumPy (the oracle as it stands, stricter than fp32)",
            "sample": desc, "seconds": round(s, 2)}


def run_reference(args, world, rank, pg):
    if rank != 0:
        return None
    sp = synth.workload(args.workload)
    per_step = []
    total_n, total_s, desc = 0, 0.0, ""
    for i in range(args.warmup + args.steps):
        n, s, desc = run_oracle_sample(sp, args.ref_step_s, rng_seed=i)
        if i >= args.warmup:
            per_step.append(s / n)
            total_n += n
            total_s += s
    value = total_n / total_s
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total_s / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "seq_len": sp.seq_kv, "global_batch": sp.batch,
                       "parallelism": "single process on host cores (oracle)"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle_threads(),
                             "kind": "oracle",
                             "precision": "fp64 NumPy (the oracle as it stands, stricter than fp32)",
                             "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="msa", choices=["msa", "reference"])
    ap.add_argument("--workload", default="prefill_128k")
    ap.add_argument("--shard", default="sequence", choices=["sequence", "group"],
                    help="sequence: one independent sequence per GPU (weak scaling); "
                         "group: the GPUs split the KV groups of one sequence (strong)")
    ap.add_argument("--decode-workload", default="decode_128k_b32")
    ap.add_argument("--skip-long", action="store_true")
    ap.add_argument("--skip-decode", action="store_true")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-topk-micro", action="store_true")
    ap.add_argument("--skip-dense", action="store_true")
    ap.add_argument("--alignment", action="store_true",
                    help="also time msa_forward_alignment (the KL variant) on the workload")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-step-s", type=float, default=4.0)
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "msa":
        args.warmup = 3
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        line = run_reference(args, world, rank, None)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    world, rank, local, pg = dist_setup(args)
    res, sp = run_msa(args, world, rank, pg)
    grouped = args.shard == "group"
    if grouped:
        sp = synth.workload(args.workload)
        parallelism = (f"group-sharded over {world} GPU(s): {sp.n_kv_heads // world} KV groups "
                       f"each, index keys replicated; decode and 1M sections: independent "
                       f"sequences per GPU")
    else:
        parallelism = f"dp{world} (independent sequences)"
    if rank == 0:
        line = {"metric": METRIC, "value": res["value"], "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
                "higher_is_better": True, "scaling": "strong" if grouped else "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": args.workload, "seq_len": sp.seq_kv,
                           "global_batch": sp.batch * (1 if grouped else world),
                           "heads": f"{sp.n_q_heads}q/{sp.n_kv_heads}kv",
                           "head_dim": sp.head_dim, "index_dim": sp.index_dim, "block": sp.block,
                           "topk": sp.topk, "parallelism": parallelism,
                           "l2": l2_note(sp)},
                "gpu_launches": res["gpu_launches"], "roofline": res["roofline"],
                "stages": res["stages"], "kernels_ms_per_launch": res["kernels_ms_per_launch"],
                "clocks": res["clocks"]}
        for key in ("step_roofline", "e2e", "dense_gqa_prefill", "alignment_forward",
                    "topk_microbench", "decode", "ctx_1m"):
            if key in res:
                line[key] = res[key]
        if world == 1 and not args.skip_cpu:
            line["cpu_baseline"] = cpu_baseline(sp, args.cpu_budget)
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
