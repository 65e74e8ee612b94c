"""bench.py's algorithmic-work accounting against closed forms.

These numbers are the numerators of every roofline fraction the benchmark
prints, so they are pinned here by hand-derived totals for the named
workloads.
"""
import importlib.util
import os

import numpy as np
import pytest
import torch

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_index_flops_closed_form(bench):
    # causal prefill from position 0: 2*G*d_i * sum_{t<T} (t+1) = G*d_i*T*(T+1)
    sp = synth.workload("prefill_128k")
    T = sp.seq_q
    assert bench.index_flops(sp) == sp.n_kv_heads * sp.index_dim * T * (T + 1)
    assert bench.index_flops(sp) == pytest.approx(8.80e12, rel=1e-3)
    # the 1M chunk: positions N-8192 .. N-1
    sp = synth.workload("prefill_1m_chunk8k")
    p = np.arange(sp.q_offset, sp.q_offset + sp.seq_q, dtype=np.float64)
    assert bench.index_flops(sp) == 2 * sp.n_kv_heads * sp.index_dim * (p + 1).sum()
    assert bench.index_flops(sp) == pytest.approx(8.76e12, rel=1e-3)


def test_selected_attention_flops_closed_form(bench):
    # every (token, group) attends min(k, b_t + 1) blocks; the first 15 blocks
    # of tokens hold 1..15 of them, every later token 16
    sp = synth.workload("prefill_128k")
    T, G, k = sp.seq_q, sp.n_kv_heads, sp.topk
    bt = np.arange(T) // 128
    count = np.minimum(k, bt + 1)
    sel = torch.full((1, T, G, k), -1, dtype=torch.int32)
    for c in range(1, k + 1):
        rows = torch.from_numpy(count >= c)
        sel[0, rows, :, c - 1] = 0
    per_group = 128 * sum(range(1, 16)) + (T - 15 * 128) * 16
    assert int((sel >= 0).sum()) == G * per_group
    r = sp.n_q_heads // G
    assert bench.selected_attention_flops(sp, sel) == 4 * r * sp.head_dim * 128 * G * per_group
    assert bench.selected_attention_flops(sp, sel) == pytest.approx(8.73e12, rel=1e-3)


def test_decode_bytes_closed_form(bench):
    sp = synth.workload("decode_128k_b32")
    assert bench.decode_kv_bytes(sp) == 256 * 2 ** 20          # 32 x 8 x 16 blocks x 32 KB
    # top-k: 4 B per causal block before the local one, 4 B per selected slot
    bt = (sp.seq_kv - 1) // 128
    assert bench.topk_bytes(sp) == sp.batch * sp.n_kv_heads * (4 * bt + 4 * sp.topk)


def test_prefill_step_bound_is_the_sum_of_stage_bounds(bench):
    sp = synth.workload("tiny_prefill_2k")
    sel = torch.zeros((1, sp.seq_q, sp.n_kv_heads, sp.topk), dtype=torch.int32)
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops": 2000.0, "bf16_tflops_sustained": 1000.0}
    out = bench.prefill_step_bound(sp, sel, peaks, ms=2.0)
    want = 1e3 * (bench.index_flops(sp) / 1e15 + bench.topk_bytes(sp) / 1e12
                  + bench.selected_attention_flops(sp, sel) / 1e15)
    assert out["ms_at_bounds"] == pytest.approx(want, abs=1e-3)
    assert out["frac"] == pytest.approx(want / 2.0, abs=1e-4)
