"""Helpers shared by the GPU parity tests (inputs, oracle calls, comparisons)."""
import numpy as np
import torch

import oracle as O
import synth

# Tolerances of the attention outputs against the fp64 oracle, both sides fed
# the same selection (bf16 inputs and outputs, fp32 accumulation).
MAX_ABS = 1e-2
MEAN_ABS = 1e-3
# Log-sum-exp (natural log): the kernels round P to bf16 before summing the
# row normaliser l, so |d lse| = |d l| / l <= 2^-9 from that rounding alone,
# plus fp32 accumulation; 4e-3 leaves a 2x margin.
LSE_ABS = 4e-3
# Index-alignment KL.  P_main(j) is built from the same l sums, so each block
# mass has relative error eps <= 2 * 2^-9 (numerator and normaliser).  With
# sum_j dP_main(j) = 0, dKL = sum_j dP_main(j) ln(P_main(j) / P_index(j)), and
# sum_j P_main |ln(P_main / P_index)| <= KL + 2 (the terms with P_main < P_index
# add at most sum P_index <= 1 in absolute value), so |dKL| <= eps (KL + 2);
# the tolerance doubles eps.
KL_REL = 8e-3


def spec(batch, seq_q, seq_kv, q_offset, H, G, d, di, topk, seed=7, planted=0):
    return synth.WorkloadSpec(batch, seq_q, seq_kv, q_offset, H, G, d, di, 128, topk,
                              seed=seed, planted=planted)


def inputs_cpu(sp, names=("q", "k", "v", "q_idx", "k_idx")):
    return synth.make_inputs(sp, "cpu", names)


def positions(sp):
    return np.arange(sp.q_offset, sp.q_offset + sp.seq_q)


def oracle_pooled(sp, inp, b):
    return O.index_pooled(inp.q_idx[b], inp.k_idx[b], positions(sp), sp.block)


def oracle_sel(sp, pooled):
    return O.block_topk(pooled, positions(sp), sp.block, sp.topk)


def check_pooled(gpu, ref, sp):
    """Bit-exact on causal blocks, -inf above the local block."""
    g = gpu.double().cpu().numpy()
    assert g.shape == ref.shape, (g.shape, ref.shape)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isneginf(g), np.isneginf(ref)), "-inf pattern differs"
    bad = np.argwhere(fin & (g != ref))
    assert bad.size == 0, f"{len(bad)} pooled mismatches, first {bad[:5].tolist()}: " \
        f"gpu {g[tuple(bad[0])]} ref {ref[tuple(bad[0])]}"


def check_attn(o_gpu, o_ref, what=""):
    g = o_gpu.double().cpu().numpy()
    err = np.abs(g - o_ref)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= MAX_ABS and mean <= MEAN_ABS, f"{what}: max abs {mx:.3e}, mean abs {mean:.3e}"
    return mx, mean


def oracle_attention(sp, inp, sel_np, b):
    return O.sparse_attention(inp.q[b], inp.k[b], inp.v[b], sel_np, positions(sp), sp.block)


def cuda(t):
    return t.contiguous().cuda()
