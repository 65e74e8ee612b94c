"""Failure detection on the GPU without a fault: the bounded waits.

Every wait of the kernels is bounded; an expired wait sets bit 0 of the
device error word, the kernel stops its roles, lets the loads already in
flight land and returns, and the context stays usable.  The test sets the
bound to 0 (every wait that is not complete at its first probe expires at
once), runs the sparse decode attention, which must wait for its K/V
loads, and checks that the call returns, that msa_device_status reports
the expiry, and that with the default bound restored the same call is
correct again.  Nothing here faults, traps or hangs the GPU.
"""
import numpy as np
import pytest
import torch

import block_sparse_gqa_05_b200 as M
from tests.gpu_helpers import (spec, inputs_cpu, oracle_pooled, oracle_sel, check_attn,
                               oracle_attention, cuda)

pytestmark = pytest.mark.gpu

DEFAULT_LIMIT_NS = 2_000_000_000


def test_expired_wait_is_reported_and_the_context_recovers():
    # 8 sequences x 8 groups x 16 blocks: several blocks per CTA of the
    # persistent decode grid, so its loader waits for a ring stage to free
    sp = spec(8, 1, 4096, 4095, 64, 8, 128, 64, 16, seed=81)
    inp = inputs_cpu(sp)
    sel_np = np.stack([oracle_sel(sp, oracle_pooled(sp, inp, b)) for b in range(sp.batch)])
    q, k, v, sel = cuda(inp.q), cuda(inp.k), cuda(inp.v), cuda(torch.from_numpy(sel_np))
    sh = M.Shape.of(sp)
    assert M.device_status() == 0
    try:
        M.set_wait_limit_ns(0)
        M.sparse_attn_decode(sh, q, k, v, sel)
        torch.cuda.synchronize()          # the kernel returned
        flags = M.device_status()
    finally:
        M.set_wait_limit_ns(DEFAULT_LIMIT_NS)
    assert flags & 1, f"no expired wait reported (flags {flags})"
    o, _ = M.sparse_attn_decode(sh, q, k, v, sel)
    torch.cuda.synchronize()
    assert M.device_status() == 0
    o_ref = np.stack([oracle_attention(sp, inp, sel_np[b], b)[0] for b in range(sp.batch)])
    check_attn(o, o_ref, "decode after the expired wait")


def test_expired_wait_in_the_prefill_kernels():
    # the whole prefill layer: the index-score GEMM with the fused top-k and
    # the KV-outer attention, both tcgen05 kernels whose roles drain their
    # loads and MMAs and leave their named barriers together on an expiry
    sp = spec(1, 640, 2048, 1408, 16, 2, 128, 64, 8, seed=82)
    inp = inputs_cpu(sp)
    dev = [cuda(t) for t in (inp.q, inp.k, inp.v, inp.q_idx, inp.k_idx)]
    sh = M.Shape.of(sp)
    assert M.device_status() == 0
    try:
        M.set_wait_limit_ns(0)
        M.forward(sh, *dev)
        torch.cuda.synchronize()
        flags = M.device_status()
    finally:
        M.set_wait_limit_ns(DEFAULT_LIMIT_NS)
    assert flags & 1, f"no expired wait reported (flags {flags})"
    o, _, sel = M.forward(sh, *dev)
    torch.cuda.synchronize()
    assert M.device_status() == 0
    sref = oracle_sel(sp, oracle_pooled(sp, inp, 0))
    assert np.array_equal(sel[0].cpu().numpy(), sref)
    check_attn(o[0], oracle_attention(sp, inp, sref, 0)[0], "prefill after the expired wait")
