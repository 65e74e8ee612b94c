"""msa_sparse_attn_decode_static: decode attention that allocates nothing.

Callers that cannot allocate device memory on the decode path (a memory
manager that owns every device buffer in a fixed arena, or a serving loop that
must not call cudaMalloc/cudaFree because they synchronise the device) use
this entry point: its split-K scratch is a static device array inside the
library.  The test calls it through the C ABI with caller-owned outputs,
twice in a row (every call reuses the same static array), and checks each
result against the fp64 oracle fed the same selection at the parity
tolerance, and bit for bit against msa_sparse_attn_decode (caller-provided
workspace): the two run the same kernel with the same split of the work, so
only the scratch address differs.  This file is collected last so that a run
stopping at the first failure has already run the rest.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_gqa_05_b200 as M
from block_sparse_gqa_05_b200 import msa as B
from tests.gpu_helpers import (spec, inputs_cpu, oracle_pooled, oracle_sel, check_attn, cuda,
                               oracle_attention, LSE_ABS)

pytestmark = pytest.mark.gpu


def _call_static(sh, q, k, v, sel, o, lse):
    L = B.lib()
    return L.msa_sparse_attn_decode_static(
        ctypes.byref(sh), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
        ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(sel.data_ptr()),
        ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_static_scratch_decode_matches_workspace_entry_point():
    sp = spec(3, 1, 5000, 4999, 16, 2, 128, 64, 16, seed=61, planted=2)
    inp = inputs_cpu(sp)
    sel_np = np.stack([oracle_sel(sp, oracle_pooled(sp, inp, b)) for b in range(sp.batch)])
    sel = cuda(torch.from_numpy(sel_np))
    q, k, v = cuda(inp.q), cuda(inp.k), cuda(inp.v)
    sh = M.Shape.of(sp)
    # the fp64 oracle, fed the same selection
    refs = [oracle_attention(sp, inp, sel_np[b], b) for b in range(sp.batch)]
    o_orc = np.stack([r[0] for r in refs])
    lse_orc = np.stack([r[1] for r in refs])
    # the entry point with a caller-provided workspace
    o_ws, lse_ws = M.sparse_attn_decode(sh, q, k, v, sel)
    torch.cuda.synchronize()
    for _ in range(2):
        o = torch.full_like(q, float("nan"))
        lse = torch.full((sp.batch, 1, sp.n_q_heads), float("nan"), device="cuda")
        assert _call_static(sh, q, k, v, sel, o, lse) == 0
        torch.cuda.synchronize()
        check_attn(o, o_orc, "static-scratch decode vs oracle")
        assert np.abs(lse.double().cpu().numpy() - lse_orc).max() < LSE_ABS
        assert torch.equal(o, o_ws), "static-scratch and workspace decode differ"
        assert torch.equal(lse, lse_ws), "static-scratch and workspace lse differ"
    assert M.device_status() == 0


def test_static_scratch_rejects_shapes_beyond_its_size():
    # 2^20 sequences x 8 groups: the per-(sequence, group) counters alone
    # need more than the static array holds
    sp = spec(1 << 20, 1, 255, 254, 16, 8, 128, 64, 2)
    sh = M.Shape.of(sp)
    assert M.workspace_size(sh, M.OP_SPARSE_DECODE) > 24 * 2**20
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    assert _call_static(sh, dummy, dummy, dummy, dummy, dummy, dummy) == 4
