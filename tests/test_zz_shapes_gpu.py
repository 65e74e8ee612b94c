"""A sweep of the supported shape space through msa_forward (prefill and
decode), each case small, against the oracle: KV-group counts 1 to 32, head
ratios 1 to 16, both head dims and index dims, k from 1 to 64, ragged tails,
q_offset > 0 and batch > 1.  Selections bit-exact, outputs within the
attention tolerance."""
import numpy as np
import pytest
import torch

import block_sparse_gqa_05_b200 as M
from tests.gpu_helpers import (spec, inputs_cpu, oracle_pooled, oracle_sel, check_attn,
                               oracle_attention, cuda, LSE_ABS)

pytestmark = pytest.mark.gpu

#            B    T     N    q_off   H   G   d   d_i  k
CASES = [
    spec(1, 300, 1000, 700, 2, 2, 128, 32, 4, seed=101),      # r = 1, d = 128
    spec(2, 200, 900, 700, 4, 2, 64, 64, 3, seed=102),        # r = 2
    spec(1, 260, 2000, 1740, 64, 16, 64, 32, 8, seed=103),    # G = 16, r = 4
    spec(1, 130, 1500, 1370, 32, 32, 64, 32, 5, seed=104),    # G = 32, r = 1
    spec(1, 200, 3000, 2800, 32, 2, 128, 64, 16, seed=105),   # r = 16, d = 128
    spec(1, 250, 5000, 4750, 16, 2, 64, 64, 64, seed=106),    # k = 64
    spec(2, 129, 129, 0, 8, 2, 128, 32, 2, seed=107),         # one block and one key past it
    spec(1, 300, 2000, 1700, 16, 4, 128, 64, 1, seed=108),    # k = 1: the local block alone
    spec(5, 1, 2500, 2499, 32, 2, 128, 32, 16, seed=109),     # decode, r = 16
    spec(4, 1, 1000, 999, 32, 32, 64, 64, 8, seed=110),       # decode, G = 32
]


@pytest.mark.parametrize("sp", CASES, ids=lambda sp: f"B{sp.batch}T{sp.seq_q}N{sp.seq_kv}"
                         f"H{sp.n_q_heads}G{sp.n_kv_heads}d{sp.head_dim}di{sp.index_dim}k{sp.topk}")
def test_forward_shape(sp):
    inp = inputs_cpu(sp)
    o, lse, sel = M.forward(M.Shape.of(sp), cuda(inp.q), cuda(inp.k), cuda(inp.v),
                            cuda(inp.q_idx), cuda(inp.k_idx))
    torch.cuda.synchronize()
    assert M.device_status() == 0
    o_ref, l_ref = [], []
    for b in range(sp.batch):
        sref = oracle_sel(sp, oracle_pooled(sp, inp, b))
        assert np.array_equal(sel[b].cpu().numpy(), sref), f"selection b={b}"
        ob, lb = oracle_attention(sp, inp, sref, b)
        o_ref.append(ob)
        l_ref.append(lb)
    check_attn(o, np.stack(o_ref), "shape sweep")
    assert np.abs(lse.double().cpu().numpy() - np.stack(l_ref)).max() < LSE_ABS
