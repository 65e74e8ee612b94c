"""The helpers of the full-size GPU parity tests, checked on the host against
the oracle: the host re-sort of pooled scores against block_topk (integer
scores with many ties, k = 1, 5, 16, 33, q_offset > 0), and the attention
reference over a row's renumbered selected blocks against the oracle's
attention over the whole sequence."""
import numpy as np
import torch

import oracle as O
from tests.gpu_helpers import spec, inputs_cpu, oracle_pooled, oracle_sel
from tests.test_gpu_fullsize import compact_attention_ref, host_resort


def test_host_resort_matches_oracle_topk():
    rng = np.random.default_rng(0)
    for R, G, nb, k, off in [(300, 2, 40, 16, 0), (64, 8, 71, 16, 8000), (50, 3, 20, 33, 0),
                             (40, 2, 10, 1, 0), (90, 4, 30, 5, 1000)]:
        pos = np.arange(off, off + R)
        pooled = np.full((R, G, nb), -np.inf)
        for r in range(R):
            bt = pos[r] // 128
            pooled[r, :, :bt + 1] = rng.integers(-3, 4, size=(G, bt + 1))
        ref = O.block_topk(pooled, pos, 128, k)
        got = host_resort(torch.from_numpy(pooled).float(), pos, 128, k).numpy()
        assert np.array_equal(ref, got), (R, G, nb, k)


def test_compact_attention_matches_oracle():
    for sp in [spec(1, 300, 1000, 700, 16, 4, 64, 64, 5, seed=11),
               spec(1, 200, 3000, 2800, 16, 2, 128, 64, 16, seed=12)]:
        inp = inputs_cpu(sp)
        sel = oracle_sel(sp, oracle_pooled(sp, inp, 0))
        pos = np.arange(sp.q_offset, sp.q_offset + sp.seq_q)
        o_ref, _ = O.sparse_attention(inp.q[0], inp.k[0], inp.v[0], sel, pos, sp.block)
        for t in [0, 1, 57, sp.seq_q - 1]:
            oc = compact_attention_ref(sp, inp.q[0, t], inp.k[0], inp.v[0], sel[t], int(pos[t]))
            assert np.allclose(oc, o_ref[t], atol=1e-12)
