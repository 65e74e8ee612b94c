"""Group sharding of the layer (host side and the oracle's group independence).

The layer has no exchange step between KV groups: the index query, the top-k
and the selection are per group, and only the index keys are read by every
group.  These tests check the shard bookkeeping and that the oracle run on
each rank's groups reproduces the matching slice of the unsharded layer,
exactly: the property that lets ranks split the groups with no collective.
"""
import numpy as np
import pytest

import block_sparse_gqa_05_b200 as M
import oracle as O
import synth


FULL = M.Shape(1, 131072, 131072, 0, 64, 8, 128, 64, 128, 16)


@pytest.mark.parametrize("world", [1, 2, 4, 8])
def test_shards_partition_heads_and_groups(world):
    heads, groups = [], []
    for rank in range(world):
        gs = M.group_shard(FULL, rank, world)
        s = gs.shape
        assert (s.n_kv_heads, s.n_q_heads) == (8 // world, 64 // world)
        assert s.n_q_heads // s.n_kv_heads == 8                       # r unchanged
        assert gs.heads == (gs.groups[0] * 8, gs.groups[1] * 8)       # heads follow groups
        for f in ("batch", "seq_q", "seq_kv", "q_offset", "head_dim", "index_dim", "block",
                  "topk"):
            assert getattr(s, f) == getattr(FULL, f)
        assert M.workspace_size(s, M.OP_FORWARD) > 0                  # a valid shape
        heads += list(range(*gs.heads))
        groups += list(range(*gs.groups))
    assert heads == list(range(64)) and groups == list(range(8))


@pytest.mark.parametrize("rank,world", [(0, 3), (2, 2), (-1, 2), (0, 0)])
def test_bad_shards_rejected(rank, world):
    with pytest.raises(ValueError):
        M.group_shard(FULL, rank, world)


def _small():
    return synth.WorkloadSpec(1, 260, 1200, 940, 16, 4, 64, 32, 128, 4, seed=5)


def test_shard_inputs_are_the_layout_slices():
    sp = _small()
    inp = synth.make_inputs(sp)
    gs = M.group_shard(M.Shape.of(sp), 1, 2)
    q, k, v, qi, ki = M.shard_inputs(gs, inp.q, inp.k, inp.v, inp.q_idx, inp.k_idx)
    assert q.equal(inp.q[:, :, 8:16]) and q.is_contiguous()
    assert k.equal(inp.k[:, 2:4]) and v.equal(inp.v[:, 2:4]) and k.is_contiguous()
    assert qi.equal(inp.q_idx[:, :, 2:4]) and qi.is_contiguous()
    assert ki is inp.k_idx                                         # replicated, not copied


@pytest.mark.parametrize("world", [2, 4])
def test_oracle_layer_is_group_independent(world):
    sp = _small()
    inp = synth.make_inputs(sp)
    pos = np.arange(sp.q_offset, sp.q_offset + sp.seq_q)
    O_full, L_full, sel_full, pooled_full = O.msa_forward(
        inp.q[0], inp.k[0], inp.v[0], inp.q_idx[0], inp.k_idx[0], pos, sp.block, sp.topk)
    for rank in range(world):
        gs = M.group_shard(M.Shape.of(sp), rank, world)
        q, k, v, qi, ki = M.shard_inputs(gs, inp.q, inp.k, inp.v, inp.q_idx, inp.k_idx)
        o, lse, sel, pooled = O.msa_forward(q[0], k[0], v[0], qi[0], ki[0], pos, sp.block,
                                            sp.topk)
        h0, h1 = gs.heads
        g0, g1 = gs.groups
        assert np.array_equal(sel, sel_full[:, g0:g1])
        assert np.array_equal(pooled, pooled_full[:, g0:g1], equal_nan=True)
        assert np.array_equal(o, O_full[:, h0:h1]) and np.array_equal(lse, L_full[:, h0:h1])
