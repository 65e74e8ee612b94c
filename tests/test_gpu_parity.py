"""GPU parity of every libmsa entry point against the CPU oracle (through the C ABI).

Index scores and selections are compared bit for bit (integer-valued index
inputs make every score exact in fp32); attention outputs, fed the same
selection on both sides, within max-abs 1e-2 / mean-abs 1e-3 of the fp64
oracle.  Shapes span several tiles and ragged tails.
"""
import numpy as np
import pytest
import torch

import block_sparse_gqa_05_b200 as M
import oracle as O
import synth
from tests.gpu_helpers import (spec, inputs_cpu, positions, oracle_pooled, oracle_sel,
                               check_pooled, check_attn, oracle_attention, cuda, LSE_ABS,
                               KL_REL)

pytestmark = pytest.mark.gpu

TINY = synth.workload("tiny_prefill_2k")
# batch 2, rows T*G not a multiple of 128, q_offset > 0, N not a multiple of 128
RAGGED = spec(2, 300, 1000, 700, 16, 4, 64, 64, 5, seed=11)
RAGGED_R8 = spec(2, 300, 1000, 700, 16, 2, 128, 64, 5, seed=12)


@pytest.fixture(scope="module")
def tiny_inputs():
    return inputs_cpu(TINY)


@pytest.fixture(scope="module")
def tiny_oracle(tiny_inputs):
    pooled = oracle_pooled(TINY, tiny_inputs, 0)
    sel = oracle_sel(TINY, pooled)
    return pooled, sel


# ------------------------------------------------------------ index scores
def test_index_scores_tiny(tiny_inputs, tiny_oracle):
    sh = M.Shape.of(TINY)
    pooled = M.index_scores(sh, cuda(tiny_inputs.q_idx), cuda(tiny_inputs.k_idx))
    torch.cuda.synchronize()
    check_pooled(pooled[0], tiny_oracle[0], TINY)


@pytest.mark.parametrize("sp", [RAGGED, spec(1, 640, 9000, 8000, 8, 8, 64, 64, 16, seed=3),
                                spec(1, 513, 513, 0, 8, 1, 64, 32, 4, seed=4)])
def test_index_scores_ragged(sp):
    inp = inputs_cpu(sp, ("q_idx", "k_idx"))
    pooled = M.index_scores(M.Shape.of(sp), cuda(inp.q_idx), cuda(inp.k_idx))
    torch.cuda.synchronize()
    for b in range(sp.batch):
        check_pooled(pooled[b], oracle_pooled(sp, inp, b), sp)


@pytest.mark.parametrize("sp", [spec(3, 1, 3000, 2999, 16, 8, 128, 64, 16, seed=5),
                                spec(2, 1, 1100, 1099, 8, 2, 64, 32, 4, seed=6),
                                spec(2, 3, 700, 690, 8, 4, 64, 64, 4, seed=8)])
def test_index_scores_decode_scan(sp):
    inp = inputs_cpu(sp, ("q_idx", "k_idx"))
    pooled = M.index_scores(M.Shape.of(sp), cuda(inp.q_idx), cuda(inp.k_idx))
    torch.cuda.synchronize()
    for b in range(sp.batch):
        check_pooled(pooled[b], oracle_pooled(sp, inp, b), sp)


# ------------------------------------------------------------------ top-k
def test_topk_on_oracle_pooled(tiny_oracle):
    pooled, sel_ref = tiny_oracle
    sh = M.Shape.of(TINY)
    pl = torch.from_numpy(pooled.astype(np.float32))[None]
    sel = M.block_topk(sh, cuda(pl))
    torch.cuda.synchronize()
    assert np.array_equal(sel[0].cpu().numpy(), sel_ref)


def _random_pooled(sp, gen, lo, hi, integer=True):
    nb = sp.nb
    if integer:
        x = torch.randint(lo, hi + 1, (sp.batch, sp.seq_q, sp.n_kv_heads, nb), generator=gen).float()
    else:
        x = torch.randn((sp.batch, sp.seq_q, sp.n_kv_heads, nb), generator=gen)
    return x


@pytest.mark.parametrize("sp,lo,hi", [
    (spec(1, 4096, 4096 + 9000, 9000, 8, 8, 64, 64, 16), -3, 3),        # heavy ties
    (spec(1, 2000, 2000 + 1100, 1100, 8, 4, 64, 64, 16), -200, 200),    # nb % 4 != 0
    (spec(2, 300, 5000, 4700, 16, 8, 64, 64, 64), -5, 5),               # k = 64: general merge
    (spec(1, 500, 6000, 5500, 16, 8, 64, 64, 33), -1000, 1000),         # k-1 = 32
    (spec(64, 1, 300000, 299999, 64, 8, 64, 64, 16), -50, 50),          # 2344 blocks: 3 chunks
    (spec(16, 1, 300000, 299999, 64, 8, 64, 64, 16), 0, 0),             # all equal, long rows
    (spec(1, 1500, 1500, 0, 8, 8, 64, 64, 1), -3, 3),                   # k = 1: local only
    # few long rows: one CTA per row, lists merged across its warps
    (spec(4, 1, 300000, 299999, 16, 8, 64, 64, 64), -5, 5),             # k = 64, heavy ties
    (spec(3, 1, 300000, 299999, 16, 8, 64, 64, 33), -1000, 1000),       # k-1 = 32
    (spec(2, 1, 1 << 20, (1 << 20) - 1, 64, 8, 64, 64, 16), -50, 50),   # 8192 blocks
    (spec(8, 1, 140000, 139999, 64, 8, 64, 64, 16), -50, 50),           # 1094 blocks: 3 warps busy
])
def test_topk_random_scores(sp, lo, hi):
    gen = torch.Generator().manual_seed(sp.seq_q + sp.topk)
    pl = _random_pooled(sp, gen, lo, hi)
    sel = M.block_topk(M.Shape.of(sp), cuda(pl))
    torch.cuda.synchronize()
    got = sel.cpu().numpy()
    for b in range(sp.batch):
        ref = O.block_topk(pl[b].double().numpy(), positions(sp), sp.block, sp.topk)
        assert np.array_equal(got[b], ref), np.argwhere(got[b] != ref)[:5]


def test_topk_real_valued_scores():
    sp = spec(1, 3000, 3000 + 20000, 20000, 8, 8, 64, 64, 16)
    gen = torch.Generator().manual_seed(99)
    pl = _random_pooled(sp, gen, 0, 0, integer=False)
    sel = M.block_topk(M.Shape.of(sp), cuda(pl))
    torch.cuda.synchronize()
    ref = O.block_topk(pl[0].double().numpy(), positions(sp), sp.block, sp.topk)
    assert np.array_equal(sel[0].cpu().numpy(), ref)


# ------------------------------------------------------- sparse attention
def test_sparse_prefill_tiny(tiny_inputs, tiny_oracle):
    _, sel_ref = tiny_oracle
    sh = M.Shape.of(TINY)
    sel = cuda(torch.from_numpy(sel_ref)[None])
    o, lse = M.sparse_attn_prefill(sh, cuda(tiny_inputs.q), cuda(tiny_inputs.k),
                                   cuda(tiny_inputs.v), sel)
    torch.cuda.synchronize()
    O_ref, L_ref = oracle_attention(TINY, tiny_inputs, sel_ref, 0)
    check_attn(o[0], O_ref, "tiny prefill")
    assert np.abs(lse[0].double().cpu().numpy() - L_ref).max() < LSE_ABS


@pytest.mark.parametrize("sp", [RAGGED, RAGGED_R8])
def test_sparse_prefill_ragged(sp):
    inp = inputs_cpu(sp)
    sels = [oracle_sel(sp, oracle_pooled(sp, inp, b)) for b in range(sp.batch)]
    sel = cuda(torch.from_numpy(np.stack(sels)))
    o, lse = M.sparse_attn_prefill(M.Shape.of(sp), cuda(inp.q), cuda(inp.k), cuda(inp.v), sel)
    torch.cuda.synchronize()
    for b in range(sp.batch):
        O_ref, L_ref = oracle_attention(sp, inp, sels[b], b)
        check_attn(o[b], O_ref, f"ragged prefill b={b}")
        assert np.abs(lse[b].double().cpu().numpy() - L_ref).max() < LSE_ABS


def test_sparse_prefill_spans_token_chunks():
    # more than one 8192-token chunk of the prefill work decomposition, ragged end
    sp = spec(1, 9000, 9100, 100, 8, 2, 64, 32, 6, seed=14, planted=2)
    inp = inputs_cpu(sp)
    sel_ref = oracle_sel(sp, oracle_pooled(sp, inp, 0))
    sel = cuda(torch.from_numpy(sel_ref)[None])
    o, lse = M.sparse_attn_prefill(M.Shape.of(sp), cuda(inp.q), cuda(inp.k), cuda(inp.v), sel)
    torch.cuda.synchronize()
    O_ref, L_ref = oracle_attention(sp, inp, sel_ref, 0)
    check_attn(o[0], O_ref, "multi-chunk prefill")
    assert np.abs(lse[0].double().cpu().numpy() - L_ref).max() < LSE_ABS


@pytest.mark.parametrize("sp", [spec(3, 1, 3000, 2999, 16, 2, 128, 64, 4, seed=21),
                                spec(2, 1, 5000, 4999, 8, 2, 64, 32, 16, seed=22),
                                spec(2, 1, 129, 128, 16, 1, 128, 64, 16, seed=23),
                                # more (sequence, group, block) items than SMs: each CTA
                                # streams several blocks, some groups finish inside one CTA
                                spec(32, 1, 3000, 2999, 16, 8, 64, 32, 4, seed=24),
                                spec(12, 1, 9000, 8999, 16, 4, 128, 64, 16, seed=25)])
def test_sparse_decode(sp):
    inp = inputs_cpu(sp)
    sels = [oracle_sel(sp, oracle_pooled(sp, inp, b)) for b in range(sp.batch)]
    sel = cuda(torch.from_numpy(np.stack(sels)))
    o, lse = M.sparse_attn_decode(M.Shape.of(sp), cuda(inp.q), cuda(inp.k), cuda(inp.v), sel)
    torch.cuda.synchronize()
    for b in range(sp.batch):
        O_ref, L_ref = oracle_attention(sp, inp, sels[b], b)
        check_attn(o[b], O_ref, f"decode b={b}")
        assert np.abs(lse[b].double().cpu().numpy() - L_ref).max() < LSE_ABS


@pytest.mark.parametrize("sp", [spec(2, 1, 4000, 3999, 16, 2, 128, 64, 4, seed=31),
                                # 2504 blocks: every (sequence, group) spans many CTAs
                                spec(2, 1, 40000, 39999, 8, 4, 128, 64, 4, seed=36)])
def test_dense_decode(sp):
    inp = inputs_cpu(sp)
    o, lse = M.dense_attn_decode(M.Shape.of(sp), cuda(inp.q), cuda(inp.k), cuda(inp.v))
    torch.cuda.synchronize()
    for b in range(sp.batch):
        O_ref, L_ref = O.dense_attention(inp.q[b], inp.k[b], inp.v[b], positions(sp))
        check_attn(o[b], O_ref, f"dense decode b={b}")
        assert np.abs(lse[b].double().cpu().numpy() - L_ref).max() < LSE_ABS


@pytest.mark.parametrize("sp", [spec(1, 1000, 1000, 0, 8, 2, 64, 32, 4, seed=32),
                                spec(2, 300, 1000, 700, 16, 2, 128, 64, 4, seed=33),
                                spec(1, 130, 5000, 4870, 16, 8, 128, 64, 4, seed=34)])
def test_dense_prefill(sp):
    inp = inputs_cpu(sp)
    o, lse = M.dense_attn_prefill(M.Shape.of(sp), cuda(inp.q), cuda(inp.k), cuda(inp.v))
    torch.cuda.synchronize()
    for b in range(sp.batch):
        O_ref, L_ref = O.dense_attention(inp.q[b], inp.k[b], inp.v[b], positions(sp))
        check_attn(o[b], O_ref, f"dense prefill b={b}")
        assert np.abs(lse[b].double().cpu().numpy() - L_ref).max() < LSE_ABS


def test_dense_prefill_growing_logits_rescale():
    # key norms grow along the sequence, so row maxima keep rising block after
    # block and the accumulated output has to be rescaled
    sp = spec(1, 256, 2048, 1792, 8, 1, 64, 32, 4, seed=35)
    inp = inputs_cpu(sp)
    ramp = torch.linspace(0.2, 6.0, sp.seq_kv).view(1, 1, -1, 1)
    k = (inp.k.float() * ramp).to(torch.bfloat16)
    o, lse = M.dense_attn_prefill(M.Shape.of(sp), cuda(inp.q), cuda(k), cuda(inp.v))
    torch.cuda.synchronize()
    O_ref, L_ref = O.dense_attention(inp.q[0], k[0], inp.v[0], positions(sp))
    check_attn(o[0], O_ref, "dense prefill with rescales")
    assert np.abs(lse[0].double().cpu().numpy() - L_ref).max() < LSE_ABS


# ------------------------------------------------------------- whole layer
def test_forward_tiny(tiny_inputs, tiny_oracle):
    pooled_ref, sel_ref = tiny_oracle
    sh = M.Shape.of(TINY)
    o, lse, sel = M.forward(sh, cuda(tiny_inputs.q), cuda(tiny_inputs.k), cuda(tiny_inputs.v),
                            cuda(tiny_inputs.q_idx), cuda(tiny_inputs.k_idx))
    torch.cuda.synchronize()
    assert np.array_equal(sel[0].cpu().numpy(), sel_ref)
    O_ref, _ = oracle_attention(TINY, tiny_inputs, sel_ref, 0)
    check_attn(o[0], O_ref, "forward tiny")


@pytest.mark.parametrize("sp,mode", [
    (spec(1, 700, 4000, 3300, 16, 8, 64, 64, 16, seed=71), "ties"),     # G = 8, index values in {-1, 0, 1}
    (spec(1, 300, 3001, 2701, 8, 1, 64, 32, 17, seed=72), "ties"),     # G = 1: a row tile spans a block edge; k = 17
    (spec(2, 260, 5000, 4740, 16, 4, 64, 64, 32, seed=73), "random"),  # k = 32, the longest fused list
    (spec(1, 400, 3000, 2600, 16, 8, 64, 64, 16, seed=74), "equal"),   # every score equal
    (spec(1, 600, 600, 0, 16, 8, 128, 64, 16, seed=75), "random"),     # rows with fewer than k causal blocks
])
def test_forward_fused_topk(sp, mode):
    """The prefill forward selects blocks inside the index-score kernel (no
    pooled scores in memory).  Its selection must equal, bit for bit, the
    oracle's and the standalone msa_index_scores + msa_block_topk pipeline's,
    tie order included."""
    inp = inputs_cpu(sp)
    if mode == "ties":
        inp.q_idx = inp.q_idx.float().clamp(-1, 1).to(torch.bfloat16)
        inp.k_idx = inp.k_idx.float().clamp(-1, 1).to(torch.bfloat16)
    elif mode == "equal":
        inp.q_idx = torch.zeros_like(inp.q_idx)
    sh = M.Shape.of(sp)
    assert M.workspace_size(sh, M.OP_FORWARD) < M.workspace_size(sh, M.OP_FORWARD_ALIGNMENT)
    qi, ki = cuda(inp.q_idx), cuda(inp.k_idx)
    o, lse, sel = M.forward(sh, cuda(inp.q), cuda(inp.k), cuda(inp.v), qi, ki)
    sel_two = M.block_topk(sh, M.index_scores(sh, qi, ki))
    torch.cuda.synchronize()
    assert M.device_status() == 0
    assert torch.equal(sel, sel_two), "fused and two-kernel selections differ"
    for b in range(sp.batch):
        sref = oracle_sel(sp, oracle_pooled(sp, inp, b))
        assert np.array_equal(sel[b].cpu().numpy(), sref), f"selection b={b}"
    O_ref, _ = oracle_attention(sp, inp, oracle_sel(sp, oracle_pooled(sp, inp, 0)), 0)
    check_attn(o[0], O_ref, "fused top-k forward")


def test_forward_decode():
    sp = spec(4, 1, 20000, 19999, 16, 2, 128, 64, 16, seed=41, planted=4)
    inp = inputs_cpu(sp)
    o, lse, sel = M.forward(M.Shape.of(sp), cuda(inp.q), cuda(inp.k), cuda(inp.v),
                            cuda(inp.q_idx), cuda(inp.k_idx))
    torch.cuda.synchronize()
    for b in range(sp.batch):
        sref = oracle_sel(sp, oracle_pooled(sp, inp, b))
        assert np.array_equal(sel[b].cpu().numpy(), sref)
        O_ref, _ = oracle_attention(sp, inp, sref, b)
        check_attn(o[b], O_ref, f"forward decode b={b}")


@pytest.mark.parametrize("sp", [
    RAGGED,                                                          # r = 4, d = 64, k = 5
    spec(1, 640, 9000, 8000, 8, 8, 128, 64, 16, seed=62),            # r = 1
    spec(1, 400, 3000, 2600, 16, 2, 128, 64, 16, seed=63, planted=2),  # r = 8, d = 128
    spec(2, 1, 3000, 2999, 16, 2, 128, 64, 4, seed=64),              # T = 1 on the prefill path
    spec(1, 200, 1000, 800, 8, 2, 64, 32, 1, seed=65),               # k = 1: KL = 0
])
def test_forward_alignment_kl(sp):
    """kl against the oracle's alignment KL on the oracle's pooled scores and
    selection; o and sel as msa_forward returns them."""
    inp = inputs_cpu(sp)
    sh = M.Shape.of(sp)
    o, lse, sel, kl = M.forward_alignment(sh, cuda(inp.q), cuda(inp.k), cuda(inp.v),
                                          cuda(inp.q_idx), cuda(inp.k_idx))
    torch.cuda.synchronize()
    assert M.device_status() == 0
    for b in range(sp.batch):
        pooled = oracle_pooled(sp, inp, b)
        sref = oracle_sel(sp, pooled)
        assert np.array_equal(sel[b].cpu().numpy(), sref)
        O_ref, _ = oracle_attention(sp, inp, sref, b)
        check_attn(o[b], O_ref, f"alignment forward b={b}")
        kl_ref = O.index_alignment_kl(inp.q[b], inp.k[b], inp.v[b], sref, pooled, positions(sp),
                                      sp.block)
        got = kl[b].double().cpu().numpy()
        assert np.all(np.isfinite(got))
        err = np.abs(got - kl_ref)
        bad = np.argwhere(err > KL_REL * (kl_ref + 2.0))
        assert bad.size == 0, f"b={b}: {len(bad)} kl mismatches, first {bad[:3].tolist()}: " \
            f"gpu {got[tuple(bad[0])]} ref {kl_ref[tuple(bad[0])]}"
        if sp.topk == 1:                     # one block: both distributions are (1)
            assert np.abs(kl_ref).max() <= 1e-12 and np.abs(got).max() <= 1e-5


@pytest.mark.parametrize("world", [2, 4])
def test_group_sharded_forward(world):
    """Every rank's group shard as its own msa_forward (run one after another on
    one GPU: the shards never wait on one another): selection bit-exact with the
    oracle on the shard and with the unsharded run's groups, outputs against the
    oracle on the shard."""
    sp = spec(1, 300, 1000, 700, 16, 4, 64, 64, 5, seed=71)
    inp = inputs_cpu(sp)
    sh = M.Shape.of(sp)
    _, _, sel_full = M.forward(sh, cuda(inp.q), cuda(inp.k), cuda(inp.v), cuda(inp.q_idx),
                               cuda(inp.k_idx))
    pos = positions(sp)
    for rank in range(world):
        gs = M.group_shard(sh, rank, world)
        q, k, v, qi, ki = M.shard_inputs(gs, inp.q, inp.k, inp.v, inp.q_idx, inp.k_idx)
        o, _, sel = M.forward_group_shard(gs, cuda(q), cuda(k), cuda(v), cuda(qi), cuda(ki))
        torch.cuda.synchronize()
        sref = O.block_topk(O.index_pooled(qi[0], ki[0], pos, sp.block), pos, sp.block, sp.topk)
        g0, g1 = gs.groups
        assert np.array_equal(sel[0].cpu().numpy(), sref)
        assert torch.equal(sel[0].cpu(), sel_full[0, :, g0:g1].cpu())
        O_ref, _ = O.sparse_attention(q[0], k[0], v[0], sref, pos, sp.block)
        check_attn(o[0], O_ref, f"group shard {rank}/{world}")
    assert M.device_status() == 0


def test_device_status_clean():
    assert M.device_status() == 0


# ------------------------------------------------- ragged batched decode
def _ragged_case(sp, lens):
    inp = inputs_cpu(sp)
    sh = M.Shape.of(sp)
    seq_lens = cuda(torch.tensor(lens, dtype=torch.int32))
    o, lse, sel = M.forward_decode_ragged(sh, cuda(inp.q), cuda(inp.k), cuda(inp.v),
                                          cuda(inp.q_idx), cuda(inp.k_idx), seq_lens)
    torch.cuda.synchronize()
    return inp, o, lse, sel


@pytest.mark.parametrize("sp,lens", [
    (spec(6, 1, 9000, 8999, 16, 4, 128, 64, 16, seed=51, planted=4),
     [1, 127, 128, 129, 5000, 9000]),
    (spec(5, 1, 3000, 2999, 8, 4, 64, 32, 4, seed=52), [2, 300, 640, 2999, 3000]),
])
def test_forward_decode_ragged(sp, lens):
    inp, o, lse, sel = _ragged_case(sp, lens)
    assert M.device_status() == 0
    o_ref, l_ref = [], []
    for b, n in enumerate(lens):
        pos = np.array([n - 1])
        pooled = O.index_pooled(inp.q_idx[b], inp.k_idx[b], pos, sp.block)
        sref = O.block_topk(pooled, pos, sp.block, sp.topk)
        assert np.array_equal(sel[b].cpu().numpy(), sref), f"sel b={b} len={n}"
        ob, lb = O.sparse_attention(inp.q[b], inp.k[b], inp.v[b], sref, pos, sp.block)
        o_ref.append(ob)
        l_ref.append(lb)
    # the tolerance applies to the call's whole output (a sequence with two
    # keys alone has too few values for a mean)
    check_attn(o, np.stack(o_ref), "ragged decode")
    assert np.abs(lse.double().cpu().numpy() - np.stack(l_ref)).max() < LSE_ABS


@pytest.mark.parametrize("sp,lens", [
    (spec(4, 1, 3000, 2999, 16, 2, 128, 64, 4, seed=54), [1, 130, 1000, 2050]),
    (spec(3, 1, 2000, 1999, 8, 4, 64, 32, 5, seed=55), [7, 500, 1999]),
])
def test_forward_decode_ragged_ignores_rows_past_length(sp, lens):
    """Cache rows past each sequence's length hold NaN and Inf (memory a
    serving cache has not written yet): selections and outputs are those of
    the oracle on the clean cache."""
    inp = inputs_cpu(sp)
    k, v, ki = inp.k.clone(), inp.v.clone(), inp.k_idx.clone()
    for b, n in enumerate(lens):
        k[b, :, n:] = float("nan")
        v[b, :, n::2] = float("inf")
        v[b, :, n + 1::2] = float("nan")
        ki[b, n:] = float("nan")
    sh = M.Shape.of(sp)
    seq_lens = cuda(torch.tensor(lens, dtype=torch.int32))
    o, lse, sel = M.forward_decode_ragged(sh, cuda(inp.q), cuda(k), cuda(v), cuda(inp.q_idx),
                                          cuda(ki), seq_lens)
    torch.cuda.synchronize()
    assert M.device_status() == 0
    o_ref = []
    for b, n in enumerate(lens):
        pos = np.array([n - 1])
        sref = O.block_topk(O.index_pooled(inp.q_idx[b], inp.k_idx[b], pos, sp.block), pos,
                            sp.block, sp.topk)
        assert np.array_equal(sel[b].cpu().numpy(), sref), f"sel b={b} len={n}"
        o_ref.append(O.sparse_attention(inp.q[b], inp.k[b], inp.v[b], sref, pos, sp.block)[0])
    check_attn(o, np.stack(o_ref), "ragged decode over a poisoned tail")
    assert torch.isfinite(lse).all()


def test_forward_decode_ragged_length_out_of_range():
    # lengths 0 and capacity+5 are clamped to 1 and capacity; the kernels flag them
    sp = spec(2, 1, 1000, 999, 8, 2, 64, 32, 4, seed=53)
    inp, o, lse, sel = _ragged_case(sp, [0, 1005])
    flags = M.device_status()
    assert flags & 2, flags
    for b, n in enumerate([1, 1000]):
        pos = np.array([n - 1])
        sref = O.block_topk(O.index_pooled(inp.q_idx[b], inp.k_idx[b], pos, sp.block), pos,
                            sp.block, sp.topk)
        assert np.array_equal(sel[b].cpu().numpy(), sref)
        O_ref, _ = O.sparse_attention(inp.q[b], inp.k[b], inp.v[b], sref, pos, sp.block)
        check_attn(o[b], O_ref, f"clamped ragged decode b={b}")
