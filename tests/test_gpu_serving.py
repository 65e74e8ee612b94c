"""GPU parity for what a serving stack brings: paged caches, selections and
page tables from outside the library (bad entries are dropped and flagged,
never used as indices), and large-model head counts whose combine tables
outgrow the default shared memory.  Through the C ABI, against the oracle.
"""
import numpy as np
import pytest
import torch

import block_sparse_gqa_05_b200 as M
import oracle as O
from tests.gpu_helpers import (spec, inputs_cpu, positions, oracle_pooled, oracle_sel,
                               check_attn, oracle_attention, cuda, LSE_ABS)

pytestmark = pytest.mark.gpu


def _paged_caches(sp, inp, lens, extra, seed):
    """Pages of one 128-row block, dealt to the sequences' live blocks by a
    seeded shuffle; unused pages and rows past the capacity hold NaN; table
    entries past each length are -1 (never read)."""
    B, G, nb, N = sp.batch, sp.n_kv_heads, sp.nb, sp.seq_kv
    P = B * nb + extra
    perm = np.random.default_rng(seed).permutation(P)
    table = np.full((B, nb), -1, dtype=np.int32)
    nan = float("nan")
    kp = torch.full((P, G, 128, sp.head_dim), nan, dtype=torch.bfloat16)
    vp = torch.full((P, G, 128, sp.head_dim), nan, dtype=torch.bfloat16)
    kip = torch.full((P, 128, sp.index_dim), nan, dtype=torch.bfloat16)
    for b, n in enumerate(lens):
        for j in range((n + 127) // 128):
            pg = int(perm[b * nb + j])
            table[b, j] = pg
            r1 = min((j + 1) * 128, N)
            kp[pg, :, :r1 - j * 128] = inp.k[b, :, j * 128:r1]
            vp[pg, :, :r1 - j * 128] = inp.v[b, :, j * 128:r1]
            kip[pg, :r1 - j * 128] = inp.k_idx[b, j * 128:r1]
    return kp, vp, kip, table


@pytest.mark.parametrize("sp,lens,extra", [
    (spec(4, 1, 3000, 2999, 16, 2, 128, 64, 4, seed=56), [1, 130, 1500, 3000], 5),
    (spec(3, 1, 2048, 2047, 8, 4, 64, 32, 5, seed=57, planted=2), [7, 1000, 2048], 3),
])
def test_forward_decode_paged(sp, lens, extra):
    """Paged caches hold the contiguous caches' blocks in shuffled pages: the
    result is bit-identical to the ragged call on the contiguous caches, and
    selections and outputs match the oracle."""
    inp = inputs_cpu(sp)
    kp, vp, kip, table = _paged_caches(sp, inp, lens, extra, seed=sp.seed)
    sh = M.Shape.of(sp)
    seq_lens = cuda(torch.tensor(lens, dtype=torch.int32))
    o, lse, sel = M.forward_decode_paged(sh, cuda(inp.q), cuda(kp), cuda(vp), cuda(inp.q_idx),
                                         cuda(kip), seq_lens, cuda(torch.from_numpy(table)))
    torch.cuda.synchronize()
    assert M.device_status() == 0                  # no table entry past a length was read
    o_r, lse_r, sel_r = M.forward_decode_ragged(sh, cuda(inp.q), cuda(inp.k), cuda(inp.v),
                                                cuda(inp.q_idx), cuda(inp.k_idx), seq_lens)
    torch.cuda.synchronize()
    assert torch.equal(sel, sel_r)
    assert torch.equal(o, o_r) and torch.equal(lse, lse_r)
    o_ref = []
    for b, n in enumerate(lens):
        pos = np.array([n - 1])
        sref = O.block_topk(O.index_pooled(inp.q_idx[b], inp.k_idx[b], pos, sp.block), pos,
                            sp.block, sp.topk)
        assert np.array_equal(sel[b].cpu().numpy(), sref), f"sel b={b} len={n}"
        o_ref.append(O.sparse_attention(inp.q[b], inp.k[b], inp.v[b], sref, pos, sp.block)[0])
    check_attn(o, np.stack(o_ref), "paged decode")


def test_forward_decode_paged_bad_page_is_flagged():
    # a page id past the pool is clamped to the last page and flagged (bit 2);
    # the other sequences are unaffected
    sp = spec(2, 1, 1024, 1023, 8, 2, 64, 32, 4, seed=58)
    inp = inputs_cpu(sp)
    lens = [1024, 600]
    kp, vp, kip, table = _paged_caches(sp, inp, lens, 2, seed=58)
    table[0, 0] = kp.shape[0] + 3
    sh = M.Shape.of(sp)
    o, _, sel = M.forward_decode_paged(sh, cuda(inp.q), cuda(kp), cuda(vp), cuda(inp.q_idx),
                                       cuda(kip), cuda(torch.tensor(lens, dtype=torch.int32)),
                                       cuda(torch.from_numpy(table)))
    flags = M.device_status()
    assert flags & 4, flags
    pos = np.array([lens[1] - 1])
    sref = O.block_topk(O.index_pooled(inp.q_idx[1], inp.k_idx[1], pos, sp.block), pos, sp.block,
                        sp.topk)
    assert np.array_equal(sel[1].cpu().numpy(), sref)
    O_ref, _ = O.sparse_attention(inp.q[1], inp.k[1], inp.v[1], sref, pos, sp.block)
    check_attn(o[1], O_ref, "paged decode next to a bad page")


def test_sparse_prefill_ignores_and_flags_bad_selection():
    """Caller selections with a block past the pool, a block past the query's
    own, and a row with no block at all: the bad entries are dropped (bit 3 of
    the device error word), the rest is the oracle on what remains, and the
    empty row gives o = 0, lse = -inf."""
    sp = spec(1, 300, 1000, 700, 16, 4, 64, 64, 5, seed=59)
    inp = inputs_cpu(sp)
    sel_ok = oracle_sel(sp, oracle_pooled(sp, inp, 0))
    bad = sel_ok.copy()
    bt = positions(sp) // sp.block
    bad[0, 0, -1] = sp.nb + 7                 # past every block of the cache
    bad[1, 1, -1] = bt[1] + 1                 # the block after the query's
    bad[2] = -1                               # nothing selected
    o, lse = M.sparse_attn_prefill(M.Shape.of(sp), cuda(inp.q), cuda(inp.k), cuda(inp.v),
                                   cuda(torch.from_numpy(bad)[None]))
    flags = M.device_status()
    assert flags & 8, flags
    keep = bad.copy()
    keep[0, 0, -1] = keep[1, 1, -1] = -1
    keep[2] = sel_ok[2]                       # any selection: row 2 is checked separately
    O_ref, L_ref = oracle_attention(sp, inp, keep, 0)
    rows = np.array([t for t in range(sp.seq_q) if t != 2])
    check_attn(o[0, torch.as_tensor(rows, device=o.device)], O_ref[rows], "bad selection")
    got_l = lse[0].double().cpu().numpy()
    assert np.abs(got_l[rows] - L_ref[rows]).max() < LSE_ABS
    assert torch.count_nonzero(o[0, 2]).item() == 0 and np.all(np.isneginf(got_l[2]))


@pytest.mark.parametrize("sp", [
    spec(1, 200, 9000, 8800, 128, 8, 64, 32, 64, seed=60),   # combine tables of 66 KB
    spec(1, 150, 6000, 5850, 16, 4, 128, 64, 33, seed=62),   # k - 1 = 32, d = 128
])
def test_forward_many_heads_and_slots(sp):
    """Many heads x many slots: the combine's per-token tables outgrow the
    default 48 KB of shared memory (first case) and k is not a power of two
    (second); selections bit-exact, outputs against the oracle."""
    inp = inputs_cpu(sp)
    o, lse, sel = M.forward(M.Shape.of(sp), cuda(inp.q), cuda(inp.k), cuda(inp.v),
                            cuda(inp.q_idx), cuda(inp.k_idx))
    torch.cuda.synchronize()
    assert M.device_status() == 0
    sref = oracle_sel(sp, oracle_pooled(sp, inp, 0))
    assert np.array_equal(sel[0].cpu().numpy(), sref)
    O_ref, L_ref = oracle_attention(sp, inp, sref, 0)
    check_attn(o[0], O_ref, "many heads and slots")
    assert np.abs(lse[0].double().cpu().numpy() - L_ref).max() < LSE_ABS


@pytest.mark.parametrize("sp,extra", [
    # fused top-k in the index scores, r = 8, d = 128, last page 80 rows deep
    (spec(2, 300, 2000, 1700, 16, 2, 128, 64, 16, seed=91, planted=2), 5),
    # k = 33: index scores then the standalone top-k; d = 64, r = 2
    (spec(1, 520, 1500, 980, 8, 4, 64, 32, 33, seed=92), 3),
    # a single 128-row query tile, last page 76 rows deep
    (spec(2, 64, 1100, 1036, 16, 2, 128, 64, 4, seed=93), 2),
])
def test_forward_prefill_paged(sp, extra):
    """A chunk of query rows over paged caches (shuffled pages; rows past N
    and unused pages hold NaN): bit-identical to msa_forward on the contiguous
    caches, and selections and outputs match the oracle."""
    inp = inputs_cpu(sp)
    kp, vp, kip, table = _paged_caches(sp, inp, [sp.seq_kv] * sp.batch, extra, seed=sp.seed)
    sh = M.Shape.of(sp)
    o, lse, sel = M.forward_prefill_paged(sh, cuda(inp.q), cuda(kp), cuda(vp), cuda(inp.q_idx),
                                          cuda(kip), cuda(torch.from_numpy(table)))
    torch.cuda.synchronize()
    assert M.device_status() == 0
    o_c, lse_c, sel_c = M.forward(sh, cuda(inp.q), cuda(inp.k), cuda(inp.v), cuda(inp.q_idx),
                                  cuda(inp.k_idx))
    torch.cuda.synchronize()
    assert torch.equal(sel, sel_c), "paged and contiguous selections differ"
    assert torch.equal(o, o_c) and torch.equal(lse, lse_c), "paged and contiguous outputs differ"
    o_ref = []
    for b in range(sp.batch):
        sref = oracle_sel(sp, oracle_pooled(sp, inp, b))
        assert np.array_equal(sel[b].cpu().numpy(), sref), f"sel b={b}"
        o_ref.append(oracle_attention(sp, inp, sref, b)[0])
    check_attn(o, np.stack(o_ref), "paged chunked prefill")


def test_forward_prefill_paged_bad_page_is_flagged():
    # a page id past the pool is clamped to the last page and flagged (bit 2)
    sp = spec(1, 256, 1024, 768, 8, 2, 64, 32, 4, seed=94)
    inp = inputs_cpu(sp)
    kp, vp, kip, table = _paged_caches(sp, inp, [sp.seq_kv], 2, seed=94)
    table[0, 1] = kp.shape[0] + 7
    sh = M.Shape.of(sp)
    M.forward_prefill_paged(sh, cuda(inp.q), cuda(kp), cuda(vp), cuda(inp.q_idx), cuda(kip),
                            cuda(torch.from_numpy(table)))
    torch.cuda.synchronize()
    assert M.device_status() & 4


@pytest.mark.parametrize("sp", [
    spec(4, 1, 70000, 69999, 16, 2, 128, 64, 16, seed=91, planted=4),   # CTA-per-row top-k
    spec(16, 1, 9000, 8999, 32, 4, 64, 32, 8, seed=92),                  # warp-per-row top-k
])
def test_forward_decode_in_cuda_graph(sp):
    """A decode step captured in a CUDA graph (as a serving loop replays it):
    the top-k and the decode attention launch as programmatic dependents of
    the kernel before them, which the graph keeps as programmatic edges.
    Replays give the eager call's bits, and the eager call matches the
    oracle."""
    inp = inputs_cpu(sp)
    sh = M.Shape.of(sp)
    q, k, v, qi, ki = (cuda(inp.q), cuda(inp.k), cuda(inp.v), cuda(inp.q_idx), cuda(inp.k_idx))
    ws = M.alloc_workspace(sh, M.OP_FORWARD)
    o_e, lse_e, sel_e = M.forward(sh, q, k, v, qi, ki, ws=ws)
    torch.cuda.synchronize()
    assert M.device_status() == 0
    o = torch.full_like(o_e, float("nan"))
    lse = torch.full_like(lse_e, float("nan"))
    sel = torch.full_like(sel_e, -7)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for _ in range(3):
                M.forward(sh, q, k, v, qi, ki, o=o, lse=lse, sel=sel, ws=ws, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(4):
        g.replay()
    torch.cuda.synchronize()
    assert M.device_status() == 0
    assert torch.equal(sel, sel_e)
    assert torch.equal(o, o_e)
    assert torch.equal(lse, lse_e)
    for b in range(sp.batch):
        sref = oracle_sel(sp, oracle_pooled(sp, inp, b))
        assert np.array_equal(sel_e[b].cpu().numpy(), sref)
        O_ref, _ = oracle_attention(sp, inp, sref, b)
        check_attn(o_e[b], O_ref, f"graph decode b={b}")
    del g
