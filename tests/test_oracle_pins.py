"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test fixes a result by a route other than the oracle's own code: hand-built
inputs with known answers, a library routine (torch SDPA) for a special case
the method reduces to, closed forms, brute-force definitions on tiny inputs,
and numbers the pages print.  A plausible slip in the oracle (a dropped scale,
an off-by-one causal bound, a wrong group index, a reversed tie-break) fails
at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- index branch

def test_pooled_onehot_key_known_values():
    # one key j* = 3*e_2 among zero keys; group 0 queries 2*e_2, group 1 queries -e_2
    N, B, di = 40, 8, 4
    jstar = 13                                   # block 1 (keys 8..15)
    k_idx = np.zeros((N, di)); k_idx[jstar, 2] = 3.0
    q_idx = np.zeros((3, 2, di)); q_idx[:, 0, 2] = 2.0; q_idx[:, 1, 2] = -1.0
    pos = [12, 13, 39]                           # before j*, at j*, far after
    pooled = O.index_pooled(q_idx, k_idx, pos, B)
    assert pooled.shape == (3, 2, 5)
    # p=12: j* is in the future -> block 1 scores 0 (keys 8..12 all zero)
    assert pooled[0, 0, 1] == 0.0 and pooled[0, 1, 1] == 0.0
    assert np.all(np.isneginf(pooled[0, :, 2:]))
    # p=13: j* now causal: group 0 sees 6, group 1 sees max(0, -3) = 0
    assert pooled[1, 0, 1] == 6.0 and pooled[1, 1, 1] == 0.0
    # p=39: every block causal, only block 1 is non-zero for group 0
    assert list(pooled[2, 0]) == [0.0, 6.0, 0.0, 0.0, 0.0]
    assert list(pooled[2, 1]) == [0.0, 0.0, 0.0, 0.0, 0.0]


def test_pooled_partial_local_block_uses_causal_keys_only():
    N, B, di = 16, 8, 2
    rng = np.random.default_rng(0)
    k_idx = rng.integers(-3, 4, size=(N, di)).astype(float)
    k_idx[11] = [100.0, 0.0]                     # huge key just after p
    q_idx = np.array([[[1.0, 0.0]]])
    pooled = O.index_pooled(q_idx, k_idx, [10], B)
    assert pooled[0, 0, 1] == max(k_idx[8:11, 0])   # keys 8,9,10 only
    assert pooled[0, 0, 0] == max(k_idx[0:8, 0])


def test_pooled_brute_force_tiny():
    rng = np.random.default_rng(1)
    N, B, di, G = 21, 4, 3, 2
    k_idx = rng.integers(-3, 4, size=(N, di)).astype(float)
    pos = [0, 3, 4, 9, 20]
    q_idx = rng.integers(-3, 4, size=(len(pos), G, di)).astype(float)
    pooled = O.index_pooled(q_idx, k_idx, pos, B)
    for r, p in enumerate(pos):
        for g in range(G):
            for b in range(6):
                best = -math.inf
                for j in range(N):
                    if j // B == b and j <= p:
                        best = max(best, sum(q_idx[r, g, c] * k_idx[j, c] for c in range(di)))
                assert pooled[r, g, b] == best


# ------------------------------------------------------------- block selection

def test_select_all_equal_takes_lowest_indices_plus_local():
    sel = O.select_blocks(np.zeros(20), b_t=12, k=5)
    assert list(sel) == [0, 1, 2, 3, 12]


def test_select_increasing_takes_latest():
    sel = O.select_blocks(np.arange(20, dtype=float), b_t=12, k=5)
    assert list(sel) == [8, 9, 10, 11, 12]


def test_select_tie_at_boundary_lower_index_wins():
    s = np.array([5, 9, 7, 9, 7, 7, 1, 0], dtype=float)
    # local = 7; top-3 of blocks 0..6: 9(b1), 9(b3), then 7 at b2/b4/b5 -> b2
    assert list(O.select_blocks(s, b_t=7, k=4)) == [1, 2, 3, 7]


def test_select_matches_beaten_by_count_definition():
    rng = np.random.default_rng(2)
    for trial in range(50):
        nb = int(rng.integers(2, 40))
        b_t = int(rng.integers(0, nb))
        k = int(rng.integers(1, 10))
        s = rng.integers(-5, 6, size=nb).astype(float)      # many ties
        # definition: block b < b_t is kept iff fewer than k-1 blocks beat it,
        # where c beats b if s_c > s_b, or s_c == s_b and c < b
        keep = [b for b in range(b_t)
                if sum(1 for c in range(b_t) if s[c] > s[b] or (s[c] == s[b] and c < b)) < k - 1]
        want = sorted(keep + [b_t])
        sel = O.select_blocks(s, b_t, k)
        got = [int(x) for x in sel if x >= 0]
        assert got == want
        assert all(x == -1 for x in sel[len(got):])


def test_select_local_forced_even_if_lowest_and_k1():
    s = np.array([10, 10, 10, -100], dtype=float)
    assert list(O.select_blocks(s, b_t=3, k=2)) == [0, 3]
    assert list(O.select_blocks(s, b_t=3, k=1)) == [3]


def test_select_fewer_blocks_than_k_pads():
    assert list(O.select_blocks(np.ones(3), b_t=2, k=6)) == [0, 1, 2, -1, -1, -1]
    assert list(O.select_blocks(np.ones(1), b_t=0, k=4)) == [0, -1, -1, -1]


def test_topk_rows_use_each_rows_local_block():
    B = 4
    pooled = np.zeros((3, 2, 6))
    pooled[:, 1, 0] = 5.0
    sel = O.block_topk(pooled, [0, 9, 23], B, k=2)
    assert sel[0, 0].tolist() == [0, -1]
    assert sel[1, 0].tolist() == [0, 2] and sel[1, 1].tolist() == [0, 2]
    assert sel[2, 0].tolist() == [0, 5]


def test_budget_golden():
    gold = json.load(open(os.path.join(GOLD, "budget_and_flops.json")))["budget"]
    k, B = gold["blocks"], gold["block_tokens"]
    assert k * B == gold["total_tokens"]
    # a query at the last token of block b_t >= k-1 attends exactly k*B keys
    b_t = 40
    p = (b_t + 1) * B - 1
    sel = O.select_blocks(np.random.default_rng(3).normal(size=64), b_t, k)
    assert len(O.attended_keys(sel, p, B, 64 * B)) == gold["total_tokens"]
    # elsewhere in the block: (k-1)*B + (p mod B) + 1
    for p in (b_t * B, b_t * B + 57):
        assert len(O.attended_keys(sel, p, B, 64 * B)) == (k - 1) * B + p % B + 1


def test_flops_ratio_golden():
    gold = json.load(open(os.path.join(GOLD, "budget_and_flops.json")))["flops_ratio_1m"]
    s = gold["shapes"]
    ratio = O.attention_flops_ratio(gold["context_tokens"], s["H"], s["d"], s["G"],
                                    s["d_idx"], s["k"], s["B"])
    assert abs(ratio - 256.0 / 9.0) < 1e-12
    assert abs(ratio - gold["value"]) / gold["value"] < gold["rel_tol"]


# ------------------------------------------------------------------ main branch

def _sdpa_causal_gqa(q, k, v):
    # q [T,H,d], k/v [G,N,d], positions 0..T-1 (T == N): torch library routine in fp64
    T, H, d = q.shape
    G = k.shape[0]
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(k).repeat_interleave(H // G, dim=0)[None]
    vt = torch.from_numpy(v).repeat_interleave(H // G, dim=0)[None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    return o[0].permute(1, 0, 2).numpy()


def test_k_covering_all_blocks_equals_dense_causal_gqa():
    rng = np.random.default_rng(4)
    T, H, G, d, B = 37, 6, 2, 8, 8                 # 5 blocks, ragged tail
    q = rng.normal(size=(T, H, d)); k = rng.normal(size=(G, T, d)); v = rng.normal(size=(G, T, d))
    qi = rng.integers(-3, 4, size=(T, G, 4)); ki = rng.integers(-3, 4, size=(T, 4))
    pos = np.arange(T)
    Os, _, sel, _ = O.msa_forward(q, k, v, qi, ki, pos, B, topk=5)
    ref = _sdpa_causal_gqa(q, k, v)
    assert np.abs(Os - ref).max() < 1e-12
    Od, _ = O.dense_attention(q, k, v, pos)
    assert np.abs(Od - ref).max() < 1e-12
    # each row selected every causal block
    for t in range(T):
        assert [x for x in sel[t, 0] if x >= 0] == list(range(t // B + 1))


def test_sparse_attention_is_dense_over_selected_keys():
    # drop the unselected blocks from K/V and compare with SDPA over the rest
    rng = np.random.default_rng(5)
    H, G, d, B, N = 4, 1, 8, 4, 24
    k = rng.normal(size=(G, N, d)); v = rng.normal(size=(G, N, d))
    q = rng.normal(size=(1, H, d))
    p = 21
    sel = np.array([[[1, 3, 5, -1]]])
    keys = [4, 5, 6, 7, 12, 13, 14, 15, 20, 21]
    Os, L = O.sparse_attention(q, k, v, sel, [p], B)
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(k[:, keys]).repeat_interleave(H, dim=0)[None]
    vt = torch.from_numpy(v[:, keys]).repeat_interleave(H, dim=0)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)[0].permute(1, 0, 2).numpy()
    assert np.abs(Os - ref).max() < 1e-12
    # lse closed form
    logits = q[0] @ k[0, keys].T / math.sqrt(d)
    assert np.abs(L[0] - np.log(np.exp(logits).sum(axis=1))).max() < 1e-12


def test_sparse_attention_equals_block_masked_sdpa():
    # many rows, several groups, random selections: the oracle's gathered-key
    # attention against SDPA over every key with a boolean mask built from the
    # definition (key j of group g is attended by row t iff block(j) is in
    # sel[t, g] and j <= p_t); ragged tail (N not a multiple of B)
    rng = np.random.default_rng(15)
    T, H, G, d, B, N, k = 40, 6, 2, 8, 8, 61, 3
    q = rng.normal(size=(T, H, d)); kk = rng.normal(size=(G, N, d)); v = rng.normal(size=(G, N, d))
    pos = rng.integers(0, N, size=T)
    pos[:3] = [0, N - 1, 2 * B]
    sel = np.full((T, G, k), -1, dtype=np.int32)
    for t in range(T):
        bt = pos[t] // B
        for g in range(G):
            others = rng.permutation(bt)[:k - 1]
            sel[t, g, :len(others) + 1] = sorted(list(others) + [bt])
    Os, L = O.sparse_attention(q, kk, v, sel, pos, B)
    r = H // G
    mask = np.zeros((H, T, N), dtype=bool)
    for t in range(T):
        for h in range(H):
            blocks = set(int(b) for b in sel[t, h // r] if b >= 0)
            mask[h, t] = [(j // B in blocks) and j <= pos[t] for j in range(N)]
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(kk).repeat_interleave(r, dim=0)[None]
    vt = torch.from_numpy(v).repeat_interleave(r, dim=0)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=torch.from_numpy(mask)[None])[0].permute(1, 0, 2).numpy()
    assert np.abs(Os - ref).max() < 1e-12
    logits = np.einsum("thd,hnd->htn", q, np.repeat(kk, r, axis=0)) / math.sqrt(d)
    lse = np.log(np.where(mask, np.exp(logits), 0.0).sum(axis=2)).T
    assert np.abs(L - lse).max() < 1e-12


def test_two_key_closed_form_and_scale():
    d = 4
    q = np.zeros((1, 1, d)); q[0, 0, 0] = 2.0            # logit = 2 * k0 / sqrt(4)
    k = np.zeros((1, 2, d)); k[0, 0, 0] = 1.0
    v = np.zeros((1, 2, d)); v[0, 0, 1] = 1.0; v[0, 1, 2] = 1.0
    Os, L = O.sparse_attention(q, k, v, np.array([[[0]]]), [1], block=8)
    w0 = math.e / (math.e + 1.0)
    assert abs(Os[0, 0, 1] - w0) < 1e-15 and abs(Os[0, 0, 2] - (1 - w0)) < 1e-15
    assert abs(L[0, 0] - math.log(math.e + 1.0)) < 1e-15


def test_zero_query_is_mean_of_attended_values():
    rng = np.random.default_rng(6)
    G, N, d, B = 2, 32, 5, 8
    v = rng.normal(size=(G, N, d)); k = rng.normal(size=(G, N, d))
    q = np.zeros((1, 4, d))
    sel = np.array([[[0, 2, 3], [1, 3, -1]]])
    p = 29
    Os, _ = O.sparse_attention(q, k, v, sel, [p], B)
    for g in range(G):
        keys = O.attended_keys(sel[0, g], p, B, N)
        assert np.abs(Os[0, 2 * g:2 * g + 2] - v[g, keys].mean(axis=0)).max() < 1e-14
    assert len(O.attended_keys(sel[0, 0], p, B, N)) == 8 + 8 + 6


def test_head_to_group_mapping_is_contiguous():
    G, H, N, d, B = 3, 6, 16, 4, 8
    rng = np.random.default_rng(7)
    v = np.zeros((G, N, d))
    for g in range(G):
        v[g] = g + 1.0                                   # group-constant values
    k = rng.normal(size=(G, N, d)); q = rng.normal(size=(1, H, d))
    sel = np.array([[[0, 1]] * G])
    Os, _ = O.sparse_attention(q, k, v, sel, [15], B)
    for h in range(H):
        assert np.abs(Os[0, h] - (h // 2 + 1.0)).max() < 1e-14


def test_softmax_weights_sum_to_one_and_single_key():
    rng = np.random.default_rng(8)
    q = rng.normal(size=(2, 2, 4)); k = rng.normal(size=(1, 10, 4)); v = rng.normal(size=(1, 10, 4))
    sel = np.array([[[0, -1]], [[0, 1]]])
    Os, _, W = O.sparse_attention(q, k, v, sel, [0, 9], 5, return_weights=True)
    assert np.abs(Os[0] - v[0, 0]).max() < 1e-15                # position 0: only key 0
    for row in W:
        for keys, w in row:
            assert np.abs(w.sum(axis=1) - 1.0).max() < 1e-14


def test_topk_selection_on_planted_synthetic_block():
    # one block whose token scores far above the rest must be selected by every later query
    rng = np.random.default_rng(9)
    B, nb, di = 8, 12, 4
    ki = rng.integers(-1, 2, size=(nb * B, di)).astype(float)
    ki[3 * B + 5] = [3, 3, 3, 3]
    pos = np.arange(4 * B, nb * B)
    qi = np.tile(np.array([3.0, 3.0, 3.0, 3.0]), (len(pos), 1, 1))
    sel = O.block_topk(O.index_pooled(qi, ki, pos, B), pos, B, k=2)
    assert np.all(sel[:, 0, 0] == 3)
    assert np.all(sel[:, 0, 1] == pos // B)


# ------------------------------------------------------- alignment diagnostic

def test_alignment_single_block_is_zero():
    # k = 1: both distributions sit on the local block alone
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 4, 8))
    k = rng.standard_normal((2, 40, 8))
    v = rng.standard_normal((2, 40, 8))
    sel = np.array([[[3], [3]]], dtype=np.int32)
    pooled = rng.standard_normal((1, 2, 5))
    kl = O.index_alignment_kl(q, k, v, sel, pooled, np.array([29]), 8)
    assert np.abs(kl).max() <= 1e-12          # the head weights sum to 1 up to rounding


def test_alignment_uniform_keys_closed_form():
    # identical keys -> uniform attention over the attended keys: block masses
    # are key counts (8, 8, and the 6 causal keys 24..29 of local block 3);
    # equal pooled scores -> uniform index distribution over the 3 blocks
    B, N, d = 8, 40, 4
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, 2, d))
    k = np.tile(rng.standard_normal((1, 1, d)), (1, N, 1))
    v = rng.standard_normal((1, N, d))
    sel = np.array([[[0, 2, 3]]], dtype=np.int32)
    pooled = np.full((1, 1, 5), 7.0)
    kl = O.index_alignment_kl(q, k, v, sel, pooled, np.array([29]), B)
    p = np.array([8, 8, 6]) / 22.0
    assert kl[0, 0] == pytest.approx(float(np.sum(p * np.log(p * 3.0))), rel=1e-12)


def test_alignment_averages_heads_and_direction():
    # head 0 sees only block 0, head 1 only block 1 -> P_main = (1/2, 1/2);
    # index logits (log 3, 0) -> P_index = (3/4, 1/4);
    # KL(P_main || P_index) = 1/2 log(4/3) (the reverse direction differs)
    B, N, d = 8, 16, 2
    k = np.zeros((1, N, d))
    k[0, :8, 0] = 50.0
    k[0, 8:, 1] = 50.0
    q = np.array([[[20.0, 0.0], [0.0, 20.0]]])
    v = np.zeros((1, N, d))
    sel = np.array([[[0, 1]]], dtype=np.int32)
    pooled = np.array([[[math.log(3.0), 0.0]]])
    kl = O.index_alignment_kl(q, k, v, sel, pooled, np.array([15]), B)
    assert kl[0, 0] == pytest.approx(0.5 * math.log(4.0 / 3.0), abs=1e-12)
    reverse = 0.75 * math.log(1.5) + 0.25 * math.log(0.5)
    assert abs(kl[0, 0] - reverse) > 1e-3
