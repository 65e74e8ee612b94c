"""Plain fp64 CPU oracle of the MiniMax Sparse Attention (MSA) hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code with
the CUDA library and imports nothing from it.

What it computes, step by step, in the order the pages describe the method
(page names: P1 Notion note "Minimax sparse Attention"; P2 hamidun.com "MiniMax
lança MSA: atenção esparsa acelera em 28 vezes…"; P3 yhxrc.cn article on the
MSA figure; P4 lumi-systems AI news on MSA; P5 lefilia.fr "MiniMax Sparse
Attention (MSA) : attention block-sparse à deux branches…"):

1. ``index_pooled`` -- index branch scoring (P3, section 第一步 "index branch"):
   one index query per GQA group, one index key per KV token shared by all
   heads, token score = raw dot product q_idx . k_idx over causal keys, then a
   max over each B-token block.  Blocks with no causal key are -inf.
2. ``select_blocks`` / ``block_topk`` -- per query and per group, keep the top
   scoring blocks (P3 第一步 "TopK"; P4, passage on one independent top-k
   subset per GQA group), with the local block always included (P5, paragraph on the
   local block) in a budget of k blocks of B tokens (P5: 16 x 128 = 2048).
3. ``sparse_attention`` -- main branch (P3, section 第二步 "sparse branch"; P2
   "Como o MSA funciona"): exact softmax attention of every query head over
   the real K/V of its group's selected blocks; every head of a group uses that
   group's selection (P3: Q1/Q2/Q3 share I1, Q4/Q5/Q6 share I2).
4. ``dense_attention`` -- causal GQA (P1, GQA definition) for the
   "k >= number of causal blocks" invariant and the dense baseline.
5. ``index_alignment_kl`` -- the divergence P1 (bullet "KL Loss Alignment")
   trains the index branch on, computed forward-only as a diagnostic: the
   main branch's attention distribution over the selected blocks against the
   index branch's distribution over the same blocks.

Readings where the pages are silent:
  * index score: raw dot product, no scale / activation (P3 names only Q_idx.K_idx;
    only the ordering is used);
  * blocks are aligned at absolute position 0: block b = [bB, (b+1)B);
  * local block = the block b_t = floor(p_t / B) that contains the query;
  * k counts the local block: sel = {b_t} + top-(k-1) of blocks 0..b_t-1;
  * ties: equal pooled scores -> the lower block index wins;
  * fewer than k causal blocks -> all of them, padded with -1;
  * sel is written in ascending block order, -1 padding last;
  * attention scale 1/sqrt(d); head h belongs to group floor(h / (H/G));
  * selection is decided on the pooled scores rounded to float32 (the
    kernel's precision); with the integer-valued index inputs of the workloads
    every score is an exact integer, so this rounding is the identity.

  * alignment (P1 gives no formula): per (query, group), P_main(b) = the
    attention mass of selected block b averaged over the group's heads,
    P_index(b) = softmax over the selected blocks of the raw pooled index
    scores (no temperature), KL(P_main || P_index) in natural log.

Precision: float64 throughout.  Pins (tests/test_oracle_pins.py), each
independent of this module's code: pooled scores by brute force and one-hot
keys; the selection by a beaten-by-count definition with ties; the attention
by torch SDPA (causal GQA when k covers every block, gathered keys, and a
boolean block mask built from the definition over random selections) and by
closed forms; the alignment KL by closed forms.  The pages print no worked
example of an attention output, so none of the pins is a page value.
"""
from __future__ import annotations

import math

import numpy as np


def _f64(x) -> np.ndarray:
    """Convert a torch tensor (any dtype, any device) or array to float64 numpy."""
    if hasattr(x, "detach"):
        return x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def local_block(p: int, block: int) -> int:
    """Block containing absolute position p (blocks aligned at position 0)."""
    return p // block


def index_pooled(q_idx, k_idx, positions, block: int) -> np.ndarray:
    """Block max-pooled index scores.

    q_idx [R, G, d_i] (one index query per group per query row), k_idx [N, d_i]
    (shared by all heads), positions [R] = absolute position p of each query row.
    Returns pooled [R, G, nb] float64, nb = ceil(N / block):
      pooled[r, g, b] = max over causal keys j (j <= p_r) of block b of
                        sum_c q_idx[r, g, c] * k_idx[j, c];  -inf if none.
    """
    q = _f64(q_idx)
    kk = _f64(k_idx)
    pos = np.asarray(positions, dtype=np.int64)
    R, G, _ = q.shape
    N = kk.shape[0]
    nb = (N + block - 1) // block
    out = np.full((R, G, nb), -np.inf)
    for r in range(R):
        p = int(pos[r])
        n_causal = min(p + 1, N)
        s = q[r] @ kk[:n_causal].T                       # [G, n_causal] token scores
        for b in range((n_causal + block - 1) // block):
            lo, hi = b * block, min((b + 1) * block, n_causal)
            out[r, :, b] = s[:, lo:hi].max(axis=1)
    return out


def select_blocks(pooled_row, b_t: int, k: int) -> np.ndarray:
    """Selection of one (query, group): int32 [k].

    The local block b_t always; plus the top-(k-1) of blocks 0..b_t-1 ordered by
    (score descending, block index ascending); ascending order; -1 padding.
    """
    scores = np.asarray(pooled_row, dtype=np.float64).astype(np.float32)
    cand = np.arange(b_t, dtype=np.int64)
    # np.lexsort sorts by the last key first: primary = -score, secondary = index
    order = np.lexsort((cand, -scores[:b_t].astype(np.float64)))
    chosen = list(cand[order][: max(0, min(k - 1, b_t))]) + [b_t]
    chosen.sort()
    out = np.full(k, -1, dtype=np.int32)
    out[: len(chosen)] = chosen
    return out


def block_topk(pooled, positions, block: int, k: int) -> np.ndarray:
    """sel [R, G, k] int32 for every row of ``pooled`` [R, G, nb]."""
    pl = _f64(pooled)
    pos = np.asarray(positions, dtype=np.int64)
    R, G, _ = pl.shape
    sel = np.empty((R, G, k), dtype=np.int32)
    for r in range(R):
        b_t = local_block(int(pos[r]), block)
        for g in range(G):
            sel[r, g] = select_blocks(pl[r, g], b_t, k)
    return sel


def attended_keys(sel_row, p: int, block: int, n_kv: int) -> np.ndarray:
    """Key positions one (query, group) attends: selected blocks, causal part."""
    keys = []
    for b in sorted(int(x) for x in sel_row if x >= 0):
        keys.extend(range(b * block, min((b + 1) * block, p + 1, n_kv)))
    return np.asarray(keys, dtype=np.int64)


def _softmax_attend(qh, kb, vb, scale):
    """Exact softmax attention of query rows qh [r, d] over keys kb/vb [n, d]."""
    logits = (qh @ kb.T) * scale                  # [r, n]
    m = logits.max(axis=1, keepdims=True)
    w = np.exp(logits - m)
    l = w.sum(axis=1, keepdims=True)
    o = (w @ vb) / l
    lse = (m + np.log(l))[:, 0]
    return o, lse, w / l


def sparse_attention(q, k, v, sel, positions, block: int, scale: float | None = None,
                     return_weights: bool = False):
    """Main branch: O [R, H, d] and lse [R, H] (natural log), float64.

    q [R, H, d] query rows at absolute positions ``positions``; k, v [G, N, d]
    (one sequence); sel [R, G, k] block lists (-1 = unused slot).  Query head h
    uses group g = h // (H // G) and that group's selection.
    """
    qq, kk, vv = _f64(q), _f64(k), _f64(v)
    sl = np.asarray(sel)
    pos = np.asarray(positions, dtype=np.int64)
    R, H, d = qq.shape
    G, N, _ = kk.shape
    r = H // G
    sc = (1.0 / math.sqrt(d)) if scale is None else scale
    O = np.zeros((R, H, d))
    L = np.zeros((R, H))
    weights = []
    for i in range(R):
        p = int(pos[i])
        wrow = []
        for g in range(G):
            keys = attended_keys(sl[i, g], p, block, N)
            o, lse, w = _softmax_attend(qq[i, g * r:(g + 1) * r], kk[g, keys], vv[g, keys], sc)
            O[i, g * r:(g + 1) * r] = o
            L[i, g * r:(g + 1) * r] = lse
            wrow.append((keys, w))
        weights.append(wrow)
    if return_weights:
        return O, L, weights
    return O, L


def dense_attention(q, k, v, positions, scale: float | None = None):
    """Causal GQA attention over every key j <= p (float64): O [R, H, d], lse [R, H]."""
    qq, kk, vv = _f64(q), _f64(k), _f64(v)
    pos = np.asarray(positions, dtype=np.int64)
    R, H, d = qq.shape
    G, N, _ = kk.shape
    r = H // G
    sc = (1.0 / math.sqrt(d)) if scale is None else scale
    O = np.zeros((R, H, d))
    L = np.zeros((R, H))
    for i in range(R):
        n = min(int(pos[i]) + 1, N)
        for g in range(G):
            o, lse, _ = _softmax_attend(qq[i, g * r:(g + 1) * r], kk[g, :n], vv[g, :n], sc)
            O[i, g * r:(g + 1) * r] = o
            L[i, g * r:(g + 1) * r] = lse
    return O, L


def msa_forward(q, k, v, q_idx, k_idx, positions, block: int, topk: int):
    """Whole layer for one sequence: (O, lse, sel, pooled)."""
    pooled = index_pooled(q_idx, k_idx, positions, block)
    sel = block_topk(pooled, positions, block, topk)
    O, L = sparse_attention(q, k, v, sel, positions, block)
    return O, L, sel, pooled


def index_alignment_kl(q, k, v, sel, pooled, positions, block: int,
                       scale: float | None = None) -> np.ndarray:
    """KL(P_main || P_index) per (query row, group), float64 [R, G].

    P_main(b): for each head of group g, the sum of its attention weights
    (``sparse_attention``'s normalised weights) over the keys of selected
    block b, averaged over the group's heads.  P_index(b): softmax over the
    selected blocks of pooled[r, g, b].  Terms with P_main(b) = 0 contribute 0.
    """
    sl = np.asarray(sel)
    pl = _f64(pooled)
    R, G, _ = sl.shape
    _, _, weights = sparse_attention(q, k, v, sel, positions, block, scale, return_weights=True)
    out = np.zeros((R, G))
    for i in range(R):
        for g in range(G):
            keys, w = weights[i][g]                       # w [r, n] rows sum to 1
            blocks = [int(b) for b in sl[i, g] if b >= 0]
            p_main = np.array([w[:, (keys // block) == b].sum(axis=1).mean() for b in blocks])
            logits = np.array([pl[i, g, b] for b in blocks])
            p_idx = np.exp(logits - logits.max())
            p_idx /= p_idx.sum()
            nz = p_main > 0
            out[i, g] = float(np.sum(p_main[nz] * (np.log(p_main[nz]) - np.log(p_idx[nz]))))
    return out


def attention_flops_ratio(n_ctx: int, H: int, d: int, G: int, d_idx: int,
                          k: int, block: int) -> float:
    """Dense-GQA over MSA attention FLOPs averaged over a causal prefill of n_ctx.

    Dense: 4*H*d per (query, key) pair over mean key count n_ctx/2.  MSA: the
    main branch attends k*block keys per query and the index branch costs
    2*G*d_idx per (query, key) pair.  (Our accounting of the pages' 28.4x.)
    """
    mean_keys = n_ctx / 2.0
    dense = 4.0 * H * d * mean_keys
    msa = 4.0 * H * d * k * block + 2.0 * G * d_idx * mean_keys
    return dense / msa
