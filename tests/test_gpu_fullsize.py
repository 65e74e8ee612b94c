"""Parity at the full benchmark sizes, through msa_forward as bench.py runs it.

For every full-size configuration (32K, 128K and 1M-chunk prefill; 32 x 128K
and 4 x 1M decode):
  * the whole selection is compared, bit for bit, with a re-sort on the host
    of the pooled scores msa_index_scores returns: (score descending, block
    index ascending) over the causal blocks before the local one, plus the
    local block, ascending, -1 padding.  Index inputs are integers, so pooled
    scores are exact integers and the keys score*2^20 + (2^20-1-index) are
    exact and distinct in float64;
  * pooled scores of sampled query rows are compared bit for bit with the
    fp64 oracle;
  * attention outputs of sampled rows are compared with the fp64 oracle fed
    the same selection (max-abs 1e-2, mean-abs 1e-3).  Only the selected
    blocks of a row are copied to the host: they are renumbered in ascending
    order (the local block last) and the query position is moved into the
    last one, which leaves every mask unchanged.
"""
import numpy as np
import pytest
import torch

import block_sparse_gqa_05_b200 as M
import oracle as O
import synth
from tests.gpu_helpers import MAX_ABS, MEAN_ABS

pytestmark = pytest.mark.gpu

ROW_CHUNK = 1 << 13
IDX_SPAN = float(1 << 20)   # above any block index


def host_resort(pooled, positions, block, k):
    """Selection of every row of GPU pooled scores [R, G, nb], on the host."""
    R, G, nb = pooled.shape
    out = torch.empty((R, G, k), dtype=torch.int32)
    idx = torch.arange(nb, dtype=torch.float64)
    for r0 in range(0, R, ROW_CHUNK):
        r1 = min(R, r0 + ROW_CHUNK)
        pl = pooled[r0:r1].double().cpu()
        bt = torch.as_tensor(positions[r0:r1] // block, dtype=torch.int64)
        cand = (idx[None, None, :] < bt[:, None, None]).expand(-1, G, -1)   # blocks 0 .. b_t-1
        key = torch.where(cand, pl * IDX_SPAN + (IDX_SPAN - 1.0 - idx),
                          torch.tensor(-np.inf, dtype=torch.float64))
        kk = min(k - 1, nb)
        top = torch.topk(key, kk, dim=-1).indices if kk > 0 else torch.empty((r1 - r0, G, 0),
                                                                              dtype=torch.int64)
        valid = torch.gather(cand, 2, top)
        chosen = torch.where(valid, top, torch.full_like(top, nb + 1))   # drop missing candidates
        allb = torch.cat([chosen, bt[:, None, None].expand(-1, G, 1)], dim=2)
        srt = torch.sort(allb, dim=-1).values[..., :k]
        if srt.shape[-1] < k:
            srt = torch.cat([srt, torch.full((*srt.shape[:2], k - srt.shape[-1]), nb + 1)], -1)
        out[r0:r1] = torch.where(srt > nb, torch.full_like(srt, -1), srt).to(torch.int32)
    return out


def sample_rows(sp, n, seed):
    T = sp.seq_q
    fixed = [0, 1, 127, 128, 129, 1023, 1024, 2047, 2048, 2049, T // 2, T - 2, T - 1]
    rng = np.random.default_rng(seed)
    extra = rng.choice(T, size=max(0, n - len(fixed)), replace=False)
    return np.unique(np.clip(np.concatenate([fixed, extra]), 0, T - 1))


def compact_attention_ref(sp, q_row, k_seq, v_seq, sel_row, p):
    """fp64 oracle attention of one query row over only its selected blocks."""
    B = sp.block
    n = int((sel_row[0] >= 0).sum())            # same count in every group
    for g in range(sp.n_kv_heads):
        assert int((sel_row[g] >= 0).sum()) == n
    kc, vc = [], []
    for g in range(sp.n_kv_heads):
        blocks = torch.as_tensor(sorted(int(b) for b in sel_row[g] if b >= 0),
                                 dtype=torch.int64, device=k_seq.device)
        rows = (blocks[:, None] * B + torch.arange(B, device=k_seq.device)[None, :]).reshape(-1)
        rows = rows.clamp(max=sp.seq_kv - 1)     # the causal mask never reaches past p
        kc.append(k_seq[g, rows].cpu())
        vc.append(v_seq[g, rows].cpu())
    kc, vc = torch.stack(kc), torch.stack(vc)
    p_c = (n - 1) * B + p % B                    # the local block is the last one
    sel_c = np.tile(np.arange(n, dtype=np.int32), (sp.n_kv_heads, 1))
    o, _ = O.sparse_attention(q_row[None], kc, vc, sel_c[None], np.array([p_c]), B)
    return o[0]


def run_case(name, n_pool_rows, n_attn_rows):
    sp = synth.workload(name)
    inp = synth.make_inputs(sp, "cuda")
    sh = M.Shape.of(sp)
    o, _, sel = M.forward(sh, inp.q, inp.k, inp.v, inp.q_idx, inp.k_idx, want_lse=False)
    pooled = M.index_scores(sh, inp.q_idx, inp.k_idx)
    torch.cuda.synchronize()
    assert M.device_status() == 0
    pos = np.arange(sp.q_offset, sp.q_offset + sp.seq_q)
    for b in range(sp.batch):
        # whole selection against the host re-sort of the GPU pooled scores
        ref = host_resort(pooled[b], pos, sp.block, sp.topk)
        got = sel[b].cpu()
        bad = (got != ref).any(dim=-1).nonzero()
        assert bad.numel() == 0, f"{name} b={b}: {bad.shape[0]} rows differ, first {bad[:3].tolist()}"
        # pooled scores of sampled rows against the oracle
        rows = sample_rows(sp, n_pool_rows, seed=b) if sp.seq_q > n_pool_rows else np.arange(sp.seq_q)
        k_idx = inp.k_idx[b].cpu()
        q_rows = inp.q_idx[b, torch.as_tensor(rows, device=inp.q_idx.device)].cpu()
        pref = O.index_pooled(q_rows, k_idx, pos[rows], sp.block)
        pg = pooled[b, torch.as_tensor(rows, device=pooled.device)].double().cpu().numpy()
        fin = np.isfinite(pref)
        assert np.array_equal(np.isneginf(pg), np.isneginf(pref)), f"{name}: -inf pattern"
        assert np.array_equal(pg[fin], pref[fin]), f"{name}: pooled differs on sampled rows"
        # outputs of sampled rows against the oracle over the same selection
        arows = rows[:n_attn_rows] if len(rows) > n_attn_rows else rows
        errs = []
        for t in arows:
            ref_o = compact_attention_ref(sp, inp.q[b, int(t)].cpu(), inp.k[b], inp.v[b],
                                          sel[b, int(t)].cpu().numpy(), int(pos[t]))
            errs.append(ref_o - o[b, int(t)].double().cpu().numpy())
        err = np.abs(np.stack(errs))
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, \
            f"{name}: max abs {err.max():.3e}, mean abs {err.mean():.3e}"
    del inp, o, sel, pooled
    torch.cuda.empty_cache()


def test_ragged_decode_full_size():
    """32 sequences in a 128K-capacity cache with seeded lengths in [1, 131072]
    (both ends included): whole selection against the host re-sort, every
    output against the oracle."""
    sp = synth.workload("decode_128k_b32")
    inp = synth.make_inputs(sp, "cuda")
    sh = M.Shape.of(sp)
    rng = np.random.default_rng(7)
    lens = rng.integers(1, sp.seq_kv + 1, size=sp.batch)
    lens[:3] = [1, 128, sp.seq_kv]
    seq_lens = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o, _, sel = M.forward_decode_ragged(sh, inp.q, inp.k, inp.v, inp.q_idx, inp.k_idx, seq_lens,
                                        want_lse=False)
    torch.cuda.synchronize()
    assert M.device_status() == 0
    for b in range(sp.batch):
        pos = np.array([int(lens[b]) - 1])
        pooled = O.index_pooled(inp.q_idx[b].cpu(), inp.k_idx[b].cpu(), pos, sp.block)
        ref = host_resort(torch.from_numpy(pooled).float(), pos, sp.block, sp.topk)
        assert torch.equal(sel[b].cpu(), ref), f"b={b} len={lens[b]}"
        assert np.array_equal(ref.numpy(), O.block_topk(pooled, pos, sp.block, sp.topk))
        ref_o = compact_attention_ref(sp, inp.q[b, 0].cpu(), inp.k[b], inp.v[b],
                                      sel[b, 0].cpu().numpy(), int(pos[0]))
        err = np.abs(ref_o - o[b, 0].double().cpu().numpy())
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (b, err.max(), err.mean())


@pytest.mark.parametrize("name,n_pool,n_attn", [
    ("prefill_32k", 48, 48),
    ("prefill_128k", 48, 48),
    ("prefill_1m_chunk8k", 16, 16),
    ("decode_128k_b32", 1, 1),
    ("decode_1m_b4", 1, 1),
])
def test_full_size(name, n_pool, n_attn):
    run_case(name, n_pool, n_attn)
