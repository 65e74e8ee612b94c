"""The binding's argument checks, on the host (the library is replaced by a
stub that accepts every call, so no device is needed).

Every entry point is called with arrays in the C-ABI layouts of a small
workload (which must pass), then with a wrong dtype and with too few
elements (which must raise before reaching the library)."""
import ctypes

import pytest
import torch

import block_sparse_gqa_05_b200.msa as msa
import synth


@pytest.fixture
def calls(monkeypatch):
    seen = []

    class Stub:
        def __getattr__(self, name):
            def fn(*args):
                seen.append(name)
                return 0
            return fn

    monkeypatch.setattr(msa, "lib", lambda: Stub())
    monkeypatch.setattr(msa, "_ptr",
                        lambda t: None if t is None else ctypes.c_void_p(t.data_ptr()))
    monkeypatch.setattr(msa, "_stream", lambda s: None)
    return seen


def _prefill():
    sp = synth.WorkloadSpec(2, 130, 1000, 870, 16, 4, 64, 32, 128, 5)
    return sp, msa.Shape.of(sp), synth.make_inputs(sp)


def _decode():
    sp = synth.WorkloadSpec(3, 1, 1000, 999, 16, 4, 64, 32, 128, 5)
    return sp, msa.Shape.of(sp), synth.make_inputs(sp)


def test_every_entry_point_accepts_its_layouts(calls):
    sp, sh, x = _prefill()
    pooled = msa.index_scores(sh, x.q_idx, x.k_idx)
    assert pooled.shape == (2, 130, 4, sh.nb) and pooled.dtype == torch.float32
    sel = msa.block_topk(sh, pooled)
    assert sel.shape == (2, 130, 4, 5) and sel.dtype == torch.int32
    msa.sparse_attn_prefill(sh, x.q, x.k, x.v, sel)
    msa.forward(sh, x.q, x.k, x.v, x.q_idx, x.k_idx)
    o, lse, sel2, kl = msa.forward_alignment(sh, x.q, x.k, x.v, x.q_idx, x.k_idx)
    assert kl.shape == (2, 130, 4) and lse.shape == (2, 130, 16)
    msa.dense_attn_prefill(sh, x.q, x.k, x.v)
    sp, sh, x = _decode()
    sel = torch.zeros((3, 1, 4, 5), dtype=torch.int32)
    lens = torch.tensor([1, 500, 1000], dtype=torch.int32)
    msa.sparse_attn_decode(sh, x.q, x.k, x.v, sel)
    msa.sparse_attn_decode_static(sh, x.q, x.k, x.v, sel)
    msa.dense_attn_decode(sh, x.q, x.k, x.v)
    msa.forward_decode_ragged(sh, x.q, x.k, x.v, x.q_idx, x.k_idx, lens)
    P = 3 * sh.nb
    kp = torch.zeros((P, 4, 128, 64), dtype=torch.bfloat16)
    kip = torch.zeros((P, 128, 32), dtype=torch.bfloat16)
    table = torch.zeros((3, sh.nb), dtype=torch.int32)
    msa.forward_decode_paged(sh, x.q, kp, kp.clone(), x.q_idx, kip, lens, table)
    assert calls.count("msa_forward_decode_paged") == 1 and "msa_forward_alignment" in calls


def test_wrong_dtype_or_size_is_rejected_before_the_library(calls):
    sp, sh, x = _prefill()
    sel = torch.zeros((2, 130, 4, 5), dtype=torch.int32)
    with pytest.raises(ValueError, match="sel: expected torch.int32"):
        msa.sparse_attn_prefill(sh, x.q, x.k, x.v, sel.long())
    with pytest.raises(ValueError, match="q: expected torch.bfloat16"):
        msa.sparse_attn_prefill(sh, x.q.float(), x.k, x.v, sel)
    with pytest.raises(ValueError, match="k: .* elements"):
        msa.forward(sh, x.q, x.k[:, :2], x.v, x.q_idx, x.k_idx)
    with pytest.raises(ValueError, match="o: .* elements"):
        msa.forward(sh, x.q, x.k, x.v, x.q_idx, x.k_idx, o=x.q[:1])
    with pytest.raises(ValueError, match="pooled: expected torch.float32"):
        msa.block_topk(sh, torch.zeros((2, 130, 4, sh.nb), dtype=torch.float16))
    sp, sh, x = _decode()
    with pytest.raises(ValueError, match="seq_lens: expected torch.int32"):
        msa.forward_decode_ragged(sh, x.q, x.k, x.v, x.q_idx, x.k_idx,
                                  torch.tensor([1, 2, 3], dtype=torch.int64))
    kp = torch.zeros((4, 4, 128, 64), dtype=torch.bfloat16)
    kip = torch.zeros((3, 128, 32), dtype=torch.bfloat16)       # one page short
    with pytest.raises(ValueError, match="kidx_pages: .* elements"):
        msa.forward_decode_paged(sh, x.q, kp, kp, x.q_idx, kip,
                                 torch.ones(3, dtype=torch.int32),
                                 torch.zeros((3, sh.nb), dtype=torch.int32))
    assert set(calls) <= {"msa_workspace_size"}             # no compute call was made


def test_workspace_size_is_passed_in_bytes(calls, monkeypatch):
    sp, sh, x = _prefill()
    seen = {}

    class Stub:
        def msa_sparse_attn_prefill(self, *args):
            seen["bytes"] = args[-2]
            return 0

    monkeypatch.setattr(msa, "lib", lambda: Stub())
    ws = torch.zeros(100, dtype=torch.float32)
    msa.sparse_attn_prefill(sh, x.q, x.k, x.v, torch.zeros((2, 130, 4, 5), dtype=torch.int32),
                            ws=ws)
    assert seen["bytes"] == 400
