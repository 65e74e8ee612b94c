"""Pins of the seeded input generator (CPU)."""
import json
import os

import torch

import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_splitmix64_matches_published_outputs_from_state_zero():
    gold = json.load(open(os.path.join(GOLD, "splitmix64_seed0.json")))
    # tensor-vectorised mixing from state 0 reproduces the published sequence
    from synth.gen import _s64, _GOLDEN
    z = (torch.arange(1, 4, dtype=torch.int64) * _s64(_GOLDEN))
    from synth.gen import _lsr, _M1, _M2
    z = (z ^ _lsr(z, 30)) * _s64(_M1)
    z = (z ^ _lsr(z, 27)) * _s64(_M2)
    z = z ^ _lsr(z, 31)
    got = [int(x) & ((1 << 64) - 1) for x in z.tolist()]
    assert got == [int(h, 16) for h in gold["state0_outputs_hex"]]


def test_vector_words_match_scalar_reference():
    idx = torch.tensor([0, 1, 2, 1000, 123456789, (1 << 40) + 7], dtype=torch.int64)
    w = synth.splitmix64_words(11, synth.TID_K, idx)
    for i, x in zip(idx.tolist(), w.tolist()):
        assert (x & ((1 << 64) - 1)) == synth.splitmix64_words_py(11, synth.TID_K, i)


def test_distributions():
    idx = torch.arange(0, 1 << 18, dtype=torch.int64)
    w = synth.splitmix64_words(3, synth.TID_Q, idx)
    n = synth.normal01(w)
    assert abs(n.mean().item()) < 0.01 and abs(n.std().item() - 1.0) < 0.01
    iu = synth.int_uniform(w, -3, 3)
    assert iu.min().item() == -3 and iu.max().item() == 3
    counts = torch.bincount(iu + 3).double() / iu.numel()
    assert (counts - 1 / 7).abs().max().item() < 0.005


def test_subset_regeneration_matches_whole_tensor():
    spec = synth.workload("tiny_prefill_2k")
    full = synth.make_tensor(spec, "q")
    idx = torch.tensor([0, 17, 5000, full.numel() - 1])
    sub = synth.values_at(spec, "q", idx).float().to(torch.bfloat16)
    assert torch.equal(sub, full.view(-1)[idx])


def test_planting_recipe():
    spec = synth.WorkloadSpec(1, 1024, 1024, 0, 8, 2, 16, 8, 128, 4, seed=9, planted=3)
    inp = synth.make_inputs(spec, names=("q_idx", "k_idx"))
    lay = inp.plant
    for g in range(2):
        assert len(lay.blocks[0][g]) == 3 and max(lay.blocks[0][g]) <= spec.nb - 2
        for pos in lay.tokens[0][g]:
            row = inp.k_idx[0, pos].float()
            assert row[:4].tolist() == lay.signs[0][g] and row[4:].abs().sum() == 0
        # first half of this group's index queries carries the sign pattern
        qh = inp.q_idx[0, :, g, :4].float()
        sg = torch.tensor(lay.signs[0][g]).float().sign()
        assert torch.all(qh * sg >= 0) and qh.abs().max() <= 3
    # subset regeneration applies the planting too
    pos = lay.tokens[0][1][0]
    idx = torch.arange(pos * 8, pos * 8 + 8)
    assert torch.equal(synth.values_at(spec, "k_idx", idx, lay).float(), inp.k_idx[0, pos].float())
