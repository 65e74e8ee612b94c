"""Counter-based seeded generator for the synthetic MSA workloads.

Every element of every input tensor is a pure function of (seed, tensor id,
flat element index), so any subset of a tensor can be regenerated on the host
without materialising the rest, and the same call gives the same bits on CPU
and on CUDA for the integer-valued tensors (index queries and keys).

Bits: element i of tensor ``tid`` under ``seed`` is the (i+1)-th output of the
SplitMix64 generator (Steele, Lea & Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014; constants as in Vigna's public-domain reference)
started from the state ``mix(seed << 16 ^ tid)``.  It is evaluated with wrapping
int64 tensor arithmetic (logical shifts are emulated with masks).

Distributions (the workloads' recipe):
  * Q, K, V: standard normal by the Box-Muller transform on the word's two
    32-bit halves, in float64, rounded to float32 and then to bf16 (RNE).
    Float64 ``log``/``cos`` are not bit-identical across devices, so a device
    draw may differ from a host draw by one bf16 ulp with probability ~2^-45
    per element; tests that need identical bits copy device data to the host.
  * index queries/keys: integers in [-3, 3] (``lo + floor(7*u)`` done in integer
    arithmetic), stored exactly in bf16.
  * planting (workloads with ``planted > 0``): for each (sequence, group) a sign
    pattern v in {-3,+3}^(d_i/2); that group's index queries take
    ``sign(v_c) * U{0..3}`` in the first d_i/2 coordinates; ``planted`` distinct
    blocks in [0, nb-2] each get one token whose index key is (v, 0, ..., 0).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

TID_Q, TID_K, TID_V, TID_QIDX, TID_KIDX, TID_PLANT = 1, 2, 3, 4, 5, 6

_GOLDEN = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_U64 = (1 << 64) - 1


def _s64(x: int) -> int:
    x &= _U64
    return x - (1 << 64) if x >= (1 << 63) else x


def _mix_py(z: int) -> int:
    z &= _U64
    z = ((z ^ (z >> 30)) * _M1) & _U64
    z = ((z ^ (z >> 27)) * _M2) & _U64
    return z ^ (z >> 31)


def stream_state(seed: int, tid: int) -> int:
    """Initial SplitMix64 state of tensor ``tid`` under ``seed`` (Python int)."""
    return _mix_py(((seed & 0xFFFFFFFFFFFF) << 16) ^ tid)


def splitmix64_words_py(seed: int, tid: int, idx: int) -> int:
    """Reference scalar: word ``idx`` as an unsigned Python int."""
    z = (stream_state(seed, tid) + (idx + 1) * _GOLDEN) & _U64
    return _mix_py(z)


def _lsr(z: torch.Tensor, s: int) -> torch.Tensor:
    return (z >> s) & ((1 << (64 - s)) - 1)


def splitmix64_words(seed: int, tid: int, idx: torch.Tensor) -> torch.Tensor:
    """Words for flat indices ``idx`` (int64 tensor) as int64 bit patterns."""
    base = _s64(stream_state(seed, tid))
    z = (idx + 1) * _s64(_GOLDEN) + base
    z = (z ^ _lsr(z, 30)) * _s64(_M1)
    z = (z ^ _lsr(z, 27)) * _s64(_M2)
    return z ^ _lsr(z, 31)


def uniform01(w: torch.Tensor) -> torch.Tensor:
    """float64 in [0, 1) from the top 53 bits."""
    return _lsr(w, 11).to(torch.float64) * (2.0 ** -53)


def int_uniform(w: torch.Tensor, lo: int, hi: int) -> torch.Tensor:
    """Integer uniform on [lo, hi] from the top 32 bits (exact integer math)."""
    return lo + ((_lsr(w, 32) * (hi - lo + 1)) >> 32)


def normal01(w: torch.Tensor) -> torch.Tensor:
    """Standard normal (float64) by Box-Muller on the two 32-bit halves."""
    u1 = (_lsr(w, 32).to(torch.float64) + 0.5) * (2.0 ** -32)
    u2 = (w & 0xFFFFFFFF).to(torch.float64) * (2.0 ** -32)
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)


@dataclass
class WorkloadSpec:
    """Shapes and seed of one synthetic workload (layouts of the C ABI).

    q      [batch, seq_q, H, d]       k, v  [batch, G, seq_kv, d]
    q_idx  [batch, seq_q, G, d_i]     k_idx [batch, seq_kv, d_i]
    """
    batch: int
    seq_q: int
    seq_kv: int
    q_offset: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    index_dim: int
    block: int = 128
    topk: int = 16
    seed: int = 1
    planted: int = 0

    @property
    def nb(self) -> int:
        return (self.seq_kv + self.block - 1) // self.block

    def shape_of(self, name: str):
        b, t, n = self.batch, self.seq_q, self.seq_kv
        h, g, d, di = self.n_q_heads, self.n_kv_heads, self.head_dim, self.index_dim
        return {"q": (b, t, h, d), "k": (b, g, n, d), "v": (b, g, n, d),
                "q_idx": (b, t, g, di), "k_idx": (b, n, di)}[name]


@dataclass
class PlantLayout:
    signs: list = field(default_factory=list)     # [batch][G] -> list of +-3 (len d_i/2)
    blocks: list = field(default_factory=list)    # [batch][G] -> sorted block ids
    tokens: list = field(default_factory=list)    # [batch][G] -> token positions


def plant_layout(spec: WorkloadSpec) -> PlantLayout:
    """Sign patterns, planted blocks and planted token positions (host side)."""
    lay = PlantLayout()
    if spec.planted <= 0:
        return lay
    half = spec.index_dim // 2
    nb = spec.nb
    if nb < spec.planted + 1:
        raise ValueError("too few blocks to plant into")
    ctr = 0

    def word():
        nonlocal ctr
        w = splitmix64_words_py(spec.seed, TID_PLANT, ctr)
        ctr += 1
        return w

    for b in range(spec.batch):
        sgn_b, blk_b, tok_b, used_tok = [], [], [], set()
        for g in range(spec.n_kv_heads):
            sgn_b.append([3 if (word() >> 63) else -3 for _ in range(half)])
            chosen = []
            while len(chosen) < spec.planted:
                blk = ((word() >> 32) * (nb - 1)) >> 32          # uniform in [0, nb-2]
                if blk in chosen:
                    continue
                pos = blk * spec.block + (((word() >> 32) * spec.block) >> 32)
                if pos in used_tok:
                    continue
                chosen.append(blk)
                used_tok.add(pos)
                tok_b.append((g, blk, pos))
            blk_b.append(sorted(chosen))
        lay.signs.append(sgn_b)
        lay.blocks.append(blk_b)
        lay.tokens.append([sorted(p for (gg, _, p) in tok_b if gg == g)
                           for g in range(spec.n_kv_heads)])
    return lay


def values_at(spec: WorkloadSpec, name: str, flat_idx: torch.Tensor,
              lay: PlantLayout | None = None) -> torch.Tensor:
    """float64 values of tensor ``name`` at flat indices (device of ``flat_idx``)."""
    dev = flat_idx.device
    if name in ("q", "k", "v"):
        tid = {"q": TID_Q, "k": TID_K, "v": TID_V}[name]
        return normal01(splitmix64_words(spec.seed, tid, flat_idx))
    if name == "q_idx":
        w = splitmix64_words(spec.seed, TID_QIDX, flat_idx)
        val = int_uniform(w, -3, 3)
        if spec.planted > 0:
            lay = lay or plant_layout(spec)
            di, G = spec.index_dim, spec.n_kv_heads
            half = di // 2
            c = flat_idx % di
            g = (flat_idx // di) % G
            b = flat_idx // (di * G * spec.seq_q)
            sg = torch.tensor(lay.signs, dtype=torch.int64, device=dev)   # [B, G, half]
            first = c < half
            cc = torch.where(first, c, torch.zeros_like(c))
            sign = sg[b, g, cc].sign()
            val = torch.where(first, sign * int_uniform(w, 0, 3), val)
        return val.to(torch.float64)
    if name == "k_idx":
        val = int_uniform(splitmix64_words(spec.seed, TID_KIDX, flat_idx), -3, 3)
        if spec.planted > 0:
            lay = lay or plant_layout(spec)
            di = spec.index_dim
            half = di // 2
            c = flat_idx % di
            row = flat_idx // di                       # b * seq_kv + j
            for b in range(spec.batch):
                for g in range(spec.n_kv_heads):
                    v = torch.tensor(lay.signs[b][g] + [0] * (di - half),
                                     dtype=torch.int64, device=dev)
                    for pos in lay.tokens[b][g]:
                        hit = row == (b * spec.seq_kv + pos)
                        val = torch.where(hit, v[c], val)
        return val.to(torch.float64)
    raise KeyError(name)


def make_tensor(spec: WorkloadSpec, name: str, device="cpu",
                lay: PlantLayout | None = None, chunk: int = 1 << 24) -> torch.Tensor:
    """Whole bf16 tensor ``name`` in the C-ABI layout, generated in chunks."""
    shape = spec.shape_of(name)
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    total = flat.numel()
    if name == "k_idx" and spec.planted > 0:
        lay = lay or plant_layout(spec)
    for s in range(0, total, chunk):
        e = min(total, s + chunk)
        idx = torch.arange(s, e, dtype=torch.int64, device=device)
        if name == "k_idx" and spec.planted > 0:
            # planting is applied once below; draw the plain integers here
            v = int_uniform(splitmix64_words(spec.seed, TID_KIDX, idx), -3, 3).to(torch.float64)
        elif name == "q_idx" and spec.planted > 0:
            v = values_at(spec, name, idx, lay or plant_layout(spec))
        else:
            v = values_at(spec, name, idx)
        flat[s:e] = v.to(torch.float32).to(torch.bfloat16)
    if name == "k_idx" and spec.planted > 0:
        half = spec.index_dim // 2
        for b in range(spec.batch):
            for g in range(spec.n_kv_heads):
                row = torch.tensor(lay.signs[b][g] + [0] * (spec.index_dim - half),
                                   dtype=torch.float32).to(torch.bfloat16).to(device)
                for pos in lay.tokens[b][g]:
                    out[b, pos, :] = row
    return out


@dataclass
class MsaInputs:
    spec: WorkloadSpec
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    q_idx: torch.Tensor
    k_idx: torch.Tensor
    plant: PlantLayout


def make_inputs(spec: WorkloadSpec, device="cpu",
                names=("q", "k", "v", "q_idx", "k_idx")) -> MsaInputs:
    lay = plant_layout(spec)
    t = {n: (make_tensor(spec, n, device, lay) if n in names else None)
         for n in ("q", "k", "v", "q_idx", "k_idx")}
    return MsaInputs(spec, t["q"], t["k"], t["v"], t["q_idx"], t["k_idx"], lay)
