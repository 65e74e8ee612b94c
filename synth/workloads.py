"""The named synthetic workloads (shapes, seeds, planting) used by tests and bench.

Seeds 1..5 go to the five workloads in order.  Shapes follow the layouts of
the C ABI (see ``synth.gen.WorkloadSpec``).
"""
from .gen import WorkloadSpec

_H, _G, _D, _DI = 64, 8, 128, 64

WORKLOADS = {
    # 2048-token causal prefill, 8 query heads / 2 KV heads, d=64, index dim 32, k=4
    "tiny_prefill_2k": WorkloadSpec(1, 2048, 2048, 0, 8, 2, 64, 32, 128, 4, seed=1, planted=0),
    # 32K causal prefill, 64/8 heads, d=128, index dim 64, k=16, 4 planted blocks per group
    "prefill_32k": WorkloadSpec(1, 32768, 32768, 0, _H, _G, _D, _DI, 128, 16, seed=2, planted=4),
    # 128K causal prefill, same shapes
    "prefill_128k": WorkloadSpec(1, 131072, 131072, 0, _H, _G, _D, _DI, 128, 16, seed=3, planted=4),
    # 32 sequences x 128K cache, one new query token each (query sits at position L-1)
    "decode_128k_b32": WorkloadSpec(32, 1, 131072, 131071, _H, _G, _D, _DI, 128, 16, seed=4, planted=4),
    # last 8192-query chunk of a 1M-token causal context
    "prefill_1m_chunk8k": WorkloadSpec(1, 8192, 1048576, 1048576 - 8192, _H, _G, _D, _DI, 128, 16,
                                       seed=5, planted=4),
    # 4 sequences x 1M cache, one query each
    "decode_1m_b4": WorkloadSpec(4, 1, 1048576, 1048575, _H, _G, _D, _DI, 128, 16, seed=5, planted=4),
    # small cases of the same shapes, sized for profiler captures (a few GB on the device)
    "prefill_16k": WorkloadSpec(1, 16384, 16384, 0, _H, _G, _D, _DI, 128, 16, seed=7, planted=4),
    "decode_16k_b8": WorkloadSpec(8, 1, 16384, 16383, _H, _G, _D, _DI, 128, 16, seed=8, planted=4),
    # a decode with more than 512 candidate blocks per row and few rows (the
    # top-k's CTA-per-row kernel), at ~3 GB of caches
    "decode_80k_b8": WorkloadSpec(8, 1, 81920, 81919, _H, _G, _D, _DI, 128, 16, seed=9, planted=4),
}


def workload(name: str, **overrides) -> WorkloadSpec:
    base = WORKLOADS[name]
    d = dict(base.__dict__)
    d.update(overrides)
    return WorkloadSpec(**d)
