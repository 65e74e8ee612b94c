"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This package holds no arithmetic of the attention method itself: it only draws
the tensors (Q, K, V, index queries, index keys) that both sides read.
"""
from .gen import (  # noqa: F401
    TID_Q, TID_K, TID_V, TID_QIDX, TID_KIDX, TID_PLANT,
    splitmix64_words, splitmix64_words_py, stream_state,
    uniform01, normal01, int_uniform,
    WorkloadSpec, PlantLayout, plant_layout, values_at, make_tensor,
    MsaInputs, make_inputs,
)
from .workloads import WORKLOADS, workload  # noqa: F401
