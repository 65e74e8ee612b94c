"""B200 (sm_100a) kernels for the MiniMax Sparse Attention hot path.

The compute lives in ``libmsa.so`` (built from ``csrc/`` by ``build.py``);
``msa`` is its ctypes binding.
"""
from . import msa  # noqa: F401
from .msa import (  # noqa: F401
    Shape, MsaError, lib, workspace_size, alloc_workspace, index_scores, block_topk,
    sparse_attn_prefill, sparse_attn_decode, sparse_attn_decode_static, forward,
    forward_decode_ragged, forward_decode_paged, forward_prefill_paged, forward_alignment, dense_attn_prefill, dense_attn_decode, device_status, set_wait_limit_ns, profile_enable,
    profile_read, OP_INDEX_SCORES, OP_BLOCK_TOPK, OP_SPARSE_PREFILL, OP_SPARSE_DECODE, OP_FORWARD,
    OP_DENSE_PREFILL, OP_DENSE_DECODE, OP_FORWARD_ALIGNMENT, OP_FORWARD_PREFILL_PAGED,
)
from . import shard  # noqa: F401,E402
from .shard import GroupShard, group_shard, shard_inputs, forward_group_shard  # noqa: F401,E402
