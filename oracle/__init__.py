"""CPU oracle (test infrastructure only; see ``oracle.msa_oracle``)."""
from .msa_oracle import (  # noqa: F401
    local_block, index_pooled, select_blocks, block_topk, attended_keys,
    sparse_attention, dense_attention, msa_forward, index_alignment_kl, attention_flops_ratio,
)
