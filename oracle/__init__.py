"""CPU oracle for the DeepSeek Sparse Attention (DSA) forward path.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it. It shares no code with the CUDA library; both sides only
consume the same seeded inputs.
"""

from .dsa_oracle import (  # noqa: F401
    bf16_round,
    e4m3_decode,
    e4m3_encode,
    quantize_indexer_query,
    indexer_scores,
    topk_select,
    topk_rows,
    sparse_mla_token,
    sparse_mla,
    dense_causal_mqa,
    resolve_kv_rows,
    dsa_forward,
    indexer_kl_token,
    sparse_indexer_kl,
    dense_indexer_kl,
    mla_up_project,
    mha_head_attention,
    masked_mha,
    absorb_mha_query,
)
