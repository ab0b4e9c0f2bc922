"""CPU float64 oracle for the CSA2 hot path.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and
bench.py's CPU-baseline / reference arm, never by the product library.
"""
from .csa2_oracle import (  # noqa: F401
    bf16_bits_to_float, round_to_bf16, compress, index_scores, select_top,
    gather_pool_ids, sparse_attn, e2m1_value, e4m3_value, fp4_pack, fp4_unpack,
    run_group, FP4_BLOCK, swa_attn, lse_merge, sparse_attn_swa, compress_hca, dense_attn,
    index_scores_fp4,
)
