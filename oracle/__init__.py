"""fp64 CPU oracle of the SLA / SLA2 forward and backward passes.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
CPU-baseline leg of bench.py, never by the package block_sparse_linear_pool_b200.
See oracle/sla.py for the step-by-step restatement and its citations.
"""
from .sla import (  # noqa: F401
    OracleParams,
    EPS_DEFAULT,
    block_counts,
    num_blocks,
    block_range,
    smooth_keys,
    mean_pool,
    compressed_logits,
    compressed_attention,
    classify,
    soft_topk,
    predict_mask,
    critical_lut,
    feature_map,
    linear_block_stats,
    quantize_e4m3,
    quantize_int8,
    LOWBIT_MAX,
    LOG2E,
    lowbit_tile,
    pv_fp8_scales,
    pv_fp8_values,
    sparse_branch_fp8_pv,
    forward_given_mask,
    forward,
    mask_grading,
    feature_map_backward,
    backward_given_mask,
)
