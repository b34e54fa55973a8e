"""SLA / SLA2 forward on B200 (sm_100a).

The compute lives in the C-ABI library ``libsla.so`` (csrc/, declared in
include/sla.h).  ``block_sparse_linear_pool_b200.binding`` marshals torch
tensors into its calls; ``inputs`` draws seeded synthetic inputs.
"""
