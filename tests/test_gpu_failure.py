"""Failure detection on the GPU without a fault.

Every wait in every kernel is bounded: when it runs out, the kernel records a
code in the workspace's error word and returns, and sla_get_device_status
reports it.  These tests make that happen on purpose, in ways that cannot
fault: a wait on a barrier nothing completes, and a LUT entry out of range
(the kernels check every index before use and skip it).
"""
import time

import pytest
import torch

from block_sparse_linear_pool_b200 import binding as bnd
from block_sparse_linear_pool_b200.build import build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    bnd.lib()


def test_a_wait_that_never_completes_reports_a_timeout():
    ws = bnd.new_workspace(256, "cuda")
    t0 = time.time()
    assert bnd.lib().sla_selftest_wait_timeout(bnd._ptr(ws), bnd._stream()) == 0
    code, detail = bnd.sla_get_device_status(ws)
    assert code == 5 and detail == 3  # SLA_ERR_DEVICE_TIMEOUT, a hand-off that never completed
    assert time.time() - t0 < 30
    # the word is cleared by the read, and the context still works
    assert bnd.sla_get_device_status(ws) == (0, 0)
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum()) == 8.0


def test_an_out_of_range_lut_entry_is_reported_not_followed():
    g = torch.Generator().manual_seed(0)
    B, H, N, d = 1, 1, 1024, 64
    Q, K, V = (torch.randn(B, H, N, d, generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    cfg = bnd.SlaConfig(k_h=0.1, k_l=0.5, combine="alpha")
    ws = bnd.new_workspace(bnd.sla_workspace_size(bnd.make_params(Q, cfg, K, V)), "cuda")
    mc, lut = bnd.sla_predict_mask(Q, K, cfg, workspace=ws)
    hz = bnd.sla_precompute_linear(K, V, cfg, None, workspace=ws)
    lut[0, 3, 0] = 1 << 20  # far past T_kv
    alpha = torch.full((1, 1), 0.8)
    bnd.sla_forward(Q, K, V, mc, lut, hz, cfg, alpha=alpha, workspace=ws)
    code, detail = bnd.sla_get_device_status(ws)
    assert code == 6 and detail == 4  # SLA_ERR_DEVICE_BAD_INDEX
    # with the entry repaired the same workspace runs clean again
    mc2, lut2 = bnd.sla_predict_mask(Q, K, cfg, workspace=ws)
    bnd.sla_forward(Q, K, V, mc2, lut2, hz, cfg, alpha=alpha, workspace=ws)
    assert bnd.sla_get_device_status(ws) == (0, 0)
