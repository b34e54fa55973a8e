"""sla_predict_mask_noalloc: mask prediction for callers that cannot allocate
device memory, with its scratch in the library's static device array.

Collected last on purpose: if it fails, a run stopped at the first failure has
already run every other test.  It must pass alone in a fresh process and after
the other tests (the static scratch keeps the previous call's contents).
"""
import ctypes

import pytest
import torch

from block_sparse_linear_pool_b200 import binding as bnd
from block_sparse_linear_pool_b200 import inputs as I
from block_sparse_linear_pool_b200.build import build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    bnd.lib()


def _compare_twice(Q, K, cfg, Wq=None, Wk=None):
    ref_mc, ref_lut = bnd.sla_predict_mask(Q, K, cfg, Wq, Wk)
    for _ in range(2):  # two calls in a row share (and reuse) the static scratch
        mc, lut = bnd.sla_predict_mask_noalloc(Q, K, cfg, Wq, Wk)
        torch.cuda.synchronize()
        # integer outputs: bit-exact against the workspace entry point
        assert torch.equal(mc, ref_mc)
        assert torch.equal(lut, ref_lut)


def test_noalloc_matches_workspace_entry_point_tiny():
    data, w = I.make_workload("tiny_sla")
    Q, K = data["Q"].cuda(), data["K"].cuda()
    _compare_twice(Q, K, bnd.SlaConfig(k_h=w["k_h"], k_l=w["k_l"]))


def test_noalloc_matches_workspace_entry_point_router_and_smooth_k():
    data, w = I.make_workload("wan1.3b_sla2")
    Q, K = data["Q"].cuda(), data["K"].cuda()
    cfg = bnd.SlaConfig(k_h=w["k_h"], k_l=w["k_l"], combine="alpha", smooth_k=True)
    _compare_twice(Q, K, cfg, data["Wq"].cuda(), data["Wk"].cuda())


def test_noalloc_rejects_problems_larger_than_its_scratch():
    # 14B-720P shape with a router needs ~97 MB of scratch: refused before any launch
    p = bnd.sla_params_t()
    L = bnd.lib()
    L.sla_params_default(ctypes.byref(p), 1, 40, 75600, 128, 0.03, 0.8, 1)
    buf = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    w = torch.zeros(128, 128, dtype=torch.float32, device="cuda")
    ptr = ctypes.c_void_p(buf.data_ptr())
    code = L.sla_predict_mask_noalloc(ctypes.byref(p), ptr, ptr, ctypes.c_void_p(w.data_ptr()),
                                      ctypes.c_void_p(w.data_ptr()), ptr, ptr, None)
    assert code == 3  # SLA_ERR_WORKSPACE
