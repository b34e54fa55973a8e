"""The C-ABI library loads, exports every declared symbol and validates its
arguments on the host (no GPU needed: nothing here launches a kernel)."""
import ctypes
import os
import re

import pytest

from block_sparse_linear_pool_b200 import binding as bnd
from block_sparse_linear_pool_b200.build import build

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build()
    return bnd.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "sla.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sla_[a-z_]+)\s*\(", src)))


def test_header_declarations_match_binding_exports():
    assert _declared() == sorted(bnd.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    for name in _declared():
        assert hasattr(L, name), name


def _params(B=1, H=2, N=1024, d=64, kh=0.1, kl=0.6, combine=0):
    p = bnd.sla_params_t()
    bnd.lib().sla_params_default(ctypes.byref(p), B, H, N, d, kh, kl, combine)
    return p


@pytest.mark.parametrize("N,kh,kl", [(1024, 0.10, 0.60), (32760, 0.05, 0.75), (32760, 0.03, 0.80),
                                     (75600, 0.03, 0.80), (130, 1.0, 0.0), (64, 0.0, 1.0),
                                     (4000, 0.29, 0.5)])
def test_block_counts_follow_the_oracle_rule(L, N, kh, kl):
    Tq, Tkv, nh, nl = bnd.sla_block_counts(_params(N=N, kh=kh, kl=kl))
    T = O.num_blocks(N, 64)
    assert (Tq, Tkv) == (T, T)
    assert (nh, nl) == O.block_counts(T, kh, kl)


def test_invalid_arguments_are_rejected_before_any_launch(L):
    p = _params()
    p.d = 96
    assert L.sla_block_counts(ctypes.byref(p), None, None, None, None) == 2  # UNSUPPORTED
    p = _params()
    p.b_q = 32
    assert L.sla_block_counts(ctypes.byref(p), None, None, None, None) == 2
    p = _params()
    p.k_h = 1.5
    assert L.sla_block_counts(ctypes.byref(p), None, None, None, None) == 1  # INVALID_ARG
    p = _params()
    p.stride_q[2] = 60  # not a multiple of 8 / smaller than d
    assert L.sla_block_counts(ctypes.byref(p), None, None, None, None) == 1
    p = _params()
    p.phi = 2  # no such feature map
    assert L.sla_block_counts(ctypes.byref(p), None, None, None, None) == 1
    p = _params()
    p.linear_over_all = 7
    assert L.sla_block_counts(ctypes.byref(p), None, None, None, None) == 1
    p = _params()
    p.pv_prec = 3
    assert L.sla_block_counts(ctypes.byref(p), None, None, None, None) == 1
    p = _params(d=64)
    p.pv_prec = 1  # FP8 P V is built for d = 128
    assert L.sla_block_counts(ctypes.byref(p), None, None, None, None) == 2
    for qk, want in ((1, 2), (2, 2), (3, 1)):  # 8-bit Q K^T is built for d = 128; no format 3
        p = _params(d=64)
        p.qk_prec = qk
        assert L.sla_block_counts(ctypes.byref(p), None, None, None, None) == want
    p = _params(d=128)
    p.qk_prec = 2  # INT8 Q K^T at d = 128
    assert L.sla_block_counts(ctypes.byref(p), None, None, None, None) == 0
    p = _params()
    ws = (ctypes.c_uint8 * 1024)()
    # NULL tensors
    assert L.sla_predict_mask(ctypes.byref(p), None, None, None, None, None, None, ws, 1024, None) == 1
    assert L.sla_forward(ctypes.byref(p), None, None, None, None, None, None, None, None, None, ws,
                         1024, None) == 1
    # SLA2 without alpha
    p2 = _params(combine=1)
    dummy = ctypes.c_void_p(4096)
    assert L.sla_forward(ctypes.byref(p2), dummy, dummy, dummy, dummy, dummy, dummy, None, None,
                         dummy, ws, 1024, None) == 1
    # workspace too small
    assert L.sla_forward(ctypes.byref(p), dummy, dummy, dummy, dummy, dummy, dummy, None, None,
                         dummy, ctypes.c_void_p(4096), 16, None) == 3
    # backward: NULL gradient outputs, then a workspace that is too small
    args = [dummy] * 12 + [None] * 6
    assert L.sla_backward(ctypes.byref(p), *args[:9], dummy, dummy, dummy, None, None, None, None,
                          None, None, ctypes.c_void_p(1 << 20), 1 << 40, None) == 1
    need = bnd.sla_backward_workspace_size(p)
    assert L.sla_backward(ctypes.byref(p), *[dummy] * 15, None, None, None,
                          ctypes.c_void_p(1 << 20), need - 1, None) == 3
    # router probabilities and SoftTop-k: NULL / misaligned buffers, tau not positive and finite
    assert L.sla_router_probs(ctypes.byref(p), dummy, dummy, None, None, None, ws, 1024, None) == 1
    assert L.sla_router_probs(ctypes.byref(p), dummy, dummy, None, None, ctypes.c_void_p(4100), ws,
                              1024, None) == 1
    assert L.sla_router_probs(ctypes.byref(p), dummy, dummy, None, None, dummy,
                              ctypes.c_void_p(4096), 16, None) == 3
    # (a subnormal tau would make 1 / tau overflow in the kernel's fp32 arithmetic)
    for tau in (0.0, -1.0, float("nan"), float("inf"), 1e-39, 1e-45):
        assert L.sla_soft_topk(ctypes.byref(p), dummy, ctypes.c_float(tau), dummy, dummy, None) == 1
    assert L.sla_soft_topk(ctypes.byref(p), None, ctypes.c_float(0.1), dummy, dummy, None) == 1
    assert L.sla_soft_topk(ctypes.byref(p), dummy, ctypes.c_float(0.1), dummy, None, None) == 1


def test_defaults_are_the_pages_main_method(L):
    p = _params()
    assert (p.phi, p.linear_over_all, p.qk_prec, p.smooth_k, p.pv_prec) == (0, 0, 0, 0, 0)
    assert abs(p.eps - 1e-5) < 1e-12


def test_workspace_sizes_grow_with_the_problem(L):
    small, big = _params(N=1024), _params(N=32760, H=12, d=128)
    assert bnd.sla_workspace_size(small) < bnd.sla_workspace_size(big)
    assert bnd.sla_attention_workspace_size(big) > bnd.sla_workspace_size(big)
    T = O.num_blocks(32760, 64)
    assert bnd.sla_hz_size(big) == 12 * T * (128 * 128 + 128) * 2


def test_status_strings(L):
    for code, name in bnd.STATUS.items():
        assert L.sla_status_string(code).decode() == name
    assert L.sla_abi_version() == 104
