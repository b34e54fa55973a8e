"""Thin ctypes binding of libsla.so (include/sla.h) for torch tensors.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of the library.  torch provides device memory and the current stream.
The functions carry the C names; outputs and workspaces are allocated here
with torch (the library itself allocates nothing).  If libsla.so is missing,
every call raises: there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsla.so")

SLA_COMBINE_PROJ, SLA_COMBINE_ALPHA = 0, 1
SLA_QK_BF16, SLA_QK_FP8_E4M3, SLA_QK_INT8 = 0, 1, 2
_QK_PREC = {"bf16": SLA_QK_BF16, "fp8_e4m3": SLA_QK_FP8_E4M3, "int8": SLA_QK_INT8}
SLA_PHI_SOFTMAX, SLA_PHI_ELU1 = 0, 1

STATUS = {
    0: "SLA_OK", 1: "SLA_ERR_INVALID_ARG", 2: "SLA_ERR_UNSUPPORTED", 3: "SLA_ERR_WORKSPACE",
    4: "SLA_ERR_CUDA", 5: "SLA_ERR_DEVICE_TIMEOUT", 6: "SLA_ERR_DEVICE_BAD_INDEX",
}

# Every symbol include/sla.h declares (checked by the CPU tests).
EXPORTS = (
    "sla_params_default", "sla_block_counts", "sla_workspace_size", "sla_hz_size",
    "sla_predict_mask", "sla_precompute_linear", "sla_forward", "sla_attention_workspace_size",
    "sla_attention", "sla_aggregate_marginal", "sla_fused_forward",
    "sla_attention_host_workspace_size", "sla_attention_host", "sla_backward",
    "sla_get_device_status", "sla_status_string", "sla_abi_version",
    "sla_predict_mask_noalloc", "sla_forward_train", "sla_backward_workspace_size",
    "sla_selftest_wait_timeout", "sla_router_probs", "sla_soft_topk",
    "sla_pair_query_blocks", "sla_fused_forward_paired", "sla_workspace_pairs",
)


class SlaError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS.get(code, code)}")
        self.code = code


class sla_params_t(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int), ("d", ctypes.c_int),
        ("b_q", ctypes.c_int), ("b_kv", ctypes.c_int),
        ("k_h", ctypes.c_float), ("k_l", ctypes.c_float),
        ("combine", ctypes.c_int), ("qk_prec", ctypes.c_int), ("smooth_k", ctypes.c_int),
        ("eps", ctypes.c_float),
        ("stride_q", ctypes.c_int64 * 3), ("stride_k", ctypes.c_int64 * 3),
        ("stride_v", ctypes.c_int64 * 3), ("stride_o", ctypes.c_int64 * 3),
        ("phi", ctypes.c_int), ("linear_over_all", ctypes.c_int), ("pv_prec", ctypes.c_int),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built: run `python -m block_sparse_linear_pool_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(sla_params_t)
        vp, sz = ctypes.c_void_p, ctypes.c_size_t
        L.sla_params_default.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_float, ctypes.c_float, ctypes.c_int]
        L.sla_params_default.restype = None
        ip = ctypes.POINTER(ctypes.c_int)
        L.sla_block_counts.argtypes = [P, ip, ip, ip, ip]
        for f in ("sla_workspace_size", "sla_hz_size", "sla_attention_workspace_size",
                  "sla_attention_host_workspace_size", "sla_backward_workspace_size"):
            getattr(L, f).argtypes = [P, ctypes.POINTER(sz)]
        L.sla_predict_mask.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sla_precompute_linear.argtypes = [P, vp, vp, vp, vp, vp, sz, vp]
        L.sla_forward.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sla_attention.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sla_aggregate_marginal.argtypes = [P, vp, vp, vp, sz, vp]
        L.sla_fused_forward.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sla_fused_forward_paired.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sla_pair_query_blocks.argtypes = [P, vp, vp, sz, vp]
        L.sla_workspace_pairs.argtypes = [P, ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t)]
        L.sla_attention_host.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sla_predict_mask_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp, vp]
        L.sla_forward_train.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sla_backward.argtypes = [P] + [vp] * 18 + [vp, sz, vp]
        L.sla_get_device_status.argtypes = [vp, vp, ip]
        L.sla_selftest_wait_timeout.argtypes = [vp, vp]
        L.sla_router_probs.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sla_soft_topk.argtypes = [P, vp, ctypes.c_float, vp, vp, vp]
        L.sla_status_string.argtypes = [ctypes.c_int]
        L.sla_status_string.restype = ctypes.c_char_p
        for f in EXPORTS:
            if f not in ("sla_params_default", "sla_status_string"):
                getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(code: int, where: str):
    if code != 0:
        raise SlaError(code, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _strides(t: torch.Tensor):
    s = t.stride()
    if s[3] != 1:
        raise ValueError("the head dimension must be contiguous")
    return (ctypes.c_int64 * 3)(s[0], s[1], s[2])


@dataclass
class SlaConfig:
    """Settings of one forward ([SLA] §4 notation table; [SLA2] §3-5)."""
    k_h: float
    k_l: float
    combine: str = "proj"     # "proj" (SLA) or "alpha" (SLA2)
    qk: str = "bf16"          # "bf16", "fp8_e4m3" or "int8" (Q K^T of critical blocks, [SLA2] §5)
    smooth_k: bool = False
    eps: float = 1e-5
    phi: str = "softmax"      # "softmax" ([SLA] Fig. 4) or "elu1" ([SLA] Table 2 ablation)
    linear_over_all: bool = False  # linear branch over every key block ([SLA] §7 item 2)
    pv: str = "bf16"          # "bf16" or "fp8_e4m3" (P V of critical blocks, [SLA2] §5)


def make_params(Q: torch.Tensor, cfg: SlaConfig, K=None, V=None, O=None) -> sla_params_t:
    B, H, N, d = Q.shape
    p = sla_params_t()
    lib().sla_params_default(ctypes.byref(p), B, H, N, d, cfg.k_h, cfg.k_l,
                             SLA_COMBINE_PROJ if cfg.combine == "proj" else SLA_COMBINE_ALPHA)
    if cfg.qk not in _QK_PREC:
        raise ValueError(f"qk must be one of {sorted(_QK_PREC)}, not {cfg.qk!r}")
    p.qk_prec = _QK_PREC[cfg.qk]
    p.smooth_k = int(cfg.smooth_k)
    p.eps = cfg.eps
    if cfg.phi not in ("softmax", "elu1"):
        raise ValueError(f"phi must be 'softmax' or 'elu1', not {cfg.phi!r}")
    p.phi = SLA_PHI_SOFTMAX if cfg.phi == "softmax" else SLA_PHI_ELU1
    p.linear_over_all = int(cfg.linear_over_all)
    if cfg.pv not in ("bf16", "fp8_e4m3"):
        raise ValueError(f"pv must be 'bf16' or 'fp8_e4m3', not {cfg.pv!r}")
    p.pv_prec = 0 if cfg.pv == "bf16" else 1
    p.stride_q = _strides(Q)
    p.stride_k = _strides(K if K is not None else Q)
    p.stride_v = _strides(V if V is not None else Q)
    if O is not None:
        p.stride_o = _strides(O)
    return p


def sla_block_counts(p: sla_params_t):
    out = [ctypes.c_int() for _ in range(4)]
    _check(lib().sla_block_counts(ctypes.byref(p), *[ctypes.byref(x) for x in out]), "sla_block_counts")
    return tuple(x.value for x in out)  # T_q, T_kv, n_h, n_l


def _size(fn: str, p: sla_params_t) -> int:
    n = ctypes.c_size_t()
    _check(getattr(lib(), fn)(ctypes.byref(p), ctypes.byref(n)), fn)
    return n.value


def sla_workspace_size(p: sla_params_t) -> int:
    return _size("sla_workspace_size", p)


def sla_hz_size(p: sla_params_t) -> int:
    return _size("sla_hz_size", p)


def sla_attention_workspace_size(p: sla_params_t) -> int:
    return _size("sla_attention_workspace_size", p)


def new_workspace(nbytes: int, device) -> torch.Tensor:
    """Zero-initialised workspace (the first word is the device error word)."""
    return torch.zeros(nbytes, dtype=torch.uint8, device=device)


def _f32(t: Optional[torch.Tensor], device):
    return None if t is None else t.to(device=device, dtype=torch.float32).contiguous()


def sla_predict_mask(Q, K, cfg: SlaConfig, Wq=None, Wk=None, workspace=None):
    """Returns (mc int8 [B*H, T_q, T_kv], lut int32 [B*H, T_q, n_h])."""
    p = make_params(Q, cfg, K=K)
    Tq, Tkv, nh, _ = sla_block_counts(p)
    BH = Q.shape[0] * Q.shape[1]
    mc = torch.empty((BH, Tq, Tkv), dtype=torch.int8, device=Q.device)
    lut = torch.empty((BH, Tq, nh), dtype=torch.int32, device=Q.device)
    ws = workspace if workspace is not None else new_workspace(sla_workspace_size(p), Q.device)
    Wq, Wk = _f32(Wq, Q.device), _f32(Wk, Q.device)
    _check(lib().sla_predict_mask(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(Wq), _ptr(Wk), _ptr(mc),
                                  _ptr(lut), _ptr(ws), ws.numel(), _stream()), "sla_predict_mask")
    return mc, lut


def sla_router_probs(Q, K, cfg: SlaConfig, Wq=None, Wk=None, workspace=None):
    """P_c fp32 [B*H, T_q, T_kv]: the row softmax of the router's compressed logits."""
    p = make_params(Q, cfg, K=K)
    Tq, Tkv, _, _ = sla_block_counts(p)
    BH = Q.shape[0] * Q.shape[1]
    Pc = torch.empty((BH, Tq, Tkv), dtype=torch.float32, device=Q.device)
    ws = workspace if workspace is not None else new_workspace(sla_workspace_size(p), Q.device)
    Wq, Wk = _f32(Wq, Q.device), _f32(Wk, Q.device)
    _check(lib().sla_router_probs(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(Wq), _ptr(Wk), _ptr(Pc),
                                  _ptr(ws), ws.numel(), _stream()), "sla_router_probs")
    return Pc


def sla_soft_topk(Pc, Q, cfg: SlaConfig, tau: float):
    """SoftTop-k of P_c ([B*H, T_q, T_kv] fp32; Q gives the problem's shape):
    returns (M fp32 like Pc, lambda fp32 [B*H, T_q])."""
    p = make_params(Q, cfg)
    Tq, Tkv, _, _ = sla_block_counts(p)
    BH = Q.shape[0] * Q.shape[1]
    if tuple(Pc.shape) != (BH, Tq, Tkv) or Pc.dtype != torch.float32 or not Pc.is_contiguous():
        raise ValueError(f"Pc must be contiguous fp32 {(BH, Tq, Tkv)}")
    M = torch.empty_like(Pc)
    lam = torch.empty((BH, Tq), dtype=torch.float32, device=Pc.device)
    _check(lib().sla_soft_topk(ctypes.byref(p), _ptr(Pc), ctypes.c_float(tau), _ptr(M), _ptr(lam),
                               _stream()), "sla_soft_topk")
    return M, lam


def sla_precompute_linear(K, V, cfg: SlaConfig, proj_w=None, workspace=None):
    """Returns hz bf16 [B*H, T_kv, d*d + d] (see include/sla.h for the layout)."""
    p = make_params(K, cfg, K=K, V=V)
    _, Tkv, _, _ = sla_block_counts(p)
    BH, d = K.shape[0] * K.shape[1], K.shape[3]
    hz = torch.empty((BH, Tkv, d * d + d), dtype=torch.bfloat16, device=K.device)
    ws = workspace if workspace is not None else new_workspace(sla_workspace_size(p), K.device)
    proj_w = _f32(proj_w, K.device)
    _check(lib().sla_precompute_linear(ctypes.byref(p), _ptr(K), _ptr(V), _ptr(proj_w), _ptr(hz),
                                       _ptr(ws), ws.numel(), _stream()), "sla_precompute_linear")
    return hz


def sla_forward(Q, K, V, mc, lut, hz, cfg: SlaConfig, proj_b=None, alpha=None, out=None,
                workspace=None):
    """O bf16 [B, H, N, d]."""
    O = out if out is not None else torch.empty_like(Q)
    p = make_params(Q, cfg, K=K, V=V, O=O)
    ws = workspace if workspace is not None else new_workspace(sla_workspace_size(p), Q.device)
    proj_b, alpha = _f32(proj_b, Q.device), _f32(alpha, Q.device)
    _check(lib().sla_forward(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(mc), _ptr(lut), _ptr(hz),
                             _ptr(proj_b), _ptr(alpha), _ptr(O), _ptr(ws), ws.numel(), _stream()),
           "sla_forward")
    return O


def sla_forward_train(Q, K, V, mc, lut, hz, cfg: SlaConfig, proj_b=None, alpha=None, workspace=None):
    """sla_forward plus what the backward needs: (O, lse fp32 [B*H, N], o_sparse fp32 [B*H, N, d])."""
    O = torch.empty_like(Q)
    p = make_params(Q, cfg, K=K, V=V, O=O)
    B, H, N, d = Q.shape
    lse = torch.empty((B * H, N), dtype=torch.float32, device=Q.device)
    os_ = torch.empty((B * H, N, d), dtype=torch.float32, device=Q.device)
    ws = workspace if workspace is not None else new_workspace(sla_workspace_size(p), Q.device)
    proj_b, alpha = _f32(proj_b, Q.device), _f32(alpha, Q.device)
    _check(lib().sla_forward_train(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(mc), _ptr(lut),
                                   _ptr(hz), _ptr(proj_b), _ptr(alpha), _ptr(O), _ptr(lse), _ptr(os_),
                                   _ptr(ws), ws.numel(), _stream()), "sla_forward_train")
    return O, lse, os_


def sla_backward_workspace_size(p: sla_params_t) -> int:
    return _size("sla_backward_workspace_size", p)


def sla_backward(Q, K, V, mc, lut, hz, o_sparse, lse, dO, cfg: SlaConfig, proj_w=None, proj_b=None,
                 alpha=None, workspace=None):
    """Gradients of sum(O * dO): dict with dQ, dK, dV (bf16 like Q, K, V) and
    dproj_w, dproj_b (SLA) or dalpha (SLA2), fp32."""
    dev = Q.device
    dQ, dK, dV = torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V)
    p = make_params(Q, cfg, K=K, V=V, O=dO)
    d = Q.shape[-1]
    B, H = Q.shape[:2]
    proj = cfg.combine == "proj"
    dW = torch.empty((d, d), dtype=torch.float32, device=dev) if proj else None
    db = torch.empty(d, dtype=torch.float32, device=dev) if proj else None
    da = None if proj else torch.empty(B * H, dtype=torch.float32, device=dev)
    ws = workspace if workspace is not None else new_workspace(sla_backward_workspace_size(p), dev)
    args = [_f32(x, dev) for x in (proj_w, proj_b, alpha)]
    _check(lib().sla_backward(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(mc), _ptr(lut), _ptr(hz),
                              *[_ptr(x) for x in args], _ptr(o_sparse), _ptr(lse), _ptr(dO), _ptr(dQ), _ptr(dK),
                              _ptr(dV), _ptr(dW), _ptr(db), _ptr(da), _ptr(ws), ws.numel(), _stream()),
           "sla_backward")
    out = {"dQ": dQ, "dK": dK, "dV": dV}
    if proj:
        out.update(dproj_w=dW, dproj_b=db)
    else:
        out["dalpha"] = da.view(B, H)
    return out, ws


def sla_attention(Q, K, V, cfg: SlaConfig, proj_w=None, proj_b=None, alpha=None, Wq=None, Wk=None,
                  out=None, workspace=None):
    """The whole forward in one library call.  O bf16 [B, H, N, d]."""
    O = out if out is not None else torch.empty_like(Q)
    p = make_params(Q, cfg, K=K, V=V, O=O)
    ws = workspace if workspace is not None else new_workspace(sla_attention_workspace_size(p), Q.device)
    dev = Q.device
    args = [_f32(x, dev) for x in (proj_w, proj_b, alpha, Wq, Wk)]
    _check(lib().sla_attention(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), *[_ptr(x) for x in args],
                               _ptr(O), _ptr(ws), ws.numel(), _stream()), "sla_attention")
    return O


def sla_attention_host_workspace_size(p: sla_params_t) -> int:
    return _size("sla_attention_host_workspace_size", p)


def sla_aggregate_marginal(p: sla_params_t, mc, hz, workspace):
    """[H_i^T | Z_i] of every query block into `workspace` (first half of sla_forward)."""
    _check(lib().sla_aggregate_marginal(ctypes.byref(p), _ptr(mc), _ptr(hz), _ptr(workspace),
                                        workspace.numel(), _stream()), "sla_aggregate_marginal")


def sla_fused_forward(p: sla_params_t, Q, K, V, lut, O, workspace, proj_b=None, alpha=None):
    """The fused kernel (second half of sla_forward); proj_b / alpha fp32 on the device."""
    _check(lib().sla_fused_forward(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(lut), _ptr(proj_b),
                                   _ptr(alpha), _ptr(O), _ptr(workspace), workspace.numel(), _stream()),
           "sla_fused_forward")


def sla_pair_query_blocks(p: sla_params_t, lut, workspace):
    """Which two query blocks share a tile of the fused kernel (first step of
    sla_fused_forward); the pairs stay in `workspace`."""
    _check(lib().sla_pair_query_blocks(ctypes.byref(p), _ptr(lut), _ptr(workspace), workspace.numel(),
                                       _stream()), "sla_pair_query_blocks")


def sla_fused_forward_paired(p: sla_params_t, Q, K, V, lut, O, workspace, proj_b=None, alpha=None):
    """The fused kernel on the pairs already in `workspace` (second step of sla_fused_forward)."""
    _check(lib().sla_fused_forward_paired(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(lut),
                                          _ptr(proj_b), _ptr(alpha), _ptr(O), _ptr(workspace),
                                          workspace.numel(), _stream()), "sla_fused_forward_paired")


def sla_workspace_pairs(p: sla_params_t, workspace) -> torch.Tensor:
    """The block pairs in `workspace` as an int32 [B*H, ceil(T_q / 2), 2] view."""
    off, cnt = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().sla_workspace_pairs(ctypes.byref(p), ctypes.byref(off), ctypes.byref(cnt)),
           "sla_workspace_pairs")
    B, H = p.B, p.H
    return workspace[off.value:off.value + cnt.value * 8].view(torch.int32).view(B * H, -1, 2)


def sla_attention_host(p: sla_params_t, Qh, Kh, Vh, Oh, workspace, proj_w=None, proj_b=None,
                       alpha=None, Wq=None, Wk=None):
    """Host-memory activations (pinned CPU tensors); parameters are device tensors."""
    for t in (Qh, Kh, Vh, Oh):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("host variant takes contiguous CPU tensors")
    _check(lib().sla_attention_host(ctypes.byref(p), _ptr(Qh), _ptr(Kh), _ptr(Vh), _ptr(proj_w),
                                    _ptr(proj_b), _ptr(alpha), _ptr(Wq), _ptr(Wk), _ptr(Oh),
                                    _ptr(workspace), workspace.numel(), _stream()), "sla_attention_host")


def sla_get_device_status(workspace) -> int:
    detail = ctypes.c_int()
    code = lib().sla_get_device_status(_ptr(workspace), _stream(), ctypes.byref(detail))
    return code, detail.value


def sla_predict_mask_noalloc(Q, K, cfg: SlaConfig, Wq=None, Wk=None):
    """sla_predict_mask with the library's static scratch instead of a workspace."""
    p = make_params(Q, cfg, K=K)
    Tq, Tkv, nh, _ = sla_block_counts(p)
    BH = Q.shape[0] * Q.shape[1]
    mc = torch.empty((BH, Tq, Tkv), dtype=torch.int8, device=Q.device)
    lut = torch.empty((BH, Tq, nh), dtype=torch.int32, device=Q.device)
    Wq, Wk = _f32(Wq, Q.device), _f32(Wk, Q.device)
    _check(lib().sla_predict_mask_noalloc(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(Wq), _ptr(Wk),
                                          _ptr(mc), _ptr(lut), _stream()), "sla_predict_mask_noalloc")
    return mc, lut
