"""GPU parity of the backward (through the C ABI) against the fp64 oracle.

The CUDA path runs sla_predict_mask, sla_precompute_linear, sla_forward_train
and sla_backward; the oracle's analytic backward (pinned by finite
differences) gets the same bf16 inputs and the GPU's own M_c.  Every gradient
is held to the forward's output tolerances, relative to the largest reference
magnitude of that gradient: max-abs 2e-2 and mean-abs 2e-3.
"""
import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_linear_pool_b200 import binding as bnd
from block_sparse_linear_pool_b200 import inputs as I
from block_sparse_linear_pool_b200.build import build

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    bnd.lib()


def _np(t):
    return None if t is None else t.detach().float().cpu().numpy().astype(np.float64)


def _small(B, H, N, d, seed):
    g = torch.Generator().manual_seed(seed)
    T = -(-N // 64)
    x = {}
    for name in ("Q", "K", "V"):
        base = torch.randn(B, H, N, d, generator=g)
        mean = torch.randn(B, H, T, d, generator=g).repeat_interleave(64, dim=2)[:, :, :N]
        x[name] = (base + mean * 0.7).to(torch.bfloat16)
    x["proj_w"] = torch.randn(d, d, generator=g) * 0.05
    x["proj_b"] = torch.randn(d, generator=g) * 0.1
    x["alpha"] = torch.rand(B, H, generator=g) * 0.35 + 0.6
    x["dO"] = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    return x


def _compare(got, ref, what):
    g, r = _np(got), np.asarray(ref, dtype=np.float64)
    scale = np.abs(r).max()
    err = np.abs(g - r)
    if scale == 0:  # a gradient that is exactly zero (e.g. dProj when no block is marginal)
        assert err.max() == 0, f"{what}: the reference is exactly zero, the GPU gives max |x| = {err.max():.3e}"
        return 0.0
    assert err.max() <= MAX_ABS * scale, f"{what}: max-abs {err.max():.3e} > {MAX_ABS}*{scale:.3e}"
    assert err.mean() <= MEAN_ABS * scale, f"{what}: mean-abs {err.mean():.3e} > {MEAN_ABS}*{scale:.3e}"
    return err.max() / scale


def _run(data, cfg):
    dev = "cuda"
    Q, K, V, dO = (data[k].to(dev) for k in ("Q", "K", "V", "dO"))
    proj = cfg.combine == "proj"
    proj_w = data["proj_w"] if proj else None
    proj_b = data["proj_b"] if proj else None
    alpha = None if proj else data["alpha"]
    ws = bnd.new_workspace(bnd.sla_workspace_size(bnd.make_params(Q, cfg, K, V)), dev)
    mc, lut = bnd.sla_predict_mask(Q, K, cfg, workspace=ws)
    hz = bnd.sla_precompute_linear(K, V, cfg, proj_w, workspace=ws)
    out, lse, osp = bnd.sla_forward_train(Q, K, V, mc, lut, hz, cfg, proj_b=proj_b, alpha=alpha,
                                          workspace=ws)
    # the forward with the LSE output writes the same O as sla_forward
    out_plain = bnd.sla_forward(Q, K, V, mc, lut, hz, cfg, proj_b=proj_b, alpha=alpha, workspace=ws)
    grads, bws = bnd.sla_backward(Q, K, V, mc, lut, hz, osp, lse, dO, cfg, proj_w=proj_w, proj_b=proj_b,
                                  alpha=alpha)
    torch.cuda.synchronize()
    for w in (ws, bws):
        code, detail = bnd.sla_get_device_status(w)
        assert code == 0, (code, detail)
    assert torch.equal(out, out_plain)
    B, H, N, d = Q.shape
    T = mc.shape[-1]
    Mc = mc.cpu().numpy().reshape(B, H, T, T)
    p = O.OracleParams(k_h=cfg.k_h, k_l=cfg.k_l, combine=cfg.combine, eps=cfg.eps, phi=cfg.phi,
                       linear_over_all=cfg.linear_over_all)
    ref = O.backward_given_mask(_np(Q), _np(K), _np(V), Mc, _np(dO), p, proj_w=_np(proj_w),
                                proj_b=_np(proj_b), alpha=_np(alpha))
    # the stored sparse-branch output against the oracle's
    _, ref_os, _ = O.forward_given_mask(_np(Q), _np(K), _np(V), Mc, p, proj_w=_np(proj_w),
                                        proj_b=_np(proj_b), alpha=_np(alpha), return_branches=True)
    _compare(osp.view(B, H, N, d), ref_os, "o_sparse")
    rel = {}
    for k in ("dQ", "dK", "dV"):
        rel[k] = _compare(grads[k], ref[k], k)
    if proj:
        rel["dproj_w"] = _compare(grads["dproj_w"], ref["dproj_w"], "dproj_w")
        rel["dproj_b"] = _compare(grads["dproj_b"], ref["dproj_b"], "dproj_b")
    else:
        rel["dalpha"] = _compare(grads["dalpha"], ref["dalpha"], "dalpha")
    # the LSE against the oracle's definition on the GPU mask
    qs = _np(Q).reshape(B * H, N, d)
    ks = _np(K).reshape(B * H, N, d)
    lref = np.empty((B * H, N))
    for bh in range(B * H):
        for i in range(T):
            rs, re = O.block_range(i, 64, N)
            idx = np.concatenate([np.arange(*O.block_range(int(j), 64, N))
                                  for j in np.nonzero(Mc.reshape(B * H, T, T)[bh, i] == 1)[0]])
            s = qs[bh, rs:re] @ ks[bh, idx].T / np.sqrt(d)
            m = s.max(axis=1)
            lref[bh, rs:re] = m + np.log(np.exp(s - m[:, None]).sum(axis=1))
    np.testing.assert_allclose(_np(lse), lref, atol=2e-3)
    return rel


@pytest.mark.parametrize("B,H,N,d,kh,kl,combine", [
    (1, 2, 1024, 64, 0.10, 0.60, "alpha"),
    (1, 1, 1000, 64, 0.10, 0.50, "proj"),     # ragged tail (40 tokens)
    (2, 1, 130, 128, 0.34, 0.33, "proj"),     # 3 blocks, tail of 2 tokens, B > 1
    (1, 3, 2049, 128, 0.05, 0.70, "alpha"),   # tail of 1 token, odd T
    (1, 1, 640, 128, 1.0, 0.0, "proj"),       # k_h = 100%: dense attention
    (1, 2, 768, 64, 0.25, 0.75, "alpha"),     # no marginal blocks
    (1, 2, 3000, 128, 0.10, 0.40, "proj"),
])
def test_backward_small_shapes(B, H, N, d, kh, kl, combine):
    data = _small(B, H, N, d, seed=N + d + 11)
    _run(data, bnd.SlaConfig(k_h=kh, k_l=kl, combine=combine))


@pytest.mark.parametrize("phi,over_all,combine", [
    ("elu1", False, "proj"),
    ("softmax", True, "alpha"),
    ("elu1", True, "proj"),
])
def test_backward_code_variants(phi, over_all, combine):
    data = _small(1, 2, 1500, 128, seed=77)
    _run(data, bnd.SlaConfig(k_h=0.1, k_l=0.4, combine=combine, phi=phi, linear_over_all=over_all))


@pytest.mark.parametrize("name", ["wan1.3b_sla", "wan1.3b_sla2"])
def test_backward_wan13b_one_head_full_length(name):
    # one head of the Wan2.1-1.3B workload at its full length (N = 32760)
    data, w = I.make_workload(name, H=1)
    g = torch.Generator().manual_seed(123)
    data["dO"] = torch.randn(data["Q"].shape, generator=g).to(torch.bfloat16)
    if w["combine"] == "alpha":
        data["proj_w"] = data["proj_b"] = None
    cfg = bnd.SlaConfig(k_h=w["k_h"], k_l=w["k_l"], combine=w["combine"])
    _run(data, cfg)
