"""GPU parity of the router probabilities and SoftTop-k ("SLA2: Sparse-Linear
Attention with Learnable Routing and QAT", §4 Learnable Router, §6 Training with
SLA2) through the C ABI against the fp64 oracle.

P_c is compared with the oracle's compressed attention on the same bf16 inputs
(relative 2e-4: fp32 pooled means and logits).  SoftTop-k is compared with the
oracle run on the GPU's own P_c: weights within 2e-4, row sums within 1e-3 of
n_h, and lambda within what the row's slope determines (|d lambda| times
sum M (1 - M) / tau <= 1e-3).  With a small temperature the weights above 1/2
are the hard mask's critical blocks.
"""
import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_linear_pool_b200 import binding as bnd
from block_sparse_linear_pool_b200 import inputs as I
from block_sparse_linear_pool_b200.build import build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    bnd.lib()


def _np(t):
    return None if t is None else t.detach().double().cpu().numpy()


def _small(B, H, N, d, seed):
    g = torch.Generator().manual_seed(seed)
    T = -(-N // 64)
    x = {}
    for name in ("Q", "K"):
        base = torch.randn(B, H, N, d, generator=g)
        mean = torch.randn(B, H, T, d, generator=g).repeat_interleave(64, dim=2)[:, :, :N]
        x[name] = (base + mean * 0.7).to(torch.bfloat16)
    x["Wq"] = (torch.rand(d, d, generator=g) * 2 - 1) / d ** 0.5
    x["Wk"] = (torch.rand(d, d, generator=g) * 2 - 1) / d ** 0.5
    return x


def _check(data, cfg, taus, router):
    Q, K = data["Q"].cuda(), data["K"].cuda()
    Wq, Wk = (data["Wq"], data["Wk"]) if router else (None, None)
    Pc = bnd.sla_router_probs(Q, K, cfg, Wq, Wk)
    torch.cuda.synchronize()
    p = O.OracleParams(k_h=cfg.k_h, k_l=cfg.k_l, smooth_k=cfg.smooth_k)
    B, H, N, d = Q.shape
    Pref = O.compressed_attention(O.compressed_logits(_np(Q), _np(K), p, _np(Wq), _np(Wk)))
    Pref = Pref.reshape(B * H, *Pref.shape[-2:])
    Pg = _np(Pc)
    np.testing.assert_allclose(Pg, Pref, rtol=2e-4, atol=1e-7)
    T = Pg.shape[-1]
    n_h, _ = O.block_counts(T, cfg.k_h, cfg.k_l)
    for tau_rel in taus:
        tau = tau_rel / T  # the mean probability is 1 / T
        M, lam = bnd.sla_soft_topk(Pc, Q, cfg, tau)
        torch.cuda.synchronize()
        Mref, lref = O.soft_topk(Pg, n_h, tau)
        Mg, lg = _np(M), _np(lam)
        assert np.abs(Mg - Mref).max() <= 2e-4, (tau_rel, np.abs(Mg - Mref).max())
        assert np.abs(Mg.sum(-1) - n_h).max() <= 1e-3
        slope = (Mref * (1 - Mref)).sum(-1) / tau
        assert (np.abs(lg - lref) * slope).max() <= 1e-3
    # a small temperature gives back the hard Top-k on rows with a clear cut
    mc, _ = bnd.sla_predict_mask(Q, K, cfg, Wq, Wk)
    tau = 1e-4 / T
    M, _ = bnd.sla_soft_topk(Pc, Q, cfg, tau)
    srt = -np.sort(-Pg, axis=-1)
    clear = (srt[..., n_h - 1] - srt[..., n_h]) > 100 * tau
    assert clear.any()
    hard = mc.cpu().numpy() == 1
    soft = _np(M) > 0.5
    assert np.array_equal(soft[clear], hard[clear])


@pytest.mark.parametrize("B,H,N,d,kh,router,smooth", [
    (1, 2, 1024, 64, 0.10, False, False),
    (1, 2, 1024, 64, 0.10, True, False),
    (2, 1, 1000, 128, 0.05, True, True),   # ragged tail, B > 1
    (1, 1, 4160, 128, 0.30, False, True),  # T = 65, n_h = 19
])
def test_soft_topk_small(B, H, N, d, kh, router, smooth):
    data = _small(B, H, N, d, seed=N + d)
    cfg = bnd.SlaConfig(k_h=kh, k_l=0.5, combine="alpha" if router else "proj", smooth_k=smooth)
    _check(data, cfg, taus=(0.2, 1.0, 5.0), router=router)


def test_soft_topk_wan13b_sla2_one_head_full_length():
    data, w = I.make_workload("wan1.3b_sla2", H=1)
    cfg = bnd.SlaConfig(k_h=w["k_h"], k_l=w["k_l"], combine=w["combine"])
    _check(data, cfg, taus=(0.5, 2.0), router=data.get("Wq") is not None)
