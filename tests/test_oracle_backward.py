"""Pins of the oracle's analytic backward (CPU only).

The backward is pinned to things other than itself:
  * central finite differences of the (separately pinned) forward oracle, for
    every input it differentiates (Q, K, V, Proj weight and bias, alpha), both
    combines, both feature maps and the all-blocks linear variant;
  * with k_h = 100% and alpha = 1 the forward is dense softmax attention, so
    dQ, dK, dV must equal torch autograd through scaled_dot_product_attention
    in float64.
"""
import numpy as np
import pytest
import torch

import oracle as O


def _random_mask(rng, B, H, T, n_h, n_l):
    """Every row: n_h critical, n_l negligible, the rest marginal, at random places."""
    Mc = np.zeros((B, H, T, T), dtype=np.int8)
    for idx in np.ndindex(B, H, T):
        perm = rng.permutation(T)
        Mc[idx][perm[:n_h]] = 1
        Mc[idx][perm[T - n_l:]] = -1
    return Mc


def _problem(seed, B=1, H=2, N=150, d=8, n_h=1, n_l=1):
    rng = np.random.default_rng(seed)
    T = O.num_blocks(N, 64)
    x = {n: rng.standard_normal((B, H, N, d)) for n in ("Q", "K", "V", "dO")}
    x["Mc"] = _random_mask(rng, B, H, T, n_h, n_l)
    x["W"] = rng.standard_normal((d, d)) * 0.3
    x["b"] = rng.standard_normal(d) * 0.1
    x["alpha"] = rng.uniform(0.2, 0.9, size=(B, H))
    return x, rng


def _loss(x, p, **over):
    y = dict(x)
    y.update(over)
    O_ = O.forward_given_mask(y["Q"], y["K"], y["V"], y["Mc"], p, proj_w=y["W"], proj_b=y["b"],
                              alpha=y["alpha"])
    return float((O_ * y["dO"]).sum())


@pytest.mark.parametrize("seed,combine,phi,over_all", [
    (1, "proj", "softmax", False),
    (2, "alpha", "softmax", False),
    (3, "proj", "elu1", False),
    (4, "alpha", "elu1", True),
    (5, "proj", "softmax", True),
])
def test_backward_matches_finite_differences(seed, combine, phi, over_all):
    # N = 150: blocks of 64, 64 and a partial block of 22 tokens
    x, rng = _problem(seed=seed)
    p = O.OracleParams(combine=combine, phi=phi, linear_over_all=over_all, eps=1e-3)
    g = O.backward_given_mask(x["Q"], x["K"], x["V"], x["Mc"], x["dO"], p, proj_w=x["W"],
                              proj_b=x["b"], alpha=x["alpha"])
    names = [("Q", "dQ"), ("K", "dK"), ("V", "dV")]
    names += [("W", "dproj_w"), ("b", "dproj_b")] if combine == "proj" else [("alpha", "dalpha")]
    h = 1e-5
    for name, gname in names:
        for _ in range(2):
            delta = rng.standard_normal(x[name].shape)
            fd = (_loss(x, p, **{name: x[name] + h * delta}) -
                  _loss(x, p, **{name: x[name] - h * delta})) / (2 * h)
            an = float((g[gname] * delta).sum())
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, fd, an)


def test_dense_case_equals_autograd_of_dense_attention():
    # k_h = 100%: every block critical; alpha = 1 leaves the sparse branch alone
    rng = np.random.default_rng(5)
    B, H, N, d = 1, 2, 200, 16
    Q, K, V, dO = (rng.standard_normal((B, H, N, d)) for _ in range(4))
    T = O.num_blocks(N, 64)
    Mc = np.ones((B, H, T, T), dtype=np.int8)
    p = O.OracleParams(k_h=1.0, k_l=0.0, combine="alpha")
    g = O.backward_given_mask(Q, K, V, Mc, dO, p, alpha=np.ones((B, H)))
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (Q, K, V))
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)
    out.backward(torch.tensor(dO))
    for mine, ref in ((g["dQ"], tq.grad), (g["dK"], tk.grad), (g["dV"], tv.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=1e-9, atol=1e-11)


def test_feature_map_backward_matches_autograd():
    rng = np.random.default_rng(9)
    X = rng.standard_normal((40, 12)) * 2
    dF = rng.standard_normal((40, 12))
    for kind, fn in (("softmax", lambda t: torch.softmax(t, -1)),
                     ("elu1", lambda t: torch.nn.functional.elu(t) + 1)):
        t = torch.tensor(X, requires_grad=True)
        fn(t).backward(torch.tensor(dF))
        got = O.feature_map_backward(X, O.feature_map(X, kind), dF, kind)
        np.testing.assert_allclose(got, t.grad.numpy(), rtol=1e-12, atol=1e-13)
