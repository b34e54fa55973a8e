"""Pins of the fp64 oracle against what the pages and mathematics fix.

Nothing here compares the oracle with itself: every expected value comes from a
hand derivation (tests/golden), a closed form, a library routine that computes
a special case (torch's scaled_dot_product_attention, softmax, F.linear, the
float8_e4m3fn cast) or a brute-force N x N formulation.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _token_mask(Mc, value, b, N):
    """Expand a block mask row set to tokens: True where M_c == value."""
    m = (Mc == value)
    m = np.repeat(np.repeat(m, b, axis=-2), b, axis=-1)
    return m[..., :N, :N]


# ---------------------------------------------------------------- counts
@pytest.mark.parametrize("T,kh,kl,exp", [
    (16, 0.10, 0.60, (1, 9)),
    (512, 0.05, 0.75, (25, 384)),
    (512, 0.03, 0.80, (15, 409)),
    (1182, 0.03, 0.80, (35, 945)),
    (8, 1.0, 0.0, (8, 0)),       # k_h = 100%: every block critical
    (8, 0.0, 0.0, (1, 0)),       # at least one critical block
    (8, 0.0, 1.0, (1, 7)),       # k_l = 100% capped so one block stays critical
])
def test_block_counts(T, kh, kl, exp):
    assert O.block_counts(T, kh, kl) == exp


# ---------------------------------------------------------------- pooling
def test_mean_pool_ramp_with_partial_tail():
    N, b = 150, 64
    X = np.arange(N, dtype=np.float64)[None, :, None] * np.ones((1, 1, 3))
    P = O.mean_pool(X, b)
    # means of 0..63, 64..127, 128..149
    np.testing.assert_array_equal(P[0, :, 0], [31.5, 95.5, 138.5])
    C = np.full((2, 130, 4), 2.5)
    np.testing.assert_array_equal(O.mean_pool(C, 64), np.full((2, 3, 4), 2.5))


# ---------------------------------------------------------------- classification
def _golden_mask_cases():
    cases, lines = [], [l.split("#")[0].strip() for l in open(os.path.join(GOLDEN, "mask_classify.txt"))]
    lines = [l for l in lines if l]
    for k in range(0, len(lines), 3):
        _, T, nh, nl = lines[k].split()
        P = np.array([float(x) for x in lines[k + 1].split()])
        M = np.array([int(x) for x in lines[k + 2].split()], dtype=np.int8)
        assert len(P) == int(T) == len(M)
        cases.append((P, int(nh), int(nl), M))
    return cases


@pytest.mark.parametrize("case", _golden_mask_cases())
def test_classify_golden(case):
    P, nh, nl, M = case
    np.testing.assert_array_equal(O.classify(P[None], nh, nl)[0], M)


def test_classify_brute_force_definition():
    rng = np.random.default_rng(5)
    for trial in range(200):
        T = int(rng.integers(1, 10))
        nh = int(rng.integers(1, T + 1))
        nl = int(rng.integers(0, T - nh + 1))
        P = rng.integers(0, 4, size=T).astype(float)  # many ties
        M = O.classify(P[None], nh, nl)[0]
        assert (M == 1).sum() == nh and (M == -1).sum() == nl
        key = lambda j: (-P[j], j)  # total order of the reading
        crit = [j for j in range(T) if M[j] == 1]
        negl = [j for j in range(T) if M[j] == -1]
        rest = [j for j in range(T) if M[j] != 1]
        nonneg = [j for j in range(T) if M[j] != -1]
        if crit and rest:
            assert max(key(j) for j in crit) < min(key(j) for j in rest)
        if negl and nonneg:
            assert min(key(j) for j in negl) > max(key(j) for j in nonneg)


def test_ranking_on_logits_equals_ranking_on_softmax():
    L = _rand((3, 7, 11), 1)
    nh, nl = O.block_counts(11, 0.2, 0.5)
    np.testing.assert_array_equal(O.classify(L, nh, nl), O.classify(O.compressed_attention(L), nh, nl))


def test_compressed_softmax_matches_torch():
    L = _rand((2, 5, 9), 2, 3.0)
    np.testing.assert_allclose(O.compressed_attention(L), torch.softmax(torch.from_numpy(L), -1).numpy(),
                               rtol=0, atol=1e-15)


def test_router_follows_linear_layer_convention():
    B, H, N, d, b = 1, 2, 200, 8, 32
    Q, K = _rand((B, H, N, d), 3), _rand((B, H, N, d), 4)
    Wq, Wk = _rand((d, d), 5), _rand((d, d), 6)
    p = O.OracleParams(b_q=b, b_kv=b)
    L = O.compressed_logits(Q, K, p, Wq, Wk)
    Qc = torch.from_numpy(O.mean_pool(Q, b))
    Kc = torch.from_numpy(O.mean_pool(K, b))
    ref = F.linear(Qc, torch.from_numpy(Wq)) @ F.linear(Kc, torch.from_numpy(Wk)).transpose(-1, -2) / math.sqrt(d)
    np.testing.assert_allclose(L, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_smooth_k_leaves_mask_unchanged():
    B, H, N, d = 1, 2, 640, 16
    Q, K = _rand((B, H, N, d), 7), _rand((B, H, N, d), 8) + 3.0  # K with a large common mean
    p0 = O.OracleParams(k_h=0.2, k_l=0.3)
    p1 = O.OracleParams(k_h=0.2, k_l=0.3, smooth_k=True)
    M0, L0, _ = O.predict_mask(Q, K, p0)
    M1, _, _ = O.predict_mask(Q, K, p1)
    nh, nl = O.block_counts(L0.shape[-1], 0.2, 0.3)
    g = O.mask_grading(L0, nh, nl, 1e-9)
    assert g.mean() > 0.9
    np.testing.assert_array_equal(M0[g], M1[g])


# ---------------------------------------------------------------- feature map and block statistics
def test_feature_map_against_torch():
    X = _rand((4, 9, 16), 9, 2.0)
    np.testing.assert_allclose(O.feature_map(X, "softmax"), torch.softmax(torch.from_numpy(X), -1).numpy(),
                               atol=1e-15)
    np.testing.assert_allclose(O.feature_map(X, "elu1"), (F.elu(torch.from_numpy(X)) + 1).numpy(), atol=1e-15)
    np.testing.assert_allclose(O.feature_map(X + 7.0), O.feature_map(X), atol=1e-14)


def test_linear_stats_invariants_and_outer_products():
    N, d, b = 150, 6, 64
    K, V = _rand((N, d), 10), _rand((N, d), 11)
    h, z = O.linear_block_stats(K, V, b)
    fk = torch.softmax(torch.from_numpy(K), -1).numpy()
    for j in range(3):
        s, e = j * b, min(N, (j + 1) * b)
        # sum over a of phi(k)_a = 1 per token
        np.testing.assert_allclose(h[j].sum(axis=0), V[s:e].sum(axis=0), atol=1e-12)
        np.testing.assert_allclose(z[j].sum(), e - s, atol=1e-12)
        outer = sum(np.outer(fk[t], V[t]) for t in range(s, e))
        np.testing.assert_allclose(h[j], outer, atol=1e-12)


# ---------------------------------------------------------------- degenerate limits of the whole forward
def _sdpa(Q, K, V, mask=None):
    return F.scaled_dot_product_attention(torch.from_numpy(Q), torch.from_numpy(K), torch.from_numpy(V),
                                          attn_mask=None if mask is None else torch.from_numpy(mask)).numpy()


@pytest.mark.parametrize("N", [200, 256])
def test_kh_100_percent_is_dense_attention(N):
    B, H, d = 1, 2, 16
    Q, K, V = _rand((B, H, N, d), 12), _rand((B, H, N, d), 13), _rand((B, H, N, d), 14)
    W = _rand((d, d), 15)
    p = O.OracleParams(k_h=1.0, k_l=0.0)
    out, Mc = O.forward(Q, K, V, p, proj_w=W)
    assert (Mc == 1).all()
    np.testing.assert_allclose(out, _sdpa(Q, K, V), atol=1e-12)
    p2 = O.OracleParams(k_h=1.0, k_l=0.0, combine="alpha")
    alpha = np.array([[0.3, 0.8]])
    out2, _ = O.forward(Q, K, V, p2, alpha=alpha)
    np.testing.assert_allclose(out2, alpha[..., None, None] * _sdpa(Q, K, V), atol=1e-12)


def test_no_marginal_blocks_is_block_sparse_attention():
    B, H, N, d, b = 1, 2, 300, 8, 64
    Q, K, V = _rand((B, H, N, d), 16), _rand((B, H, N, d), 17), _rand((B, H, N, d), 18)
    p = O.OracleParams(k_h=0.4, k_l=0.6, combine="alpha")  # T=5 -> n_h=2, n_l=3, no marginal
    out, Mc = O.forward(Q, K, V, p, alpha=np.ones((1, 2)))
    assert not (Mc == 0).any()
    ref = _sdpa(Q, K, V, _token_mask(Mc, 1, b, N))
    np.testing.assert_allclose(out, ref, atol=1e-12)
    # SLA combine with Proj = 0 gives the same
    p_proj = O.OracleParams(k_h=0.4, k_l=0.6)
    out3 = O.forward_given_mask(Q, K, V, Mc, p_proj, proj_w=np.zeros((d, d)))
    np.testing.assert_allclose(out3, ref, atol=1e-12)


@pytest.mark.parametrize("phi,over_all", [("softmax", False), ("elu1", False), ("softmax", True)])
def test_linear_branch_equals_masked_quadratic_form(phi, over_all):
    B, H, N, d, b = 1, 1, 200, 8, 32
    Q, K, V = _rand((B, H, N, d), 19), _rand((B, H, N, d), 20), _rand((B, H, N, d), 21)
    p = O.OracleParams(b_q=b, b_kv=b, k_h=0.15, k_l=0.3, combine="alpha", phi=phi,
                       linear_over_all=over_all)
    out, Mc = O.forward(Q, K, V, p, alpha=np.zeros((1, 1)))  # alpha = 0 isolates O^l
    fq = O.feature_map(Q[0, 0], phi) if phi == "elu1" else torch.softmax(torch.from_numpy(Q[0, 0]), -1).numpy()
    fk = O.feature_map(K[0, 0], phi) if phi == "elu1" else torch.softmax(torch.from_numpy(K[0, 0]), -1).numpy()
    A = fq @ fk.T
    if not over_all:
        A = A * _token_mask(Mc[0, 0], 0, b, N)
    ref = (A @ V[0, 0]) / (A.sum(axis=1, keepdims=True) + 1e-5)
    np.testing.assert_allclose(out[0, 0], ref, atol=1e-12)


def test_decomposition_identity_eq1():
    B, H, N, d, b = 1, 1, 130, 4, 32
    Q, K = _rand((B, H, N, d), 22), _rand((B, H, N, d), 23)
    Mc, _, _ = O.predict_mask(Q, K, O.OracleParams(b_q=b, b_kv=b, k_h=0.2, k_l=0.2))
    P = torch.softmax(torch.from_numpy(Q[0, 0] @ K[0, 0].T / 2.0), -1).numpy()
    M = _token_mask(Mc[0, 0], 1, b, N).astype(np.float64)
    np.testing.assert_array_equal(P * M + P * (1 - M), P)


def test_alpha_endpoints_and_linearity():
    B, H, N, d = 1, 2, 260, 8
    Q, K, V = _rand((B, H, N, d), 24), _rand((B, H, N, d), 25), _rand((B, H, N, d), 26)
    p = O.OracleParams(k_h=0.2, k_l=0.4, combine="alpha")
    Mc, _, _ = O.predict_mask(Q, K, p)
    a = np.array([[0.25, 0.9]])
    o_a = O.forward_given_mask(Q, K, V, Mc, p, alpha=a)
    o_1 = O.forward_given_mask(Q, K, V, Mc, p, alpha=np.ones((1, 2)))
    o_0 = O.forward_given_mask(Q, K, V, Mc, p, alpha=np.zeros((1, 2)))
    np.testing.assert_allclose(o_a, a[..., None, None] * o_1 + (1 - a[..., None, None]) * o_0, atol=1e-12)
    # alpha = 1 is pure block-sparse attention over the critical blocks
    np.testing.assert_allclose(o_1, _sdpa(Q, K, V, _token_mask(Mc, 1, 64, N)), atol=1e-12)


def test_proj_is_a_linear_layer_on_the_linear_branch():
    B, H, N, d = 1, 2, 200, 8
    Q, K, V = _rand((B, H, N, d), 27), _rand((B, H, N, d), 28), _rand((B, H, N, d), 29)
    W, bias = _rand((d, d), 30), _rand((d,), 31)
    p = O.OracleParams(k_h=0.25, k_l=0.25)
    Mc, _, _ = O.predict_mask(Q, K, p)
    o = O.forward_given_mask(Q, K, V, Mc, p, proj_w=W, proj_b=bias)
    pa = O.OracleParams(k_h=0.25, k_l=0.25, combine="alpha")
    o_s = O.forward_given_mask(Q, K, V, Mc, pa, alpha=np.ones((1, 2)))
    o_l = O.forward_given_mask(Q, K, V, Mc, pa, alpha=np.zeros((1, 2)))
    ref = o_s + F.linear(torch.from_numpy(o_l), torch.from_numpy(W), torch.from_numpy(bias)).numpy()
    np.testing.assert_allclose(o, ref, atol=1e-12)


def test_linear_branch_is_a_shrunk_convex_combination():
    B, H, N, d = 1, 1, 512, 8
    Q, K, V = _rand((B, H, N, d), 32), _rand((B, H, N, d), 33), _rand((B, H, N, d), 34)
    p = O.OracleParams(k_h=0.125, k_l=0.25, combine="alpha")
    out, Mc = O.forward(Q, K, V, p, alpha=np.zeros((1, 1)))
    lo = np.minimum(V[0, 0].min(axis=0), 0) - 1e-12
    hi = np.maximum(V[0, 0].max(axis=0), 0) + 1e-12
    assert ((out[0, 0] >= lo) & (out[0, 0] <= hi)).all()


def test_hand_computed_tiny_forward():
    vals = {}
    for line in open(os.path.join(GOLDEN, "tiny_forward.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        key, rest = line.split(None, 1)
        vals[key] = np.array([[float(x) for x in r.split()] for r in rest.split("|")])
    Q, K, V = (vals[k][None, None] for k in ("Q", "K", "V"))
    Mc = vals["Mc"].astype(np.int8)[None, None]
    eps = float(vals["eps"][0, 0])
    p = O.OracleParams(b_q=2, b_kv=2, combine="alpha", eps=eps)
    _, Os, Ol = O.forward_given_mask(Q, K, V, Mc, p, alpha=np.full((1, 1), 0.5), return_branches=True)
    np.testing.assert_allclose(Os[0, 0], vals["Os"], atol=1e-14)
    np.testing.assert_allclose(Ol[0, 0], vals["Ol_num"] / (vals["Ol_den"] + eps), atol=1e-14)


# ---------------------------------------------------------------- FP8 E4M3 quantiser
def test_quantize_e4m3_hand_values():
    x = np.array([1.0625, 1.1875, 448.0, 500.0, -500.0, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -10, 0.0, -3.3])
    exp = np.array([1.0, 1.25, 448.0, 448.0, -448.0, 2.0 ** -9, 0.0, 2.0 ** -8, 0.0, -3.25])
    np.testing.assert_array_equal(O.quantize_e4m3(x), exp)


def test_quantize_e4m3_matches_torch_float8():
    rng = np.random.default_rng(35)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.1, 1.0, 30.0, 150.0)])
    x = np.clip(x, -448, 448)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.quantize_e4m3(x), ref)


def test_mask_grading_excludes_near_ties():
    L = np.array([[0.0, 1.0, 1.00005, 2.0, -3.0]])
    g = O.mask_grading(L, 2, 1)
    # thresholds: top-2 -> midpoint(1.00005, 1.0); bottom-1 -> midpoint(-3, 0)
    np.testing.assert_array_equal(g[0], [True, False, False, True, True])


# ---------------------------------------------------------------- low-bit Q, K tiles
def _tiles_with_different_ranges(seed, d=32):
    """Three 64-row tiles and a partial one whose magnitudes differ by orders of
    magnitude, so that a per-tensor scale or a scale taken over the wrong rows
    cannot pass."""
    rng = np.random.default_rng(seed)
    parts = [rng.standard_normal((64, d)) * s for s in (0.01, 1.0, 40.0)] + [rng.standard_normal((20, d)) * 3.0]
    X = np.concatenate(parts)
    return torch.from_numpy(X).to(torch.bfloat16).double().numpy()  # bf16 values, as the kernels see them


def _torch_tile_dequant(X, fmt):
    """Per-64-row-tile quantisation with torch: E4M3 through the float8_e4m3fn cast,
    INT8 through round-half-even and clamping; scale max|tile| / R."""
    R = 448.0 if fmt == "fp8_e4m3" else 127.0
    out = np.empty_like(X)
    for s in range(0, X.shape[0], 64):
        t = torch.from_numpy(X[s:s + 64]).float()
        amax = t.abs().max()
        y = t * (torch.tensor(R, dtype=torch.float32) / amax)
        code = y.to(torch.float8_e4m3fn).double() if fmt == "fp8_e4m3" else torch.round(y).clamp(-127, 127).double()
        out[s:s + 64] = (code * (amax / R).double()).numpy()
    return out


@pytest.mark.parametrize("fmt", ["fp8_e4m3", "int8"])
def test_lowbit_tile_per_64_row_tile_against_torch(fmt):
    X = _tiles_with_different_ranges(40)
    got = np.concatenate([O.lowbit_tile(X[s:s + 64], fmt) for s in range(0, X.shape[0], 64)])
    np.testing.assert_array_equal(got, _torch_tile_dequant(X, fmt))


@pytest.mark.parametrize("fmt", ["fp8_e4m3", "int8"])
def test_lowbit_tile_error_bounds_and_range(fmt):
    # each tile's largest element maps to the format's largest code, and every
    # element is within the format's rounding bound of its own tile's scale:
    # E4M3 half a step (2^-4 relative in the normal range, 2^-10 s below it),
    # INT8 half a step (s / 2).  A swapped (448 / max) or per-tensor scale breaks both.
    X = _tiles_with_different_ranges(41)
    R = O.LOWBIT_MAX[fmt]
    for s in range(0, X.shape[0], 64):
        t = X[s:s + 64]
        q = O.lowbit_tile(t, fmt)
        amax = np.abs(t).max()
        sc = amax / R
        assert abs(np.abs(q).max() - amax) <= 1e-6 * amax
        err = np.abs(q - t)
        if fmt == "int8":
            assert (err <= 0.5 * sc * (1 + 1e-4)).all()  # + the fp32 rounding of x * (R / max)
            codes = q / np.float64(np.float32(amax) / np.float32(R))
            np.testing.assert_allclose(codes, np.round(codes), atol=1e-9)
        else:
            normal = np.abs(t) >= 2.0 ** -6 * sc
            assert (err[normal] <= 2.0 ** -4 * np.abs(t[normal]) * (1 + 1e-4)).all()
            assert (err[~normal] <= 2.0 ** -10 * sc * (1 + 1e-4)).all()


def test_lowbit_tile_int8_exact_on_its_grid():
    c = 0.37
    ints = np.random.default_rng(42).integers(-127, 128, size=(64, 16)).astype(np.float64)
    ints[0, 0] = 127.0
    X = ints * c
    np.testing.assert_allclose(O.lowbit_tile(X, "int8"), X, rtol=1e-6, atol=0)


def _sparse_case(seed, N=200, d=16, alpha_one=True):
    rng = np.random.default_rng(seed)
    B, H = 1, 1
    T = O.num_blocks(N, 64)
    Q = np.concatenate([rng.standard_normal((B, H, 64, d)) * s for s in (0.3, 2.0, 0.05, 8.0)], axis=2)[:, :, :N]
    K = np.concatenate([rng.standard_normal((B, H, 64, d)) * s for s in (5.0, 0.1, 1.0, 0.7)], axis=2)[:, :, :N]
    V = rng.standard_normal((B, H, N, d)) * np.linspace(0.2, 3.0, d)
    Q, K, V = (torch.from_numpy(x).to(torch.bfloat16).double().numpy() for x in (Q, K, V))
    Mc = np.full((B, H, T, T), -1, dtype=np.int8)
    for i in range(T):  # two critical blocks per row (no marginal ones), a different pair per row
        Mc[0, 0, i, [(i + 1) % T, (3 * i) % T if (3 * i) % T != (i + 1) % T else (i + 2) % T]] = 1
    return Q, K, V, Mc


@pytest.mark.parametrize("fmt", ["fp8_e4m3", "int8"])
def test_lowbit_qk_forward_is_block_sparse_attention_on_dequantised_tiles(fmt):
    # brute force: Q, K dequantised tile by tile with torch, N x N scores with -inf
    # outside the critical blocks, torch SDPA; alpha = 1 and no marginal blocks.
    Q, K, V, Mc = _sparse_case(43)
    N = Q.shape[2]
    Qd = _torch_tile_dequant(Q[0, 0], fmt)
    Kd = _torch_tile_dequant(K[0, 0], fmt)
    allow = torch.from_numpy(_token_mask(Mc[0, 0], 1, 64, N))
    ref = F.scaled_dot_product_attention(torch.from_numpy(Qd)[None], torch.from_numpy(Kd)[None],
                                         torch.from_numpy(V[0, 0])[None], attn_mask=allow)[0].numpy()
    p = O.OracleParams(combine="alpha")
    got = O.forward_given_mask(Q, K, V, Mc, p, alpha=np.ones((1, 1)), qk=fmt)[0, 0]
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-12)
    # and the quantisation is not the identity
    plain = O.forward_given_mask(Q, K, V, Mc, p, alpha=np.ones((1, 1)))[0, 0]
    assert np.abs(got - plain).max() > 1e-4 * np.abs(plain).max()


# ---------------------------------------------------------------- FP8 P V emulation
def _golden_fp8_pv():
    vals = {}
    for line in open(os.path.join(GOLDEN, "fp8_pv_tiny.txt")):
        line = line.split("#")[0].strip()
        if line:
            k, rest = line.split(None, 1)
            vals[k] = np.array([[float(x) for x in r.split()] for r in rest.split("|")])
    return vals


def test_fp8_pv_hand_worked_case():
    g = _golden_fp8_pv()
    V = g["V"]
    np.testing.assert_array_equal(O.pv_fp8_values(V), g["Vhat"])
    np.testing.assert_array_equal(O.pv_fp8_scales(V), [1 / 448, 3 / 448])
    s = g["x"] * math.log(2.0)  # scores in natural-log units
    got = O.sparse_branch_fp8_pv(s, g["Vhat"], O.pv_fp8_scales(V))
    np.testing.assert_allclose(got, g["o"], rtol=1e-13)


def test_fp8_pv_forward_against_n_by_n_brute_force():
    # the whole N x N score matrix, -inf outside the critical blocks; per row
    # M = ceil(max s log2 e), P = 2^(s log2 e - M); E4M3 by torch's float8 cast
    Q, K, V, Mc = _sparse_case(44)
    N, d = Q.shape[2], Q.shape[3]
    allow = _token_mask(Mc[0, 0], 1, 64, N)
    S = np.where(allow, (Q[0, 0] @ K[0, 0].T) / math.sqrt(d), -np.inf)
    x = S * math.log2(math.e)
    M = np.ceil(x.max(axis=1, keepdims=True))
    P = np.where(allow, np.exp2(x - M), 0.0)
    f8 = lambda a: torch.from_numpy(a).to(torch.float8_e4m3fn).double().numpy()  # noqa: E731
    V32 = torch.from_numpy(V[0, 0]).float()
    amax = V32.abs().max(dim=0).values
    Vhat = f8((V32 * (torch.tensor(448.0) / amax)).double().numpy())
    ref = (f8(448.0 * P) @ Vhat) * (amax.double().numpy() / 448.0) / 448.0 / P.sum(axis=1, keepdims=True)
    p = O.OracleParams(combine="alpha")
    got = O.forward_given_mask(Q, K, V, Mc, p, alpha=np.ones((1, 1)), pv_fp8=True)[0, 0]
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-13)


def test_fp8_pv_is_independent_of_token_order_and_whole_power_of_two_shifts():
    rng = np.random.default_rng(45)
    s = rng.standard_normal((8, 300)) * 3.0
    V = rng.standard_normal((300, 16))
    vh, sV = O.pv_fp8_values(V), O.pv_fp8_scales(V)
    base = O.sparse_branch_fp8_pv(s, vh, sV)
    perm = rng.permutation(300)
    np.testing.assert_allclose(O.sparse_branch_fp8_pv(s[:, perm], vh[perm], sV), base, rtol=1e-13, atol=1e-15)
    # adding 3 ln 2 to a row moves M by exactly 3 and leaves every P (and o) unchanged
    np.testing.assert_allclose(O.sparse_branch_fp8_pv(s + 3 * math.log(2.0), vh, sV), base, rtol=1e-13, atol=1e-15)
    # ... while a shift that is not a whole power of two changes the rounding
    assert np.abs(O.sparse_branch_fp8_pv(s + 0.3, vh, sV) - base).max() > 0


def test_fp8_pv_is_exact_when_p_and_v_are_on_the_grid():
    # Q = 0: every score is 0, so M = 0 and P = 1 (E4M3(448) is exact); V in
    # {0, +-1, 2, 4, 8} has per-channel amax 8 and V / s_V in {0, +-56, 112, 224, 448},
    # all E4M3 values.
    rng = np.random.default_rng(11)
    B, H, N, d = 1, 1, 192, 8
    Q = np.zeros((B, H, N, d))
    K = rng.standard_normal((B, H, N, d))
    V = rng.choice([-8.0, -4.0, -2.0, -1.0, 0.0, 1.0, 2.0, 4.0, 8.0], size=(B, H, N, d))
    V[..., 0, :] = 8.0  # every channel reaches 8
    T = O.num_blocks(N, 64)
    Mc = np.full((B, H, T, T), -1, dtype=np.int8)
    Mc[..., 0] = 1
    Mc[..., 1] = 1
    p = O.OracleParams(combine="alpha")
    a = np.ones((B, H))
    exact = O.forward_given_mask(Q, K, V, Mc, p, alpha=a)
    fp8 = O.forward_given_mask(Q, K, V, Mc, p, alpha=a, pv_fp8=True)
    np.testing.assert_allclose(fp8, exact, rtol=0, atol=1e-12)


def test_fp8_pv_without_rounding_is_softmax_attention(monkeypatch):
    # with the quantiser replaced by the identity, the FP8 P V form is plain softmax
    # attention over the critical tokens (up to the fp32 rounding of V * 448 / max|V|)
    rng = np.random.default_rng(12)
    B, H, N, d = 1, 2, 200, 16
    Q, K, V = (rng.standard_normal((B, H, N, d)) for _ in range(3))
    T = O.num_blocks(N, 64)
    Mc = np.zeros((B, H, T, T), dtype=np.int8)
    Mc[..., ::2] = 1
    p = O.OracleParams(combine="alpha")
    a = np.ones((B, H))
    exact = O.forward_given_mask(Q, K, V, Mc, p, alpha=a)
    import oracle.sla as S
    monkeypatch.setattr(S, "quantize_e4m3", lambda x: np.asarray(x, dtype=np.float64))
    ident = S.forward_given_mask(Q, K, V, Mc, p, alpha=a, pv_fp8=True)
    np.testing.assert_allclose(ident, exact, rtol=1e-6, atol=1e-6)
