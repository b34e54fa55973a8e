"""Plain fp64 CPU oracle of the Sparse-Linear Attention forward and backward passes
(SLA and SLA2).

TEST INFRASTRUCTURE ONLY.  This module is the independent checker of the CUDA
path: it shares no code, constants or helpers with the package
``block_sparse_linear_pool_b200`` and must never be imported by it.  Only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import it.  It is slow on purpose: every step is written out in the order the
pages give it, in float64, with numpy primitives (matmul, sort, exp) only.

Sources, cited by page title and section:
  [SLA]  "SLA: Beyond Sparsity in Diffusion Transformers via Fine-Tunable
         Sparse-Linear Attention" (detail page, arXiv 2509.24006): §2 Q2 (the
         algorithm, steps 1-4), §3 Fig. 4 (the forward flowchart), §4 (notation
         table, Eq. 1, Eq. 3-4, Eq. 6, the six checks), §5 Table 2 (phi ablation),
         §7 (code cross-reference: Proj init, linear-over-all-tokens variant,
         smooth-K, exp2 online softmax, LUT-driven loop).
  [SLA2] "SLA2: Sparse-Linear Attention with Learnable Routing and QAT"
         (summary page, arXiv 2602.12675): §3 SLA2 Design (alpha combine),
         §4 Learnable Router (pooling, proj_q/proj_k, row-wise Top-k),
         §5 Quantization-aware Training (low-bit Q/K with scales), App. A
         (backward pass: dH_i, dZ_i accumulated into the marginal blocks).

Readings taken where the pages are silent:
  * the last block may be partial (N not a multiple of b): its pooled mean is
    over its real tokens only and no padding token enters any sum;
  * block counts: n_h = max(1, floor(k_h*T + 1e-9)),
    n_l = min(floor(k_l*T + 1e-9), T - n_h), per row;
  * Top-k / Bottom-k is row-wise ([SLA2] §4), ranking by compressed attention
    weight, descending, ties broken by the lower key-block index first; the
    bottom n_l of that same order are negligible;
  * the 1e-5 epsilon ([SLA] §4 check 5) is added to the linear denominator;
  * Proj follows the nn.Linear convention Proj(x) = x W^T + b and is shared by
    all heads; router projections are bias-free d x d maps shared by all heads;
  * alpha is one scalar per head;
  * the backward treats M_c as a constant (hard Top-k has no gradient) and
    returns gradients for Q, K, V and the combine's parameters only.

  * SoftTop-k ([SLA2] §4, §6) keeps n_h (the hard Top-k's count) per row and
    applies its sigmoid to P_c.

Low-bit emulations ([SLA2] §5): ``lowbit_tile`` (Q, K per 64-row tile, E4M3
or INT8) and ``sparse_branch_fp8_pv`` (E4M3 P and V) are pinned against
torch's float8_e4m3fn cast, hand-worked values and N x N brute force.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

EPS_DEFAULT = 1e-5


# --------------------------------------------------------------------------
# Parameters
# --------------------------------------------------------------------------
@dataclass
class OracleParams:
    """Hyper-parameters of one SLA / SLA2 forward ([SLA] §4 notation table)."""

    b_q: int = 64
    b_kv: int = 64
    k_h: float = 0.05           # critical fraction per row
    k_l: float = 0.10           # negligible fraction per row
    combine: str = "proj"       # "proj" (SLA, [SLA] Eq. 6) or "alpha" (SLA2, [SLA2] §3)
    eps: float = EPS_DEFAULT    # [SLA] §4 check 5
    smooth_k: bool = False      # [SLA] §7 item 3 (code only)
    linear_over_all: bool = False  # [SLA] §7 item 2 (code variant)
    phi: str = "softmax"        # "softmax" ([SLA] Fig. 4) or "elu1" ([SLA] Table 2)


def block_counts(T_kv: int, k_h: float, k_l: float) -> tuple[int, int]:
    """Number of critical (n_h) and negligible (n_l) key blocks per query row.

    [SLA] §2 Q2 step 2 gives the critical and negligible shares as
    percentages; [SLA2] §4 / §6 make the count per row (k% of the N/b_k
    blocks).  Reading: floor, with at least one critical block so that the
    sparse softmax is defined.
    """
    n_h = max(1, int(np.floor(k_h * T_kv + 1e-9)))
    n_l = min(int(np.floor(k_l * T_kv + 1e-9)), T_kv - n_h)
    n_l = max(n_l, 0)
    return n_h, n_l


def num_blocks(N: int, b: int) -> int:
    return -(-N // b)


def block_range(i: int, b: int, N: int) -> tuple[int, int]:
    """Token range [start, stop) of block i; the last block may be partial."""
    return i * b, min((i + 1) * b, N)


# --------------------------------------------------------------------------
# Step 1: compressed attention prediction ([SLA] §2 Q2 step 1, Fig. 4)
# --------------------------------------------------------------------------
def smooth_keys(K: np.ndarray) -> np.ndarray:
    """K minus its mean over tokens ([SLA] §7 item 3: zero-mean K before the mask)."""
    K = np.asarray(K, dtype=np.float64)
    return K - K.mean(axis=-2, keepdims=True)


def mean_pool(X: np.ndarray, b: int) -> np.ndarray:
    """Mean of X over consecutive blocks of b tokens: [..., N, d] -> [..., T, d].

    [SLA] §2 Q2 step 1 and Fig. 4 (mean_pool); [SLA2] §4 (pooling adjacent
    tokens before routing).  A partial last block is averaged over its real
    tokens.
    """
    X = np.asarray(X, dtype=np.float64)
    N = X.shape[-2]
    T = num_blocks(N, b)
    out = np.empty(X.shape[:-2] + (T, X.shape[-1]), dtype=np.float64)
    for i in range(T):
        s, e = block_range(i, b, N)
        out[..., i, :] = X[..., s:e, :].sum(axis=-2) / (e - s)
    return out


def compressed_logits(Q, K, p: OracleParams, Wq=None, Wk=None) -> np.ndarray:
    """pool(Q) . pool(K)^T / sqrt(d), with SLA2's router projections if given.

    [SLA] §2 Q2 step 1 / Fig. 4: P_c = Softmax(pool(Q) pool(K)^T / sqrt(d)).
    [SLA2] §4: proj_q, proj_k (d -> d) transform the pooled Q and K first.
    Returns the pre-softmax logits [..., T_q, T_kv].
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    d = Q.shape[-1]
    if p.smooth_k:
        K = smooth_keys(K)
    Qc = mean_pool(Q, p.b_q)
    Kc = mean_pool(K, p.b_kv)
    if Wq is not None:
        Qc = Qc @ np.asarray(Wq, dtype=np.float64).T
    if Wk is not None:
        Kc = Kc @ np.asarray(Wk, dtype=np.float64).T
    return (Qc @ np.swapaxes(Kc, -1, -2)) / np.sqrt(d)


def compressed_attention(logits: np.ndarray) -> np.ndarray:
    """Row softmax of the compressed logits: P_c ([SLA] Fig. 4)."""
    m = logits.max(axis=-1, keepdims=True)
    e = np.exp(logits - m)
    return e / e.sum(axis=-1, keepdims=True)


def classify(Pc: np.ndarray, n_h: int, n_l: int) -> np.ndarray:
    """Three-way block classification M_c in {1, 0, -1} ([SLA] §2 Q2 step 2).

    Per row ([SLA2] §4: Top-k is taken within each row): order the
    key blocks by P_c descending, ties by lower index first; the first n_h are
    critical (1), the last n_l negligible (-1), the rest marginal (0).
    """
    Pc = np.asarray(Pc, dtype=np.float64)
    T = Pc.shape[-1]
    flat = Pc.reshape(-1, T)
    Mc = np.zeros(flat.shape, dtype=np.int8)
    idx = np.arange(T)
    for r in range(flat.shape[0]):
        order = np.lexsort((idx, -flat[r]))  # primary: -P ascending; secondary: index
        rank = np.empty(T, dtype=np.int64)
        rank[order] = idx
        Mc[r, rank < n_h] = 1
        if n_l > 0:
            Mc[r, rank >= T - n_l] = -1
    return Mc.reshape(Pc.shape)


def soft_topk(Pc: np.ndarray, n_h: int, tau: float, iters: int = 200):
    """SLA2's SoftTop-k, the differentiable stand-in for the router's hard
    row-wise Top-k during training ([SLA2] §4 Learnable Router, §6 Training with
    SLA2: a sigmoid with temperature tau and a per-row threshold lambda_i found
    by binary search so that the row keeps the Top-k row sum).

    M[i, j] = sigmoid((Pc[i, j] - lambda_i) / tau), with lambda_i the root of
    f(lambda) = sum_j sigmoid((Pc[i, j] - lambda) / tau) - n_h.  f falls
    monotonically from T (lambda -> -inf) to 0 (lambda -> +inf), so bisection on
    [min_j Pc - 50 tau, max_j Pc + 50 tau] (where every term is within e^-50 of
    1, respectively 0) finds it; `iters` halvings run it to fp64 resolution.

    Readings: the target row sum is n_h, the hard Top-k's count, so that
    tau -> 0 gives back the hard mask's critical set; the sigmoid acts on P_c,
    the quantity the hard Top-k ranks.  Returns (M, lambda) in float64.
    """
    from scipy.special import expit
    if not tau > 0:
        raise ValueError("tau must be positive")
    Pc = np.asarray(Pc, dtype=np.float64)
    T = Pc.shape[-1]
    flat = Pc.reshape(-1, T)
    M = np.empty_like(flat)
    lam = np.empty(flat.shape[0])
    for r in range(flat.shape[0]):
        row = flat[r]
        lo, hi = row.min() - 50.0 * tau, row.max() + 50.0 * tau
        for _ in range(iters):
            mid = 0.5 * (lo + hi)
            if expit((row - mid) / tau).sum() > n_h:
                lo = mid
            else:
                hi = mid
        lam[r] = 0.5 * (lo + hi)
        M[r] = expit((row - lam[r]) / tau)
    return M.reshape(Pc.shape), lam.reshape(Pc.shape[:-1])


def predict_mask(Q, K, p: OracleParams, Wq=None, Wk=None):
    """Compressed mask prediction, Fig. 4 left: returns (M_c, logits, P_c)."""
    logits = compressed_logits(Q, K, p, Wq, Wk)
    Pc = compressed_attention(logits)
    T_kv = logits.shape[-1]
    n_h, n_l = block_counts(T_kv, p.k_h, p.k_l)
    return classify(Pc, n_h, n_l), logits, Pc


def critical_lut(Mc: np.ndarray) -> np.ndarray:
    """Per query block, the critical key-block indices in ascending order
    ([SLA] §7 item 5: the kernel walks a per-row list of critical blocks)."""
    n_h = int((Mc[(0,) * (Mc.ndim - 1)] == 1).sum())
    out = np.zeros(Mc.shape[:-1] + (n_h,), dtype=np.int32)
    flat_m = Mc.reshape(-1, Mc.shape[-1])
    flat_o = out.reshape(-1, n_h)
    for r in range(flat_m.shape[0]):
        flat_o[r] = np.nonzero(flat_m[r] == 1)[0]
    return out


# --------------------------------------------------------------------------
# Step 3 ingredients: feature map and per-block linear statistics
# --------------------------------------------------------------------------
def feature_map(X: np.ndarray, kind: str = "softmax") -> np.ndarray:
    """phi applied per token over the head dimension.

    "softmax" is the map of [SLA] Fig. 4 (a softmax feature map); "elu1" is
    elu(x) + 1, the ablation of [SLA] Table 2.
    """
    X = np.asarray(X, dtype=np.float64)
    if kind == "softmax":
        m = X.max(axis=-1, keepdims=True)
        e = np.exp(X - m)
        return e / e.sum(axis=-1, keepdims=True)
    if kind == "elu1":
        return np.where(X > 0, X + 1.0, np.exp(np.minimum(X, 0.0)))
    raise ValueError(kind)


def linear_block_stats(K, V, b_kv: int, phi: str = "softmax"):
    """h_j = phi(K_j)^T V_j  (d x d) and z_j = rowsum(phi(K_j)^T) (d).

    [SLA] §2 Q2 step 3 and Fig. 4 ("h_j = phi(K_j)^T V_j, z_j =
    rowsum(phi(K_j)^T)").  Only the real tokens of a partial block count.
    Returns h [..., T, d, d] (index [j, a, b]) and z [..., T, d].
    """
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    N, d = K.shape[-2], K.shape[-1]
    T = num_blocks(N, b_kv)
    fK = feature_map(K, phi)
    h = np.empty(K.shape[:-2] + (T, d, V.shape[-1]), dtype=np.float64)
    z = np.empty(K.shape[:-2] + (T, d), dtype=np.float64)
    for j in range(T):
        s, e = block_range(j, b_kv, N)
        h[..., j, :, :] = np.swapaxes(fK[..., s:e, :], -1, -2) @ V[..., s:e, :]
        z[..., j, :] = fK[..., s:e, :].sum(axis=-2)
    return h, z


# --------------------------------------------------------------------------
# Steps 3-4: the per-query-block computation and the combination
# --------------------------------------------------------------------------
def quantize_e4m3(x: np.ndarray) -> np.ndarray:
    """Round to the nearest FP8 E4M3 value (ties to even), saturating at 448.

    Written from the OCP 8-bit floating point specification: 1 sign bit,
    4 exponent bits (bias 7), 3 mantissa bits; normal numbers 2^-6 .. 448,
    subnormals m * 2^-9.  Used by the low-bit path of [SLA2] §5.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), 448.0)
    # exponent of the quantisation step: 2^(e-3) for a in [2^e, 2^(e+1)), e >= -6
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -6.0)
    step = np.exp2(e - 3.0)
    q = np.round(a / step) * step  # np.round is round-half-to-even
    q = np.minimum(q, 448.0)
    return np.sign(x) * q


def quantize_int8(y: np.ndarray) -> np.ndarray:
    """Round to the nearest integer (ties to even) and clamp to [-127, 127]: the
    symmetric INT8 code of a value already divided by its scale ([SLA2] §5 names
    INT8 beside FP8 as the low-bit format)."""
    return np.clip(np.round(np.asarray(y, dtype=np.float64)), -127.0, 127.0)


LOWBIT_MAX = {"fp8_e4m3": 448.0, "int8": 127.0}


def lowbit_tile(X: np.ndarray, fmt: str) -> np.ndarray:
    """Quantise one 64-row tile of Q or K with one scale per tile and return the
    dequantised values ([SLA2] §5: Q and K are mapped to a low-bit format with
    scales before Q K^T, and the product is rescaled).

    The scale is s = max|X| / R with R = 448 (the largest finite E4M3 value) or
    127 (symmetric INT8).  The code of each element is an integer decision, so it
    is taken on the fp32 value X * (R / max|X|) (both factors and the product
    rounded to fp32), which is the precision a GPU kernel takes it in; the
    dequantised value is code * s."""
    R = np.float32(LOWBIT_MAX[fmt])
    X32 = np.asarray(X, dtype=np.float32)
    amax = np.float32(np.abs(X32).max()) if X32.size else np.float32(0)
    if amax == 0:
        return np.zeros(X32.shape, dtype=np.float64)
    inv = R / amax                       # fp32 division
    y = (X32 * inv).astype(np.float64)   # fp32 product, exact in fp64
    code = quantize_e4m3(y) if fmt == "fp8_e4m3" else quantize_int8(y)
    return code * np.float64(amax / R)


def pv_fp8_scales(Vh: np.ndarray) -> np.ndarray:
    """Per-channel scale of one head's V for the FP8 P V product: max_t |V[t, c]| / 448
    (1 where a channel is all zero).  [SLA2] §5 quantises P and V with scales and
    dequantises their product; with one scale per channel both scales factor out of
    the sum over keys."""
    amax = np.abs(np.asarray(Vh, dtype=np.float32)).max(axis=0)
    return np.where(amax > 0, amax.astype(np.float64) / 448.0, 1.0)


def pv_fp8_values(Vh: np.ndarray) -> np.ndarray:
    """E4M3 codes of one head's V on its per-channel scale, V / s_V, the division
    taken as the fp32 product V * (448 / max|V[:, c]|) (an integer decision in
    the kernel's precision)."""
    V32 = np.asarray(Vh, dtype=np.float32)
    amax = np.abs(V32).max(axis=0)
    inv = np.where(amax > 0, np.float32(448.0) / np.where(amax > 0, amax, np.float32(1)), np.float32(0))
    return quantize_e4m3((V32 * inv.astype(np.float32)).astype(np.float64))


LOG2E = 1.4426950408889634


def sparse_branch_fp8_pv(s: np.ndarray, vhat: np.ndarray, sV: np.ndarray) -> np.ndarray:
    """o^s of a set of query rows with the FP8 P V product ([SLA2] §5: P and V are
    quantised with scales and their product is dequantised).

    s: the rows' scaled scores over their critical tokens [rows, C]; vhat: the
    E4M3 codes of those tokens' V on the per-channel scale sV [C, d].
    Per row, P is taken against the row's maximum score rounded up to a whole
    power of two: with x = s log2(e) and M = ceil(max x), P = 2^(x - M), so
    1/2 < max P <= 1 and the row's P scale is an exact power of two.  P is
    quantised as E4M3(448 P), the product with V^ is dequantised by sV / 448,
    and the row sum uses the unquantised P:
        o^s = (E4M3(448 P) V^) sV / 448 / sum(P).
    The result depends only on the set of critical tokens, not on the order in
    which a kernel visits them."""
    x = np.asarray(s, dtype=np.float64) * LOG2E
    M = np.ceil(x.max(axis=1, keepdims=True))
    P = np.exp2(x - M)
    acc = quantize_e4m3(448.0 * P) @ np.asarray(vhat, dtype=np.float64)
    return acc * np.asarray(sV, dtype=np.float64)[None, :] / 448.0 / P.sum(axis=1, keepdims=True)


def forward_given_mask(Q, K, V, Mc, p: OracleParams, proj_w=None, proj_b=None, alpha=None,
                       qblocks: Optional[Sequence[int]] = None, heads: Optional[Sequence] = None,
                       qk: str = "bf16", return_branches: bool = False, pv_fp8: bool = False):
    """SLA / SLA2 output for a given compressed mask M_c.

    Q, K, V: [B, H, N, d] (any float dtype; upcast to float64).
    Mc: int8 [B, H, T_q, T_kv].
    For each query block i ([SLA] §2 Q2 step 3, Fig. 4 "Fused kernel"):
      * critical blocks (M_c = 1): exact softmax attention over their tokens,
        O^s = diag(l)^-1 O^s_acc  (two-pass softmax: max, then exp / sum);
      * marginal blocks (M_c = 0): H_i = sum h_j, Z_i = sum z_j and
        O^l = phi(Q_i) H_i / (phi(Q_i) Z_i + eps)  ([SLA] Eq. 3-4, §4 check 5);
      * negligible blocks (M_c = -1) contribute nothing.
    Combination ([SLA] Eq. 6 / [SLA2] §3):
      "proj":  O = O^s + O^l W^T + b
      "alpha": O = alpha_h O^s + (1 - alpha_h) O^l
    `qblocks` / `heads` restrict the work to a sample (rows of other blocks are
    left as NaN).  `qk` = "fp8_e4m3" or "int8" quantises Q and K per 64-row
    tile (``lowbit_tile``) before Q K^T ([SLA2] §5); `pv_fp8` computes the sparse
    branch's P V with E4M3 P and V (``sparse_branch_fp8_pv``); both emulate the
    low-bit path.
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    B, H, N, d = Q.shape
    dv = V.shape[-1]
    T_q = num_blocks(N, p.b_q)
    T_kv = num_blocks(N, p.b_kv)
    assert Mc.shape == (B, H, T_q, T_kv), Mc.shape
    scale = 1.0 / np.sqrt(d)
    O = np.full((B, H, N, dv), np.nan)
    Os = np.full((B, H, N, dv), np.nan)
    Ol = np.full((B, H, N, dv), np.nan)
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(H)]
    qsel = range(T_q) if qblocks is None else qblocks
    W = None if proj_w is None else np.asarray(proj_w, dtype=np.float64)
    bias = None if proj_b is None else np.asarray(proj_b, dtype=np.float64)

    for (bb, hh) in heads:
        h_stats, z_stats = linear_block_stats(K[bb, hh], V[bb, hh], p.b_kv, p.phi)
        fQ = feature_map(Q[bb, hh], p.phi)
        if pv_fp8:
            sV = pv_fp8_scales(V[bb, hh])
            Vhat = pv_fp8_values(V[bb, hh])
        if qk not in ("bf16", "fp8_e4m3", "int8"):
            raise ValueError(qk)
        for i in qsel:
            qs, qe = block_range(i, p.b_q, N)
            q = Q[bb, hh, qs:qe]
            row = Mc[bb, hh, i]
            # --- sparse branch over critical blocks
            crit = np.nonzero(row == 1)[0]
            if qk != "bf16":
                q = lowbit_tile(q, qk)
            keys, vals, vhat = [], [], []
            for j in crit:
                ks, ke = block_range(int(j), p.b_kv, N)
                kj = K[bb, hh, ks:ke]
                if qk != "bf16":
                    kj = lowbit_tile(kj, qk)
                keys.append(kj)
                vals.append(V[bb, hh, ks:ke])
                if pv_fp8:
                    vhat.append(Vhat[ks:ke])
            if keys:
                kk = np.concatenate(keys, axis=0)
                s = (q @ kk.T) * scale
            if keys and pv_fp8:
                o_s = sparse_branch_fp8_pv(s, np.concatenate(vhat, axis=0), sV)
            elif keys:
                vv = np.concatenate(vals, axis=0)
                m = s.max(axis=1, keepdims=True)
                e = np.exp(s - m)
                o_s = (e @ vv) / e.sum(axis=1, keepdims=True)
            else:
                o_s = np.zeros((qe - qs, dv))
            # --- linear branch over marginal blocks
            marg = np.arange(T_kv) if p.linear_over_all else np.nonzero(row == 0)[0]
            Hi = h_stats[marg].sum(axis=0) if len(marg) else np.zeros((d, dv))
            Zi = z_stats[marg].sum(axis=0) if len(marg) else np.zeros(d)
            fq = fQ[qs:qe]
            o_l = (fq @ Hi) / ((fq @ Zi) + p.eps)[:, None]
            # --- combine
            if p.combine == "proj":
                proj = o_l @ W.T if W is not None else np.zeros_like(o_l)
                if bias is not None:
                    proj = proj + bias
                o = o_s + proj
            elif p.combine == "alpha":
                a = float(np.asarray(alpha, dtype=np.float64).reshape(B, H)[bb, hh]) \
                    if np.ndim(alpha) else float(alpha)
                o = a * o_s + (1.0 - a) * o_l
            else:
                raise ValueError(p.combine)
            O[bb, hh, qs:qe] = o
            Os[bb, hh, qs:qe] = o_s
            Ol[bb, hh, qs:qe] = o_l
    if return_branches:
        return O, Os, Ol
    return O


def forward(Q, K, V, p: OracleParams, proj_w=None, proj_b=None, alpha=None, Wq=None, Wk=None,
            **kw):
    """Full SLA / SLA2 forward: predict M_c, then the fused computation.

    Returns (O, M_c)."""
    Mc, _, _ = predict_mask(Q, K, p, Wq, Wk)
    return forward_given_mask(Q, K, V, Mc, p, proj_w, proj_b, alpha, **kw), Mc


def mask_grading(logits: np.ndarray, n_h: int, n_l: int, gap: float = 1e-4) -> np.ndarray:
    """Which mask entries are decided by more than `gap` on the logit scale.

    An entry is graded when its logit lies farther than `gap` from both the
    top-k threshold (midpoint of the n_h-th and (n_h+1)-th largest) and the
    bottom-k threshold (midpoint of the n_l-th and (n_l+1)-th smallest).
    Returns a boolean array shaped like `logits`.
    """
    L = np.asarray(logits, dtype=np.float64)
    T = L.shape[-1]
    srt = -np.sort(-L, axis=-1)  # descending
    big = np.inf
    t_hi = 0.5 * (srt[..., n_h - 1] + srt[..., n_h]) if n_h < T else np.full(L.shape[:-1], -big)
    if n_l > 0:
        t_lo = 0.5 * (srt[..., T - n_l - 1] + srt[..., T - n_l])
    else:
        t_lo = np.full(L.shape[:-1], big)
    dh = np.abs(L - t_hi[..., None])
    dl = np.abs(L - t_lo[..., None])
    return (dh > gap) & (dl > gap)


# --------------------------------------------------------------------------
# Backward pass given the mask ([SLA] §4 check 6; [SLA2] App. A)
# --------------------------------------------------------------------------
def feature_map_backward(X: np.ndarray, fX: np.ndarray, dF: np.ndarray, kind: str = "softmax"):
    """Gradient through phi, per token over the head dimension.

    softmax: d x = phi * (d phi - <phi, d phi>);  elu + 1: d x = d phi * (1 if x > 0 else e^x).
    """
    X = np.asarray(X, dtype=np.float64)
    if kind == "softmax":
        return fX * (dF - (fX * dF).sum(axis=-1, keepdims=True))
    if kind == "elu1":
        return dF * np.where(X > 0, 1.0, np.exp(np.minimum(X, 0.0)))
    raise ValueError(kind)


def backward_given_mask(Q, K, V, Mc, dO, p: OracleParams, proj_w=None, proj_b=None, alpha=None):
    """Gradients of L = sum(O * dO) for the forward of ``forward_given_mask``.

    The mask M_c is a constant of the backward (hard Top-k / Bottom-k has no
    gradient; SLA2 trains its router through a soft Top-k that is not part of
    this path).  Both pages describe the same split ([SLA] §4 check 6,
    [SLA2] App. A): the sparse branch takes the FlashAttention backward over
    the critical blocks, and the linear branch forms dH_i, dZ_i per query block,
    accumulates them into every marginal key block's dh_j, dz_j (the mirror of
    the forward's H_i = sum h_j), and goes back through h_j = phi(K_j)^T V_j,
    z_j = colsum phi(K_j) and through phi.

    With o_s = P V (P the row softmax over critical keys), o_l = num / den,
    num = phi(q) H_i, den = phi(q) . Z_i + eps, and the combine's
      proj:  O = o_s + o_l W^T + b    ->  do_s = dO, do_l = dO W, dW = dO^T o_l, db = sum dO
      alpha: O = a o_s + (1 - a) o_l  ->  do_s = a dO, do_l = (1 - a) dO,
                                          da = sum (o_s - o_l) . dO
    sparse:  dP = do_s V^T, D = rowsum(do_s * o_s), dS = P (dP - D),
             dq = dS K / sqrt(d), dk = dS^T q / sqrt(d), dv = P^T do_s
    linear:  g = do_l / den, gden = -(do_l . o_l) / den,
             d phi(q) = g H_i^T + gden Z_i,  dH_i = phi(q)^T g,  dZ_i = gden^T phi(q),
             dh_j = sum over query blocks with j marginal of dH_i (dz_j likewise),
             d phi(k_t) = dh_j v_t + dz_j,  dv_t += dh_j^T phi(k_t)   (t in block j)
    Returns a dict with dQ, dK, dV [B,H,N,d], dproj_w [d,d], dproj_b [d] and
    dalpha [B,H] (zeros for the combine that does not use them).
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    dO = np.asarray(dO, dtype=np.float64)
    B, H, N, d = Q.shape
    dv_dim = V.shape[-1]
    T_q = num_blocks(N, p.b_q)
    T_kv = num_blocks(N, p.b_kv)
    assert Mc.shape == (B, H, T_q, T_kv), Mc.shape
    scale = 1.0 / np.sqrt(d)
    W = None if proj_w is None else np.asarray(proj_w, dtype=np.float64)
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    dW = np.zeros((dv_dim, dv_dim))
    db = np.zeros(dv_dim)
    dalpha = np.zeros((B, H))
    for bb in range(B):
        for hh in range(H):
            q, k, v, do = Q[bb, hh], K[bb, hh], V[bb, hh], dO[bb, hh]
            h_stats, z_stats = linear_block_stats(k, v, p.b_kv, p.phi)
            fQ = feature_map(q, p.phi)
            fK = feature_map(k, p.phi)
            dfQ = np.zeros_like(q)
            dfK = np.zeros_like(k)
            dh = np.zeros_like(h_stats)
            dz = np.zeros_like(z_stats)
            for i in range(T_q):
                qs, qe = block_range(i, p.b_q, N)
                qi, doi = q[qs:qe], do[qs:qe]
                row = Mc[bb, hh, i]
                # forward quantities of this block
                crit = np.nonzero(row == 1)[0]
                idx = np.concatenate([np.arange(*block_range(int(j), p.b_kv, N)) for j in crit])
                s = (qi @ k[idx].T) * scale
                e = np.exp(s - s.max(axis=1, keepdims=True))
                P = e / e.sum(axis=1, keepdims=True)
                o_s = P @ v[idx]
                marg = np.arange(T_kv) if p.linear_over_all else np.nonzero(row == 0)[0]
                Hi = h_stats[marg].sum(axis=0) if len(marg) else np.zeros((d, dv_dim))
                Zi = z_stats[marg].sum(axis=0) if len(marg) else np.zeros(d)
                fq = fQ[qs:qe]
                den = fq @ Zi + p.eps
                o_l = (fq @ Hi) / den[:, None]
                # the combine
                if p.combine == "proj":
                    do_s = doi
                    do_l = doi @ W if W is not None else np.zeros_like(doi)
                    dW += doi.T @ o_l
                    db += doi.sum(axis=0)
                elif p.combine == "alpha":
                    a = float(np.asarray(alpha, dtype=np.float64).reshape(B, H)[bb, hh]) \
                        if np.ndim(alpha) else float(alpha)
                    do_s = a * doi
                    do_l = (1.0 - a) * doi
                    dalpha[bb, hh] += ((o_s - o_l) * doi).sum()
                else:
                    raise ValueError(p.combine)
                # sparse branch: FlashAttention backward over the critical tokens
                dP = do_s @ v[idx].T
                Drow = (do_s * o_s).sum(axis=1, keepdims=True)
                dS = P * (dP - Drow)
                dQ[bb, hh, qs:qe] += (dS @ k[idx]) * scale
                dK[bb, hh, idx] += (dS.T @ qi) * scale
                dV[bb, hh, idx] += P.T @ do_s
                # linear branch
                g = do_l / den[:, None]
                gden = -(do_l * o_l).sum(axis=1) / den
                dfQ[qs:qe] += g @ Hi.T + gden[:, None] * Zi[None, :]
                dHi = fq.T @ g
                dZi = (gden[:, None] * fq).sum(axis=0)
                for j in marg:
                    dh[j] += dHi
                    dz[j] += dZi
            for j in range(T_kv):
                ks, ke = block_range(j, p.b_kv, N)
                dfK[ks:ke] += v[ks:ke] @ dh[j].T + dz[j][None, :]
                dV[bb, hh, ks:ke] += fK[ks:ke] @ dh[j]
            dQ[bb, hh] += feature_map_backward(q, fQ, dfQ, p.phi)
            dK[bb, hh] += feature_map_backward(k, fK, dfK, p.phi)
    return {"dQ": dQ, "dK": dK, "dV": dV, "dproj_w": dW, "dproj_b": db, "dalpha": dalpha}
