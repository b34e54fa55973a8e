"""Host-side accounting of bench.py, checked on the CPU: the work model behind the
headline number (algorithmic FLOPs of a step, the fused kernel's issued FLOPs on
the union of each tile's two critical lists), the roofline arithmetic, and the
rule that a DRAM-traffic figure is reported only for the kernel source it was
measured on."""
import hashlib
import os
import sys
from types import SimpleNamespace

import numpy as np
import pytest

sys.path.insert(0, os.path.join(os.path.dirname(os.path.abspath(__file__)), ".."))
import bench  # noqa: E402


def _dims(BH, N, d, Tq, Tkv, nh, nl):
    return dict(BH=BH, N=N, d=d, Tq=Tq, Tkv=Tkv, nh=nh, nl=nl)


def test_work_model_union_and_counts():
    # two heads, four query blocks, two critical key blocks per query block
    d, N, Tq, Tkv, nh, nl, BH = 64, 256, 4, 4, 2, 1, 2
    lut = np.array([[[0, 1], [1, 2], [3, 0], [3, 2]],
                    [[0, 1], [0, 1], [2, 3], [1, 0]]], dtype=np.int32)
    pairs = np.array([[[0, 1], [2, 3]], [[0, 2], [1, 3]]], dtype=np.int32)
    w = bench.work_model(SimpleNamespace(combine="proj"), _dims(BH, N, d, Tq, Tkv, nh, nl), lut, pairs)
    # unions, counted by hand: head 0 {0,1,2}, {0,2,3}; head 1 {0,1,2,3}, {0,1}
    assert w["union_total"] == 3 + 3 + 4 + 2
    assert w["n_tiles"] == 4
    assert w["critical_entries"] == Tq * nh * BH == 16
    # one critical (query block, key block) pair is Q K^T + P V over 64 x 64 x d
    per_pair = 2 * (2 * 64 * 64 * d)
    assert w["fused_pairs_alg"] == 16 * per_pair
    assert w["fused_alg"] == 16 * per_pair + BH * N * 2 * d * d
    # a tile issues both MMAs at M = 128 for every union entry, plus the two
    # linear-branch chains (M = 128, N = d, K = d)
    assert w["fused_issued"] == 12 * 2 * (2 * 128 * 64 * d) + 4 * 2 * (2 * 128 * d * d)
    # SLA: h_j and the folded Proj product, 2 d^2 each per key token
    assert w["kv_alg"] == 2 * (2 * N * d * d * BH)
    # one marginal block per query block (T_kv - n_h - n_l), one add per element of [h|z]
    assert w["marg_alg"] == Tq * 1 * (d * d + d) * BH
    assert w["logits"] == 2 * Tq * Tkv * d * BH
    assert w["step_alg"] == w["fused_alg"] + w["kv_alg"] + w["marg_alg"] + w["logits"]
    assert w["dense_equiv"] == 4 * N * N * d * BH
    # SLA2 (alpha combine): no Proj product, the router's two d x d maps per pooled row
    w2 = bench.work_model(SimpleNamespace(combine="alpha"), _dims(BH, N, d, Tq, Tkv, nh, nl), lut, pairs)
    assert w2["kv_alg"] == 2 * N * d * d * BH
    assert w2["logits"] == 2 * Tq * Tkv * d * BH + 4 * Tq * d * d * BH


def test_work_model_adjacent_pairs_and_odd_tail():
    # without a pairs buffer the tiles are (0, 1), (2, 3), (4, -1): the last block alone
    d, N, Tq, Tkv, nh, nl, BH = 64, 320, 5, 5, 1, 1, 1
    lut = np.array([[[0], [1], [1], [4], [2]]], dtype=np.int32)
    w = bench.work_model(SimpleNamespace(combine="proj"), _dims(BH, N, d, Tq, Tkv, nh, nl), lut)
    assert w["n_tiles"] == 3
    assert w["union_total"] == 2 + 2 + 1


def test_rooflines_fractions():
    wk = {"fused_alg": 2.0e12, "fused_pairs_alg": 1.6e12, "fused_issued": 3.0e12,
          "bytes": {"predict_mask": 2.0e8, "precompute_linear": 4.0e8, "aggregate_marginal": 8.0e8}}
    rec = {"work": wk, "qk": "bf16", "pv": "bf16",
           "stage_ms": {"fused_kernel": 2.0, "predict_mask": 0.1, "precompute_linear": 0.1,
                        "aggregate_marginal": 0.2}}
    peaks = {"bf16_tflops": 1600.0, "hbm_gbs": 6400.0}
    r = bench.rooflines(rec, peaks, "measured")
    assert r["fused_kernel"]["achieved"] == pytest.approx(1000.0)
    assert r["fused_kernel"]["peak"] == pytest.approx(1600.0)
    assert r["fused_kernel"]["frac"] == pytest.approx(0.625)
    assert r["fused_kernel"]["issued_frac"] == pytest.approx(1500.0 / 1600.0, abs=1e-4)
    assert r["predict_mask"]["achieved"] == pytest.approx(2000.0)
    assert r["aggregate_marginal"]["frac"] == pytest.approx(4000.0 / 6400.0)
    # an 8-bit Q K^T doubles the rate of half the pair FLOPs: peak = the harmonic mix
    rec8 = dict(rec, qk="fp8_e4m3")
    r8 = bench.rooflines(rec8, peaks, "measured")
    t_unit = 0.8e12 / 2 + 0.8e12 + 0.4e12
    assert r8["fused_kernel"]["peak"] == pytest.approx(round(1600.0 * 2.0e12 / t_unit, 1))


def test_traffic_figure_only_for_the_profiled_source(tmp_path, monkeypatch):
    src_dir = tmp_path / "block_sparse_linear_pool_b200" / "csrc"
    src_dir.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    src = src_dir / "fused_pt.cu"
    src.write_bytes(b"// kernel source as profiled\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (tmp_path / "profiles" / "fused_pt_wl_traffic.txt").write_text(
        "# comment = ignored\nkernel_source = fused_pt.cu\n"
        f"source_sha256_16 = {sha}\ndram_bytes_per_launch = 123456\nheads = 12\nqk = bf16\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.delenv("SLA_FUSED_SCHEDULE", raising=False)
    assert bench.fused_traffic_per_launch("wl", 12, "bf16") == 123456.0
    assert bench.fused_traffic_per_launch("wl", 6, "bf16") is None       # other head count
    assert bench.fused_traffic_per_launch("wl", 12, "int8") is None      # other Q K^T type
    assert bench.fused_traffic_per_launch("other", 12, "bf16") is None   # no summary
    src.write_bytes(b"// kernel source changed since\n")
    assert bench.fused_traffic_per_launch("wl", 12, "bf16") is None
