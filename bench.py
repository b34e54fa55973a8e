#!/usr/bin/env python
"""Benchmark of the SLA / SLA2 forward on B200.

One step = one pass of the whole forward over one synthetic batch: compressed
mask prediction (pool, router, row-wise selection), per-block linear
statistics, marginal aggregation and the fused sparse + linear kernel.  Inputs
are resident in HBM when the timed region starts.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun, one process per GPU): every rank runs its own independent
problem of the same shape (the forward has no cross-head or cross-batch
exchange), so per-GPU work is fixed and `scaling` is "weak"; the time is the
max over ranks of CUDA-event time, and `value` counts the FLOPs of all ranks.

`--impl reference` times the fp64 CPU oracle instead, on a bounded sample of
the same workload (rank 0 only).  Prints ONE JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_linear_pool_b200 import binding as bnd  # noqa: E402
from block_sparse_linear_pool_b200 import inputs as I  # noqa: E402

METRIC = "SLA forward ms and executed TFLOPS (% tensor peak) at N=32760,d=128, 95-97% sparse"
UNIT = "TFLOP/s"
WORKLOAD = "wan1.3b_sla"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# --------------------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled in the background."""

    FIELDS = ("index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str | None):
        self.bus_id = bus_id
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 10:
                    continue
                if self.bus_id and self.bus_id.lower() not in parts[1].lower():
                    continue
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i].lower() == "active"})
        loaded = [x for x in sm if x > 0.5 * max(sm)] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": float(rows[0][3]) if rows[0][3].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(float(r[4]) for r in rows if r[4].replace(".", "").isdigit())}


def bus_id_of(dev):
    try:
        pr = torch.cuda.get_device_properties(dev)
        return f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}"
    except Exception:
        return None


def split_schedule() -> bool:
    return os.environ.get("SLA_FUSED_SCHEDULE", "") == "split"


def fused_kernel_name(qk: str, pv: str) -> str:
    """The fused kernel the library runs for these precisions (the persistent
    kernel for bf16, the one-tile-per-CTA kernel for the 8-bit products, the
    split-union kernel when that schedule is selected)."""
    if qk != "bf16" or pv != "bf16":
        return "sla_fused_kernel"
    return "sla_fused_sk_kernel" if split_schedule() else "sla_fused_pt_kernel"


def fused_traffic_per_launch(workload: str, heads: int, qk: str):
    """DRAM bytes per launch of the persistent fused kernel from the committed ncu
    summary, or None if the summary is for another workload or the kernel source
    changed since those counters were taken."""
    path = os.path.join(ROOT, "profiles", f"fused_pt_{workload}_traffic.txt")
    src = os.path.join(ROOT, "block_sparse_linear_pool_b200", "csrc", "fused_pt.cu")
    if not os.path.exists(path) or split_schedule():
        return None
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    vals = {}
    for line in open(path):
        if "=" in line and not line.startswith("#"):
            k, v = line.split("=", 1)
            vals[k.strip()] = v.strip()
    if vals.get("source_sha256_16") != sha:
        return None
    if vals.get("heads") != str(heads) or vals.get("qk", "bf16") != qk:
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except Exception:
        return None


# --------------------------------------------------------------------------- work accounting
def work_model(cfg, dims, lut_np, pairs_np=None):
    """Algorithmic and issued work of one step.

    Algorithmic FLOPs (what the method needs, counted once):
      fused     Q K^T + P V over the critical pairs, 4*64*64*d each, plus
                phi(Q) H (2 d^2 per query row) and, for the SLA combine, the Proj
                product (2 d^2 per row; folded into h_j here, executed by kv_prep);
      kv_prep   h_j = phi(K_j)^T V_j, 2 d^2 per key token;
      marginal  one add per (query block, marginal key block, element of [h|z]);
      logits    pooled Q_c K_c^T, 2 d per (query block, key block), plus the
                router's two d x d maps per pooled row (SLA2).
    Issued FLOPs add what the kernels execute beyond that: the fused kernel's
    masked halves (a tile walks the union of its two blocks' critical lists:
    U entries per tile, counted on the pairs the kernel used) and the dense
    0/1 aggregation GEMM (128 x 256 tiles, K padded to 64)."""
    BH, N, d, Tq, Tkv, nh, nl = (dims[k] for k in ("BH", "N", "d", "Tq", "Tkv", "nh", "nl"))
    NN = d * d + d
    lut = lut_np.reshape(BH, Tq, nh)
    if pairs_np is None:  # adjacent pairs
        pairs_np = np.stack([np.arange(0, Tq, 2), np.where(np.arange(1, Tq + 1, 2) < Tq,
                                                           np.arange(1, Tq + 1, 2), -1)], axis=1)
        pairs_np = np.broadcast_to(pairs_np, (BH,) + pairs_np.shape)
    U = 0
    for bh in range(BH):
        for a, b in pairs_np[bh].tolist():
            s = set(lut[bh, a].tolist())
            if b >= 0:
                s |= set(lut[bh, b].tolist())
            U += len(s)
    n_cta = int(pairs_np.shape[0] * pairs_np.shape[1])
    proj = cfg.combine == "proj"
    fused_pairs = 4 * 64 * 64 * d * Tq * nh * BH
    fused_alg = fused_pairs + 2 * N * d * d * BH
    fused_issued = U * 2 * (2 * 128 * 64 * d) + n_cta * 2 * (2 * 128 * d * d)
    kv_alg = 2 * N * d * d * BH + (2 * N * d * d * BH if proj else 0)
    n_m = Tkv - nh - nl
    marg_alg = Tq * n_m * NN * BH
    marg_issued = 2 * (math.ceil(Tq / 128) * 128) * (math.ceil(NN / 256) * 256) * (math.ceil(Tkv / 64) * 64) * BH
    logits = 2 * Tq * Tkv * d * BH + (4 * Tq * d * d * BH if cfg.combine == "alpha" else 0)
    step_alg = fused_alg + kv_alg + marg_alg + logits
    act = BH * N * d * 2  # one bf16 [B, H, N, d] tensor
    hz_bytes = BH * Tkv * NN * 2
    return {"fused_alg": fused_alg, "fused_pairs_alg": fused_pairs, "fused_issued": fused_issued,
            "kv_alg": kv_alg, "marg_alg": marg_alg, "marg_issued": marg_issued, "logits": logits,
            "step_alg": step_alg, "step_issued": fused_issued + kv_alg + marg_issued + logits,
            "union_total": U, "n_tiles": n_cta, "critical_entries": Tq * nh * BH,
            "dense_equiv": 4 * N * N * d * BH,
            # algorithmic HBM bytes of the bandwidth-bound stages
            "bytes": {"predict_mask": 2 * act, "precompute_linear": 2 * act + hz_bytes,
                      "aggregate_marginal": 2 * hz_bytes}}


# --------------------------------------------------------------------------- our arm
def reduce_over_ranks(ms_total: float, flops_per_step: float, device):
    """Whole-job figures of a data-parallel run: the slowest rank's timed-region
    duration (max over ranks) and the algorithmic FLOPs of one step summed over
    the ranks' independent problems.  Every rank must call this, in the same order."""
    t_ms = torch.tensor([ms_total], dtype=torch.float64, device=device)
    t_fl = torch.tensor([flops_per_step], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t_ms, op=torch.distributed.ReduceOp.MAX)
    torch.distributed.all_reduce(t_fl, op=torch.distributed.ReduceOp.SUM)
    return float(t_ms.item()), float(t_fl.item())


STAGES = ["predict_mask", "precompute_linear", "aggregate_marginal", "pair_query_blocks", "fused_kernel"]


def measure(workload, qk, pv, steps, warmup, dev, rank=0, world=1, heads=None, burn=0.0, sampler=None,
            keep=False):
    """Times `steps` steps of one workload on this rank's GPU.  Returns a record
    (ms per step, stage ms, work, fused roofline) and, with keep, the inputs."""
    torch.cuda.set_device(dev)
    over = {} if heads is None else {"H": heads}
    data, w = I.make_workload(workload, device=f"cuda:{dev}", problem=rank, **over)
    cfg = bnd.SlaConfig(k_h=w["k_h"], k_l=w["k_l"], combine=w["combine"], qk=qk, pv=pv)
    Q, K, V = (data[k].to(dev) for k in ("Q", "K", "V"))
    O = torch.empty_like(Q)
    f32 = lambda t: None if t is None else t.to(dev).float().contiguous()  # noqa: E731
    proj_w, proj_b = f32(data.get("proj_w")), f32(data.get("proj_b"))
    alpha, Wq, Wk = f32(data.get("alpha")), f32(data.get("Wq")), f32(data.get("Wk"))
    L = bnd.lib()
    p = bnd.make_params(Q, cfg, K, V, O)
    Tq, Tkv, nh, nl = bnd.sla_block_counts(p)
    B, H, N, d = Q.shape
    BH = B * H
    ws = bnd.new_workspace(bnd.sla_workspace_size(p), dev)
    mc = torch.empty((BH, Tq, Tkv), dtype=torch.int8, device=dev)
    lut = torch.empty((BH, Tq, nh), dtype=torch.int32, device=dev)
    hz = torch.empty((BH, Tkv, d * d + d), dtype=torch.bfloat16, device=dev)
    P = bnd._ptr
    pw = proj_w if cfg.combine == "proj" else None
    st = bnd._stream
    wsz = ws.numel()
    pp = bnd.ctypes.byref(p)
    calls = [
        lambda: L.sla_predict_mask(pp, P(Q), P(K), P(Wq), P(Wk), P(mc), P(lut), P(ws), wsz, st()),
        lambda: L.sla_precompute_linear(pp, P(K), P(V), P(pw), P(hz), P(ws), wsz, st()),
        lambda: L.sla_aggregate_marginal(pp, P(mc), P(hz), P(ws), wsz, st()),
        lambda: L.sla_pair_query_blocks(pp, P(lut), P(ws), wsz, st()),
        lambda: L.sla_fused_forward_paired(pp, P(Q), P(K), P(V), P(lut), P(proj_b), P(alpha), P(O), P(ws),
                                           wsz, st()),
    ]
    router = Wq is not None or Wk is not None
    launches = {"predict_mask": 3 + (1 if router else 0), "precompute_linear": 1, "aggregate_marginal": 2,
                "pair_query_blocks": 3 if (qk == "bf16" and pv == "bf16") else 2,
                "fused_kernel": 1 + (1 if qk != "bf16" else 0) + (2 if pv != "bf16" else 0)}

    def step(ev=None):
        for i, c in enumerate(calls):
            if ev is not None:
                ev[i].record()
            code = c()
            if code != 0:
                raise bnd.SlaError(code, STAGES[i])
        if ev is not None:
            ev[len(calls)].record()

    for _ in range(max(warmup, 3)):
        step()
    torch.cuda.synchronize()
    code, detail = bnd.sla_get_device_status(ws)
    if code != 0:
        raise RuntimeError(f"device status {code} ({detail}) after warm-up")
    pairs = bnd.sla_workspace_pairs(p, ws).cpu().numpy()
    wk = work_model(cfg, dict(BH=BH, N=N, d=d, Tq=Tq, Tkv=Tkv, nh=nh, nl=nl), lut.cpu().numpy(), pairs)

    if sampler is not None:
        sampler.start()
    t_end = time.time() + burn
    while time.time() < t_end:
        step()
        torch.cuda.synchronize()
    nst = len(calls) + 1
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nst)] for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    start.record()
    for k in range(steps):
        step(evs[k])
    end.record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop() if sampler is not None else None
    ms_total = start.elapsed_time(end)
    stage_ms = [sum(evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(steps)) / steps
                for i in range(len(calls))]
    code, detail = bnd.sla_get_device_status(ws)
    if code != 0:
        raise RuntimeError(f"device status {code} ({detail}) after timing")
    rec = {"workload": workload, "qk": qk, "pv": pv, "B": B, "H": H, "N": N, "d": d, "T": Tq, "n_h": nh,
           "n_l": nl, "sparsity": round(1 - nh / Tkv, 4), "ms_total": ms_total, "steps": steps,
           "ms_per_step": ms_total / steps, "stage_ms": dict(zip(STAGES, stage_ms)), "work": wk,
           "launches_per_step": launches, "clocks": clocks}
    ctx = None
    if keep:
        ctx = dict(Q=Q, K=K, V=V, cfg=cfg, data=data, w=w, wk=wk, params=(proj_w, proj_b, alpha, Wq, Wk),
                   dev=dev)
    return rec, ctx


def rooflines(rec, peaks, peak_kind):
    """Achieved / peak per stage: the fused kernel against the bf16 tensor peak on
    its algorithmic FLOPs (the FP8 / INT8 paths' own peak is twice that), the
    bandwidth-bound stages against the HBM copy peak on their algorithmic bytes."""
    wk, sm = rec["work"], rec["stage_ms"]
    # an 8-bit product runs at twice the bf16 rate (the recipe's nominal ratio): the
    # fused kernel's peak is the harmonic mix over Q K^T, P V and the bf16 phi(Q) H
    half = wk["fused_pairs_alg"] / 2
    rest = wk["fused_alg"] - 2 * half
    t_unit = half / (2.0 if rec["qk"] != "bf16" else 1.0) + half / (2.0 if rec["pv"] != "bf16" else 1.0) + rest
    tens = round(float(peaks["bf16_tflops"]) * wk["fused_alg"] / t_unit, 1)
    hbm = float(peaks["hbm_gbs"])
    out = {}
    f_ms = sm["fused_kernel"]
    ach = wk["fused_alg"] / (f_ms * 1e-3) / 1e12
    out["fused_kernel"] = {"bound": "tensor", "achieved": round(ach, 2), "peak": tens, "unit": "TFLOP/s",
                           "frac": round(ach / tens, 4),
                           "issued_tflops": round(wk["fused_issued"] / (f_ms * 1e-3) / 1e12, 2),
                           "issued_frac": round(wk["fused_issued"] / (f_ms * 1e-3) / 1e12 / tens, 4)}
    for s in ("predict_mask", "precompute_linear", "aggregate_marginal"):
        gbs = wk["bytes"][s] / (sm[s] * 1e-3) / 1e9
        out[s] = {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                  "frac": round(gbs / hbm, 4)}
    return out


def workload_summary(rec, peaks, peak_kind):
    ms = rec["ms_per_step"]
    wk = rec["work"]
    return {"workload": rec["workload"], "qk": rec["qk"], "pv": rec["pv"],
            "shape": f"B={rec['B']}, H={rec['H']}, N={rec['N']}, d={rec['d']}, n_h={rec['n_h']}, "
                     f"n_l={rec['n_l']}, sparsity {rec['sparsity']}",
            "ms_per_step": round(ms, 4), "algorithmic_tflops": round(wk["step_alg"] / (ms * 1e-3) / 1e12, 2),
            "dense_equiv_tflops": round(wk["dense_equiv"] / (ms * 1e-3) / 1e12, 1),
            "stage_ms": {k: round(v, 4) for k, v in rec["stage_ms"].items()},
            "roofline": rooflines(rec, peaks, peak_kind)}


def run_e2e(ctx, steps):
    """Same metric through the host-buffer C-ABI call: H2D copies of Q, K, V and the
    D2H copy of O are inside the timed region."""
    Q, cfg, dev = ctx["Q"], ctx["cfg"], ctx["dev"]
    proj_w, proj_b, alpha, Wq, Wk = ctx["params"]
    Qh, Kh, Vh = (ctx[k].cpu().pin_memory() for k in ("Q", "K", "V"))
    Oh = torch.empty_like(Qh).pin_memory()
    p = bnd.make_params(Qh, cfg, Kh, Vh, Oh)
    ws = bnd.new_workspace(bnd.sla_attention_host_workspace_size(p), dev)
    pw = proj_w if cfg.combine == "proj" else None
    for _ in range(2):
        bnd.sla_attention_host(p, Qh, Kh, Vh, Oh, ws, pw, proj_b, alpha, Wq, Wk)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        bnd.sla_attention_host(p, Qh, Kh, Vh, Oh, ws, pw, proj_b, alpha, Wq, Wk)
    b.record()
    torch.cuda.synchronize()
    code, _ = bnd.sla_get_device_status(ws)
    if code != 0:
        raise RuntimeError(f"device status {code} in e2e")
    ms = a.elapsed_time(b) / steps
    act = Qh.numel() * Qh.element_size()
    return {"value": round(ctx["wk"]["step_alg"] / (ms * 1e-3) / 1e12, 3), "unit": UNIT,
            "ms_per_step": round(ms, 3), "h2d_bytes_per_step": 3 * act, "d2h_bytes_per_step": act,
            "api": "sla_attention_host (pinned host Q, K, V, O)"}


def run_train(ctx, steps=10, warmup=3, dense=True):
    """Forward + backward of the same workload (the fine-tuning step): the four
    forward stages with the LSE output, then sla_backward with dO ~ N(0, 1) bf16.
    Also times dense attention's forward + backward (torch SDPA) on the same inputs."""
    Q, K, V, cfg, dev = ctx["Q"], ctx["K"], ctx["V"], ctx["cfg"], ctx["dev"]
    proj_w, proj_b, alpha, Wq, Wk = ctx["params"]
    L, P = bnd.lib(), bnd._ptr
    B, H, N, d = Q.shape
    O = torch.empty_like(Q)
    p = bnd.make_params(Q, cfg, K, V, O)
    Tq, Tkv, nh, nl = bnd.sla_block_counts(p)
    BH = B * H
    ws = bnd.new_workspace(bnd.sla_workspace_size(p), dev)
    bws = bnd.new_workspace(bnd.sla_backward_workspace_size(p), dev)
    mc = torch.empty((BH, Tq, Tkv), dtype=torch.int8, device=dev)
    lut = torch.empty((BH, Tq, nh), dtype=torch.int32, device=dev)
    hz = torch.empty((BH, Tkv, d * d + d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((BH, N), dtype=torch.float32, device=dev)
    osp = torch.empty((BH, N, d), dtype=torch.float32, device=dev)
    g = torch.Generator(device=dev).manual_seed(7)
    dO = torch.randn(Q.shape, generator=g, device=dev).to(torch.bfloat16)
    dQ, dK, dV = torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V)
    proj = cfg.combine == "proj"
    dW = torch.empty((d, d), dtype=torch.float32, device=dev) if proj else None
    db = torch.empty(d, dtype=torch.float32, device=dev) if proj else None
    da = None if proj else torch.empty(BH, dtype=torch.float32, device=dev)
    pw = proj_w if proj else None
    st = bnd._stream
    names = ["predict_mask", "precompute_linear", "forward_train", "backward"]

    def stage(i):
        if i == 0:
            return L.sla_predict_mask(bnd.ctypes.byref(p), P(Q), P(K), P(Wq), P(Wk), P(mc), P(lut),
                                      P(ws), ws.numel(), st())
        if i == 1:
            return L.sla_precompute_linear(bnd.ctypes.byref(p), P(K), P(V), P(pw), P(hz), P(ws),
                                           ws.numel(), st())
        if i == 2:
            return L.sla_forward_train(bnd.ctypes.byref(p), P(Q), P(K), P(V), P(mc), P(lut), P(hz),
                                       P(proj_b), P(alpha), P(O), P(lse), P(osp), P(ws), ws.numel(), st())
        return L.sla_backward(bnd.ctypes.byref(p), P(Q), P(K), P(V), P(mc), P(lut), P(hz), P(pw),
                              P(proj_b), P(alpha), P(osp), P(lse), P(dO), P(dQ), P(dK), P(dV), P(dW),
                              P(db), P(da), P(bws), bws.numel(), st())

    def step(ev=None):
        for i in range(4):
            if ev is not None:
                ev[i].record()
            code = stage(i)
            if code != 0:
                raise bnd.SlaError(code, names[i])
        if ev is not None:
            ev[4].record()

    for _ in range(max(warmup, 1)):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    for k in range(steps):
        step(evs[k])
    torch.cuda.synchronize()
    for w_ in (ws, bws):
        code, detail = bnd.sla_get_device_status(w_)
        if code != 0:
            raise RuntimeError(f"device status {code} ({detail}) in the training step")
    stage_ms = [sum(evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(steps)) / steps for i in range(4)]
    res = {"workload": "forward + backward of the bench workload, dO ~ N(0, 1) bf16",
           "ms_per_step": round(sum(stage_ms), 4),
           "stage_ms": {n: round(x, 4) for n, x in zip(names, stage_ms)}}
    # the backward's algorithmic work: the sparse branch's FlashAttention backward over
    # the critical pairs (dQ: S, dP, dS K = 6*64*64*d; dK, dV: S^T, dP^T, dV, dK =
    # 8*64*64*d per pair) and the linear branch's d x d products (query side 3, key
    # side 4, dW 1 per token: 16 N d^2 per head)
    crit = Tq * nh * BH
    bwd_alg = 14 * 64 * 64 * d * crit + 16 * N * d * d * BH
    peaks, _ = load_peaks()
    ach = bwd_alg / (stage_ms[3] * 1e-3) / 1e12
    res["backward_roofline"] = {"kernels": "all of sla_backward", "bound": "tensor", "achieved": round(ach, 2),
                                "peak": float(peaks["bf16_tflops"]), "unit": "TFLOP/s",
                                "frac": round(ach / float(peaks["bf16_tflops"]), 4),
                                "algorithmic_flops": bwd_alg}
    # dense attention forward + backward on the same inputs
    if not dense:
        return res
    try:
        from torch.nn.attention import SDPBackend, sdpa_kernel
        q, k_, v = (t.detach().clone().requires_grad_(True) for t in (Q, K, V))
        with sdpa_kernel([SDPBackend.CUDNN_ATTENTION, SDPBackend.FLASH_ATTENTION]):
            for _ in range(2):
                torch.nn.functional.scaled_dot_product_attention(q, k_, v).backward(dO)
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(5):
                torch.nn.functional.scaled_dot_product_attention(q, k_, v).backward(dO)
            b.record()
            torch.cuda.synchronize()
        res["dense_fwd_bwd_ms"] = round(a.elapsed_time(b) / 5, 3)
        res["speedup_vs_dense"] = round(res["dense_fwd_bwd_ms"] / res["ms_per_step"], 2)
    except Exception as e:  # backend not available for this shape
        res["dense_fwd_bwd_ms"] = f"unavailable: {type(e).__name__}"
    return res


def run_train_main(args):
    """`--train`: the forward + backward step of the workload as its own JSON line."""
    dev = 0
    torch.cuda.set_device(dev)
    over = {} if args.heads is None else {"H": args.heads}
    data, w = I.make_workload(args.workload, device=f"cuda:{dev}", **over)
    cfg = bnd.SlaConfig(k_h=w["k_h"], k_l=w["k_l"], combine=w["combine"])
    Q, K, V = (data[k].to(dev) for k in ("Q", "K", "V"))
    f32 = lambda t: None if t is None else t.to(dev).float().contiguous()  # noqa: E731
    params = tuple(f32(data.get(k)) for k in ("proj_w", "proj_b", "alpha", "Wq", "Wk"))
    ctx = dict(Q=Q, K=K, V=V, cfg=cfg, dev=dev, params=params)
    r = run_train(ctx, steps=args.steps, warmup=args.warmup, dense=not args.no_extras)
    B, H, N, d = Q.shape
    return {"metric": "SLA forward + backward step ms", "value": r["ms_per_step"], "unit": "ms",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "higher_is_better": False,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"{args.workload} (B={B}, H={H}, N={N}, d={d}) forward + backward, "
                                   "dO ~ N(0, 1) bf16"},
            **{k: v for k, v in r.items() if k not in ("workload", "ms_per_step")}}


def run_dense(ctx, iters=10):
    """Dense bf16 softmax attention on the same inputs (torch SDPA, cuDNN else flash)."""
    from torch.nn.attention import SDPBackend, sdpa_kernel
    Q, K, V = ctx["Q"], ctx["K"], ctx["V"]
    out = {}
    for name, be in (("cudnn", SDPBackend.CUDNN_ATTENTION), ("flash", SDPBackend.FLASH_ATTENTION)):
        try:
            with sdpa_kernel([be]):
                for _ in range(3):
                    torch.nn.functional.scaled_dot_product_attention(Q, K, V)
                torch.cuda.synchronize()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                for _ in range(iters):
                    torch.nn.functional.scaled_dot_product_attention(Q, K, V)
                b.record()
                torch.cuda.synchronize()
            ms = a.elapsed_time(b) / iters
            out[name] = {"ms": round(ms, 3),
                         "tflops": round(ctx["wk"]["dense_equiv"] / (ms * 1e-3) / 1e12, 1)}
        except Exception as e:  # backend not available for this shape
            out[name] = {"error": str(e).splitlines()[0][:120]}
    return out


# --------------------------------------------------------------------------- oracle arm
def oracle_head(data, w, hh):
    """The fp64 oracle's whole forward of one head (mask prediction, linear
    statistics, every query block); returns its seconds and BLAS threads."""
    import oracle as Or
    from threadpoolctl import threadpool_info
    p = Or.OracleParams(k_h=w["k_h"], k_l=w["k_l"], combine=w["combine"])
    np_ = lambda t: None if t is None else t.float().cpu().numpy().astype(np.float64)  # noqa: E731
    sl = slice(hh, hh + 1)
    Q, K, V = (np_(data[k][:, sl]) for k in ("Q", "K", "V"))
    t0 = time.perf_counter()
    Mc, _, _ = Or.predict_mask(Q, K, p, np_(data.get("Wq")), np_(data.get("Wk")))
    alpha = data.get("alpha")
    Or.forward_given_mask(Q, K, V, Mc, p, proj_w=np_(data.get("proj_w")), proj_b=np_(data.get("proj_b")),
                          alpha=None if alpha is None else np_(alpha)[:, sl])
    secs = time.perf_counter() - t0
    cores = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    return secs, cores


def head_work(workload, data, w):
    """Algorithmic FLOPs of one head of the workload (the unit both CPU legs time)."""
    import oracle as Or
    B, H, N, d = data["Q"].shape
    T = Or.num_blocks(N, 64)
    nh, nl = Or.block_counts(T, w["k_h"], w["k_l"])
    cfg = bnd.SlaConfig(k_h=w["k_h"], k_l=w["k_l"], combine=w["combine"])
    lut = np.zeros((1, T, nh), dtype=np.int32)  # the count of critical pairs is all that is used
    wk = work_model(cfg, dict(BH=1, N=N, d=d, Tq=T, Tkv=T, nh=nh, nl=nl), lut,
                    np.zeros((1, 0, 2), dtype=np.int64))
    return wk["step_alg"], H


SAMPLE_RULE = ("one whole head per sample (mask prediction, linear statistics and every query block of "
               "that head), heads taken in order; value = that head's algorithmic FLOPs / its seconds")


def cpu_baseline(ctx, budget_s=15.0):
    """The oracle on the GPU machine's host cores, timed on whole heads until ~budget_s."""
    flops_head, H = head_work(WORKLOAD, ctx["data"], ctx["w"])
    tot, n, cores = 0.0, 0, 1
    while n < H and (n == 0 or tot < budget_s):
        s, cores = oracle_head(ctx["data"], ctx["w"], n)
        tot += s
        n += 1
    return {"value": round(flops_head * n / tot / 1e12, 6), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n} of {H} heads ({tot:.1f} s); " + SAMPLE_RULE,
            "s_per_head": round(tot / n, 3),
            "full_step_s": {"value": round(tot / n * H, 1), "extrapolated": True}}


def run_reference(args):
    """`--impl reference`: the fp64 oracle (the pages ship no code; the oracle is
    this build's reference arm) on the host cores, one whole head per step."""
    data, w = I.make_workload(args.workload)
    B, H, N, d = data["Q"].shape
    flops_head, _ = head_work(args.workload, data, w)
    for k in range(args.warmup):
        oracle_head(data, w, k % H)
    tot, cores = 0.0, 1
    for k in range(args.steps):
        s, cores = oracle_head(data, w, k % H)
        tot += s
    ms = tot / args.steps * 1e3
    value = flops_head * args.steps / tot / 1e12
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT,
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 1), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{args.workload} (B={B}, H={H}, N={N}, d={d}, k_h={w['k_h']}, "
                                   f"k_l={w['k_l']}, {w['combine']} combine)",
                       "step": "one whole head of the workload (a bounded sample)"},
            "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": SAMPLE_RULE,
                             "full_step_s": {"value": round(ms / 1e3 * H, 1), "extrapolated": True}},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# the other workloads of the metric, each as its own record in the bench line
EXTRA_WORKLOADS = [("wan1.3b_sla2", "bf16", "bf16"), ("wan14b_720p_sla2", "bf16", "bf16"),
                   ("wan14b_720p_sla2", "fp8_e4m3", "bf16"), ("wan14b_720p_sla2", "int8", "bf16"),
                   ("wan14b_720p_sla2", "int8", "fp8_e4m3")]


# --------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(I.WORKLOADS))
    ap.add_argument("--no-extras", action="store_true",
                    help="skip e2e, the other workloads, dense, training and CPU baselines")
    ap.add_argument("--qk", choices=["bf16", "fp8_e4m3", "int8"], default="bf16",
                    help="precision of Q K^T on critical blocks (fp8_e4m3, int8: d = 128 only)")
    ap.add_argument("--pv", choices=["bf16", "fp8_e4m3"], default="bf16",
                    help="precision of P V on critical blocks (fp8_e4m3: d = 128 only)")
    ap.add_argument("--heads", type=int, default=None, help="override the workload's head count "
                    "(profiling runs only; the bench line uses the workload as named)")
    ap.add_argument("--train", action="store_true",
                    help="time the training step (forward with the backward's residuals + sla_backward) "
                         "instead of the forward; one GPU")
    ap.add_argument("--burn", type=float, default=0.5,
                    help="seconds of untimed steps before the timed region (clock sampling)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    bnd.lib()
    if args.train:
        if rank == 0:
            print(json.dumps(run_train_main(args)), flush=True)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device(f"cuda:{local}"))
    sampler = ClockSampler(bus_id_of(local)) if rank == 0 else None
    rec, ctx = measure(args.workload, args.qk, args.pv, args.steps, args.warmup, local, rank, world,
                       args.heads, args.burn, sampler, keep=True)
    ms_total, job_flops = rec["ms_total"], rec["work"]["step_alg"]
    if world > 1:
        ms_total, job_flops = reduce_over_ranks(ms_total, job_flops, torch.device(f"cuda:{local}"))
    if rank == 0:
        peaks, peak_kind = load_peaks()
        wk = rec["work"]
        ms_step = ms_total / args.steps
        rl = rooflines(rec, peaks, peak_kind)
        fr = rl["fused_kernel"]
        B, H, N, d = rec["B"], rec["H"], rec["N"], rec["d"]
        cfg = ctx["cfg"]
        res = {
            "metric": METRIC, "value": round(job_flops / (ms_step * 1e-3) / 1e12, 3),
            "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16" if args.qk == "bf16" and args.pv == "bf16" else f"bf16+{args.qk}/{args.pv}",
            "data": "synthetic",
            "config": {"workload": f"{args.workload} (B={B}, H={H}, N={N}, d={d}, k_h={cfg.k_h}, "
                                   f"k_l={cfg.k_l}, {cfg.combine} combine)",
                       "B": B, "H": H, "N": N, "d": d, "n_h": rec["n_h"], "n_l": rec["n_l"], "T": rec["T"],
                       "sparsity": rec["sparsity"],
                       "l2": "inputs larger than L2 (Q, K, V = 302 MB vs 126 MB L2); no flush",
                       "parallelism": f"{world} independent problems, one per GPU (no collective)"},
            "value_note": "algorithmic FLOPs of the step (critical Q K^T + P V, phi(Q) H, Proj, h_j, "
                          "marginal adds, compressed logits) / time; issued FLOPs are under 'work'",
            "stage_ms": {n: round(x, 4) for n, x in rec["stage_ms"].items()},
            "work": {"step_algorithmic_flops": wk["step_alg"], "step_issued_flops": wk["step_issued"],
                     "fused_algorithmic_flops": wk["fused_alg"], "fused_issued_flops": wk["fused_issued"],
                     "union_entries": wk["union_total"], "critical_entries": wk["critical_entries"],
                     "tiles": wk["n_tiles"], "marginal_gemm_issued_flops": wk["marg_issued"],
                     "dense_equivalent_flops": wk["dense_equiv"]},
            "dense_equiv_tflops": round(wk["dense_equiv"] / (ms_step * 1e-3) / 1e12, 2),
            "roofline": {"kernel": fused_kernel_name(args.qk, args.pv), "timed": "sla_fused_forward_paired alone (CUDA events "
                         "around it inside the timed loop)", "bound": "tensor", "achieved": fr["achieved"],
                         "peak": fr["peak"], "unit": "TFLOP/s", "frac": fr["frac"],
                         "traffic": fused_traffic_per_launch(args.workload, H, args.qk if args.pv == "bf16"
                                                             else "fp8 P V"),
                         "peak_note": f"dense bf16 GEMM burst peak ({peak_kind})",
                         "per_launch_flops": wk["fused_alg"], "issued_frac": fr["issued_frac"]},
            "stage_roofline": {k: v for k, v in rl.items() if k != "fused_kernel"},
            "clocks": rec["clocks"],
            "gpu_launches": sum(rec["launches_per_step"].values()) * args.steps,
        }
        if not args.no_extras and world == 1:  # single-GPU measurements: no rank waits on them
            res["e2e"] = run_e2e(ctx, steps=min(args.steps, 10))
            res["dense_baseline"] = run_dense(ctx)
            best = min((v["ms"] for v in res["dense_baseline"].values() if "ms" in v), default=None)
            res["speedup_vs_dense"] = None if best is None else round(best / ms_step, 2)
            res["train_step"] = run_train(ctx)
            if world == 1:
                res["cpu_baseline"] = cpu_baseline(ctx)
            del ctx
            torch.cuda.empty_cache()
            res["workloads"] = []
            for (wl, qk, pv) in EXTRA_WORKLOADS:
                r2, _ = measure(wl, qk, pv, 10, 3, local)
                res["workloads"].append(workload_summary(r2, peaks, peak_kind))
                del r2
                torch.cuda.empty_cache()
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
