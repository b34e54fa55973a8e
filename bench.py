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


def fused_traffic_per_launch(workload: str, heads: int, qk: str):
    """DRAM bytes per launch of the fused kernel from the committed ncu summary,
    or None if the summary is for another workload or the kernel source changed
    since those counters were taken."""
    path = os.path.join(ROOT, "profiles", f"fused_{workload}_traffic.txt")
    src = os.path.join(ROOT, "block_sparse_linear_pool_b200", "csrc", "fused.cu")
    if not os.path.exists(path):
        return None
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    vals = {}
    for line in open(path):
        if "=" in line and not line.startswith("#"):
            k, v = line.split("=", 1)
            vals[k.strip()] = v.strip()
    if vals.get("fused_cu_sha256_16") != sha:
        return None
    if vals.get("heads") != str(heads) or vals.get("qk", "bf16") != qk:
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except Exception:
        return None


# --------------------------------------------------------------------------- FLOP accounting
def flop_model(cfg, dims, lut_np):
    """Executed and algorithmic FLOPs of one step.

    Executed = every tensor-core MMA the kernels issue (union entries of the fused
    kernel, padded GEMM tiles) plus the fp32 logits; algorithmic (fused) = QK^T and
    PV over the critical pairs plus phi(Q)H per query row."""
    BH, N, d, Tq, Tkv, nh, nl = (dims[k] for k in ("BH", "N", "d", "Tq", "Tkv", "nh", "nl"))
    NN = d * d + d
    # fused kernel: per CTA (pair of query blocks) U union entries x (S + PV), + 2 phi(Q)H tiles
    lut = lut_np.reshape(BH, Tq, nh)
    U = 0
    for bh in range(BH):
        for p in range(0, Tq, 2):
            s = set(lut[bh, p].tolist())
            if p + 1 < Tq:
                s |= set(lut[bh, p + 1].tolist())
            U += len(s)
    n_cta = BH * ((Tq + 1) // 2)
    fused_exec = U * 2 * (2 * 128 * 64 * d) + n_cta * 2 * (2 * 128 * d * d)
    fused_alg = 4 * 64 * 64 * d * Tq * nh * BH + 2 * N * d * d * BH
    # marginal aggregation GEMM: 128 x 256 tiles, K padded to 64
    marg_exec = 2 * (math.ceil(Tq / 128) * 128) * (math.ceil(NN / 256) * 256) * \
        (math.ceil(Tkv / 64) * 64) * BH
    marg_alg = Tq * (Tkv - nh - nl) * NN * BH  # one add per marginal (i, j, element)
    kv_exec = BH * Tkv * ((2 * 64 * d * d) * (2 if cfg.combine == "proj" else 1))
    select = 2 * Tq * Tkv * d * BH + (4 * Tq * d * d * BH if cfg.combine == "alpha" else 0)
    return {"fused_exec": fused_exec, "fused_alg": fused_alg, "marg_exec": marg_exec,
            "marg_alg": marg_alg, "kv_exec": kv_exec, "select": select, "union_total": U,
            "n_cta_fused": n_cta,
            "step_exec": fused_exec + marg_exec + kv_exec + select,
            "dense_equiv": 4 * N * N * d * BH}


# --------------------------------------------------------------------------- our arm
def reduce_over_ranks(ms_total: float, flops_per_step: float, device):
    """Whole-job figures of a data-parallel run: the slowest rank's timed-region
    duration (max over ranks) and the executed FLOPs of one step summed over the
    ranks' independent problems.  Every rank must call this, in the same order."""
    t_ms = torch.tensor([ms_total], dtype=torch.float64, device=device)
    t_fl = torch.tensor([flops_per_step], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t_ms, op=torch.distributed.ReduceOp.MAX)
    torch.distributed.all_reduce(t_fl, op=torch.distributed.ReduceOp.SUM)
    return float(t_ms.item()), float(t_fl.item())


def run_ours(args, rank, world, dev):
    torch.cuda.set_device(dev)
    over = {} if args.heads is None else {"H": args.heads}
    data, w = I.make_workload(args.workload, device=f"cuda:{dev}", problem=rank, **over)
    cfg = bnd.SlaConfig(k_h=w["k_h"], k_l=w["k_l"], combine=w["combine"], qk=args.qk, pv=args.pv)
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
    st = lambda: bnd._stream()  # noqa: E731
    wsz = ws.numel()

    def stage(i):
        if i == 0:
            return L.sla_predict_mask(bnd.ctypes.byref(p), P(Q), P(K), P(Wq), P(Wk), P(mc), P(lut),
                                      P(ws), wsz, st())
        if i == 1:
            return L.sla_precompute_linear(bnd.ctypes.byref(p), P(K), P(V), P(pw), P(hz), P(ws), wsz, st())
        if i == 2:
            return L.sla_aggregate_marginal(bnd.ctypes.byref(p), P(mc), P(hz), P(ws), wsz, st())
        return L.sla_fused_forward(bnd.ctypes.byref(p), P(Q), P(K), P(V), P(lut), P(proj_b), P(alpha),
                                   P(O), P(ws), wsz, st())

    names = ["predict_mask", "precompute_linear", "aggregate_marginal", "fused_forward"]
    launches_per_step = {"predict_mask": 3 + (2 if Wq is not None or Wk is not None else 0),
                         "precompute_linear": 1, "aggregate_marginal": 2,
                         "fused_forward": 3 + (1 if args.qk != "bf16" else 0) + (2 if args.pv != "bf16" else 0)}

    def step(ev=None):
        for i in range(4):
            if ev is not None:
                ev[i].record()
            code = stage(i)
            if code != 0:
                raise bnd.SlaError(code, names[i])
        if ev is not None:
            ev[4].record()

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    code, detail = bnd.sla_get_device_status(ws)
    if code != 0:
        raise RuntimeError(f"device status {code} ({detail}) after warm-up")
    fl = flop_model(cfg, dict(BH=BH, N=N, d=d, Tq=Tq, Tkv=Tkv, nh=nh, nl=nl), lut.cpu().numpy())

    # keep the GPU busy ~0.5 s before timing so that the clock sampler sees the loaded state
    sampler = ClockSampler(bus_id_of(dev) if rank == 0 else None)
    if rank == 0:
        sampler.start()
    t_end = time.time() + args.burn
    while time.time() < t_end:
        step()
        torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    start.record()
    for k in range(args.steps):
        step(evs[k])
    end.record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop() if rank == 0 else None
    ms_total = start.elapsed_time(end)
    stage_ms = [sum(evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(args.steps)) / args.steps
                for i in range(4)]
    job_flops = fl["step_exec"]
    if world > 1:
        ms_total, job_flops = reduce_over_ranks(ms_total, fl["step_exec"], torch.device(f"cuda:{dev}"))
    code, detail = bnd.sla_get_device_status(ws)
    if code != 0:
        raise RuntimeError(f"device status {code} ({detail}) after timing")
    ms_step = ms_total / args.steps

    result = None
    if rank == 0:
        peaks, peak_kind = load_peaks()
        fused_ms = stage_ms[3]
        ach = fl["fused_alg"] / (fused_ms * 1e-3) / 1e12
        peak = float(peaks["bf16_tflops"])
        traffic = fused_traffic_per_launch(args.workload, H, args.qk if args.pv == "bf16" else "fp8 P V")
        result = {
            "metric": METRIC, "value": round(job_flops / (ms_total * 1e-3 / args.steps) / 1e12, 3),
            "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16" if args.qk == "bf16" and args.pv == "bf16" else "bf16+e4m3",
            "data": "synthetic",
            "config": {"workload": f"{args.workload} (B={B}, H={H}, N={N}, d={d}, k_h={cfg.k_h}, "
                                   f"k_l={cfg.k_l}, {cfg.combine} combine)",
                       "B": B, "H": H, "N": N, "d": d, "n_h": nh, "n_l": nl, "T": Tq,
                       "sparsity": round(1 - nh / Tkv, 4),
                       "l2": "inputs larger than L2 (Q, K, V = 302 MB vs 126 MB L2); no flush",
                       "parallelism": f"{world} independent problems, one per GPU (no collective)"},
            "stage_ms": {n: round(x, 4) for n, x in zip(names, stage_ms)},
            "flops": {"step_executed": fl["step_exec"], "fused_executed": fl["fused_exec"],
                      "fused_algorithmic": fl["fused_alg"], "marginal_gemm_executed": fl["marg_exec"],
                      "dense_equivalent": fl["dense_equiv"], "fused_union_entries": fl["union_total"]},
            "dense_equiv_tflops": round(fl["dense_equiv"] / (ms_step * 1e-3) / 1e12, 2),
            "fused_executed_tflops": round(fl["fused_exec"] / (fused_ms * 1e-3) / 1e12, 2),
            "fused_executed_frac": round(fl["fused_exec"] / (fused_ms * 1e-3) / 1e12 / peak, 4),
            "roofline": {"kernel": "sla_fused_kernel<128>", "timed": "the fused_forward stage (pair_overlap_kernel "
                         "+ pair_match_kernel + sla_fused_kernel)", "bound": "tensor", "achieved": round(ach, 2),
                         "peak": peak, "unit": "TFLOP/s", "frac": round(ach / peak, 4),
                         "traffic": traffic,
                         "peak_note": f"dense bf16 GEMM burst peak ({peak_kind})",
                         "per_launch_flops": fl["fused_alg"]},
            "clocks": clocks,
            "gpu_launches": sum(launches_per_step.values()) * args.steps,
        }
        result["_ctx"] = dict(Q=Q, K=K, V=V, cfg=cfg, data=data, w=w, fl=fl,
                              params=(proj_w, proj_b, alpha, Wq, Wk), dev=dev)
    return result


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
    return {"value": round(ctx["fl"]["step_exec"] / (ms * 1e-3) / 1e12, 3), "unit": UNIT,
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
                         "tflops": round(ctx["fl"]["dense_equiv"] / (ms * 1e-3) / 1e12, 1)}
        except Exception as e:  # backend not available for this shape
            out[name] = {"error": str(e).splitlines()[0][:120]}
    return out


# --------------------------------------------------------------------------- oracle arm
def oracle_sample(data, w, heads, qblocks_per_head):
    """Runs the fp64 oracle on `heads` heads and the first `qblocks_per_head` query
    blocks of each; returns (seconds, fraction of the workload's (head, query
    block) units covered)."""
    import oracle as Or
    from threadpoolctl import threadpool_info
    p = Or.OracleParams(k_h=w["k_h"], k_l=w["k_l"], combine=w["combine"])
    H = data["Q"].shape[1]
    T = Or.num_blocks(data["Q"].shape[2], 64)
    nb = min(qblocks_per_head, T)
    t0 = time.perf_counter()
    for hh in range(heads):
        sl = slice(hh, hh + 1)
        Q, K, V = (data[k][:, sl].float().numpy().astype(np.float64) for k in ("Q", "K", "V"))
        np_ = lambda t: None if t is None else t.float().numpy().astype(np.float64)  # noqa: E731
        Mc, _, _ = Or.predict_mask(Q, K, p, np_(data.get("Wq")), np_(data.get("Wk")))
        alpha = data.get("alpha")
        a = None if alpha is None else np_(alpha)[:, sl]
        Or.forward_given_mask(Q, K, V, Mc, p, proj_w=np_(data.get("proj_w")),
                              proj_b=np_(data.get("proj_b")), alpha=a, qblocks=range(nb))
    secs = time.perf_counter() - t0
    cores = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    return secs, (heads * nb) / (H * T), cores


def cpu_baseline(ctx):
    secs, frac, cores = oracle_sample(ctx["data"], ctx["w"], heads=4, qblocks_per_head=10 ** 9)
    step_equiv = secs / frac
    return {"value": round(ctx["fl"]["step_exec"] / step_equiv / 1e12, 6), "unit": UNIT,
            "cores": cores, "kind": "oracle", "ms_per_step_equiv": round(step_equiv * 1e3, 1),
            "sample": f"4 of {ctx['data']['Q'].shape[1]} heads, all query blocks, mask prediction "
                      f"and linear statistics included ({secs:.1f} s); value = the step's executed "
                      f"FLOPs scaled by the covered (head, query block) fraction {frac:.3f}"}


def run_reference(args):
    data, w = I.make_workload(args.workload)
    B, H, N, d = data["Q"].shape
    # one step = 1 head, first 64 query blocks (about 1 s of fp64 work on 8 cores)
    from block_sparse_linear_pool_b200.binding import SlaConfig
    cfg = SlaConfig(k_h=w["k_h"], k_l=w["k_l"], combine=w["combine"])
    import oracle as Or
    T = Or.num_blocks(N, 64)
    nh, nl = Or.block_counts(T, cfg.k_h, cfg.k_l)
    Mc, _, _ = Or.predict_mask(data["Q"].float().numpy().astype(np.float64),
                               data["K"].float().numpy().astype(np.float64),
                               Or.OracleParams(k_h=w["k_h"], k_l=w["k_l"]),
                               None if data.get("Wq") is None else data["Wq"].numpy().astype(np.float64),
                               None if data.get("Wk") is None else data["Wk"].numpy().astype(np.float64))
    lut = Or.critical_lut(Mc)
    fl = flop_model(cfg, dict(BH=B * H, N=N, d=d, Tq=T, Tkv=T, nh=nh, nl=nl), lut)
    for _ in range(args.warmup):
        oracle_sample(data, w, 1, 64)
    tot, frac, cores = 0.0, 0.0, 1
    for _ in range(args.steps):
        s, frac, cores = oracle_sample(data, w, 1, 64)
        tot += s
    step_equiv = tot / args.steps / frac
    value = fl["step_exec"] / step_equiv / 1e12
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT,
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(step_equiv * 1e3, 1), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{args.workload} (B={B}, H={H}, N={N}, d={d}, k_h={w['k_h']}, "
                                   f"k_l={w['k_l']}, {w['combine']} combine)"},
            "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": "per step: 1 head, its first 64 query blocks, mask prediction "
                                       "and linear statistics of that head; value scaled by the "
                                       f"covered (head, query block) fraction {frac:.4f}"},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# --------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(I.WORKLOADS))
    ap.add_argument("--no-extras", action="store_true", help="skip e2e, dense baseline and CPU baseline")
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
    res = run_ours(args, rank, world, local)
    if rank == 0:
        ctx = res.pop("_ctx")
        if not args.no_extras:
            res["e2e"] = run_e2e(ctx, steps=min(args.steps, 10))
            res["dense_baseline"] = run_dense(ctx)
            res["train_step"] = run_train(ctx)
            best = min((v["ms"] for v in res["dense_baseline"].values() if "ms" in v), default=None)
            res["speedup_vs_dense"] = None if best is None else round(best / res["ms_per_step"], 2)
            if world == 1:
                res["cpu_baseline"] = cpu_baseline(ctx)
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
