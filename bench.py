#!/usr/bin/env python
"""Masked MoE-layer throughput of the BEAM layer on B200, with roofline and CPU-oracle baselines.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step = one forward of the whole layer (router, Top-K/softmax/mask, compaction, kept experts,
shared experts, combine) over one synthetic token batch resident in HBM.  N > 1 runs N
independent replicas (one per GPU, launched with torchrun), each on its own batch: the layer
has no cross-token exchange, so there is no collective on the data path (weak scaling).
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import functools
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0

# name -> (layer spec, tokens, keep rate; None = mask off / plain Top-K[, spec overrides])
WORKLOADS = {
    # reduced copy of the Mixtral-like layer (4 experts, 1024 tokens, about 1.5 GB on the
    # device) for ncu captures of the same kernels
    "profile-prefill": ("mixtral", 1024, 0.5, {"n_experts": 4}),
    "profile-decode": ("mixtral", 2, None, {"n_experts": 4}),
    # reduced Mixtral-like training step (4 experts, 2048 tokens) for ncu captures of the
    # routing-gradient kernels
    "profile-train": ("mixtral", 2048, 0.5, {"n_experts": 4}),
    # reduced fine-grained prefill (2048 tokens) for ncu captures of the small-K down GEMM
    "profile-fine": ("fine", 2048, 0.5),
    "mixtral-prefill": ("mixtral", 4096, 0.5),
    "mixtral-prefill-high": ("mixtral", 4096, 0.25),
    "mixtral-decode1": ("mixtral", 1, 0.5),
    "mixtral-decode8": ("mixtral", 8, 0.5),
    "mixtral-decode64": ("mixtral", 64, 0.5),
    "dsv2lite-prefill": ("dsv2lite", 8192, 0.45),
    "dsv2lite-decode1": ("dsv2lite", 1, 0.07),
    "dsv2lite-decode64": ("dsv2lite", 64, 0.45),
    "qwenmoe-prefill": ("qwenmoe", 16384, 0.5),
    "fine-prefill": ("fine", 8192, 0.25),
    "fine-decode32": ("fine", 32, 0.5),
    "tiny": ("tiny", 64, 0.5),
    # keep-rate sweep of the fine-grained layer (layer time vs Avg-K), plus the plain Top-K
    "fine-prefill-k100": ("fine", 8192, None),
    "fine-prefill-k50": ("fine", 8192, 0.5),
    "fine-prefill-k25": ("fine", 8192, 0.25),
    "fine-prefill-k10": ("fine", 8192, 0.1),
    "fine-seg16-prefill": ("fine_seg16", 8192, 0.5),
    "mixtral-prefill-plain": ("mixtral", 4096, None),
    "dsv2lite-prefill-high": ("dsv2lite", 8192, 0.07),
    "dsv2lite-decode1-mid": ("dsv2lite", 1, 0.45),
    "dsv2lite-decode64-high": ("dsv2lite", 64, 0.07),
    "qwenmoe-prefill-high": ("qwenmoe", 16384, 0.14),
    "mixtral-decode1-high": ("mixtral", 1, 0.25),
}
DEFAULT_WORKLOAD = "mixtral-prefill"
# supplementary points measured after the headline in the default run
EXTRA_POINTS = ["mixtral-decode1", "mixtral-decode8", "mixtral-decode64", "dsv2lite-decode1",
                "fine-decode32"]
# cross-layer routing (the mask generator) points: name -> (layer spec, MoE layers, tokens,
# segment length, keep rate).  The Stepped-MoE shape: 44 MoE layers of 212 experts (K = 16,
# D = 1536), one decision per 16-token segment, over an 8192-token context or one decode token.
GEN_POINTS = {"gen-fine44-prefill": ("fine", 44, 8192, 16, 0.5),
              "gen-fine44-decode": ("fine", 44, 1, 16, 0.5)}
# training-side points (BEAM_TRAIN forward, then the routing gradient): name -> workload
TRAIN_POINTS = {"train-mixtral-prefill": "mixtral-prefill",
                "train-dsv2lite-prefill": "dsv2lite-prefill",
                "train-fine-seg16-prefill": "fine-seg16-prefill",
                "train-profile": "profile-train"}
# every workload, one JSON line each (--sweep)
SWEEP = ["mixtral-prefill", "mixtral-prefill-high", "mixtral-prefill-plain", "mixtral-decode1",
         "mixtral-decode1-high", "mixtral-decode8", "mixtral-decode64", "dsv2lite-prefill",
         "dsv2lite-prefill-high", "dsv2lite-decode1", "dsv2lite-decode1-mid", "dsv2lite-decode64",
         "dsv2lite-decode64-high", "qwenmoe-prefill", "qwenmoe-prefill-high", "fine-prefill-k100",
         "fine-prefill-k50", "fine-prefill-k25", "fine-prefill-k10", "fine-seg16-prefill",
         "fine-decode32", "tiny"]


# ------------------------------------------------------------------ environment helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return dict(hbm=float(d["hbm_gbs"]), tc=float(d["bf16_tflops"]),
                    tc_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    except Exception:
        return dict(hbm=FALLBACK_HBM_GBS, tc=FALLBACK_BF16_TFLOPS,
                    tc_sustained=FALLBACK_BF16_TFLOPS, source="fallback")


# Sources that do not take part in a stage's kernels or launches: the forward's kernels never
# run the routing-gradient code, so its file is left out of their hash.
GRAD_SOURCES = {"route_grad.cuh"}
GRAD_STAGES = {"route_grad", "route_dw"}


def kernel_source_hash(stage: str = "") -> str:
    """Hash of the CUDA sources a stage's kernels are built and launched from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "dynamic_expert_routing_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f in GRAD_SOURCES and stage not in GRAD_STAGES:
            continue
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes of `kernel` from a committed ncu summary, if it still matches the
    current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
    except Exception:
        return None
    rec = d.get(workload, {}).get(kernel)
    if not rec or rec.get("source_hash") != kernel_source_hash(kernel):
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi samples (every 200 ms) of the SM clock and throttle reasons of one GPU."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        # raw samples: BEAM_BENCH_OUT if set, else the system temporary directory
        out = os.environ.get("BEAM_BENCH_OUT") or tempfile.gettempdir()
        self.path = os.path.join(out, f"clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", self.gpu_id], stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None:
            return None
        try:
            rows = [l.split(",") for l in open(self.path).read().strip().splitlines()]
        except Exception:
            return None
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [c.strip() for c in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def gpu_uuid(torch, dev):
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        return str(dev)


# ------------------------------------------------------------------ algorithmic work
def layer_work(spec, T, st, tc_path=True, joint=False):
    """Algorithmic bytes and FLOPs of one forward (what the method must move / compute), per
    stage.  The intermediates are counted at the precision the path keeps them in: H in fp16
    for bf16 layers (fp32 for fp32 layers); expert output rows in fp16 on the tensor-core
    path, fp32 on the streaming path.  On the tensor-core path the shared experts are a
    problem of their own (tc_shared_* stages) for larger batches; with joint=True (small
    batches) they run inside the routed launches, whose stages then carry both problems, as
    the streaming kernels always do."""
    D, E, K, F = spec.d_model, spec.n_experts, spec.top_k, spec.d_ff
    es = 4 if spec.storage == "fp32" else 2
    hs = 4 if spec.storage == "fp32" else 2
    ys = 2 if tc_path else 4
    Fsh = spec.n_shared * spec.d_ff_shared
    Tsh = T if Fsh else 0
    na, nk = st["n_active_experts"], st["n_kept"]
    Tr = math.ceil(T / spec.segment_len) if spec.segment_len > 1 else T
    w = {}
    w["router_logits"] = dict(bytes=2 * E * D * es + Tr * D * es + Tr * 2 * E * 4,
                              flops=2 * Tr * D * 2 * E)
    w["tc_router"] = w["router_logits"]
    gu_r = dict(bytes=na * 2 * F * D * es + nk * D * es + nk * F * hs, flops=4 * nk * F * D)
    gu_s = dict(bytes=2 * Fsh * D * es + Tsh * D * es + Tsh * Fsh * hs, flops=4 * Tsh * Fsh * D)
    dn_r = dict(bytes=na * D * F * es + nk * F * hs + nk * D * ys, flops=2 * nk * F * D)
    dn_s = dict(bytes=D * Fsh * es + Tsh * Fsh * hs + Tsh * D * ys, flops=2 * Tsh * Fsh * D)
    both = lambda a, b: {k: a[k] + b[k] for k in a}
    w["stream_gateup"], w["stream_down"] = both(gu_r, gu_s), both(dn_r, dn_s)
    w["tc_gateup"], w["tc_down"] = (both(gu_r, gu_s), both(dn_r, dn_s)) if joint else (gu_r, dn_r)
    w["tc_shared_gateup"], w["tc_shared_down"] = gu_s, dn_s
    w["combine"] = dict(bytes=nk * D * ys + Tsh * D * ys + T * D * 4 + T * K * 8,
                        flops=2 * nk * D)
    w["scatter_gather"] = dict(bytes=2 * nk * D * es + T * K * 12, flops=0)
    total_bytes = (na * 3 * F * D + 3 * Fsh * D + 2 * E * D) * es + T * D * es + T * D * 4
    total_flops = 2 * (nk * 3 * F * D + T * 3 * Fsh * D + Tr * D * 2 * E)
    return w, dict(bytes=total_bytes, flops=total_flops)


TENSOR_STAGES = {"tc_gateup", "tc_down", "tc_router", "tc_shared_gateup", "tc_shared_down"}


def gen_work(spec, L: int, T: int, S: int) -> dict:
    """Algorithmic work of one cross-layer routing call: the generator matrix [L*2E][D] read
    once, the segment leaders' rows of z read once, every layer's routing arrays written once
    (topk_id, gate, mask_logit, ghat: 4 B, keep: 1 B per slot; n_keep, lreg: 4 B per token;
    the active bitsets), and the logit GEMM's FLOPs."""
    es = 2 if spec.storage == "bf16" else 4
    D, E, K = spec.d_model, spec.n_experts, spec.top_k
    Tr = -(-T // max(1, S))
    cols = L * 2 * E
    bytes_ = (cols * D * es + Tr * D * es + L * T * K * (4 * 4 + 1) + L * T * 8
              + L * ((E + 31) // 32) * 4)
    return {"bytes": bytes_, "flops": 2 * Tr * D * cols}


def gen_point(torch, name, steps, warmup, device, peaks):
    """Time beam_gen_route on one GPU: each timed call has its own event pair, and between
    calls, outside the timed region, a 256 MB buffer is written and then read, so the L2 holds
    none of the call's data and no dirty lines whose write-back would land in the next call."""
    import synth
    from dynamic_expert_routing_b200 import BeamGenerator
    spec_name, L, T, S, keep = GEN_POINTS[name]
    spec = synth.SPECS[spec_name].with_(segment_len=S)
    wr, wm = synth.make_generator(spec, L, seed=0, keep_rate=keep)
    flush = torch.empty(64 << 20, dtype=torch.float32, device=device)
    with torch.cuda.stream(torch.cuda.Stream(device)):
        gen = BeamGenerator(wr.to(device), wm.to(device), spec.top_k, max_tokens=T, segment_len=S)
        del wr, wm
        z = synth.make_tokens(spec, T, seed=1, device=device)
        out = gen.route(z)
        for _ in range(warmup):
            gen.route(z, out=out)
        st = torch.cuda.current_stream()
        pairs = []
        sink = torch.empty((), dtype=torch.float32, device=device)
        for _ in range(steps):
            flush.zero_()
            torch.sum(flush, dim=0, out=sink)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(st)
            gen.route(z, out=out)
            b.record(st)
            pairs.append((a, b))
        torch.cuda.synchronize()
        gen.sync()
        ms = sum(a.elapsed_time(b) for a, b in pairs) / steps
        keep_sum = int(out["keep"].sum().item())
        act = out["active"].cpu().numpy().astype("int64") & 0xffffffff
        n_act = [sum(bin(int(w)).count("1") for w in row) for row in act]
        gen.close()
    del flush
    work = gen_work(spec, L, T, S)
    t_hbm = work["bytes"] / (peaks["hbm"] * 1e9)
    t_tc = work["flops"] / (peaks["tc"] * 1e12)
    return dict(workload=name, metric="cross-layer routing tokens/s", unit="tokens/s",
                layers=L, tokens=T, segment_len=S, keep_rate=keep,
                value=round(T / (ms * 1e-3), 2), ms_per_step=round(ms, 5),
                layer_roofline_frac=round(max(t_hbm, t_tc) / (ms * 1e-3), 4),
                bound="hbm" if t_hbm >= t_tc else "tensor",
                algorithmic_bytes=work["bytes"], algorithmic_flops=work["flops"],
                avg_k=round(keep_sum / (L * T), 4),
                mean_active_experts=round(sum(n_act) / L, 2),
                l2="flushed (256 MB written, then read) between timed calls")


# SoftTopK points (the relaxation of the mask generator's top-k): name -> (rows, experts, K, tau)
SOFTTOPK_POINTS = {"softtopk-fine8192": (8192, 212, 16, 1.0),
                   "softtopk-fine44-decode": (44, 212, 16, 1.0)}


def softtopk_point(torch, name, steps, warmup, device, peaks):
    """SoftTopK forward (y, hard mask, nu) and backward on `rows` logit rows, each call timed with
    its own event pair after an L2 flush.  Algorithmic bytes: forward 4 B read + 4 B (y) + 1 B
    (mask) written per logit and 4 B of nu per row; backward 8 B read + 4 B written per logit."""
    from dynamic_expert_routing_b200 import softtopk, softtopk_backward
    T, E, K, tau = SOFTTOPK_POINTS[name]
    g = torch.Generator(device=device)
    g.manual_seed(3)
    r = torch.randn((T, E), generator=g, device=device, dtype=torch.float32)
    dy = torch.randn((T, E), generator=g, device=device, dtype=torch.float32)
    flush = L2Flush(torch, device)
    for _ in range(warmup):
        out = softtopk(r, K, tau, nu=True)
        softtopk_backward(out["y"], dy, tau)
    st = torch.cuda.current_stream()
    fw, bw = [], []
    for _ in range(steps):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        out = softtopk(r, K, tau, nu=True)
        b.record(st)
        fw.append((a, b))
        flush()
        c, d = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c.record(st)
        softtopk_backward(out["y"], dy, tau)
        d.record(st)
        bw.append((c, d))
    torch.cuda.synchronize()
    ms_f = sum(p.elapsed_time(q) for p, q in fw) / steps
    ms_b = sum(p.elapsed_time(q) for p, q in bw) / steps
    bytes_f = T * E * 9 + T * 4
    bytes_b = T * E * 12
    return dict(workload=name, metric="SoftTopK rows/s", unit="rows/s", rows=T, experts=E, top_k=K,
                tau=tau, value=round(T / (ms_f * 1e-3), 2), ms_forward=round(ms_f, 5),
                ms_backward=round(ms_b, 5),
                forward_hbm_frac=round(bytes_f / (peaks["hbm"] * 1e9) / (ms_f * 1e-3), 4),
                backward_hbm_frac=round(bytes_b / (peaks["hbm"] * 1e9) / (ms_b * 1e-3), 4),
                algorithmic_bytes_forward=bytes_f, algorithmic_bytes_backward=bytes_b,
                l2=L2_LABEL_FLUSHED)


def grad_work(spec, T, tc_path=True) -> dict:
    """Algorithmic bytes of the routing gradient's kernels (all HBM-bound; their FLOPs are a
    few per byte).  route_grad: dy and dx rows (fp32), every Top-K slot's expert output row
    (fp16 on the tensor-core path, fp32 otherwise), the router rows read once, the routing
    arrays (ids, gate, mask logit, inv: 16 B per slot) and the per-slot outputs (pair
    gradients 8 B, d_gate_logit / d_mask_logit / s 12 B).  route_dw: the routed rows of x
    once, perm and the pair gradients, dW_r and dW_m written (the partial columns it adds up
    are scratch, not algorithmic traffic)."""
    D, E, K = spec.d_model, spec.n_experts, spec.top_k
    es = 2 if spec.storage == "bf16" else 4
    ys = 2 if tc_path else 4
    S = max(1, spec.segment_len)
    Tr = -(-T // S)
    w = {}
    w["route_grad"] = dict(bytes=2 * T * D * 4 + T * K * D * ys + 2 * E * D * es + T * K * 36,
                           flops=2 * T * K * D + 4 * Tr * K * D)
    w["route_dw"] = dict(bytes=Tr * D * es + T * K * 12 + 2 * D * E * 4, flops=4 * Tr * K * D)
    return w


def train_point(torch, name, steps, warmup, device, peaks):
    """One training step of the routing: the BEAM_TRAIN forward (every Top-K expert evaluated,
    the mask scaling the gates) and the routing gradient.  The forward and the gradient are
    timed with their own event pairs, call by call; the forward between two gradient calls
    streams the expert weights (more than the 126 MB L2), so no gradient call finds the
    previous one's data in L2."""
    wl = TRAIN_POINTS[name]
    spec, T, keep, layer, x = build_layer(torch, wl, device)
    y = torch.empty((T, spec.d_model), dtype=torch.float32, device=device)
    g = torch.Generator(device=device)
    g.manual_seed(5)
    dy = torch.randn((T, spec.d_model), generator=g, device=device, dtype=torch.float32)
    st_ = torch.cuda.current_stream()
    for _ in range(warmup):
        layer.forward(x, out=y, train=True)
        layer.backward_router(x, dy, reg_scale=0.5)
    torch.cuda.synchronize()
    fw, bw = [], []
    n0 = layer.launch_count()
    for _ in range(steps):
        a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        a.record(st_)
        layer.forward(x, out=y, train=True)
        b.record(st_)
        layer.backward_router(x, dy, reg_scale=0.5)
        c.record(st_)
        fw.append((a, b))
        bw.append((b, c))
    torch.cuda.synchronize()
    launches = (layer.launch_count() - n0) / steps
    ms_f = sum(p.elapsed_time(q) for p, q in fw) / steps
    ms_b = sum(p.elapsed_time(q) for p, q in bw) / steps
    st = layer.stats()
    # masked inference forward at the same shape, for the training forward's extra cost
    ms_inf, _ = time_steps(torch, None, layer, x, y, steps, warmup, False, 1)
    layer.profile_begin(steps)
    for _ in range(steps):
        layer.forward(x, out=y, train=True)
        layer.backward_router(x, dy, reg_scale=0.5)
    prof = layer.profile_end()
    work = grad_work(spec, T, tc_path="tc_gateup" in prof)
    kernels = {}
    for k in ("route_grad", "route_dw"):
        if k in prof:
            kernels[k] = roofline_for(k, work[k], prof[k][0] / prof[k][1], peaks, name)
    layer.close()
    grad_bytes = sum(v["bytes"] for v in work.values())
    return dict(workload=name, metric="routing-gradient tokens/s", unit="tokens/s", tokens=T,
                keep_rate=keep, value=round(T / (ms_b * 1e-3), 2), ms_per_step=round(ms_b, 5),
                roofline_frac=round(grad_bytes / (peaks["hbm"] * 1e9) / (ms_b * 1e-3), 4),
                train_forward_ms=round(ms_f, 5), inference_forward_ms=round(ms_inf, 5),
                avg_k=round(st["avg_k"], 4), evaluated_slots_per_token=round(st["n_kept"] / T, 4),
                launches_per_step=launches,
                gradient_launches=sum(prof[k][1] for k in kernels) // max(1, prof["forwards"]),
                kernels=kernels,
                l2="a training forward (expert weights > 126 MB) runs between gradient calls")


def roofline_for(stage, work, ms_per_launch, peaks, workload):
    """Roofline of one kernel against its binding resource: tensor peak for a tensor-core
    kernel whose FLOPs take longer than its bytes at HBM speed, HBM bandwidth otherwise.
    The tensor peak is the measured burst bf16 figure: every kernel here is timed inside a
    loop of steps far shorter than the seconds-long loop that settles the sustained figure (the
    clocks sampled during the timed region stay at the maximum); the sustained peak is given
    beside it (`peak_sustained`, `frac_of_sustained`).  frac = algorithmic FLOPs (or bytes) per
    launch / ms_per_launch / peak."""
    t_bytes = work["bytes"] / (peaks["hbm"] * 1e9)
    t_flops = work["flops"] / (peaks["tc"] * 1e12)
    if stage in TENSOR_STAGES and t_flops >= t_bytes:
        achieved = work["flops"] / (ms_per_launch * 1e-3) / 1e12
        peak = peaks["tc"]
        out = dict(bound="tensor", achieved=round(achieved, 2), peak=peak, unit="TFLOP/s",
                   peak_sustained=peaks["tc_sustained"],
                   frac_of_sustained=round(achieved / peaks["tc_sustained"], 4))
    else:
        achieved = work["bytes"] / (ms_per_launch * 1e-3) / 1e9
        peak = peaks["hbm"]
        out = dict(bound="hbm", achieved=round(achieved, 1), peak=peak, unit="GB/s")
    out["frac"] = round(achieved / peak, 4)
    out["traffic"] = recorded_traffic(stage, workload)
    out["kernel"] = stage
    out["ms_per_launch"] = round(ms_per_launch, 5)
    out["algorithmic_bytes"] = int(work["bytes"])
    out["algorithmic_flops"] = int(work["flops"])
    out["peak_source"] = peaks["source"] + (" (burst bf16)" if out["bound"] == "tensor" else " (HBM copy)")
    return out


# ------------------------------------------------------------------ our arm
def workload_config(spec, T, keep, world, sbytes) -> dict:
    """The `config` of a workload's JSON line, the same on both arms: the layer shape, the batch,
    the keep rate and mask setting, how the L2 is kept from serving one step from the last, and
    the parallelism (N independent replicas)."""
    return {
        "workload": f"{spec.name}-like layer, {'prefill' if T > 64 else 'decode'} T={T}, "
                    f"keep rate {keep if keep else 1.0}",
        "d_model": spec.d_model, "n_experts": spec.n_experts, "top_k": spec.top_k,
        "d_ff": spec.d_ff, "n_shared": spec.n_shared, "d_ff_shared": spec.d_ff_shared,
        "segment_len": spec.segment_len, "tokens_per_gpu": T, "keep_rate": keep,
        "mask": "off" if keep is None else "on",
        "l2": L2_LABEL_FLUSHED if sbytes < L2_FLUSH_BELOW_BYTES else
              "inputs larger than L2 (the expert weights one step reads exceed the 126 MB L2); "
              "no flush between steps",
        "parallelism": f"{world} independent replicas" if world > 1 else "single GPU",
    }


def workload_spec(name):
    import synth
    entry = WORKLOADS[name]
    spec_name, T, keep = entry[:3]
    spec = synth.SPECS[spec_name]
    if len(entry) > 3:
        spec = spec.with_(**entry[3])
    return spec, T, keep


def build_layer(torch, name, device, seed=0):
    import synth
    from dynamic_expert_routing_b200 import BeamMoE
    spec, T, keep = workload_spec(name)
    w = synth.make_layer(spec, seed=seed, keep_rate=keep if keep else 0.5, device=device)
    wd = {k: v for k, v in w.items() if isinstance(v, torch.Tensor)}
    layer = BeamMoE(wd, spec.top_k, max_tokens=T, segment_len=spec.segment_len)
    x = synth.make_tokens(spec, T, seed=seed, device=device)
    del w, wd
    torch.cuda.empty_cache()
    return spec, T, keep, layer, x


def max_over_ranks(torch, dist, value: float, world: int, device) -> float:
    """The largest `value` over all ranks (the job time of N replicas); identity for N = 1."""
    if world <= 1:
        return float(value)
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job tokens/s of N weak-scaled replicas timed by the slowest rank."""
    return tokens_per_rank * world / (ms_max * 1e-3)


# A point whose algorithmic bytes per step are below this is timed with the L2 flushed between
# steps (its working set could otherwise stay in the 126 MB L2 from one step to the next).
L2_FLUSH_BELOW_BYTES = 1 << 30
L2_LABEL_FLUSHED = "flushed between timed steps (256 MB written, then read; each step has its own event pair)"


def l2_label(step_bytes: int) -> str:
    return (L2_LABEL_FLUSHED if step_bytes < L2_FLUSH_BELOW_BYTES else
            f"inputs larger than L2 ({step_bytes / 1e6:.0f} MB of algorithmic bytes per step against "
            "the 126 MB L2); no flush between steps")


def reference_step_bytes(spec, T, keep, w, x) -> int:
    """Algorithmic bytes per step from the oracle's routing of the whole batch (the reference
    arm runs no GPU forward to read them from)."""
    import oracle
    r = oracle.route(x, w["w_router"], w["w_mask"], spec.top_k, segment_len=spec.segment_len,
                     mask_off=keep is None)
    counts, _, _, _ = oracle.compact(r, spec.n_experts)
    st = dict(n_active_experts=int((counts > 0).sum()), n_kept=int(counts.sum()))
    _, total = layer_work(spec, T, st)
    return total["bytes"]


class L2Flush:
    """Evicts the L2 between timed steps: a 256 MB buffer written, then read (no dirty line of
    it is left to be written back inside the next step's time)."""

    def __init__(self, torch, device):
        self.buf = torch.empty(64 << 20, dtype=torch.float32, device=device)
        self.sink = torch.empty((), dtype=torch.float32, device=device)
        self.torch = torch

    def __call__(self):
        self.buf.zero_()
        self.torch.sum(self.buf, dim=0, out=self.sink)


def time_steps(torch, dist, layer, x, y, steps, warmup, mask_off, world, flush=None):
    """ms per step over `steps` forwards after `warmup` ones, max over ranks.  Without `flush`
    the steps run back to back between one event pair; with it, each step has its own event
    pair and the L2 is flushed before it, outside the timed region."""
    for _ in range(warmup):
        layer.forward(x, mask_off=mask_off, out=y)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    st = torch.cuda.current_stream()
    n0 = layer.launch_count()
    if flush is None:
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(st)
        for _ in range(steps):
            layer.forward(x, mask_off=mask_off, out=y)
        b.record(st)
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / steps
    else:
        pairs = []
        for _ in range(steps):
            flush()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(st)
            layer.forward(x, mask_off=mask_off, out=y)
            b.record(st)
            pairs.append((a, b))
        torch.cuda.synchronize()
        ms = sum(a.elapsed_time(b) for a, b in pairs) / steps
    launches = layer.launch_count() - n0
    if world > 1:
        dist.barrier()
    return max_over_ranks(torch, dist, ms, world, x.device), launches


def step_bytes(torch, layer, x, y, spec, T, mask_off):
    """Algorithmic bytes of one forward of this layer on x (from one untimed forward's stats)."""
    layer.forward(x, mask_off=mask_off, out=y)
    st = layer.stats()
    _, total = layer_work(spec, T, st)
    return total["bytes"]


def point(torch, dist, name, steps, warmup, world, device, peaks, mask_off=False):
    """Measure one supplementary point (tokens/s, roofline of its dominant kernel)."""
    with torch.cuda.stream(torch.cuda.Stream(device)):
        return _point(torch, dist, name, steps, warmup, world, device, peaks, mask_off)


def _point(torch, dist, name, steps, warmup, world, device, peaks, mask_off):
    spec, T, keep, layer, x = build_layer(torch, name, device)
    y = torch.empty((T, spec.d_model), dtype=torch.float32, device=device)
    mo = mask_off or keep is None
    sb = step_bytes(torch, layer, x, y, spec, T, mo)
    flush = L2Flush(torch, device) if sb < L2_FLUSH_BELOW_BYTES else None
    ms, _ = time_steps(torch, dist, layer, x, y, steps, warmup, mo, world, flush=flush)
    st = layer.stats()
    layer.profile_begin(steps)
    for _ in range(steps):
        if flush is not None:
            flush()
        layer.forward(x, mask_off=mo, out=y)
    prof = layer.profile_end()
    work, total = layer_work(spec, T, st, tc_path="tc_gateup" in prof,
                             joint=spec.n_shared > 0 and "tc_gateup" in prof
                             and "tc_shared_gateup" not in prof)
    stage = max((k for k in prof if k != "forwards"), key=lambda k: prof[k][0])
    rl = roofline_for(stage, work.get(stage, dict(bytes=0, flops=0)),
                      prof[stage][0] / prof[stage][1], peaks, name)
    t_roof = max(total["bytes"] / (peaks["hbm"] * 1e9), total["flops"] / (peaks["tc"] * 1e12))
    layer.close()
    return dict(workload=name, tokens=T, keep_rate=keep, mask="off" if mo else "on",
                l2=l2_label(sb),
                value=round(job_throughput(T, world, ms), 2), ms_per_step=round(ms, 5),
                avg_k=round(st["avg_k"], 4), n_active_experts=st["n_active_experts"],
                layer_roofline_frac=round(t_roof / (ms * 1e-3), 4), roofline=rl,
                stage_ms_per_forward={k: round(v[0] / prof["forwards"], 5)
                                      for k, v in prof.items() if k != "forwards"})


def spread_sample(T: int, n: int):
    """n token indices of a T-token batch spread evenly over it (all of them when n >= T)."""
    import numpy as np
    n = max(1, min(T, n))
    return np.unique(np.linspace(0, T - 1, n).round().astype(np.int64))


def cpu_baseline(spec, T, keep, weights_dev, x_dev, budget_s=15.0, reference_steps=None,
                 keep_outputs=None):
    """Time the fp64 oracle on a bounded sample of the workload (tokens/s on host cores).
    keep_outputs (a dict), if given, receives the sample, the oracle's y on it, the weights and
    x on the host, for the parity leg."""
    import numpy as np
    import torch
    import oracle
    w = {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in weights_dev.items()}
    x = x_dev.cpu()
    # probe the cost of one token, then size the sample to the budget
    t0 = time.perf_counter()
    r1 = oracle.route(x[:1], w["w_router"], w["w_mask"], spec.top_k,
                      segment_len=spec.segment_len, mask_off=keep is None)
    oracle.layer(x[:1], w, r1)
    per_tok = max(time.perf_counter() - t0, 1e-4)
    threads = oracle.num_threads()
    sel = spread_sample(T, int(budget_s * threads / per_tok))
    t0 = time.perf_counter()
    # the routing of every token (cheap next to the experts; segment routing needs the
    # leaders), then Step 4 for the sampled tokens
    r = oracle.route(x, w["w_router"], w["w_mask"], spec.top_k, segment_len=spec.segment_len,
                     mask_off=keep is None)
    y_ref = oracle.layer(x, w, r, tokens=sel)
    dt = time.perf_counter() - t0
    if keep_outputs is not None:
        keep_outputs.update(sel=sel, y_ref=y_ref, w=w, x=x)
    return dict(value=round(len(sel) / dt, 4), unit="tokens/s", cores=threads, kind="oracle",
                sample=f"routing of all {T} tokens, then the experts of {len(sel)} tokens spread "
                       "evenly over the batch (tokens/s counts the sampled tokens), fp64")


def parity_leg(spec, T, keep, y_gpu, gr, ref) -> dict:
    """The timed forward's output against the fp64 oracle, outside any timed region: routing
    on every token (bit-exact ids / keep / perm on clean tokens, unclean ones counted), y on the
    CPU baseline's token sample.  A sampled token whose decision differs from the oracle's (only
    possible inside the 1e-3 margin) is compared under the GPU's decision, which must itself be
    valid within the margin; the error against the oracle's own decisions is given beside."""
    import numpy as np
    import oracle
    from tests import parity
    w, x, sel, y_own = ref["w"], ref["x"], ref["sel"], ref["y_ref"]
    mask_off = keep is None
    out = dict(routing_tokens=T, y_tokens=int(len(sel)), tolerance=(
        dict(max_abs=parity.TOL_BF16_ABS, rel_l2=parity.TOL_BF16_REL) if spec.storage == "bf16"
        else dict(rel_l2=parity.TOL_F32_REL)))
    orr = oracle.route(x, w["w_router"], w["w_mask"], spec.top_k, segment_len=spec.segment_len,
                       mask_off=mask_off)
    ok = True
    try:
        info = parity.compare_routing(gr, orr, spec.n_experts)
        parity.check_structure(gr, T, spec.top_k, spec.n_experts)
    except AssertionError as e:
        ok = False
        clean = orr.clean()
        info = dict(clean=int(clean.sum()), unclean=int((~clean).sum()))
        out["routing_error"] = str(e)[:200]
    out.update(clean=info["clean"], unclean=info["unclean"])
    ids_same = np.array([set(gr["topk_id"][t].tolist()) == set(orr.topk_id[t].tolist()) and
                         {int(e): int(k) for e, k in zip(gr["topk_id"][t], gr["keep"][t])} ==
                         {int(e): int(k) for e, k in zip(orr.topk_id[t], orr.keep[t])}
                         for t in sel])
    yg = np.asarray(y_gpu, np.float64)[sel]
    y_ref = np.array(y_own, np.float64, copy=True)
    differ = np.nonzero(~ids_same)[0]
    out["differing_tokens"] = int(differ.size)
    if differ.size:
        try:
            gdec, _ = parity.gpu_decision_routing(gr, x, w["w_router"], w["w_mask"], spec.top_k,
                                                  spec.segment_len, mask_off)
            y_ref[differ] = oracle.layer(x, w, gdec, tokens=sel[differ])
        except AssertionError as e:
            ok = False
            out["decision_error"] = str(e)[:200]
    rep = parity.y_report(yg, y_ref, spec.storage)
    own = parity.y_report(yg, y_own, spec.storage)
    out.update(max_abs=rep["max_abs"], rel_l2=rep["rel_l2"], max_abs_own_decision=own["max_abs"],
               rel_l2_own_decision=own["rel_l2"], ok=bool(ok and rep["ok"]))
    return out


def run_ours(args):
    """Headline run.  Work is issued on a dedicated (non-default) stream, so the library can
    replay each forward as a captured CUDA graph, as a serving engine would."""
    import torch
    with torch.cuda.stream(torch.cuda.Stream()):
        _run_ours(args)


def _run_ours(args):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    peaks = load_peaks()

    name = args.workload
    spec, T, keep, layer, x = build_layer(torch, name, device)
    if args.path:
        # every forward of this run on one expert path (for profiling that path's kernels)
        layer.forward = functools.partial(type(layer).forward, layer, path=args.path)
    y = torch.empty((T, spec.d_model), dtype=torch.float32, device=device)
    mask_off = keep is None
    sb = step_bytes(torch, layer, x, y, spec, T, mask_off)
    flush = L2Flush(torch, device) if sb < L2_FLUSH_BELOW_BYTES else None
    sampler = ClockSampler(gpu_uuid(torch, device))
    with sampler:
        ms, launches = time_steps(torch, dist, layer, x, y, args.steps, args.warmup, mask_off,
                                  world, flush=flush)
    clocks = sampler.summary()
    st = layer.stats()
    # per-kernel timing pass (same K steps, events around every kernel)
    layer.profile_begin(args.steps)
    for _ in range(args.steps):
        if flush is not None:
            flush()
        layer.forward(x, mask_off=mask_off, out=y)
    prof = layer.profile_end()
    # the timed forward's output and routing, for the parity leg (deterministic: every step
    # gives the same bits)
    y_head = y.cpu().numpy() if rank == 0 and world == 1 and not args.no_cpu_baseline else None
    gr_head = layer.routing(T) if y_head is not None else None
    work, total = layer_work(spec, T, st, tc_path="tc_gateup" in prof,
                             joint=spec.n_shared > 0 and "tc_gateup" in prof
                             and "tc_shared_gateup" not in prof)
    stages = {k: v for k, v in prof.items() if k != "forwards"}
    tot_ms = sum(v[0] for v in stages.values())
    dom = max(stages, key=lambda k: stages[k][0])
    rl = roofline_for(dom, work.get(dom, dict(bytes=0, flops=0)), stages[dom][0] / stages[dom][1],
                      peaks, name)
    rl["share"] = round(stages[dom][0] / tot_ms, 4)
    t_roof = max(total["bytes"] / (peaks["hbm"] * 1e9), total["flops"] / (peaks["tc"] * 1e12))

    # end to end through the host-buffer entry point (pinned memory, copies inside the region):
    # the pipelined call (chunks whose copies overlap the other chunks' forwards) for batches of
    # at least 1024 tokens, and the plain one (copy in, forward, copy out) beside it
    es = 2 if spec.storage == "bf16" else 4
    xh = x.cpu().pin_memory()
    yh = torch.empty((T, spec.d_model), dtype=torch.float32).pin_memory()

    yh16 = torch.empty((T, spec.d_model), dtype=torch.bfloat16).pin_memory()

    def e2e_time(pipeline, out=yh):
        for _ in range(max(1, args.warmup)):
            layer.forward_host(xh, out, mask_off=mask_off, pipeline=pipeline)
        if world > 1:
            dist.barrier()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        n = max(3, args.steps // 2)
        a.record()
        for _ in range(n):
            layer.forward_host(xh, out, mask_off=mask_off, pipeline=pipeline)
        b.record()
        torch.cuda.synchronize()
        return max_over_ranks(torch, dist, a.elapsed_time(b) / n, world, device)

    def e2e_async_time(out):
        # back-to-back asynchronous calls (each copies its own x in and its y out, inside the
        # timed region), finished by one host_wait; the event pair brackets the whole run
        for _ in range(max(1, args.warmup)):
            layer.forward_host(xh, out, mask_off=mask_off, asynchronous=True)
        layer.host_wait()
        if world > 1:
            dist.barrier()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        n = max(3, args.steps // 2)
        a.record()
        for _ in range(n):
            layer.forward_host(xh, out, mask_off=mask_off, asynchronous=True)
        layer.host_wait()
        b.record()
        torch.cuda.synchronize()
        return max_over_ranks(torch, dist, a.elapsed_time(b) / n, world, device)

    pipelined = T >= 1024
    e2e_sync_ms = e2e_time(pipelined)
    e2e_plain_ms = e2e_time(False) if pipelined else e2e_sync_ms
    e2e_ms = e2e_async_time(yh)
    # the same calls with y delivered in bf16 (rounded on the device), half the D2H bytes
    e2e16_ms = e2e_async_time(yh16) if spec.storage == "bf16" else None

    # mask off through the same library at the headline shape: the layer speedup from skipping
    y.zero_()
    ms_off, _ = time_steps(torch, dist, layer, x, y, args.steps, args.warmup, True, world)

    cpu = None
    par = None
    if y_head is not None:
        import synth
        wcpu = synth.make_layer(spec, seed=0, keep_rate=keep if keep else 0.5, device=device)
        ref = {}
        cpu = cpu_baseline(spec, T, keep, wcpu, x, budget_s=args.cpu_budget, keep_outputs=ref)
        del wcpu
        par = parity_leg(spec, T, keep, y_head, gr_head, ref)
        del ref
    layer.close()
    del layer, x, y
    torch.cuda.empty_cache()

    points = []
    gen_points = []
    train_points = []
    if not args.no_points:
        for p in EXTRA_POINTS:
            if p == name:
                continue
            points.append(point(torch, dist, p, max(10, args.steps), args.warmup, world, device, peaks))
        if world == 1:
            for p in GEN_POINTS:
                gen_points.append(gen_point(torch, p, max(10, args.steps), args.warmup, device, peaks))
            train_points.append(train_point(torch, "train-mixtral-prefill", max(10, args.steps),
                                            args.warmup, device, peaks))
            for p in SOFTTOPK_POINTS:
                train_points.append(softtopk_point(torch, p, max(10, args.steps), args.warmup,
                                                   device, peaks))

    if rank == 0:
        line = {
            "metric": "masked MoE-layer tokens/s",
            "value": round(job_throughput(T, world, ms), 2),
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms, 5),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16" if spec.storage == "bf16" else "f32",
            "data": "synthetic (seeded; random-init weights of the layer shape)",
            "config": dict(workload_config(spec, T, keep, world, sb),
                           **({"expert_path": args.path} if args.path else {})),
            "routing_stats": {"avg_k": round(st["avg_k"], 4), "l_reg": round(st["l_reg"], 6),
                              "n_active_experts": st["n_active_experts"], "n_kept": st["n_kept"],
                              "n_tokens_all_masked": st["n_tokens_all_masked"]},
            "parity": par,
            "roofline": rl,
            "layer_roofline_frac": round(t_roof / (ms * 1e-3), 4),
            "mask_off": {"value": round(job_throughput(T, world, ms_off), 2),
                         "ms_per_step": round(ms_off, 5),
                         "layer_speedup_from_mask": round(ms_off / ms, 4)},
            "stage_ms_per_forward": {k: round(v[0] / prof["forwards"], 5) for k, v in stages.items()},
            "e2e": {"value": round(job_throughput(T, world, e2e_ms), 2), "unit": "tokens/s",
                    "h2d_bytes_per_step": T * spec.d_model * es,
                    "d2h_bytes_per_step": T * spec.d_model * 4,
                    "call": "beam_moe_forward_host with BEAM_HOST_ASYNC, calls issued back to back "
                            "(each copies its x from pinned host memory and its y back inside the "
                            "timed region; the copies of one call overlap its neighbours' "
                            "forwards), beam_moe_host_wait at the end",
                    "synchronous_value": round(job_throughput(T, world, e2e_sync_ms), 2),
                    "synchronous_call": "beam_moe_forward_host" + (" with BEAM_HOST_PIPELINE" if pipelined else "")
                                        + ", returning after its own y copy",
                    "unpipelined_value": round(job_throughput(T, world, e2e_plain_ms), 2),
                    "y_bf16": None if e2e16_ms is None else {
                        "value": round(job_throughput(T, world, e2e16_ms), 2),
                        "d2h_bytes_per_step": T * spec.d_model * 2,
                        "call": "the same asynchronous calls with a bf16 y_host (BEAM_HOST_Y_BF16: the "
                                "combine stores y rounded to bf16, and the bf16 rows are copied)"}},
            "gpu_launches": launches,
            "clocks": clocks,
            "cpu_baseline": cpu,
            "points": points,
            "gen_points": gen_points,
            "train_points": train_points,
            "peaks": peaks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_sweep(args):
    """One JSON line per workload on one GPU: tokens/s, the layer roofline fraction, the
    dominant kernel against its roofline, and the plain Top-K (mask off) time at the shape."""
    import torch
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    peaks = load_peaks()
    for name in SWEEP:
        r = point(torch, None, name, args.steps, args.warmup, 1, device, peaks)
        if r["mask"] == "on":
            off = point(torch, None, name, args.steps, args.warmup, 1, device, peaks, mask_off=True)
            r["mask_off_ms_per_step"] = off["ms_per_step"]
            r["layer_speedup_from_mask"] = round(off["ms_per_step"] / r["ms_per_step"], 4)
        r["metric"] = "masked MoE-layer tokens/s"
        r["unit"] = "tokens/s"
        print(json.dumps(r), flush=True)
    for name in GEN_POINTS:
        print(json.dumps(gen_point(torch, name, args.steps, args.warmup, device, peaks)), flush=True)
    for name in TRAIN_POINTS:
        if name != "train-profile":
            print(json.dumps(train_point(torch, name, args.steps, args.warmup, device, peaks)),
                  flush=True)
    for name in SOFTTOPK_POINTS:
        print(json.dumps(softtopk_point(torch, name, args.steps, args.warmup, device, peaks)), flush=True)


# ------------------------------------------------------------------ reference arm (the oracle)
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    import torch
    import oracle
    import synth
    spec, T, keep = workload_spec(args.workload)
    oracle.build()
    w = synth.make_layer(spec, seed=0, keep_rate=keep if keep else 0.5,
                         device="cuda" if torch.cuda.is_available() else "cpu")
    w = {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in w.items()}
    x = synth.make_tokens(spec, T, seed=0, device="cuda" if torch.cuda.is_available() else "cpu").cpu()
    threads = oracle.num_threads()
    # one step = the oracle on a fixed sample of tokens of the batch, end to end
    t0 = time.perf_counter()
    r1 = oracle.route(x[:1], w["w_router"], w["w_mask"], spec.top_k, mask_off=keep is None)
    oracle.layer(x[:1], w, r1)
    per_tok = max(time.perf_counter() - t0, 1e-4) / threads
    budget = 150.0 / (args.steps + args.warmup)
    sel = spread_sample(T, int(budget / per_tok))

    def step():
        # the routing of every token, then Step 4 of the sampled ones (as the CPU-baseline leg)
        r = oracle.route(x, w["w_router"], w["w_mask"], spec.top_k,
                         segment_len=spec.segment_len, mask_off=keep is None)
        oracle.layer(x, w, r, tokens=sel)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    value = round(len(sel) / dt, 4)
    line = {
        "impl": "reference",
        "metric": "masked MoE-layer tokens/s",
        "value": value, "unit": "tokens/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; random-init weights of the layer shape)",
        "config": workload_config(spec, T, keep, int(os.environ.get("WORLD_SIZE", "1")),
                                  reference_step_bytes(spec, T, keep, w, x)),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"per step: routing of all {T} tokens, then the experts of "
                                   f"{len(sel)} tokens spread evenly over the batch (tokens/s counts "
                                   "the sampled tokens), fp64"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


_BYTE_UNITS = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "Tbyte": 1e12,
               "KB": 1e3, "MB": 1e6, "GB": 1e9, "B": 1}


def record_traffic(args):
    """Write the per-launch DRAM bytes of one kernel, read from an ncu CSV log of
    dram__bytes_read.sum and dram__bytes_write.sum, into profiles/traffic.json under
    (workload, stage), stamped with the hash of the kernel sources it was measured on (a later
    source change makes the bench report null until it is captured again)."""
    import csv
    import re
    pat = re.compile(args.traffic_kernel)
    per_launch = {}
    with open(args.record_traffic, newline="") as f:
        rows = [r for r in csv.reader(f) if r]
    head = next(i for i, r in enumerate(rows) if "Metric Name" in r)
    cols = {name: j for j, name in enumerate(rows[head])}
    for r in rows[head + 1:]:
        if len(r) < len(cols) or not pat.search(r[cols["Kernel Name"]]):
            continue
        name = r[cols["Metric Name"]]
        if name not in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            continue
        v = float(r[cols["Metric Value"]].replace(",", "")) * _BYTE_UNITS[r[cols["Metric Unit"]]]
        per_launch.setdefault(r[cols["ID"]], {})[name] = v
    totals = [d["dram__bytes_read.sum"] + d["dram__bytes_write.sum"] for d in per_launch.values()
              if len(d) == 2]
    if not totals:
        raise SystemExit(f"no launch of /{args.traffic_kernel}/ with both DRAM metrics")
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except FileNotFoundError:
        d = {}
    key = getattr(args, "traffic_workload", None) or args.workload
    d.setdefault(key, {})[args.traffic_stage] = {
        "dram_bytes_per_launch": int(round(sum(totals) / len(totals))),
        "launches": len(totals),
        "kernel": args.traffic_kernel,
        "source_hash": kernel_source_hash(args.traffic_stage),
        "command": args.traffic_command,
    }
    with open(path, "w") as f:
        json.dump(d, f, indent=1, sort_keys=True)
        f.write("\n")
    print(json.dumps(d[key][args.traffic_stage]))


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-points", action="store_true", help="skip the supplementary points")
    ap.add_argument("--path", choices=["stream", "tensor"], default=None,
                    help="run the workload's forwards on this expert path (default: the library's choice)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle CPU work")
    ap.add_argument("--sweep", action="store_true",
                    help="measure every workload (one JSON line each) instead of the headline")
    ap.add_argument("--train", choices=sorted(TRAIN_POINTS) + sorted(SOFTTOPK_POINTS), action="append",
                    help="measure only these training points (routing gradient or SoftTopK; one JSON line each)")
    ap.add_argument("--record-traffic", metavar="NCU_CSV",
                    help="store a kernel's DRAM bytes per launch from an ncu CSV log (no GPU work)")
    ap.add_argument("--traffic-kernel", default=r"tc_grouped_gemm_kernel<(\(int\))?0,",
                    help="regex of the kernel name in the CSV (gate/up: EPI 0, down: EPI 2)")
    ap.add_argument("--traffic-stage", default="tc_gateup", help="bench stage of that kernel")
    ap.add_argument("--traffic-command", default="", help="the ncu command that wrote the CSV")
    ap.add_argument("--traffic-workload", default=None,
                    help="workload or point key to store it under (default: --workload)")
    args = ap.parse_args()
    if args.record_traffic:
        record_traffic(args)
        return
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    elif args.train:
        import torch
        device = torch.device("cuda", 0)
        torch.cuda.set_device(device)
        with torch.cuda.stream(torch.cuda.Stream(device)):
            for name in args.train:
                if name in SOFTTOPK_POINTS:
                    print(json.dumps(softtopk_point(torch, name, args.steps, args.warmup, device,
                                                    load_peaks())), flush=True)
                else:
                    print(json.dumps(train_point(torch, name, args.steps, args.warmup, device,
                                                 load_peaks())), flush=True)
    elif args.sweep:
        run_sweep(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
