#!/usr/bin/env python
"""Benchmark of the single-GPU MoE layer: permute -> grouped SwiGLU FFN -> weighted combine.

One step = one pass of the whole hot path over one batch of synthetic tokens that are
already resident in HBM: moe_permute (histogram, scan, stable rank, row copy; maxvio
fused), moe_grouped_ffn_up_gate, moe_grouped_ffn_down, moe_unpermute_combine. The L2
is flushed before every timed step, outside the timed events (a 256 MiB write, then a
256 MiB read of another buffer so that the write's dirty lines leave L2 there).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload large]
    python bench.py --impl reference ...     (the CPU oracle on the host cores)

Multi-GPU: replicas only (one process per GPU under torchrun, each running the whole
layer on its own batch; no data-path collective). Time = max over ranks.
Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE layer tokens/sec on 1 B200; grouped-FFN TFLOP/s; permute+combine HBM GB/s"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "large"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--zero-copy", action="store_true",
                   help="forward step without x_perm: metadata-only permute, SwiGLU pass "
                        "gathering its token rows from x (cp.async gather warps)")
    p.add_argument("--shared-experts", type=int, default=0,
                   help="append N shared experts (each with the routed experts' shape) to the "
                        "routing and run them in the same launches (no e2e or training leg)")
    p.add_argument("--no-backward", action="store_true",
                   help="skip the training-step leg (forward with saved pre-activations + backward)")
    p.add_argument("--mxfp8", action="store_true",
                   help="experts in MXFP8 (E4M3 + E8M0 block scales): weights quantised once "
                        "before timing, activations quantised inside the step")
    p.add_argument("--cpu-seconds", type=float, default=10.0,
                   help="CPU work budget for the oracle baseline sample")
    p.add_argument("--no-sweep", action="store_true",
                   help="skip the maxvio sweep (skew1/skew10/skew20) that follows the large "
                        "workload")
    args = p.parse_args()
    if args.mxfp8 and (args.shared_experts or args.zero_copy):
        p.error("--mxfp8 runs its own permute-quantise path: it does not combine with "
                "--shared-experts or --zero-copy")
    return args


KERNEL_SOURCES = {
    # the files a kernel is compiled from: a recorded traffic figure holds only for them
    "up_gate": ["grouped_ffn.cu", "gemm_common.cuh", "ptx.cuh"],
    "up_gate_zc": ["grouped_ffn.cu", "gemm_common.cuh", "ptx.cuh"],
    "weight_grad": ["grouped_ffn_bwd.cu", "gemm_common.cuh", "ptx.cuh"],
    "up_gate_mx": ["grouped_ffn_mx.cu", "gemm_common.cuh", "ptx.cuh"],
}


def kernel_source_digest(kind: str) -> str | None:
    import hashlib

    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kind]:
        path = os.path.join(ROOT, "grouped_ffn_moe_b200", "csrc", name)
        if not os.path.exists(path):
            return None
        h.update(open(path, "rb").read())
    return h.hexdigest()


def profiled_traffic(kernel_key: str):
    """DRAM bytes per launch of a kernel from the ncu summary in profiles/, if it was taken
    on the current kernel sources (the summary records their sha256); else None.
    kernel_key is "<kind>/<workload>", kind a key of KERNEL_SOURCES."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path)).get(kernel_key)
    if not rec or rec.get("source_sha256") != kernel_source_digest(kernel_key.split("/")[0]):
        return None
    return rec.get("dram_bytes_per_launch")


def reduce_step_time(ms_local: float, world: int, device=None) -> float:
    """Step time of the whole job: the maximum over ranks (replicas run in lock step)."""
    if world <= 1:
        return ms_local
    import torch
    import torch.distributed as dist

    t = torch.tensor([ms_local], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, ms_step: float) -> float:
    """Whole-job tokens/s: every rank processes its own batch (weak scaling)."""
    return world * tokens_per_rank / (ms_step / 1e3)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- work model

def work_model(w, counts=None):
    """Algorithmic bytes and flops per stage (real rows only; no padding credited)."""
    S, H, Hp, E, K = w.S, w.H, w.Hp, w.E, w.K
    M = S * K
    active = E if counts is None else int((counts > 0).sum())
    m = {
        "permute_bytes": 2 * (S + M) * H + 12 * M + 8 * E,
        "permute_meta_bytes": 12 * M + 8 * E,  # metadata only (zero copy): ids in, maps out
        "combine_bytes": 2 * (M + S) * H + 8 * M,
        "active_experts": active,
    }
    if not w.identity_ffn:
        m["up_gate_flops"] = 4 * M * H * Hp
        m["up_gate_bytes"] = 2 * 2 * active * H * Hp + 2 * M * H + 2 * M * Hp
        # zero copy: the token rows come from x itself (each token's row at least once)
        m["up_gate_zc_bytes"] = 2 * 2 * active * H * Hp + 2 * S * H + 2 * M * Hp
        m["down_flops"] = 2 * M * H * Hp
        m["down_bytes"] = 2 * active * Hp * H + 2 * M * Hp + 2 * M * H
        # backward (weights read once per pass; fp32 weight gradients written once)
        m["combine_bwd_bytes"] = 2 * S * H + 4 * M * H + 8 * M
        m["permute_bwd_bytes"] = 2 * (M + S) * H + 4 * M
        m["down_bwd_flops"] = 2 * M * H * Hp
        m["down_bwd_bytes"] = 2 * active * Hp * H + 2 * M * H + 4 * 2 * M * Hp
        m["up_gate_bwd_flops"] = 4 * M * H * Hp
        m["up_gate_bwd_bytes"] = 2 * 2 * active * H * Hp + 2 * 2 * M * Hp + 2 * M * H
        m["wgrad_flops"] = 6 * M * H * Hp
        m["wgrad_bytes"] = 4 * 3 * E * H * Hp + 2 * M * (2 * H + 3 * Hp)
        # MXFP8: one byte per element plus one scale byte per 32 (weights, x_q, h_q)
        q = 33 / 32
        m["permute_mx_bytes"] = 2 * S * H + q * M * H + 12 * M + 8 * E
        m["up_gate_mx_bytes"] = q * (2 * active * H * Hp + M * H + M * Hp)
        m["down_mx_bytes"] = q * (active * Hp * H + M * Hp) + 2 * M * H
    return m


def stage_report(w, E, K, counts, mean, peaks, peak_src, mx=False, zero_copy=False,
                 shared=False):
    """Per-stage throughput and fractions of the measured peaks, and the roofline of the
    dominant kernel (the SwiGLU pass; the permutation for identity-expert workloads).
    mean: stage times in ms ("permute", "up_gate", "down", "ffn", "combine")."""
    wm = work_model(dataclasses.replace(w, E=E, K=K), counts)
    stages = {
        "permute": {"ms": mean["permute"],
                    "GB/s": wm["permute_mx_bytes" if mx else
                               ("permute_meta_bytes" if zero_copy else "permute_bytes")]
                    / (mean["permute"] / 1e3) / 1e9},
        "combine": {"ms": mean["combine"],
                    "GB/s": wm["combine_bytes"] / (mean["combine"] / 1e3) / 1e9},
    }
    if not w.identity_ffn:
        stages["up_gate"] = {"ms": mean["up_gate"],
                             "TFLOP/s": wm["up_gate_flops"] / (mean["up_gate"] / 1e3) / 1e12}
        stages["down"] = {"ms": mean["down"],
                          "TFLOP/s": wm["down_flops"] / (mean["down"] / 1e3) / 1e12}
        stages["grouped_ffn"] = {
            "ms": mean["ffn"],
            "TFLOP/s": (wm["up_gate_flops"] + wm["down_flops"]) / (mean["ffn"] / 1e3) / 1e12}
        # both fractions of each GEMM pass: of the tensor peak (for its dtype) and of HBM
        tpk = peaks["bf16_tflops"] * (2.0 if mx else 1.0)
        ug_b = wm["up_gate_mx_bytes" if mx else
                  ("up_gate_zc_bytes" if zero_copy else "up_gate_bytes")]
        dn_b = wm["down_mx_bytes" if mx else "down_bytes"]
        for key, byts in (("up_gate", ug_b), ("down", dn_b), ("grouped_ffn", ug_b + dn_b)):
            st = stages[key]
            st["GB/s"] = byts / (st["ms"] / 1e3) / 1e9
            st["frac_tensor"] = st["TFLOP/s"] / tpk
            st["frac_hbm"] = st["GB/s"] / peaks["hbm_gbs"]
        # dominant kernel: the SwiGLU (up/gate) pass
        flops, t_s = wm["up_gate_flops"], mean["up_gate"] / 1e3
        byts = wm["up_gate_mx_bytes" if mx else
                  ("up_gate_zc_bytes" if zero_copy else "up_gate_bytes")]
        kname = ("grouped_ffn_mx_kernel<true> (MXFP8 up/gate + SwiGLU + h quantisation)" if mx
                 else "grouped_ffn_kernel<3> (zero-copy up/gate + SwiGLU, gathered rows)"
                 if zero_copy else "grouped_ffn_kernel<0> (up/gate + SwiGLU)")
        # MXFP8: the measured bf16 peak times the nominal fp8:bf16 ratio (4.5 / 2.25)
        tpeak = peaks["bf16_tflops"] * (2.0 if mx else 1.0)
        ridge = tpeak * 1e12 / (peaks["hbm_gbs"] * 1e9)
        if flops / byts >= ridge:
            roof = {"kernel": kname, "bound": "tensor", "achieved": flops / t_s / 1e12,
                    "peak": tpeak, "unit": "TFLOP/s"}
        else:
            roof = {"kernel": kname, "bound": "hbm", "achieved": byts / t_s / 1e9,
                    "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        byts, t_s = wm["permute_bytes"], mean["permute"] / 1e3
        roof = {"kernel": "moe_permute (2 kernels)", "bound": "hbm", "achieved": byts / t_s / 1e9,
                "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    for key in ("permute", "combine"):
        stages[key]["frac_hbm"] = stages[key]["GB/s"] / peaks["hbm_gbs"]
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["peak_source"] = f"{peak_src} (burst)"
    if mx and roof["bound"] == "tensor":
        roof["peak_source"] = f"{peak_src} bf16 (burst) x 2, the nominal fp8:bf16 ratio"
    kind = "up_gate_mx" if mx else ("up_gate_zc" if zero_copy else "up_gate")
    # a capture holds for its own workload only (shared experts change the launch)
    roof["traffic"] = (profiled_traffic(f"{kind}/{w.name}")
                       if not (w.identity_ffn or shared) else None)
    return stages, roof


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples (every 50 ms) with host timestamps."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.samples = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gpu_id}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 8:
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        inside = [p for (t, p) in self.samples if t0 <= t <= t1]
        window = "timed region"
        if len(inside) < 3:  # short timed region: use every sample taken under load
            inside = [p for (t, p) in self.samples]
            window = "warm-up and timed region"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [v for v in (num(p[0]) for p in inside) if v is not None]
        mx = [v for v in (num(p[1]) for p in inside) if v is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for p in inside for i in range(4) if p[4 + i] == "Active"})
        pw = [v for v in (num(p[2]) for p in inside) if v is not None]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "power_w_max": max(pw) if pw else None, "samples": len(inside),
                "window": window}


# ----------------------------------------------------------------------------- L2 flush

class L2Flush:
    """Run before every step, outside the timed events: a 256 MiB write evicts the step's
    data from the 126 MB L2; a 256 MiB read of a second buffer then replaces the write's
    dirty lines with clean ones, so that their write-back to HBM happens here and not
    inside the first timed kernel of the step."""

    def __init__(self, torch, dev):
        self.torch = torch
        self.w = torch.empty(256 << 18, dtype=torch.float32, device=dev)
        self.r = torch.zeros(256 << 18, dtype=torch.float32, device=dev)
        self.out = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self, i=0):
        self.w.fill_(float(i))
        self.torch.sum(self.r, dim=0, out=self.out)


# ----------------------------------------------------------------------------- training leg

def measure_backward(moe, synth, torch, w, inp, dev, steps, warmup, flush, peaks, peak_src):
    """Training step of the layer: forward with saved pre-activations, then the backward
    (combine bwd -> down+SwiGLU bwd -> up/gate bwd -> fp32 weight gradients -> permute bwd),
    with CUDA events between the kernels; L2 flushed before every step."""
    buf = moe.LayerBuffers.allocate(w.S, w.H, w.Hp, w.E, w.K, dev, train=True)
    grads = moe.LayerGrads.allocate(w.S, w.H, w.Hp, w.E, w.K, dev)
    grad_out = synth.normal_bf16_into(torch.empty(w.S, w.H, dtype=torch.bfloat16, device=dev),
                                      w.seed, synth.TAG_GRAD)
    wg, wu, wd = inp["w_gate"], inp["w_up"], inp["w_down"]
    E, K = w.E, w.K

    def train_step(ev=None):
        rec = (lambda i: ev[i].record()) if ev is not None else (lambda i: None)
        rec(0)
        moe.moe_permute(inp["x"], inp["topk_ids"], E, buf.x_perm, buf.counts, buf.cu_seqlens,
                        buf.row_id_map, buf.perm_src, buf.maxvio, buf.max_count, buf.workspace,
                        buf.d_status)
        rec(1)
        moe.moe_grouped_ffn_up_gate_train(buf.x_perm, wg, wu, buf.cu_seqlens, buf.h, buf.gate_pre,
                                          buf.up_pre, buf.d_status)
        rec(2)
        moe.moe_grouped_ffn_down(buf.h, wd, buf.cu_seqlens, buf.y, buf.d_status)
        moe.moe_unpermute_combine(buf.y, buf.row_id_map, inp["route_w"], buf.out)
        rec(3)
        moe.moe_combine_backward(grad_out, buf.y, buf.row_id_map, inp["route_w"], grads.grad_y,
                                 grads.grad_route_w)
        rec(4)
        moe.moe_grouped_ffn_down_backward(grads.grad_y, wd, buf.gate_pre, buf.up_pre,
                                          buf.cu_seqlens, grads.d_gate, grads.d_up, buf.d_status)
        rec(5)
        moe.moe_grouped_ffn_up_gate_backward(grads.d_gate, grads.d_up, wg, wu, buf.cu_seqlens,
                                             grads.grad_x_perm, buf.d_status)
        rec(6)
        moe.moe_grouped_ffn_weight_grad(buf.x_perm, buf.h, grads.d_gate, grads.d_up, grads.grad_y,
                                        buf.cu_seqlens, grads.grad_w_gate, grads.grad_w_up,
                                        grads.grad_w_down, False, buf.d_status)
        rec(7)
        moe.moe_permute_backward(grads.grad_x_perm, buf.row_id_map, grads.grad_x, K)
        rec(8)

    for _ in range(warmup):
        flush()
        train_step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(9)] for _ in range(steps)]
    for i in range(steps):
        flush(i)
        train_step(evs[i])
    torch.cuda.synchronize()
    status = int(buf.d_status.item())
    if status != 0:
        raise RuntimeError(f"device status {status} in the training leg")
    names = ["permute", "up_gate_train", "down_and_combine", "combine_backward", "down_backward",
             "up_gate_backward", "weight_grad", "permute_backward"]
    ms = {n: sum(e[i].elapsed_time(e[i + 1]) for e in evs) / steps for i, n in enumerate(names)}
    wm = work_model(w, buf.counts.cpu().numpy())
    st = {
        "up_gate_train": {"ms": ms["up_gate_train"],
                          "TFLOP/s": wm["up_gate_flops"] / ms["up_gate_train"] / 1e9},
        "combine_backward": {"ms": ms["combine_backward"],
                             "GB/s": wm["combine_bwd_bytes"] / ms["combine_backward"] / 1e6},
        "down_backward": {"ms": ms["down_backward"],
                          "TFLOP/s": wm["down_bwd_flops"] / ms["down_backward"] / 1e9},
        "up_gate_backward": {"ms": ms["up_gate_backward"],
                             "TFLOP/s": wm["up_gate_bwd_flops"] / ms["up_gate_backward"] / 1e9},
        "weight_grad": {"ms": ms["weight_grad"],
                        "TFLOP/s": wm["wgrad_flops"] / ms["weight_grad"] / 1e9,
                        "GB/s": wm["wgrad_bytes"] / ms["weight_grad"] / 1e6},
        "permute_backward": {"ms": ms["permute_backward"],
                             "GB/s": wm["permute_bwd_bytes"] / ms["permute_backward"] / 1e6},
    }
    bwd_ms = sum(ms[n] for n in names[3:])
    # roofline of each backward GEMM pass: the slower of its tensor and HBM times
    for key, fk, bk in (("down_backward", "down_bwd_flops", "down_bwd_bytes"),
                        ("up_gate_backward", "up_gate_bwd_flops", "up_gate_bwd_bytes"),
                        ("weight_grad", "wgrad_flops", "wgrad_bytes")):
        t_tensor = wm[fk] / (peaks["bf16_tflops"] * 1e12)
        t_hbm = wm[bk] / (peaks["hbm_gbs"] * 1e9)
        bound = "tensor" if t_tensor >= t_hbm else "hbm"
        st[key]["bound"] = bound
        st[key]["frac_of_roofline"] = max(t_tensor, t_hbm) / (ms[key] / 1e3)
    dom = max(("down_backward", "up_gate_backward", "weight_grad"), key=lambda k: ms[k])
    d = st[dom]
    if d["bound"] == "tensor":
        roof = {"kernel": dom, "bound": "tensor", "achieved": d["TFLOP/s"],
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
    else:
        byts = {"down_backward": wm["down_bwd_bytes"], "up_gate_backward": wm["up_gate_bwd_bytes"],
                "weight_grad": wm["wgrad_bytes"]}[dom]
        roof = {"kernel": dom, "bound": "hbm", "achieved": byts / ms[dom] / 1e6,
                "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["peak_source"] = f"{peak_src} (burst)"
    roof["traffic"] = profiled_traffic(f"{dom}/{w.name}")
    return {"tokens_per_s": w.S / ((ms["permute"] + ms["up_gate_train"] + ms["down_and_combine"]
                                    + bwd_ms) / 1e3),
            "ms_training_step": sum(ms.values()), "ms_backward": bwd_ms,
            "forward_train_overhead_ms": ms["up_gate_train"],
            "stages": st, "roofline": roof,
            "gpu_launches_per_step": sum(moe.LAUNCHES[n] for n in (
                "moe_permute", "moe_grouped_ffn_up_gate_train", "moe_grouped_ffn_down",
                "moe_unpermute_combine", "moe_combine_backward", "moe_grouped_ffn_down_backward",
                "moe_grouped_ffn_up_gate_backward", "moe_grouped_ffn_weight_grad",
                "moe_permute_backward")),
            "weight_grad_dtype": "f32", "steps": steps, "warmup": warmup}


# ----------------------------------------------------------------------------- our arm

def run_ours(args):
    import torch
    import torch.distributed as dist

    import grouped_ffn_moe_b200 as moe
    import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = synth.WORKLOADS[args.workload]
    ns = args.shared_experts if not w.identity_ffn else 0
    inp = synth.make_layer_inputs(w, device=str(dev), n_shared=ns)
    E, K = w.E + ns, w.K + ns  # shared experts are experts E.. with one slot each per token
    buf = moe.LayerBuffers.allocate(w.S, w.H, w.Hp, E, K, dev, with_ffn=not w.identity_ffn)
    flush = L2Flush(torch, dev)
    if ns:
        ids_ext = torch.empty(w.S, K, dtype=torch.int32, device=dev)
        w_ext = torch.empty(w.S, K, dtype=torch.float32, device=dev)
        routed_mv = torch.empty(1, dtype=torch.float64, device=dev)
    ids_step = ids_ext if ns else inp["topk_ids"]
    w_step = w_ext if ns else inp["route_w"]

    mx = args.mxfp8 and not w.identity_ffn and not ns
    zero_copy = args.zero_copy and not w.identity_ffn and not mx
    if mx:
        # weights quantised once, ahead of the layer (not part of a step)
        mw = moe.MxWeights.from_bf16(inp["w_gate"], inp["w_up"], inp["w_down"])
        mxbufs = [moe.MxBuffers.allocate(w.S, w.H, w.Hp, K, dev)]
        mxbuf = mxbufs[0]
        torch.cuda.synchronize()

    def step(ev=None):
        if ev is not None:
            ev[0].record()
        if ns:
            moe.moe_append_shared(inp["topk_ids"], inp["route_w"], w.E, ns, ids_ext, w_ext)
        moe.moe_permute(inp["x"], ids_step, E, None if (zero_copy or mx) else buf.x_perm,
                        buf.counts, buf.cu_seqlens, buf.row_id_map, buf.perm_src, buf.maxvio,
                        buf.max_count, buf.workspace, buf.d_status)
        if mx:
            moe.moe_mx_permute_quantize(inp["x"], buf.row_id_map, K, mxbuf.x_q, mxbuf.x_sf)
        if ev is not None:
            ev[1].record()
        y = buf.x_perm
        if mx:
            moe.moe_grouped_ffn_up_gate_mxfp8(mxbuf.x_q, mxbuf.x_sf, mw, buf.cu_seqlens,
                                              mxbuf.h_q, mxbuf.h_sf, buf.d_status)
            if ev is not None:
                ev[2].record()
            moe.moe_grouped_ffn_down_mxfp8(mxbuf.h_q, mxbuf.h_sf, mw, buf.cu_seqlens, buf.y,
                                           buf.d_status)
            y = buf.y
        elif not w.identity_ffn:
            if zero_copy:
                moe.moe_grouped_ffn_up_gate_gather(inp["x"], buf.perm_src, K, inp["w_gate"],
                                                   inp["w_up"], buf.cu_seqlens, buf.h,
                                                   d_status=buf.d_status)
            else:
                moe.moe_grouped_ffn_up_gate(buf.x_perm, inp["w_gate"], inp["w_up"],
                                            buf.cu_seqlens, buf.h, buf.d_status)
            if ev is not None:
                ev[2].record()
            moe.moe_grouped_ffn_down(buf.h, inp["w_down"], buf.cu_seqlens, buf.y, buf.d_status)
            y = buf.y
        elif ev is not None:
            ev[2].record()
        if ev is not None:
            ev[3].record()
        moe.moe_unpermute_combine(y, buf.row_id_map, w_step, buf.out)
        if ns:  # the routed experts' imbalance
            moe.moe_maxvio(buf.counts[:w.E], w.S, w.K, routed_mv)
        if ev is not None:
            ev[4].record()

    # the metadata-only permute (zero copy) launches one kernel, not the row copy
    launches_per_step = (moe.LAUNCHES["moe_permute"] - (1 if (zero_copy or mx) else 0)
                         + moe.LAUNCHES["moe_unpermute_combine"]
                         + (moe.LAUNCHES["moe_mx_permute_quantize"] if mx else 0)
                         + (0 if w.identity_ffn else moe.LAUNCHES["moe_grouped_ffn"])
                         + (moe.LAUNCHES["moe_append_shared"] + moe.LAUNCHES["moe_maxvio"]
                            if ns else 0))

    gpu_id = str(local)
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    clocks = ClockSampler(gpu_id) if rank == 0 else None

    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize()
    if int(buf.d_status.item()) != 0:
        raise RuntimeError(f"device status {int(buf.d_status.item())} during warm-up")

    # timed region: one event pair per step, so consecutive kernels of a step overlap their
    # launch and prologue (programmatic dependent launch) as they do in use
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    for i in range(args.steps):
        flush(i)
        evs[i][0].record()
        step()
        evs[i][1].record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t1 = time.time()
    step_ms = [e[0].elapsed_time(e[1]) for e in evs]
    ms_step = reduce_step_time(sum(step_ms) / len(step_ms), world, dev)

    # stage breakdown (separate loop: events between the stages of every step)
    sevs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    for i in range(args.steps):
        flush(i)
        step(sevs[i])
    torch.cuda.synchronize()
    per = {k: [] for k in ("permute", "up_gate", "down", "ffn", "combine", "step")}
    for e in sevs:
        per["permute"].append(e[0].elapsed_time(e[1]))
        per["up_gate"].append(e[1].elapsed_time(e[2]))
        per["down"].append(e[2].elapsed_time(e[3]))
        per["ffn"].append(e[1].elapsed_time(e[3]))
        per["combine"].append(e[3].elapsed_time(e[4]))
        per["step"].append(e[0].elapsed_time(e[4]))
    mean = {k: sum(v) / len(v) for k, v in per.items()}
    status = int(buf.d_status.item())
    counts = buf.counts.cpu().numpy()
    maxvio = float((routed_mv if ns else buf.maxvio).item())

    # e2e: host (pinned) inputs -> device -> layer -> host output, every step, through the
    # public API. Served as a pipeline: step i+1's inputs go up and step i-1's output comes
    # back on copy streams while step i's kernels run (device inputs and outputs double
    # buffered); one event pair spans all K steps, so every step's copies are inside it. No
    # L2 flush between steps here: each step's inputs arrive over PCIe and the weights exceed
    # L2. The same steps run back to back on one stream give "e2e_serial".
    e2e = None
    if not args.no_e2e and not ns:
        hx = inp["x"].cpu().pin_memory()
        hids = inp["topk_ids"].cpu().pin_memory()
        hw = inp["route_w"].cpu().pin_memory()
        hout = [torch.empty(w.S, w.H, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        dx = [torch.empty_like(inp["x"]) for _ in range(2)]
        dids = [torch.empty_like(inp["topk_ids"]) for _ in range(2)]
        dw = [torch.empty_like(inp["route_w"]) for _ in range(2)]
        bufs = [buf, moe.LayerBuffers.allocate(w.S, w.H, w.Hp, E, K, dev,
                                               with_ffn=not w.identity_ffn)]
        if mx:
            mxbufs.append(moe.MxBuffers.allocate(w.S, w.H, w.Hp, K, dev))

        def layer(k, stream):
            if mx:
                return moe.moe_layer_forward_mxfp8(dx[k], dids[k], dw[k], mw, bufs[k], mxbufs[k],
                                                   stream=stream)
            return moe.moe_layer_forward(dx[k], dids[k], dw[k], inp.get("w_gate"),
                                         inp.get("w_up"), inp.get("w_down"), bufs[k],
                                         stream=stream, zero_copy=zero_copy)
        s_up, s_run, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev), \
            torch.cuda.Stream(dev)
        h2d_bytes = hx.numel() * 2 + hids.numel() * 4 + hw.numel() * 4
        d2h_bytes = hout[0].numel() * 2

        def run_pipelined(nsteps):
            ran = [None, None]   # per slot: compute done (dx, dids, dw of the slot free)
            read = [None, None]  # per slot: download done (out of the slot free)
            for i in range(nsteps):
                k = i % 2
                with torch.cuda.stream(s_up):
                    if ran[k] is not None:
                        s_up.wait_event(ran[k])
                    dx[k].copy_(hx, non_blocking=True)
                    dids[k].copy_(hids, non_blocking=True)
                    dw[k].copy_(hw, non_blocking=True)
                    up = torch.cuda.Event()
                    up.record(s_up)
                with torch.cuda.stream(s_run):
                    s_run.wait_event(up)
                    if read[k] is not None:
                        s_run.wait_event(read[k])
                    out = layer(k, s_run)
                    ran[k] = torch.cuda.Event()
                    ran[k].record(s_run)
                with torch.cuda.stream(s_down):
                    s_down.wait_event(ran[k])
                    hout[k].copy_(out, non_blocking=True)
                    read[k] = torch.cuda.Event()
                    read[k].record(s_down)

        def run_serial(nsteps):
            with torch.cuda.stream(s_run):
                for i in range(nsteps):
                    dx[0].copy_(hx, non_blocking=True)
                    dids[0].copy_(hids, non_blocking=True)
                    dw[0].copy_(hw, non_blocking=True)
                    out = layer(0, s_run)
                    hout[0].copy_(out, non_blocking=True)

        def timed(fn):
            fn(args.warmup)
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(s_up)
            s_run.wait_event(a)
            s_down.wait_event(a)
            fn(args.steps)
            s_down.wait_stream(s_up)
            s_down.wait_stream(s_run)
            b.record(s_down)
            torch.cuda.synchronize()
            return reduce_step_time(a.elapsed_time(b) / args.steps, world, dev)

        e2e_ms = timed(run_pipelined)
        last = (args.steps - 1) % 2
        if not torch.equal(hout[last].to(dev), buf.out):
            raise RuntimeError("e2e output differs from the device-resident run")
        serial_ms = timed(run_serial)
        e2e = {"value": job_throughput(w.S, world, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes,
               "ms_per_step": e2e_ms,
               "mode": "pipelined: uploads and downloads of neighbouring steps overlap this "
                       "step's kernels on separate streams; inputs fresh over PCIe every step, "
                       "weights larger than L2, no flush",
               "e2e_serial": {"value": job_throughput(w.S, world, serial_ms),
                              "ms_per_step": serial_ms}}

    backward = None
    if not w.identity_ffn and not args.no_backward and not ns and not mx:
        peaks0, src0 = load_peaks()
        backward = measure_backward(moe, synth, torch, w, inp, dev, args.steps, args.warmup, flush,
                                    peaks0, src0)

    cpu_base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu_base = (cpu_baseline_mx(w, inp, args.cpu_seconds) if mx
                    else cpu_baseline(w, inp, args.cpu_seconds))

    # flat in maxvio: the same step on the full-size geometry's skewed routings (maxvio 1, 10
    # and 20: each workload's own topk ids, route weights and x; the full-size layer's weights,
    # whose values do not change the work), timed interleaved with the default routing -- one
    # step per routing per round, the starting routing rotating from round to round, L2
    # flushed before every step -- so that clock and power drift over the run reaches all
    # four alike
    sweep = None
    if (w.name == "large" and not (mx or ns or zero_copy) and not args.no_sweep):
        names = ("large", "skew1", "skew10", "skew20")
        base_inp = inp
        variants = {"large": base_inp}
        for sname in names[1:]:
            sw = synth.WORKLOADS[sname]
            ids_np, rw_np = synth.routing_for(sw)
            v = dict(base_inp)
            v["topk_ids"] = torch.from_numpy(ids_np).to(dev)
            v["route_w"] = torch.from_numpy(rw_np).to(dev)
            v["x"] = synth.normal_bf16_into(torch.empty(sw.S, sw.H, dtype=torch.bfloat16,
                                                        device=dev), sw.seed, synth.TAG_X)
            variants[sname] = v

        def use(name):
            nonlocal inp, ids_step, w_step
            inp = variants[name]
            ids_step, w_step = inp["topk_ids"], inp["route_w"]

        mv_of = {}
        for name in names:  # warm-up, and each routing's measured maxvio
            use(name)
            for _ in range(args.warmup):
                flush()
                step()
            torch.cuda.synchronize()
            mv_of[name] = float(buf.maxvio.item())
        swevs = {n: [] for n in names}
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        for i in range(args.steps):
            for j in range(len(names)):
                name = names[(i + j) % len(names)]
                use(name)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                flush(i)
                e0.record()
                step()
                e1.record()
                swevs[name].append((e0, e1))
        torch.cuda.synchronize()
        if int(buf.d_status.item()) != 0:
            raise RuntimeError(f"device status {int(buf.d_status.item())} in the maxvio sweep")
        use("large")
        inp = base_inp
        sweep = {"method": "interleaved: one step per routing per round, rotating order, L2 "
                           "flushed before each step; skewed routings on the same weights"}
        for name in names:
            sms = reduce_step_time(sum(a.elapsed_time(b) for a, b in swevs[name]) / args.steps,
                                   world, dev)
            sweep[name] = {"ms_per_step": sms, "maxvio_measured": mv_of[name],
                           "tokens_per_s": job_throughput(w.S, world, sms)}
        t_all = [sweep[n]["ms_per_step"] for n in names]
        sweep["spread"] = (max(t_all) - min(t_all)) / min(t_all)
        variants = None

    if clocks is not None:
        clocks.stop()

    if rank == 0:
        peaks, peak_src = load_peaks()
        stages, roof = stage_report(w, E, K, counts, mean, peaks, peak_src, mx=mx,
                                    zero_copy=zero_copy, shared=bool(ns))
        line = {
            "metric": METRIC, "value": job_throughput(w.S, world, ms_step), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "mxfp8 (e4m3, e8m0 scales per 32; fp32 accumulate; bf16 y/out)" if mx
            else "bf16",
            "data": "synthetic (seeded SplitMix64/Box-Muller inputs, random-init expert weights)",
            "config": {"workload": w.name, "S": w.S, "H": w.H, "Hp": w.Hp, "E": w.E, "K": w.K,
                       "path": ("mxfp8 (permute fused with quantisation)" if mx else
                                "zero-copy (gather)" if zero_copy else "x_perm copy"),
                       "shared_experts": ns,
                       "routing": w.routing, "maxvio_measured": maxvio,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": "flushed before every step, outside the timed events: 256 MiB "
                             "write, then a 256 MiB read so the write-back happens there"},
            "stages": stages, "stage_sum_ms": mean["step"], "roofline": roof, "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "device_status": status,
            "clocks": clocks.summary(t0, t1) if clocks else None,
        }
        if backward is not None:
            line["training_step"] = backward
        if sweep is not None:
            line["maxvio_sweep"] = sweep
        if cpu_base is not None:
            line["cpu_baseline"] = cpu_base
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ----------------------------------------------------------------------------- CPU oracle

def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _oracle_sample(w, S_sample, host):
    """Oracle layer on the first S_sample tokens of the workload. host: dict of numpy bits."""
    from oracle import moe_oracle as O

    ids = host["topk_ids"][:S_sample]
    return O.moe_layer(host["x"][:S_sample], ids, host["route_w"][:S_sample], w.E, host["get"],
                       w.Hp, identity_ffn=w.identity_ffn)


def _host_inputs_from_device(w, inp):
    """Host copies (numpy bits) of one layer's inputs for the oracle. Expert weights are
    fetched from the device one expert at a time, when the oracle first asks for them, so
    that a sample of a few tokens copies only the experts it visits."""
    import numpy as np
    import torch

    def bits(t):
        return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)

    host = {"x": bits(inp["x"]), "topk_ids": inp["topk_ids"].cpu().numpy(),
            "route_w": inp["route_w"].cpu().numpy(), "get": None}
    if not w.identity_ffn:
        cache = {}

        def get(e):
            if e not in cache:
                cache[e] = (bits(inp["w_gate"][e]), bits(inp["w_up"][e]), bits(inp["w_down"][e]))
            return cache[e]
        host["get"] = get
    return host


def _host_inputs_generated(w):
    """The same inputs made on the host by the generator (counter-based draws, identical to
    the device's); an expert's weights are generated when the oracle first asks for them."""
    import synth

    ids, rw = synth.routing_for(w)
    host = {"x": synth.normal_bf16_bits(w.seed, synth.TAG_X, w.S * w.H).reshape(w.S, w.H),
            "topk_ids": ids, "route_w": rw, "get": None}
    if not w.identity_ffn:
        cache = {}

        def get(e):
            if e not in cache:
                n = w.H * w.Hp
                cache[e] = tuple(
                    synth.normal_bf16_bits(w.seed, tag, n, synth.weight_scale(w, which),
                                           offset=e * n).reshape(shape)
                    for tag, which, shape in ((synth.TAG_W_GATE, "gate", (w.H, w.Hp)),
                                              (synth.TAG_W_UP, "up", (w.H, w.Hp)),
                                              (synth.TAG_W_DOWN, "down", (w.Hp, w.H))))
            return cache[e]
        host["get"] = get
    return host


def _sample_tokens(w):
    """Tokens per oracle sample: a few seconds of host work at most per pass (the full-size
    geometry's two tokens visit 16 experts, 1.4 GB of weights)."""
    return {"tiny": 256, "medium": 128}.get(w.name, 2 if not w.identity_ffn else 1024)


def cpu_baseline(w, inp, budget_s):
    host = _host_inputs_from_device(w, inp)
    S_sample = min(w.S, _sample_tokens(w))
    done, t_start = 0, time.perf_counter()
    while True:
        _oracle_sample(w, S_sample, host)
        done += S_sample
        el = time.perf_counter() - t_start
        if el >= budget_s:
            break
    return {"value": done / el, "unit": UNIT, "cores": _cores(), "kind": "oracle",
            "sample": f"first {S_sample} tokens of workload {w.name} (full weights), "
                      f"repeated for {el:.1f} s; numpy fp64"}


def _mx_oracle_setup(w, host, n_tokens):
    """The first n_tokens tokens of the workload and the MXFP8 weights of the experts they
    visit, quantised by the oracle (ahead of timing, as the GPU run quantises its weights)."""
    import numpy as np

    from oracle import moe_oracle as O

    ids = host["topk_ids"][:n_tokens]
    qw = {}
    for e in sorted(set(int(v) for v in np.asarray(ids).ravel())):
        wg, wu, wd = host["get"](e)
        qw[e] = (O.mx_weights(wg), O.mx_weights(wu), O.mx_weights(wd))
    return ids, qw


def _oracle_sample_mx(w, host, ids, qw):
    """The oracle's MXFP8 layer on the tokens of `ids`: permutation, expert_ffn_rows_mxfp8
    per expert (x and h quantised inside), combine."""
    import numpy as np

    from oracle import moe_oracle as O

    S, K = ids.shape
    counts, cu, rmap, psrc = O.permute_metadata(ids, w.E)
    x_perm = O.permute_rows(host["x"][:S], psrc, K)
    y = np.zeros((S * K, w.H), np.uint16)
    for e in range(w.E):
        r0, r1 = int(cu[e]), int(cu[e + 1])
        if r1 > r0:
            y[r0:r1] = O.expert_ffn_rows_mxfp8(x_perm[r0:r1], *qw[e])[2]
    return O.unpermute_combine(y, rmap, host["route_w"][:S], S, K)


def cpu_baseline_mx(w, inp, budget_s, n_tokens=2):
    """The oracle's MXFP8 layer on the first n_tokens tokens, repeated for budget_s."""
    host = _host_inputs_from_device(w, inp)
    ids, qw = _mx_oracle_setup(w, host, n_tokens)
    done, t_start = 0, time.perf_counter()
    while True:
        _oracle_sample_mx(w, host, ids, qw)
        done += n_tokens
        el = time.perf_counter() - t_start
        if el >= budget_s:
            break
    return {"value": done / el, "unit": UNIT, "cores": _cores(), "kind": "oracle",
            "sample": f"first {n_tokens} tokens of workload {w.name}, MXFP8 oracle path (weights "
                      f"of their {len(qw)} experts quantised beforehand), repeated for {el:.1f} s; "
                      f"numpy fp64"}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import synth

    w = synth.WORKLOADS[args.workload]
    host = _host_inputs_generated(w)
    mx = args.mxfp8 and not w.identity_ffn
    if mx:
        S_sample = 2
        ids, qw = _mx_oracle_setup(w, host, S_sample)
        run = lambda: _oracle_sample_mx(w, host, ids, qw)  # noqa: E731
    else:
        S_sample = min(w.S, _sample_tokens(w))
        run = lambda: _oracle_sample(w, S_sample, host)  # noqa: E731
    for _ in range(args.warmup):
        run()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        run()
        times.append(time.perf_counter() - t0)
    sec = sum(times) / len(times)
    value = S_sample / sec
    sample = (f"first {S_sample} of {w.S} tokens of workload {w.name} per step (full weights); "
              f"numpy fp64 oracle" + (", MXFP8 path (the visited experts' weights quantised "
                                      "before timing)" if mx else ""))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": w.name, "S": w.S, "H": w.H, "Hp": w.Hp,
                                        "E": w.E, "K": w.K, "routing": w.routing,
                                        "path": "mxfp8" if mx else "bf16"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": _cores(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
