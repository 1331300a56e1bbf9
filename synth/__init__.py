"""Seeded synthetic inputs for the MoE layer (permute -> grouped SwiGLU FFN -> combine).

This package only draws numbers; it holds none of the layer's arithmetic. Both the
CPU oracle (in tests) and the CUDA path consume the bytes it produces.

Streams: the i-th draw of stream (seed, tag) is output i+1 of SplitMix64 (Steele,
Lea & Flood, OOPSLA 2014) started at mix64(seed * GAMMA + tag). Normals use the
cosine branch of Box-Muller with one pair of uniforms per value, in double, then
float (RN), then bf16 (RNE). Large tensors are made on the GPU by a CUDA twin of
the host generator (same formulas, no contraction); any slice can be re-made on the
host.

Workloads follow the MoonEP benchmark geometry and the page-4 worked example of the
pages this layer is built from ("MoonEP" README, Performance; "Distributed expert
parallelism", A four-rank example).
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIBDIR = os.path.join(_HERE, "_lib")
HOST_LIB = os.path.join(_LIBDIR, "libmoe_synth_host.so")
GPU_LIB = os.path.join(_LIBDIR, "libmoe_synth_gpu.so")

GAMMA = 0x9E3779B97F4A7C15

# Stream tags: one per tensor so that tensors never share draws.
TAG_X = 1
TAG_W_GATE = 2
TAG_W_UP = 3
TAG_W_DOWN = 4
TAG_ROUTE = 5
TAG_LOGIT = 6
TAG_PERM = 7
TAG_GRAD = 8


# ----------------------------------------------------------------------------- build

def build(verbose: bool = False) -> None:
    """Compile the host generator (gcc + OpenMP) and its CUDA twin (nvcc, sm_100a)."""
    import subprocess

    os.makedirs(_LIBDIR, exist_ok=True)
    src_c = os.path.join(_HERE, "csrc", "synth_host.c")
    src_cu = os.path.join(_HERE, "csrc", "synth_gpu.cu")
    cmds = [
        ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
         "-fno-fast-math", src_c, "-o", HOST_LIB, "-lm"],
        ["nvcc", "-O2", "-shared", "-Xcompiler", "-fPIC", "--fmad=false",
         "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", src_cu, "-o", GPU_LIB],
    ]
    for c in cmds:
        if verbose:
            print(" ".join(c))
        subprocess.run(c, check=True)


_host = None
_gpu = None


def _host_lib():
    global _host
    if _host is None:
        if not os.path.exists(HOST_LIB):
            build()
        lib = ctypes.CDLL(HOST_LIB)
        u64, i64, i32 = ctypes.c_uint64, ctypes.c_int64, ctypes.c_int32
        p = ctypes.c_void_p
        lib.synth_draw64.restype = u64
        lib.synth_draw64.argtypes = [u64, u64, u64]
        lib.synth_uniform.argtypes = [u64, u64, u64, i64, p]
        lib.synth_normal_f64.argtypes = [u64, u64, u64, i64, p]
        lib.synth_normal_bf16.argtypes = [u64, u64, u64, i64, ctypes.c_double, p]
        lib.synth_route.restype = i64
        lib.synth_route.argtypes = [u64, u64, i64, i32, i32, i32, ctypes.c_double, i64, p]
        _host = lib
    return _host


def _gpu_lib():
    global _gpu
    if _gpu is None:
        if not os.path.exists(GPU_LIB):
            raise RuntimeError(f"GPU generator not built: {GPU_LIB} (run synth.build())")
        lib = ctypes.CDLL(GPU_LIB)
        lib.synth_normal_bf16_gpu.restype = ctypes.c_int
        lib.synth_normal_bf16_gpu.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64,
                                              ctypes.c_int64, ctypes.c_double, ctypes.c_void_p,
                                              ctypes.c_void_p]
        _gpu = lib
    return _gpu


# ----------------------------------------------------------------------------- draws

def draw64(seed: int, tag: int, i: int) -> int:
    return int(_host_lib().synth_draw64(seed, tag, i))


def uniform(seed: int, tag: int, n: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _host_lib().synth_uniform(seed, tag, offset, n, out.ctypes.data)
    return out


def normal_f64(seed: int, tag: int, n: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _host_lib().synth_normal_f64(seed, tag, offset, n, out.ctypes.data)
    return out


def normal_bf16_bits(seed: int, tag: int, n: int, scale: float = 1.0, offset: int = 0) -> np.ndarray:
    """n bf16 values (as uint16 bit patterns) of N(0, scale^2), made on the host."""
    out = np.empty(n, dtype=np.uint16)
    if n:
        _host_lib().synth_normal_bf16(seed, tag, offset, n, float(scale), out.ctypes.data)
    return out


def normal_bf16_into(t, seed: int, tag: int, scale: float = 1.0, offset: int = 0, stream=None):
    """Fill a contiguous torch bf16 tensor with the same values normal_bf16_bits gives.

    CUDA tensors are filled by the device twin; CPU tensors by the host generator.
    """
    import torch

    assert t.dtype == torch.bfloat16 and t.is_contiguous()
    n = t.numel()
    if n == 0:
        return t
    if t.is_cuda:
        if stream is None:
            stream = torch.cuda.current_stream(t.device).cuda_stream
        rc = _gpu_lib().synth_normal_bf16_gpu(seed, tag, offset, n, float(scale), t.data_ptr(), stream)
        if rc != 0:
            raise RuntimeError(f"synth_normal_bf16_gpu failed with code {rc}")
    else:
        bits = normal_bf16_bits(seed, tag, n, scale, offset)
        t.view(torch.int16).copy_(torch.from_numpy(bits.view(np.int16)).view(t.shape))
    return t


# ----------------------------------------------------------------------------- routing

def route_es(seed: int, S: int, K: int, E: int, hot_e: int = -1, w_hot: float = 1.0,
             cap: int = 0) -> tuple[np.ndarray, int]:
    """Top-K distinct experts per token by Efraimidis-Spirakis keys (see synth_host.c)."""
    ids = np.empty(S * K, dtype=np.int32)
    hot = _host_lib().synth_route(seed, TAG_ROUTE, S, K, E, hot_e, float(w_hot), int(cap),
                                  ids.ctypes.data)
    if hot < 0:
        raise MemoryError("synth_route: allocation failed")
    return ids.reshape(S, K), int(hot)


def route_capped_for_maxvio(seed: int, S: int, K: int, E: int, target: float, hot_e: int = 0,
                            steps: int = 30) -> tuple[np.ndarray, float]:
    """Routing whose hot expert reaches cap = floor((1+target) * S*K/E).

    Every expert is capped at `cap`, so no expert exceeds it; w_hot is the smallest
    weight (bisection on [1, 1e4] at the geometric midpoint) at which the hot count
    reaches the cap. The hot count is monotone in w_hot because the uniforms are fixed.
    Returns (ids [S,K], w_hot).
    """
    cap = int(math.floor((1.0 + target) * S * K / E))
    lo, hi = 1.0, 1.0e4
    ids_hi, hot = route_es(seed, S, K, E, hot_e, hi, cap)
    if hot < cap:
        return ids_hi, hi
    best = (ids_hi, hi)
    for _ in range(steps):
        mid = math.sqrt(lo * hi)
        ids, hot = route_es(seed, S, K, E, hot_e, mid, cap)
        if hot >= cap:
            hi, best = mid, (ids, mid)
        else:
            lo = mid
    return best


def route_balanced(seed: int, S: int, K: int, E: int) -> np.ndarray:
    """Round-robin routing e(t,k) = pi((t*K + k) mod E) with a seeded relabelling pi.

    Every expert gets floor or ceil of S*K/E rows; K <= E keeps a token's experts distinct.
    """
    perm = np.arange(E, dtype=np.int64)
    for i in range(E - 1, 0, -1):  # Fisher-Yates
        j = draw64(seed, TAG_PERM, i) % (i + 1)
        perm[i], perm[j] = perm[j], perm[i]
    f = np.arange(S * K, dtype=np.int64)
    return perm[f % E].astype(np.int32).reshape(S, K)


def route_weights(seed: int, S: int, K: int) -> np.ndarray:
    """Softmax over the K slots of N(0,1) logits, computed in double, stored as float32."""
    z = normal_f64(seed, TAG_LOGIT, S * K).reshape(S, K)
    z = z - z.max(axis=1, keepdims=True)
    ez = np.exp(z)
    return (ez / ez.sum(axis=1, keepdims=True)).astype(np.float32)


# ----------------------------------------------------------------------------- configs

@dataclass(frozen=True)
class Workload:
    """One synthetic MoE-layer workload. Hp is H' (expert intermediate size)."""

    name: str
    S: int
    H: int
    Hp: int
    E: int
    K: int
    seed: int
    routing: str = "uniform"  # "uniform" | "capped" | "balanced"
    maxvio_target: float = 0.0
    hot_e: int = 0
    identity_ffn: bool = False  # permute/combine-only workloads
    note: str = field(default="", compare=False)

    @property
    def M(self) -> int:
        return self.S * self.K


def _c5(S: int, mv: float) -> Workload:
    routing = "balanced" if mv == 0 else "capped"
    return Workload(f"permute_combine_S{S}_mv{int(mv)}", S, 7168, 0, 384, 8, 6, routing, float(mv),
                    identity_ffn=True, note="identity experts; only permute and combine bytes count")


WORKLOADS: dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny", 256, 256, 512, 8, 2, 0, "uniform"),
        Workload("medium", 4096, 2048, 1408, 64, 6, 1, "uniform"),
        Workload("large", 8192, 7168, 2048, 384, 8, 2, "capped", 0.2),
        Workload("skew1", 8192, 7168, 2048, 384, 8, 3, "capped", 1.0),
        Workload("skew10", 8192, 7168, 2048, 384, 8, 4, "capped", 10.0),
        Workload("skew20", 8192, 7168, 2048, 384, 8, 5, "capped", 20.0),
        Workload("skew20_last", 8192, 7168, 2048, 384, 8, 5, "capped", 20.0, hot_e=383),
        # per-expert shape of "large" (171 rows per expert) on 32 experts: 2.8 GB of weights,
        # small enough for detailed profiler captures
        Workload("large_slice", 684, 7168, 2048, 32, 8, 2, "capped", 0.2),
        # the same per-expert shape on 8 experts (K = E: every token visits each once); the
        # training step's fp32 weight gradients stay at 1.4 GB, small enough for captures of
        # the backward kernels
        Workload("large_slice_e8", 171, 7168, 2048, 8, 8, 2, "uniform"),
    ]
    + [_c5(S, mv) for S in (1024, 4096, 16384, 65536) for mv in (0, 1, 20)]
}


def routing_for(w: Workload) -> tuple[np.ndarray, np.ndarray]:
    """(topk_ids [S,K] int32, route_w [S,K] float32) for a workload."""
    if w.routing == "uniform":
        ids, _ = route_es(w.seed, w.S, w.K, w.E)
    elif w.routing == "capped":
        ids, _ = route_capped_for_maxvio(w.seed, w.S, w.K, w.E, w.maxvio_target, w.hot_e)
    elif w.routing == "balanced":
        ids = route_balanced(w.seed, w.S, w.K, w.E)
    else:
        raise ValueError(w.routing)
    return ids, route_weights(w.seed, w.S, w.K)


def weight_scale(w: Workload, which: str) -> float:
    """1/sqrt(fan_in): fan_in = H for gate/up, H' for down."""
    return 1.0 / math.sqrt(w.H if which in ("gate", "up") else w.Hp)


def make_layer_inputs(w: Workload, device: str = "cpu", n_shared: int = 0):
    """All inputs of one layer call as torch tensors on `device`.

    Returns dict with x [S,H] bf16, topk_ids [S,K] int32, route_w [S,K] fp32 and, unless
    the workload uses identity experts, w_gate/w_up [E',H,H'] and w_down [E',H',H] bf16 with
    E' = E + n_shared: the shared experts' weights follow the routed ones in the same
    tensors (draws are counter-based, so the routed experts' weights do not change).
    """
    import torch

    ids, rw = routing_for(w)
    out = {
        "topk_ids": torch.from_numpy(ids).to(device),
        "route_w": torch.from_numpy(rw).to(device),
        "x": normal_bf16_into(torch.empty(w.S, w.H, dtype=torch.bfloat16, device=device),
                              w.seed, TAG_X),
    }
    if not w.identity_ffn:
        E2 = w.E + n_shared
        for name, tag, shape in (("w_gate", TAG_W_GATE, (E2, w.H, w.Hp)),
                                 ("w_up", TAG_W_UP, (E2, w.H, w.Hp)),
                                 ("w_down", TAG_W_DOWN, (E2, w.Hp, w.H))):
            t = torch.empty(*shape, dtype=torch.bfloat16, device=device)
            out[name] = normal_bf16_into(t, w.seed, tag, weight_scale(w, name[2:]))
    return out
