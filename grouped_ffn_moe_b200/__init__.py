"""Python binding of libmoe_b200.so (include/moe_b200.h): the single-GPU MoE hot path.

Argument marshalling only. Every step runs in the CUDA kernels of libmoe_b200.so;
PyTorch provides device memory and the current stream. There is no CPU fallback: if
the library is missing, every call raises.

Functions carry the C ABI's names:
    moe_permute, moe_grouped_ffn (= moe_grouped_ffn_up_gate + moe_grouped_ffn_down),
    moe_unpermute_combine, moe_maxvio, moe_permute_workspace_bytes, moe_status_string
plus `LayerBuffers` / `moe_layer_forward`, which allocate the layer's buffers once and
chain the three calls (permute -> grouped FFN -> combine) on one stream; the backward
(`moe_layer_backward` and its per-stage calls), the in-place token gather
(`moe_grouped_ffn_gather`), shared experts (`moe_append_shared`) and MXFP8 experts
(`moe_mx_quantize_weights`, `moe_mx_permute_quantize`, `moe_grouped_ffn_mxfp8`, with
`MxWeights` / `MxBuffers` / `moe_layer_forward_mxfp8`).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_INVALID_ARGUMENT = 1
MOE_ERR_UNSUPPORTED_SHAPE = 2
MOE_ERR_CUDA = 3
MOE_ERR_BAD_ROUTING = 4
MOE_ERR_DEVICE_TIMEOUT = 8
MOE_MAX_EXPERTS = 65535
MOE_MAX_FFN_EXPERTS = 1024

# Kernels launched by one call of each entry point (permute with a row copy).
LAUNCHES = {"moe_permute": 2, "moe_grouped_ffn": 2, "moe_grouped_ffn_up_gate": 1,
            "moe_grouped_ffn_down": 1, "moe_unpermute_combine": 1, "moe_maxvio": 1,
            "moe_combine_backward": 1, "moe_permute_backward": 1,
            "moe_grouped_ffn_up_gate_train": 1, "moe_grouped_ffn_down_backward": 1,
            "moe_grouped_ffn_up_gate_backward": 1, "moe_grouped_ffn_weight_grad": 1,
            "moe_grouped_ffn_backward": 3, "moe_grouped_ffn_gather": 2,
            "moe_grouped_ffn_up_gate_gather": 1, "moe_append_shared": 1,
            "moe_mx_quantize_weights": 1, "moe_mx_permute_quantize": 1,
            "moe_grouped_ffn_mxfp8": 2, "moe_grouped_ffn_up_gate_mxfp8": 1,
            "moe_grouped_ffn_down_mxfp8": 1}


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {moe_status_string(status)} (status {status})")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run grouped_ffn_moe_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        i32, i64, p, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_status_string.argtypes = [i32]
        L.moe_abi_version.restype = i32
        L.moe_abi_version.argtypes = []
        L.moe_permute_workspace_bytes.restype = sz
        L.moe_permute_workspace_bytes.argtypes = [i64, i32, i32]
        L.moe_permute.restype = i32
        L.moe_permute.argtypes = [p, p, i64, i64, i32, i32, p, p, p, p, p, p, p, p, sz, p, p]
        L.moe_permute_no_alloc.restype = i32
        L.moe_permute_no_alloc.argtypes = [p, p, i64, i64, i32, i32, p, p, p, p, p, p, p, p, p]
        L.moe_grouped_ffn.restype = i32
        L.moe_grouped_ffn.argtypes = [p, p, p, p, p, i64, i64, i64, i32, p, p, p, p]
        L.moe_grouped_ffn_up_gate.restype = i32
        L.moe_grouped_ffn_up_gate.argtypes = [p, p, p, p, i64, i64, i64, i32, p, p, p]
        L.moe_grouped_ffn_down.restype = i32
        L.moe_grouped_ffn_down.argtypes = [p, p, p, i64, i64, i64, i32, p, p, p]
        L.moe_unpermute_combine.restype = i32
        L.moe_unpermute_combine.argtypes = [p, p, p, i64, i64, i32, p, p]
        L.moe_combine_backward.restype = i32
        L.moe_combine_backward.argtypes = [p, p, p, p, i64, i64, i32, p, p, p]
        L.moe_permute_backward.restype = i32
        L.moe_permute_backward.argtypes = [p, p, i64, i64, i32, p, p]
        L.moe_maxvio.restype = i32
        L.moe_maxvio.argtypes = [p, i32, i64, i32, p, p, p]
        L.moe_grouped_ffn_up_gate_train.restype = i32
        L.moe_grouped_ffn_up_gate_train.argtypes = [p, p, p, p, i64, i64, i64, i32, p, p, p, p, p]
        L.moe_grouped_ffn_down_backward.restype = i32
        L.moe_grouped_ffn_down_backward.argtypes = [p, p, p, p, p, i64, i64, i64, i32, p, p, p, p]
        L.moe_grouped_ffn_up_gate_backward.restype = i32
        L.moe_grouped_ffn_up_gate_backward.argtypes = [p, p, p, p, p, i64, i64, i64, i32, p, p, p]
        L.moe_grouped_ffn_weight_grad.restype = i32
        L.moe_grouped_ffn_weight_grad.argtypes = [p, p, p, p, p, p, i64, i64, i64, i32, p, p, p,
                                                  i32, p, p]
        L.moe_grouped_ffn_gather.restype = i32
        L.moe_grouped_ffn_gather.argtypes = [p, p, i64, i32, p, p, p, p, i64, i64, i32, p, p, p, p]
        L.moe_grouped_ffn_up_gate_gather.restype = i32
        L.moe_grouped_ffn_up_gate_gather.argtypes = [p, p, i64, i32, p, p, p, i64, i64, i32, p, p,
                                                     p, p, p]
        L.moe_append_shared.restype = i32
        L.moe_append_shared.argtypes = [p, p, i64, i32, i32, i32, p, p, p]
        L.moe_grouped_ffn_backward.restype = i32
        L.moe_grouped_ffn_backward.argtypes = [p, p, p, p, p, p, p, p, i64, i64, i64, i32, p, p,
                                               p, p, p, p, p, i32, p, p]
        L.moe_mx_weight_scale_bytes.restype = sz
        L.moe_mx_weight_scale_bytes.argtypes = [i32, i64, i64]
        L.moe_mx_quantize_weights.restype = i32
        L.moe_mx_quantize_weights.argtypes = [p, i32, i64, i64, p, p, p]
        L.moe_mx_permute_quantize.restype = i32
        L.moe_mx_permute_quantize.argtypes = [p, p, i64, i64, i32, p, p, p]
        L.moe_grouped_ffn_mxfp8.restype = i32
        L.moe_grouped_ffn_mxfp8.argtypes = [p, p, p, p, p, p, p, p, p, i64, i64, i64, i32, p, p,
                                            p, p, p]
        L.moe_grouped_ffn_up_gate_mxfp8.restype = i32
        L.moe_grouped_ffn_up_gate_mxfp8.argtypes = [p, p, p, p, p, p, p, i64, i64, i64, i32, p, p,
                                                    p, p]
        L.moe_grouped_ffn_down_mxfp8.restype = i32
        L.moe_grouped_ffn_down_mxfp8.argtypes = [p, p, p, p, p, i64, i64, i64, i32, p, p, p]
        _lib = L
    return _lib


def moe_status_string(status: int) -> str:
    return lib().moe_status_string(int(status)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device=None):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn: str, status: int):
    if status != MOE_OK:
        raise MoeError(fn, status)


def _need(t, name, dtype, device=None, ndim=None):
    if t is None:
        return
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name}: expected {ndim} dims, got {t.dim()}")


def moe_permute_workspace_bytes(S: int, K: int, E: int) -> int:
    return int(lib().moe_permute_workspace_bytes(S, K, E))


def _permute_check(x, topk_ids, E, x_perm, counts, cu_seqlens, row_id_map, perm_src, maxvio,
                   max_count, d_status):
    """Dtypes, devices and sizes of moe_permute's buffers (the C ABI cannot see sizes, so a
    short buffer is refused here, before any launch). Returns (S, K, H)."""
    if topk_ids is None or counts is None or cu_seqlens is None or row_id_map is None:
        raise ValueError("topk_ids, counts, cu_seqlens and row_id_map are required")
    if topk_ids.dim() != 2 or (x is not None and x.dim() != 2):
        raise ValueError("topk_ids must be [S,K] and x [S,H]")
    S, K = topk_ids.shape
    H = x.shape[1] if x is not None else 0
    if x is not None and x.shape[0] != S:
        raise ValueError(f"x: expected {S} rows, got {x.shape[0]}")
    if x_perm is not None and (x is None or tuple(x_perm.shape) != (S * K, H)):
        raise ValueError(f"x_perm: expected {(S * K, H)} (and x), got {tuple(x_perm.shape)}")
    if counts.numel() != E or cu_seqlens.numel() != E + 1 or row_id_map.numel() != S * K:
        raise ValueError("counts/cu_seqlens/row_id_map sizes do not match (S, K, E)")
    if perm_src is not None and perm_src.numel() != S * K:
        raise ValueError("perm_src: expected S*K entries")
    for t, n in ((maxvio, "maxvio"), (max_count, "max_count"), (d_status, "d_status")):
        if t is not None and t.numel() < 1:
            raise ValueError(f"{n}: needs one element")
    dev = topk_ids.device
    _need(topk_ids, "topk_ids", torch.int32, dev, 2)
    _need(x, "x", torch.bfloat16, dev, 2)
    _need(x_perm, "x_perm", torch.bfloat16, dev, 2)
    for t, n in ((counts, "counts"), (cu_seqlens, "cu_seqlens"), (row_id_map, "row_id_map"),
                 (perm_src, "perm_src"), (max_count, "max_count"), (d_status, "d_status")):
        _need(t, n, torch.int32, dev)
    _need(maxvio, "maxvio", torch.float64, dev)
    return S, K, H


def moe_permute(x, topk_ids, E, x_perm, counts, cu_seqlens, row_id_map, perm_src=None, maxvio=None,
                max_count=None, workspace=None, d_status=None, stream=None):
    """Route top-k copies into expert-contiguous order (see include/moe_b200.h)."""
    S, K, H = _permute_check(x, topk_ids, E, x_perm, counts, cu_seqlens, row_id_map, perm_src,
                             maxvio, max_count, d_status)
    dev = topk_ids.device
    need = moe_permute_workspace_bytes(S, K, E)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().moe_permute(_ptr(x), _ptr(topk_ids), S, H, K, E, _ptr(x_perm), _ptr(counts),
                           _ptr(cu_seqlens), _ptr(row_id_map), _ptr(perm_src), _ptr(maxvio),
                           _ptr(max_count), _ptr(workspace), wbytes, _ptr(d_status),
                           _stream(stream, dev))
    _check("moe_permute", st)


MOE_NO_ALLOC_SCRATCH_BYTES = 4 << 20


def moe_permute_no_alloc(x, topk_ids, E, x_perm, counts, cu_seqlens, row_id_map, perm_src=None,
                         maxvio=None, max_count=None, d_status=None, stream=None):
    """moe_permute without a workspace argument, for callers that may not allocate device
    memory: the scratch is a fixed 4 MiB array inside the library (see include/moe_b200.h
    for the size limit and the sharing rules). Allocates nothing."""
    S, K, H = _permute_check(x, topk_ids, E, x_perm, counts, cu_seqlens, row_id_map, perm_src,
                             maxvio, max_count, d_status)
    dev = topk_ids.device
    st = lib().moe_permute_no_alloc(_ptr(x), _ptr(topk_ids), S, H, K, E, _ptr(x_perm),
                                    _ptr(counts), _ptr(cu_seqlens), _ptr(row_id_map),
                                    _ptr(perm_src), _ptr(maxvio), _ptr(max_count),
                                    _ptr(d_status), _stream(stream, dev))
    _check("moe_permute_no_alloc", st)


def moe_grouped_ffn(x_perm, w_gate, w_up, w_down, cu_seqlens, h_scratch, y, d_status=None,
                    stream=None):
    """Grouped SwiGLU expert FFN over expert-contiguous rows (see include/moe_b200.h)."""
    M, H = x_perm.shape
    E, H2, Hp = w_gate.shape
    dev = x_perm.device
    for t, n in ((x_perm, "x_perm"), (h_scratch, "h_scratch"), (y, "y")):
        _need(t, n, torch.bfloat16, dev, 2)
    for t, n in ((w_gate, "w_gate"), (w_up, "w_up"), (w_down, "w_down")):
        _need(t, n, torch.bfloat16, dev, 3)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    _need(d_status, "d_status", torch.int32, dev)
    if H2 != H or tuple(w_up.shape) != (E, H, Hp) or tuple(w_down.shape) != (E, Hp, H):
        raise ValueError("weight shapes must be w_gate/w_up [E,H,H'] and w_down [E,H',H]")
    if tuple(h_scratch.shape) != (M, Hp) or tuple(y.shape) != (M, H):
        raise ValueError("h_scratch must be [M,H'] and y [M,H]")
    if cu_seqlens.numel() != E + 1:
        raise ValueError("cu_seqlens must have E+1 entries")
    st = lib().moe_grouped_ffn(_ptr(x_perm), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
                               _ptr(cu_seqlens), M, H, Hp, E, _ptr(h_scratch), _ptr(y),
                               _ptr(d_status), _stream(stream, dev))
    _check("moe_grouped_ffn", st)


def _ffn_check(x_perm, w_gate, w_up, w_down, cu_seqlens, h_scratch, y, d_status):
    M, H = x_perm.shape
    Hp = h_scratch.shape[1]
    E = cu_seqlens.numel() - 1
    dev = x_perm.device
    for t, n in ((x_perm, "x_perm"), (h_scratch, "h_scratch"), (y, "y")):
        _need(t, n, torch.bfloat16, dev, 2)
    for t, n in ((w_gate, "w_gate"), (w_up, "w_up"), (w_down, "w_down")):
        _need(t, n, torch.bfloat16, dev, 3)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    _need(d_status, "d_status", torch.int32, dev)
    if w_gate is not None and tuple(w_gate.shape) != (E, H, Hp):
        raise ValueError(f"w_gate must be [E,H,H'] = {(E, H, Hp)}")
    if w_up is not None and tuple(w_up.shape) != (E, H, Hp):
        raise ValueError(f"w_up must be [E,H,H'] = {(E, H, Hp)}")
    if w_down is not None and tuple(w_down.shape) != (E, Hp, H):
        raise ValueError(f"w_down must be [E,H',H] = {(E, Hp, H)}")
    if h_scratch.shape[0] != M or (y is not None and tuple(y.shape) != (M, H)):
        raise ValueError("h_scratch must be [M,H'] and y [M,H]")
    return M, H, Hp, E, dev


def moe_grouped_ffn_up_gate(x_perm, w_gate, w_up, cu_seqlens, h_scratch, d_status=None,
                            stream=None):
    """First pass of moe_grouped_ffn: h = bf16(silu(x_perm W_gate[e]) * (x_perm W_up[e]))."""
    M, H, Hp, E, dev = _ffn_check(x_perm, w_gate, w_up, None, cu_seqlens, h_scratch, None, d_status)
    st = lib().moe_grouped_ffn_up_gate(_ptr(x_perm), _ptr(w_gate), _ptr(w_up), _ptr(cu_seqlens), M,
                                       H, Hp, E, _ptr(h_scratch), _ptr(d_status),
                                       _stream(stream, dev))
    _check("moe_grouped_ffn_up_gate", st)


def moe_grouped_ffn_down(h_scratch, w_down, cu_seqlens, y, d_status=None, stream=None):
    """Second pass of moe_grouped_ffn: y = bf16(h W_down[e])."""
    M, H = y.shape
    Hp = h_scratch.shape[1]
    E = cu_seqlens.numel() - 1
    dev = y.device
    _need(h_scratch, "h_scratch", torch.bfloat16, dev, 2)
    _need(y, "y", torch.bfloat16, dev, 2)
    _need(w_down, "w_down", torch.bfloat16, dev, 3)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    _need(d_status, "d_status", torch.int32, dev)
    if tuple(w_down.shape) != (E, Hp, H) or h_scratch.shape[0] != M:
        raise ValueError("w_down must be [E,H',H] and h_scratch [M,H']")
    st = lib().moe_grouped_ffn_down(_ptr(h_scratch), _ptr(w_down), _ptr(cu_seqlens), M, H, Hp, E,
                                    _ptr(y), _ptr(d_status), _stream(stream, dev))
    _check("moe_grouped_ffn_down", st)


def _gather_check(x, perm_src, K, w_gate, w_up, cu_seqlens, h_scratch, d_status):
    S, H = x.shape
    M = S * K
    Hp = h_scratch.shape[1]
    E = cu_seqlens.numel() - 1
    dev = x.device
    _need_shape(x, "x", (S, H), torch.bfloat16, dev)
    _need(perm_src, "perm_src", torch.int32, dev)
    if perm_src.numel() != M:
        raise ValueError(f"perm_src must have S*K = {M} entries")
    _need_shape(h_scratch, "h_scratch", (M, Hp), torch.bfloat16, dev)
    _need_shape(w_gate, "w_gate", (E, H, Hp), torch.bfloat16, dev)
    _need_shape(w_up, "w_up", (E, H, Hp), torch.bfloat16, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    _need(d_status, "d_status", torch.int32, dev)
    return S, H, Hp, E, M, dev


def moe_grouped_ffn_gather(x, perm_src, K, w_gate, w_up, w_down, cu_seqlens, h_scratch, y,
                           d_status=None, stream=None):
    """moe_grouped_ffn with the token rows gathered from the token-major x through perm_src
    (no x_perm): the zero-copy path (see include/moe_b200.h)."""
    S, H, Hp, E, M, dev = _gather_check(x, perm_src, K, w_gate, w_up, cu_seqlens, h_scratch,
                                        d_status)
    _need_shape(w_down, "w_down", (E, Hp, H), torch.bfloat16, dev)
    _need_shape(y, "y", (M, H), torch.bfloat16, dev)
    st = lib().moe_grouped_ffn_gather(_ptr(x), _ptr(perm_src), S, K, _ptr(w_gate), _ptr(w_up),
                                      _ptr(w_down), _ptr(cu_seqlens), H, Hp, E, _ptr(h_scratch),
                                      _ptr(y), _ptr(d_status), _stream(stream, dev))
    _check("moe_grouped_ffn_gather", st)


def moe_grouped_ffn_up_gate_gather(x, perm_src, K, w_gate, w_up, cu_seqlens, h_scratch,
                                   gate_pre=None, up_pre=None, d_status=None, stream=None):
    """First pass of moe_grouped_ffn_gather (optionally storing the pre-activations)."""
    S, H, Hp, E, M, dev = _gather_check(x, perm_src, K, w_gate, w_up, cu_seqlens, h_scratch,
                                        d_status)
    if (gate_pre is None) != (up_pre is None):
        raise ValueError("gate_pre and up_pre go together")
    for t, n in ((gate_pre, "gate_pre"), (up_pre, "up_pre")):
        if t is not None:
            _need_shape(t, n, (M, Hp), torch.bfloat16, dev)
    st = lib().moe_grouped_ffn_up_gate_gather(_ptr(x), _ptr(perm_src), S, K, _ptr(w_gate),
                                              _ptr(w_up), _ptr(cu_seqlens), H, Hp, E,
                                              _ptr(h_scratch), _ptr(gate_pre), _ptr(up_pre),
                                              _ptr(d_status), _stream(stream, dev))
    _check("moe_grouped_ffn_up_gate_gather", st)


def moe_grouped_ffn_up_gate_train(x_perm, w_gate, w_up, cu_seqlens, h_scratch, gate_pre, up_pre,
                                  d_status=None, stream=None):
    """moe_grouped_ffn_up_gate that also stores the bf16 pre-activations x W_gate, x W_up."""
    M, H, Hp, E, dev = _ffn_check(x_perm, w_gate, w_up, None, cu_seqlens, h_scratch, None, d_status)
    for t, n in ((gate_pre, "gate_pre"), (up_pre, "up_pre")):
        _need(t, n, torch.bfloat16, dev, 2)
        if tuple(t.shape) != (M, Hp):
            raise ValueError(f"{n} must be [M,H'] = {(M, Hp)}")
    st = lib().moe_grouped_ffn_up_gate_train(_ptr(x_perm), _ptr(w_gate), _ptr(w_up),
                                             _ptr(cu_seqlens), M, H, Hp, E, _ptr(h_scratch),
                                             _ptr(gate_pre), _ptr(up_pre), _ptr(d_status),
                                             _stream(stream, dev))
    _check("moe_grouped_ffn_up_gate_train", st)


def _bwd_shapes(grad_y, gate_pre, cu_seqlens):
    M, H = grad_y.shape
    Hp = gate_pre.shape[1]
    return M, H, Hp, cu_seqlens.numel() - 1, grad_y.device


def _need_shape(t, name, shape, dtype, dev):
    _need(t, name, dtype, dev)
    if t is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must be {tuple(shape)}, got {tuple(t.shape)}")


def moe_grouped_ffn_down_backward(grad_y, w_down, gate_pre, up_pre, cu_seqlens, d_gate, d_up,
                                  d_status=None, stream=None):
    """d_gate, d_up = SwiGLU backward of grad_y W_down[e]^T at the saved pre-activations."""
    M, H, Hp, E, dev = _bwd_shapes(grad_y, gate_pre, cu_seqlens)
    _need_shape(grad_y, "grad_y", (M, H), torch.bfloat16, dev)
    _need_shape(w_down, "w_down", (E, Hp, H), torch.bfloat16, dev)
    for t, n in ((gate_pre, "gate_pre"), (up_pre, "up_pre"), (d_gate, "d_gate"), (d_up, "d_up")):
        _need_shape(t, n, (M, Hp), torch.bfloat16, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    _need(d_status, "d_status", torch.int32, dev)
    st = lib().moe_grouped_ffn_down_backward(_ptr(grad_y), _ptr(w_down), _ptr(gate_pre),
                                             _ptr(up_pre), _ptr(cu_seqlens), M, H, Hp, E,
                                             _ptr(d_gate), _ptr(d_up), _ptr(d_status),
                                             _stream(stream, dev))
    _check("moe_grouped_ffn_down_backward", st)


def moe_grouped_ffn_up_gate_backward(d_gate, d_up, w_gate, w_up, cu_seqlens, grad_x_perm,
                                     d_status=None, stream=None):
    """grad_x_perm = d_gate W_gate[e]^T + d_up W_up[e]^T."""
    M, H = grad_x_perm.shape
    Hp = d_gate.shape[1]
    E = cu_seqlens.numel() - 1
    dev = grad_x_perm.device
    _need_shape(grad_x_perm, "grad_x_perm", (M, H), torch.bfloat16, dev)
    for t, n in ((d_gate, "d_gate"), (d_up, "d_up")):
        _need_shape(t, n, (M, Hp), torch.bfloat16, dev)
    for t, n in ((w_gate, "w_gate"), (w_up, "w_up")):
        _need_shape(t, n, (E, H, Hp), torch.bfloat16, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    _need(d_status, "d_status", torch.int32, dev)
    st = lib().moe_grouped_ffn_up_gate_backward(_ptr(d_gate), _ptr(d_up), _ptr(w_gate),
                                                _ptr(w_up), _ptr(cu_seqlens), M, H, Hp, E,
                                                _ptr(grad_x_perm), _ptr(d_status),
                                                _stream(stream, dev))
    _check("moe_grouped_ffn_up_gate_backward", st)


def moe_grouped_ffn_weight_grad(x_perm, h, d_gate, d_up, grad_y, cu_seqlens, grad_w_gate,
                                grad_w_up, grad_w_down, accumulate=False, d_status=None,
                                stream=None):
    """fp32 weight gradients x^T d_gate, x^T d_up, h^T grad_y per expert (written or added)."""
    M, H = x_perm.shape
    Hp = h.shape[1]
    E = cu_seqlens.numel() - 1
    dev = x_perm.device
    _need_shape(x_perm, "x_perm", (M, H), torch.bfloat16, dev)
    _need_shape(grad_y, "grad_y", (M, H), torch.bfloat16, dev)
    for t, n in ((h, "h"), (d_gate, "d_gate"), (d_up, "d_up")):
        _need_shape(t, n, (M, Hp), torch.bfloat16, dev)
    _need_shape(grad_w_gate, "grad_w_gate", (E, H, Hp), torch.float32, dev)
    _need_shape(grad_w_up, "grad_w_up", (E, H, Hp), torch.float32, dev)
    _need_shape(grad_w_down, "grad_w_down", (E, Hp, H), torch.float32, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    _need(d_status, "d_status", torch.int32, dev)
    st = lib().moe_grouped_ffn_weight_grad(_ptr(x_perm), _ptr(h), _ptr(d_gate), _ptr(d_up),
                                           _ptr(grad_y), _ptr(cu_seqlens), M, H, Hp, E,
                                           _ptr(grad_w_gate), _ptr(grad_w_up), _ptr(grad_w_down),
                                           1 if accumulate else 0, _ptr(d_status),
                                           _stream(stream, dev))
    _check("moe_grouped_ffn_weight_grad", st)


def moe_grouped_ffn_backward(x_perm, h, gate_pre, up_pre, w_gate, w_up, w_down, cu_seqlens, grad_y,
                             d_gate, d_up, grad_x_perm, grad_w_gate, grad_w_up, grad_w_down,
                             accumulate=False, d_status=None, stream=None):
    """Backward of the grouped expert FFN (see include/moe_b200.h): d_gate, d_up, grad_x_perm
    and the fp32 weight gradients, in three launches on one stream."""
    M, H, Hp, E, dev = _bwd_shapes(grad_y, gate_pre, cu_seqlens)
    for t, n in ((x_perm, "x_perm"), (grad_y, "grad_y"), (grad_x_perm, "grad_x_perm")):
        _need_shape(t, n, (M, H), torch.bfloat16, dev)
    for t, n in ((h, "h"), (gate_pre, "gate_pre"), (up_pre, "up_pre"), (d_gate, "d_gate"),
                 (d_up, "d_up")):
        _need_shape(t, n, (M, Hp), torch.bfloat16, dev)
    for t, n in ((w_gate, "w_gate"), (w_up, "w_up")):
        _need_shape(t, n, (E, H, Hp), torch.bfloat16, dev)
    _need_shape(w_down, "w_down", (E, Hp, H), torch.bfloat16, dev)
    _need_shape(grad_w_gate, "grad_w_gate", (E, H, Hp), torch.float32, dev)
    _need_shape(grad_w_up, "grad_w_up", (E, H, Hp), torch.float32, dev)
    _need_shape(grad_w_down, "grad_w_down", (E, Hp, H), torch.float32, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    _need(d_status, "d_status", torch.int32, dev)
    st = lib().moe_grouped_ffn_backward(_ptr(x_perm), _ptr(h), _ptr(gate_pre), _ptr(up_pre),
                                        _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(cu_seqlens),
                                        M, H, Hp, E, _ptr(grad_y), _ptr(d_gate), _ptr(d_up),
                                        _ptr(grad_x_perm), _ptr(grad_w_gate), _ptr(grad_w_up),
                                        _ptr(grad_w_down), 1 if accumulate else 0,
                                        _ptr(d_status), _stream(stream, dev))
    _check("moe_grouped_ffn_backward", st)


def moe_unpermute_combine(y, row_id_map, route_w, out, stream=None):
    """out[t] = sum_k route_w[t,k] * y[row_id_map[t*K+k]] (see include/moe_b200.h)."""
    S, K = route_w.shape
    dev = y.device
    _need(y, "y", torch.bfloat16, dev, 2)
    _need(out, "out", torch.bfloat16, dev, 2)
    _need(row_id_map, "row_id_map", torch.int32, dev)
    _need(route_w, "route_w", torch.float32, dev, 2)
    H = y.shape[1]
    if tuple(out.shape) != (S, H) or row_id_map.numel() != S * K:
        raise ValueError("out must be [S,H] and row_id_map S*K entries")
    st = lib().moe_unpermute_combine(_ptr(y), _ptr(row_id_map), _ptr(route_w), S, H, K, _ptr(out),
                                     _stream(stream, dev))
    _check("moe_unpermute_combine", st)


def moe_combine_backward(grad_out, y, row_id_map, route_w, grad_y, grad_w=None, stream=None):
    """grad_y[r(t,k)] = w[t,k] * grad_out[t]; grad_w[t,k] = <grad_out[t], y[r(t,k)]>."""
    S, K = route_w.shape
    dev = grad_out.device
    _need(grad_out, "grad_out", torch.bfloat16, dev, 2)
    _need(y, "y", torch.bfloat16, dev, 2)
    _need(grad_y, "grad_y", torch.bfloat16, dev, 2)
    _need(row_id_map, "row_id_map", torch.int32, dev)
    _need(route_w, "route_w", torch.float32, dev, 2)
    _need(grad_w, "grad_w", torch.float32, dev)
    H = grad_out.shape[1]
    if tuple(grad_out.shape) != (S, H) or grad_y.shape[1] != H or row_id_map.numel() != S * K:
        raise ValueError("grad_out [S,H], grad_y [M,H], row_id_map [S*K] expected")
    if grad_w is not None and (y is None or grad_w.numel() != S * K):
        raise ValueError("grad_w needs y and S*K entries")
    st = lib().moe_combine_backward(_ptr(grad_out), _ptr(y), _ptr(row_id_map), _ptr(route_w), S,
                                    H, K, _ptr(grad_y), _ptr(grad_w), _stream(stream, dev))
    _check("moe_combine_backward", st)


def moe_permute_backward(grad_x_perm, row_id_map, grad_x, K, stream=None):
    """grad_x[t] = sum_k grad_x_perm[row_id_map[t*K+k]] (dispatch backward)."""
    S, H = grad_x.shape
    dev = grad_x.device
    _need(grad_x_perm, "grad_x_perm", torch.bfloat16, dev, 2)
    _need(grad_x, "grad_x", torch.bfloat16, dev, 2)
    _need(row_id_map, "row_id_map", torch.int32, dev)
    if grad_x_perm.shape[1] != H or row_id_map.numel() != S * K:
        raise ValueError("grad_x_perm [M,H] and row_id_map [S*K] expected")
    st = lib().moe_permute_backward(_ptr(grad_x_perm), _ptr(row_id_map), S, H, K, _ptr(grad_x),
                                    _stream(stream, dev))
    _check("moe_permute_backward", st)


def moe_append_shared(topk_ids, route_w, E, n_shared, ids_out, w_out, stream=None):
    """Routing with n_shared shared experts appended (experts E .. E+n_shared-1, weight 1 in
    slots K .. K+n_shared-1; see include/moe_b200.h)."""
    S, K = topk_ids.shape
    dev = topk_ids.device
    _need_shape(topk_ids, "topk_ids", (S, K), torch.int32, dev)
    _need_shape(route_w, "route_w", (S, K), torch.float32, dev)
    _need_shape(ids_out, "ids_out", (S, K + n_shared), torch.int32, dev)
    _need_shape(w_out, "w_out", (S, K + n_shared), torch.float32, dev)
    st = lib().moe_append_shared(_ptr(topk_ids), _ptr(route_w), S, K, E, n_shared, _ptr(ids_out),
                                 _ptr(w_out), _stream(stream, dev))
    _check("moe_append_shared", st)


def moe_maxvio(counts, S, K, maxvio, max_count=None, stream=None):
    """maxvio = max_e(counts[e] * E / (S*K)) - 1 into a device double (see include/moe_b200.h)."""
    dev = counts.device
    _need(counts, "counts", torch.int32, dev)
    _need(maxvio, "maxvio", torch.float64, dev)
    _need(max_count, "max_count", torch.int32, dev)
    st = lib().moe_maxvio(_ptr(counts), counts.numel(), S, K, _ptr(maxvio), _ptr(max_count),
                          _stream(stream, dev))
    _check("moe_maxvio", st)


@dataclass
class LayerBuffers:
    """Device buffers of one layer call, allocated once and reused (static shapes)."""

    x_perm: torch.Tensor
    counts: torch.Tensor
    cu_seqlens: torch.Tensor
    row_id_map: torch.Tensor
    perm_src: torch.Tensor
    maxvio: torch.Tensor
    max_count: torch.Tensor
    workspace: torch.Tensor
    h: torch.Tensor | None
    y: torch.Tensor | None
    out: torch.Tensor
    d_status: torch.Tensor
    gate_pre: torch.Tensor | None = None  # training: saved bf16 pre-activations [M,H']
    up_pre: torch.Tensor | None = None

    @staticmethod
    def allocate(S: int, H: int, Hp: int, E: int, K: int, device, with_ffn: bool = True,
                 train: bool = False, alloc=None):
        """alloc(shape, dtype) -> tensor on `device` (default torch.empty), e.g. an allocator
        that surrounds each buffer with guard bytes."""
        M = S * K
        new = _allocator(alloc, device)
        i32, bf = torch.int32, torch.bfloat16
        train = train and with_ffn
        d_status = new((1,), i32)
        d_status.zero_()
        return LayerBuffers(
            x_perm=new((M, H), bf), counts=new((E,), i32), cu_seqlens=new((E + 1,), i32),
            row_id_map=new((M,), i32), perm_src=new((M,), i32), maxvio=new((1,), torch.float64),
            max_count=new((1,), i32),
            workspace=new((max(moe_permute_workspace_bytes(S, K, E), 16),), torch.uint8),
            h=new((M, Hp), bf) if with_ffn else None, y=new((M, H), bf) if with_ffn else None,
            out=new((S, H), bf), d_status=d_status,
            gate_pre=new((M, Hp), bf) if train else None,
            up_pre=new((M, Hp), bf) if train else None)


def _allocator(alloc, device):
    if alloc is not None:
        return alloc
    return lambda shape, dtype: torch.empty(shape, dtype=dtype, device=device)


def moe_layer_forward(x, topk_ids, route_w, w_gate, w_up, w_down, buf: LayerBuffers, stream=None,
                      zero_copy: bool = False):
    """permute -> grouped FFN -> combine on one stream; returns buf.out.

    With w_gate None the experts are the identity (y = x_perm): permute/combine only.
    zero_copy: the permutation computes the metadata only and the SwiGLU pass gathers its
    token rows from x (same results, no x_perm; inference only).
    """
    E = buf.counts.numel()
    if zero_copy and w_gate is not None and buf.gate_pre is None:
        K = topk_ids.shape[1]
        moe_permute(x, topk_ids, E, None, buf.counts, buf.cu_seqlens, buf.row_id_map,
                    buf.perm_src, buf.maxvio, buf.max_count, buf.workspace, buf.d_status, stream)
        moe_grouped_ffn_gather(x, buf.perm_src, K, w_gate, w_up, w_down, buf.cu_seqlens, buf.h,
                               buf.y, buf.d_status, stream)
        moe_unpermute_combine(buf.y, buf.row_id_map, route_w, buf.out, stream)
        return buf.out
    moe_permute(x, topk_ids, E, buf.x_perm, buf.counts, buf.cu_seqlens, buf.row_id_map,
                buf.perm_src, buf.maxvio, buf.max_count, buf.workspace, buf.d_status, stream)
    y = buf.x_perm
    if w_gate is not None:
        if buf.gate_pre is not None:
            # training: keep the pre-activations for the backward
            moe_grouped_ffn_up_gate_train(buf.x_perm, w_gate, w_up, buf.cu_seqlens, buf.h,
                                          buf.gate_pre, buf.up_pre, buf.d_status, stream)
            moe_grouped_ffn_down(buf.h, w_down, buf.cu_seqlens, buf.y, buf.d_status, stream)
        else:
            moe_grouped_ffn(buf.x_perm, w_gate, w_up, w_down, buf.cu_seqlens, buf.h, buf.y,
                            buf.d_status, stream)
        y = buf.y
    moe_unpermute_combine(y, buf.row_id_map, route_w, buf.out, stream)
    return buf.out


@dataclass
class LayerGrads:
    """Gradient buffers of one layer's backward (fp32 weight gradients laid out like the
    weights, as the training buffers of the MoonEP README's "Gradient buffers")."""

    grad_y: torch.Tensor        # [M,H] bf16
    d_gate: torch.Tensor        # [M,H'] bf16
    d_up: torch.Tensor          # [M,H'] bf16
    grad_x_perm: torch.Tensor   # [M,H] bf16
    grad_x: torch.Tensor        # [S,H] bf16
    grad_route_w: torch.Tensor  # [S,K] fp32
    grad_w_gate: torch.Tensor   # [E,H,H'] fp32
    grad_w_up: torch.Tensor     # [E,H,H'] fp32
    grad_w_down: torch.Tensor   # [E,H',H] fp32

    @staticmethod
    def allocate(S: int, H: int, Hp: int, E: int, K: int, device, alloc=None):
        M = S * K
        new = _allocator(alloc, device)
        bf, f32 = torch.bfloat16, torch.float32
        return LayerGrads(
            grad_y=new((M, H), bf), d_gate=new((M, Hp), bf), d_up=new((M, Hp), bf),
            grad_x_perm=new((M, H), bf), grad_x=new((S, H), bf), grad_route_w=new((S, K), f32),
            grad_w_gate=new((E, H, Hp), f32), grad_w_up=new((E, H, Hp), f32),
            grad_w_down=new((E, Hp, H), f32))


def moe_layer_backward(grad_out, route_w, w_gate, w_up, w_down, buf: LayerBuffers,
                       grads: LayerGrads, accumulate: bool = False, stream=None):
    """Backward of moe_layer_forward (run with LayerBuffers.allocate(..., train=True)):
    combine backward -> grouped FFN backward -> permutation backward, on one stream.
    Fills grads (grad_x, grad_route_w and the weight gradients, written or added into)."""
    if buf.gate_pre is None:
        raise ValueError("the forward did not keep pre-activations: allocate with train=True")
    K = route_w.shape[1]
    moe_combine_backward(grad_out, buf.y, buf.row_id_map, route_w, grads.grad_y,
                         grads.grad_route_w, stream)
    moe_grouped_ffn_backward(buf.x_perm, buf.h, buf.gate_pre, buf.up_pre, w_gate, w_up, w_down,
                             buf.cu_seqlens, grads.grad_y, grads.d_gate, grads.d_up,
                             grads.grad_x_perm, grads.grad_w_gate, grads.grad_w_up,
                             grads.grad_w_down, accumulate, buf.d_status, stream)
    moe_permute_backward(grads.grad_x_perm, buf.row_id_map, grads.grad_x, K, stream)
    return grads


# ----------------------------------------------------------------------------- MXFP8


def moe_mx_weight_scale_bytes(E: int, R: int, C: int) -> int:
    return int(lib().moe_mx_weight_scale_bytes(E, R, C))


def moe_mx_quantize_weights(w, w_q, w_sf, stream=None):
    """Quantise weights [E,R,C] bf16 (R the reduction dimension) to MXFP8: w_q [E,R,C] uint8
    (E4M3 codes), w_sf uint8 with moe_mx_weight_scale_bytes(E,R,C) bytes (E8M0 scales in the
    chunk order of include/moe_b200.h)."""
    _need(w, "w", torch.bfloat16, None, 3)
    dev = w.device
    _need(w_q, "w_q", torch.uint8, dev)
    _need(w_sf, "w_sf", torch.uint8, dev)
    E, R, C = w.shape
    if tuple(w_q.shape) != (E, R, C):
        raise ValueError(f"w_q: expected {(E, R, C)}, got {tuple(w_q.shape)}")
    if w_sf.numel() != moe_mx_weight_scale_bytes(E, R, C):
        raise ValueError("w_sf: expected moe_mx_weight_scale_bytes(E, R, C) bytes")
    st = lib().moe_mx_quantize_weights(_ptr(w), E, R, C, _ptr(w_q), _ptr(w_sf),
                                       _stream(stream, dev))
    _check("moe_mx_quantize_weights", st)


def mx_quantize_weights(w, stream=None):
    """Allocate and fill (w_q, w_sf) for one projection's bf16 weights [E,R,C]."""
    E, R, C = w.shape
    w_q = torch.empty(E, R, C, dtype=torch.uint8, device=w.device)
    w_sf = torch.empty(max(moe_mx_weight_scale_bytes(E, R, C), 1), dtype=torch.uint8,
                       device=w.device)
    moe_mx_quantize_weights(w, w_q, w_sf, stream)
    return w_q, w_sf


def moe_mx_permute_quantize(x, row_id_map, K, x_q, x_sf, stream=None):
    """Quantise the token rows of x [S,H] bf16 to MXFP8 and write them to their expert-grouped
    rows: x_q [S*K,H] uint8, x_sf [S*K,H/32] uint8."""
    _need(x, "x", torch.bfloat16, None, 2)
    dev = x.device
    S, H = x.shape
    _need(row_id_map, "row_id_map", torch.int32, dev)
    _need(x_q, "x_q", torch.uint8, dev, 2)
    _need(x_sf, "x_sf", torch.uint8, dev, 2)
    if row_id_map.numel() != S * K or tuple(x_q.shape) != (S * K, H) or \
            tuple(x_sf.shape) != (S * K, H // 32):
        raise ValueError("row_id_map [S*K], x_q [S*K,H] and x_sf [S*K,H/32] expected")
    st = lib().moe_mx_permute_quantize(_ptr(x), _ptr(row_id_map), S, H, K, _ptr(x_q), _ptr(x_sf),
                                       _stream(stream, dev))
    _check("moe_mx_permute_quantize", st)


@dataclass
class MxWeights:
    """One layer's expert weights in MXFP8 (codes and chunked scales per projection)."""

    w_gate_q: torch.Tensor
    w_gate_sf: torch.Tensor
    w_up_q: torch.Tensor
    w_up_sf: torch.Tensor
    w_down_q: torch.Tensor
    w_down_sf: torch.Tensor

    @staticmethod
    def from_bf16(w_gate, w_up, w_down, stream=None):
        gq, gs = mx_quantize_weights(w_gate, stream)
        uq, us = mx_quantize_weights(w_up, stream)
        dq, ds = mx_quantize_weights(w_down, stream)
        return MxWeights(gq, gs, uq, us, dq, ds)


def _mx_check(x_q, x_sf, mw: MxWeights, cu_seqlens, d_status):
    M, H = x_q.shape
    E, H2, Hp = mw.w_gate_q.shape
    dev = x_q.device
    _need(x_q, "x_q", torch.uint8, dev, 2)
    _need(x_sf, "x_sf", torch.uint8, dev, 2)
    for name in ("w_gate_q", "w_gate_sf", "w_up_q", "w_up_sf", "w_down_q", "w_down_sf"):
        _need(getattr(mw, name), name, torch.uint8, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    _need(d_status, "d_status", torch.int32, dev)
    if H2 != H or tuple(mw.w_up_q.shape) != (E, H, Hp) or tuple(mw.w_down_q.shape) != (E, Hp, H):
        raise ValueError("MXFP8 weights must be w_gate/w_up [E,H,H'] and w_down [E,H',H]")
    if tuple(x_sf.shape) != (M, H // 32) or cu_seqlens.numel() != E + 1:
        raise ValueError("x_sf must be [M,H/32] and cu_seqlens have E+1 entries")
    return M, H, Hp, E, dev


def moe_grouped_ffn_up_gate_mxfp8(x_q, x_sf, mw: MxWeights, cu_seqlens, h_q, h_sf, d_status=None,
                                  stream=None):
    """MXFP8 SwiGLU pass: h = silu(x Wg) * (x Wu) from MXFP8 operands, stored as MXFP8
    (h_q [M,H'] uint8, h_sf [M,H'/32] uint8)."""
    M, H, Hp, E, dev = _mx_check(x_q, x_sf, mw, cu_seqlens, d_status)
    _need(h_q, "h_q", torch.uint8, dev, 2)
    _need(h_sf, "h_sf", torch.uint8, dev, 2)
    if tuple(h_q.shape) != (M, Hp) or tuple(h_sf.shape) != (M, Hp // 32):
        raise ValueError("h_q must be [M,H'] and h_sf [M,H'/32]")
    st = lib().moe_grouped_ffn_up_gate_mxfp8(_ptr(x_q), _ptr(x_sf), _ptr(mw.w_gate_q),
                                             _ptr(mw.w_gate_sf), _ptr(mw.w_up_q),
                                             _ptr(mw.w_up_sf), _ptr(cu_seqlens), M, H, Hp, E,
                                             _ptr(h_q), _ptr(h_sf), _ptr(d_status),
                                             _stream(stream, dev))
    _check("moe_grouped_ffn_up_gate_mxfp8", st)


def moe_grouped_ffn_down_mxfp8(h_q, h_sf, mw: MxWeights, cu_seqlens, y, d_status=None,
                               stream=None):
    """MXFP8 down pass: y = bf16(h W_down) from MXFP8 h and W_down."""
    M, Hp = h_q.shape
    E, _, H = mw.w_down_q.shape
    dev = h_q.device
    _need(h_q, "h_q", torch.uint8, dev, 2)
    _need(h_sf, "h_sf", torch.uint8, dev, 2)
    _need(mw.w_down_q, "w_down_q", torch.uint8, dev, 3)
    _need(mw.w_down_sf, "w_down_sf", torch.uint8, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    _need(d_status, "d_status", torch.int32, dev)
    _need(y, "y", torch.bfloat16, dev, 2)
    if tuple(h_sf.shape) != (M, Hp // 32) or tuple(y.shape) != (M, H) or \
            tuple(mw.w_down_q.shape) != (E, Hp, H) or cu_seqlens.numel() != E + 1:
        raise ValueError("h_sf [M,H'/32], y [M,H], w_down_q [E,H',H], cu_seqlens [E+1] expected")
    st = lib().moe_grouped_ffn_down_mxfp8(_ptr(h_q), _ptr(h_sf), _ptr(mw.w_down_q),
                                          _ptr(mw.w_down_sf), _ptr(cu_seqlens), M, H, Hp, E,
                                          _ptr(y), _ptr(d_status), _stream(stream, dev))
    _check("moe_grouped_ffn_down_mxfp8", st)


def moe_grouped_ffn_mxfp8(x_q, x_sf, mw: MxWeights, cu_seqlens, h_q, h_sf, y, d_status=None,
                          stream=None):
    """Both MXFP8 passes (include/moe_b200.h, moe_grouped_ffn_mxfp8)."""
    M, H, Hp, E, dev = _mx_check(x_q, x_sf, mw, cu_seqlens, d_status)
    _need(h_q, "h_q", torch.uint8, dev, 2)
    _need(h_sf, "h_sf", torch.uint8, dev, 2)
    _need(y, "y", torch.bfloat16, dev, 2)
    if tuple(h_q.shape) != (M, Hp) or tuple(h_sf.shape) != (M, Hp // 32) or \
            tuple(y.shape) != (M, H):
        raise ValueError("h_q [M,H'], h_sf [M,H'/32] and y [M,H] expected")
    st = lib().moe_grouped_ffn_mxfp8(_ptr(x_q), _ptr(x_sf), _ptr(mw.w_gate_q), _ptr(mw.w_gate_sf),
                                     _ptr(mw.w_up_q), _ptr(mw.w_up_sf), _ptr(mw.w_down_q),
                                     _ptr(mw.w_down_sf), _ptr(cu_seqlens), M, H, Hp, E, _ptr(h_q),
                                     _ptr(h_sf), _ptr(y), _ptr(d_status), _stream(stream, dev))
    _check("moe_grouped_ffn_mxfp8", st)


@dataclass
class MxBuffers:
    """The MXFP8 activations of one layer call: x_q/x_sf [M,H], [M,H/32]; h_q/h_sf [M,H'],
    [M,H'/32] (uint8)."""

    x_q: torch.Tensor
    x_sf: torch.Tensor
    h_q: torch.Tensor
    h_sf: torch.Tensor

    @staticmethod
    def allocate(S: int, H: int, Hp: int, K: int, device, alloc=None):
        M = S * K
        new = _allocator(alloc, device)
        u8 = torch.uint8
        return MxBuffers(new((M, H), u8), new((M, H // 32), u8), new((M, Hp), u8),
                         new((M, Hp // 32), u8))


def moe_layer_forward_mxfp8(x, topk_ids, route_w, mw: MxWeights, buf: LayerBuffers,
                            mxbuf: MxBuffers, stream=None):
    """The layer with MXFP8 experts: routing (moe_permute, no bf16 row copy) -> permute fused
    with the activations' quantisation -> MXFP8 grouped FFN -> weighted combine; returns
    buf.out (buf.x_perm and buf.h are not used)."""
    E = buf.counts.numel()
    K = topk_ids.shape[1]
    moe_permute(x, topk_ids, E, None, buf.counts, buf.cu_seqlens, buf.row_id_map, buf.perm_src,
                buf.maxvio, buf.max_count, buf.workspace, buf.d_status, stream)
    moe_mx_permute_quantize(x, buf.row_id_map, K, mxbuf.x_q, mxbuf.x_sf, stream)
    moe_grouped_ffn_mxfp8(mxbuf.x_q, mxbuf.x_sf, mw, buf.cu_seqlens, mxbuf.h_q, mxbuf.h_sf, buf.y,
                          buf.d_status, stream)
    moe_unpermute_combine(buf.y, buf.row_id_map, route_w, buf.out, stream)
    return buf.out
