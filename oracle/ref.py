"""ctypes loader of the plain C++ oracle (moe_oracle_ref.cpp) and numpy-facing wrappers.

TEST INFRASTRUCTURE ONLY, like moe_oracle.py: tests/ use it to cross-check the numpy
oracle; `build()` compiles it with g++ next to its source (the library is not part of the
product and is never loaded by it).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moe_oracle_ref.cpp")
LIB = os.path.join(HERE, "libmoe_oracle_ref.so")

_lib = None


def build(verbose: bool = False) -> str:
    """Compile the oracle with g++ (no floating-point contraction: every product and sum is
    rounded as written)."""
    cmd = ["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-shared",
           "-fPIC", SRC, "-o", LIB]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    return LIB


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
            build()
        L = ctypes.CDLL(LIB)
        P = ctypes.c_void_p
        i64, i32 = ctypes.c_int64, ctypes.c_int32
        L.ref_round_bf16.argtypes = [P, i64, P]
        L.ref_round_bf16.restype = None
        L.ref_permute.argtypes = [P, i64, i32, i32, P, P, P, P]
        L.ref_permute.restype = ctypes.c_int
        L.ref_permute_rows.argtypes = [P, P, i64, i32, i64, P]
        L.ref_permute_rows.restype = None
        L.ref_maxvio.argtypes = [P, i32, i64, i32, P]
        L.ref_maxvio.restype = ctypes.c_double
        L.ref_grouped_ffn.argtypes = [P, P, P, P, P, i32, i64, i64, P, P]
        L.ref_grouped_ffn.restype = None
        L.ref_combine.argtypes = [P, P, P, i64, i32, i64, P]
        L.ref_combine.restype = None
        L.ref_combine_backward.argtypes = [P, P, P, P, i64, i32, i64, P, P]
        L.ref_combine_backward.restype = None
        L.ref_permute_backward.argtypes = [P, P, i64, i32, i64, P]
        L.ref_permute_backward.restype = None
        L.ref_e4m3_round.argtypes = [P, i64, P]
        L.ref_e4m3_round.restype = None
        L.ref_mx_quantize_rows.argtypes = [P, i64, i64, P, P]
        L.ref_mx_quantize_rows.restype = None
        L.ref_expert_backward.argtypes = [P] * 8 + [i64, i64, i64] + [P] * 6
        L.ref_expert_backward.restype = None
        L.ref_expert_ffn_mxfp8.argtypes = [P, P, P, P, i64, i64, i64, P, P, P]
        L.ref_expert_ffn_mxfp8.restype = None
        _lib = L
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def round_bf16(v) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    lib().ref_round_bf16(_p(v), v.size, _p(out))
    return out


def permute(topk_ids, E: int):
    """(counts, cu_seqlens, row_id_map, perm_src); ValueError on an id outside [0, E)."""
    ids = np.ascontiguousarray(topk_ids, dtype=np.int32)
    S, K = ids.shape
    counts = np.empty(E, np.int32)
    cu = np.empty(E + 1, np.int32)
    rmap = np.empty(S * K, np.int32)
    psrc = np.empty(S * K, np.int32)
    if lib().ref_permute(_p(ids), S, K, E, _p(counts), _p(cu), _p(rmap), _p(psrc)) != 0:
        raise ValueError("expert id outside [0, E)")
    return counts, cu, rmap, psrc


def permute_rows(x_bits, perm_src, K: int) -> np.ndarray:
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    ps = np.ascontiguousarray(perm_src, dtype=np.int32)
    out = np.empty((ps.size, x.shape[1]), np.uint16)
    lib().ref_permute_rows(_p(x), _p(ps), ps.size, K, x.shape[1], _p(out))
    return out


def maxvio(counts, S: int, K: int):
    c = np.ascontiguousarray(counts, dtype=np.int32)
    mc = np.zeros(1, np.int32)
    v = lib().ref_maxvio(_p(c), c.size, S, K, _p(mc))
    return v, int(mc[0])


def grouped_ffn(x_perm_bits, cu_seqlens, w_gate, w_up, w_down):
    """(h bits [M,Hp], y bits [M,H]); weights [E,H,Hp], [E,H,Hp], [E,Hp,H] as bf16 bits."""
    x = np.ascontiguousarray(x_perm_bits, dtype=np.uint16)
    wg = np.ascontiguousarray(w_gate, dtype=np.uint16)
    wu = np.ascontiguousarray(w_up, dtype=np.uint16)
    wd = np.ascontiguousarray(w_down, dtype=np.uint16)
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    M, H = x.shape
    E, _, Hp = wg.shape
    h = np.zeros((M, Hp), np.uint16)
    y = np.zeros((M, H), np.uint16)
    lib().ref_grouped_ffn(_p(x), _p(wg), _p(wu), _p(wd), _p(cu), E, H, Hp, _p(h), _p(y))
    return h, y


def combine(y_bits, row_id_map, route_w, S: int, K: int) -> np.ndarray:
    y = np.ascontiguousarray(y_bits, dtype=np.uint16)
    rm = np.ascontiguousarray(row_id_map, dtype=np.int32)
    w = np.ascontiguousarray(route_w, dtype=np.float32)
    out = np.empty((S, y.shape[1]), np.uint16)
    lib().ref_combine(_p(y), _p(rm), _p(w), S, K, y.shape[1], _p(out))
    return out


def combine_backward(grad_out_bits, y_bits, row_id_map, route_w, S: int, K: int):
    """(grad_y bits [M,H], grad_w float64 [S,K]); rows no slot maps to stay 0."""
    g = np.ascontiguousarray(grad_out_bits, dtype=np.uint16)
    y = np.ascontiguousarray(y_bits, dtype=np.uint16)
    rm = np.ascontiguousarray(row_id_map, dtype=np.int32)
    w = np.ascontiguousarray(route_w, dtype=np.float32)
    gy = np.zeros(y.shape, np.uint16)
    gw = np.zeros((S, K), np.float64)
    lib().ref_combine_backward(_p(g), _p(y), _p(rm), _p(w), S, K, y.shape[1], _p(gy), _p(gw))
    return gy, gw


def permute_backward(grad_x_perm_bits, row_id_map, S: int, K: int) -> np.ndarray:
    gxp = np.ascontiguousarray(grad_x_perm_bits, dtype=np.uint16)
    rm = np.ascontiguousarray(row_id_map, dtype=np.int32)
    out = np.empty((S, gxp.shape[1]), np.uint16)
    lib().ref_permute_backward(_p(gxp), _p(rm), S, K, gxp.shape[1], _p(out))
    return out


def e4m3_round(v) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, np.float64)
    lib().ref_e4m3_round(_p(v), v.size, _p(out))
    return out


def mx_quantize_rows(v):
    """MXFP8 along the last axis of a 2-D array: (E4M3 values [rows, L], exponents [rows, L/32])."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    rows, L = v.shape
    q = np.empty((rows, L), np.float64)
    s = np.empty((rows, L // 32), np.int32)
    lib().ref_mx_quantize_rows(_p(v), rows, L, _p(q), _p(s))
    return q, s


def expert_backward(x, g, u, h, grad_y, wg, wu, wd):
    """One expert's backward on its n rows (all bf16 bits): (d_g, d_u, grad_x bits, dWg, dWu,
    dWd as float64)."""
    arrs = [np.ascontiguousarray(a, dtype=np.uint16) for a in (x, g, u, h, grad_y, wg, wu, wd)]
    n, H = arrs[0].shape
    Hp = arrs[1].shape[1]
    d_g = np.empty((n, Hp), np.uint16)
    d_u = np.empty((n, Hp), np.uint16)
    gx = np.empty((n, H), np.uint16)
    dwg = np.empty((H, Hp))
    dwu = np.empty((H, Hp))
    dwd = np.empty((Hp, H))
    lib().ref_expert_backward(*[_p(a) for a in arrs], n, H, Hp, _p(d_g), _p(d_u), _p(gx),
                              _p(dwg), _p(dwu), _p(dwd))
    return d_g, d_u, gx, dwg, dwu, dwd


def expert_ffn_mxfp8(x, wg, wu, wd):
    """One MXFP8 expert on its n rows (bf16 bits in): (h E4M3 values, h exponents, y bits)."""
    arrs = [np.ascontiguousarray(a, dtype=np.uint16) for a in (x, wg, wu, wd)]
    n, H = arrs[0].shape
    Hp = arrs[1].shape[1]
    hq = np.empty((n, Hp))
    hs = np.empty((n, Hp // 32), np.int32)
    y = np.empty((n, H), np.uint16)
    lib().ref_expert_ffn_mxfp8(*[_p(a) for a in arrs], n, H, Hp, _p(hq), _p(hs), _p(y))
    return hq, hs, y
