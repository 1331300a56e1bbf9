"""CPU oracle of the single-GPU MoE dispatch-compute-combine layer.

TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and bench.py's CPU
baseline (and its reference arm) may import this module. The product path never does:
it shares no code, header, table or helper with this file.

It is plain, slow and meant to be checked by eye against the pages it follows:

* "Distributed expert parallelism" (open-llm-engineering), section "The
  dispatch-compute-combine lifecycle": a token picks k experts, is copied k times,
  the copies are sorted by expert, experts run grouped FFNs, then the original token
  order is restored, each result is multiplied by its route weight and the k results
  of a token are summed.
* same page, "Token permutation and metadata": expert-contiguous order
  (expert0 tokens | expert1 tokens | ...) plus the metadata that reverses it
  (original token index, slot index, per-expert counts).
* same page, "Duplicate route accumulation": a token's top-k results are added,
  never overwritten.
* "Mixture of Kittens" teaching digest, Step 1 (The Math): every routed expert is
  Down_i(SwiGLU(Up_i x, Gate_i x)); Up and Gate expand d_model to d_expert, Down
  compresses back.
* MoonEP README, "Integration" / "Weight buffer": one contiguous weight tensor per
  projection, experts addressed purely by row index, and a cu_seqlens that selects
  each expert's rows; dispatch and combine carry bf16 hidden states and fp32 route
  weights ("API walkthrough").
* MoonEP README, "Performance": maxvio = max_e(T_e / T_bar) - 1 with T_bar the
  tokens per expert under perfect balance.

Readings where the pages are silent:
  SwiGLU(Up x, Gate x) = silu(Gate x) * (Up x), silu(z) = z / (1 + exp(-z));
  Down is stored [E, H', H] and applied as h @ W_down[e];
  inside one expert, rows keep flat order f = t*K + k (stable by token, then slot);
  cu_seqlens has E+1 entries with cu[0] = 0 (MoonEP's end offsets are cu[1:]);
  no padding rows; stored tensors (x_perm, h, y, out) are bf16 as on the pages,
  everything between two stores is exact-rounded fp64 and rounded once to bf16
  (round to nearest, ties to even); T_bar = S*K/E.

Arrays: bf16 tensors are numpy uint16 bit patterns; everything else is int32,
float32 (route weights) or float64.
"""
from __future__ import annotations

import numpy as np

# ----------------------------------------------------------------------------- bf16


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact float64 values."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round float64 values once to bf16 (nearest, ties to even) and return the bits.

    bf16 keeps 8 significant bits and fp32's exponent range: a value m * 2^e
    (0.5 <= |m| < 1) is rounded to a multiple of 2^(e-8), or of 2^-133 in the
    subnormal range. Overflow gives +-inf.
    """
    v = np.asarray(v, dtype=np.float64)
    _, e = np.frexp(v)
    q = np.maximum(e.astype(np.int64) - 8, -133)
    r = np.ldexp(np.rint(np.ldexp(v, -q)), q)  # exact power-of-two scalings; rint ties to even
    with np.errstate(over="ignore"):
        f = r.astype(np.float32)  # exact: r is a bf16 value (or overflows to inf)
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def silu(z: np.ndarray) -> np.ndarray:
    """silu(z) = z * sigmoid(z) = z / (1 + exp(-z)), in float64."""
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


# ----------------------------------------------------------------------------- permute


def permute_counting_sort(topk_ids: np.ndarray, E: int):
    """Expert-contiguous permutation by a counting sort over flat slots f = t*K + k.

    Pure-Python loops: for small cases and as a cross-check of `permute_metadata`.
    Returns (counts[E], cu_seqlens[E+1], row_id_map[S*K], perm_src[S*K]).
    """
    flat = [int(v) for v in np.asarray(topk_ids).reshape(-1)]
    for e in flat:
        if not 0 <= e < E:
            raise ValueError(f"expert id {e} outside [0, {E})")
    counts = [0] * E
    for e in flat:  # per-expert token counts
        counts[e] += 1
    cu = [0] * (E + 1)
    for e in range(E):  # exclusive scan
        cu[e + 1] = cu[e] + counts[e]
    cursor = list(cu[:E])
    row_id_map = [0] * len(flat)
    perm_src = [0] * len(flat)
    for f, e in enumerate(flat):  # increasing f keeps (token, slot) order inside an expert
        row_id_map[f] = cursor[e]
        perm_src[cursor[e]] = f
        cursor[e] += 1
    i32 = lambda a: np.asarray(a, dtype=np.int32)
    return i32(counts), i32(cu), i32(row_id_map), i32(perm_src)


def permute_metadata(topk_ids: np.ndarray, E: int):
    """Same result as `permute_counting_sort`, by a stable sort of slots by expert id.

    Returns (counts[E], cu_seqlens[E+1], row_id_map[S*K], perm_src[S*K]).
    """
    flat = np.asarray(topk_ids, dtype=np.int64).reshape(-1)
    if flat.size and (flat.min() < 0 or flat.max() >= E):
        raise ValueError("expert id outside [0, E)")
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    cu = np.zeros(E + 1, dtype=np.int64)
    np.cumsum(counts, out=cu[1:])
    perm_src = np.argsort(flat, kind="stable")  # row -> flat slot
    row_id_map = np.empty_like(perm_src)
    row_id_map[perm_src] = np.arange(flat.size)  # flat slot -> row
    return (counts.astype(np.int32), cu.astype(np.int32), row_id_map.astype(np.int32),
            perm_src.astype(np.int32))


def permute_rows(x_bits: np.ndarray, perm_src: np.ndarray, K: int) -> np.ndarray:
    """x_perm[row] = x[perm_src[row] // K] (a bit copy of the token's bf16 row)."""
    return np.asarray(x_bits)[np.asarray(perm_src, dtype=np.int64) // K]


def maxvio(counts: np.ndarray, S: int, K: int):
    """maxvio = max_e(T_e / T_bar) - 1 with T_bar = S*K/E.

    Evaluated as ((double)maxcount * E) / ((double)S * K) - 1: two exact products,
    one correctly rounded division, one subtraction. Returns (maxvio, max_count).
    """
    counts = np.asarray(counts)
    E = counts.size
    mc = int(counts.max()) if E else 0
    num = float(mc) * float(E)
    den = float(S) * float(K)
    return (num / den) - 1.0, mc


# ----------------------------------------------------------------------------- expert FFN


def expert_ffn_rows(x_rows_bits: np.ndarray, w_gate_e: np.ndarray, w_up_e: np.ndarray,
                    w_down_e: np.ndarray):
    """One expert on a block of rows: h = bf16(silu(x Wg) * (x Wu)), y = bf16(h Wd).

    x_rows_bits [n,H] bf16 bits; w_gate_e, w_up_e [H,H'] and w_down_e [H',H] as bf16
    bits. Products accumulate in float64. Returns (h_bits [n,H'], y_bits [n,H]).
    """
    x = bf16_bits_to_f64(x_rows_bits)
    g = x @ bf16_bits_to_f64(w_gate_e)
    u = x @ bf16_bits_to_f64(w_up_e)
    h_bits = f64_to_bf16_bits(silu(g) * u)
    y_bits = f64_to_bf16_bits(bf16_bits_to_f64(h_bits) @ bf16_bits_to_f64(w_down_e))
    return h_bits, y_bits


def expert_down_rows(h_rows_bits: np.ndarray, w_down_e: np.ndarray) -> np.ndarray:
    """Second half of one expert on given activations: y = bf16(h Wd), float64 products."""
    return f64_to_bf16_bits(bf16_bits_to_f64(h_rows_bits) @ bf16_bits_to_f64(w_down_e))


def grouped_ffn(x_perm_bits: np.ndarray, cu_seqlens: np.ndarray, get_weights, Hp: int):
    """Grouped expert FFN over expert-contiguous rows.

    Rows [cu[e], cu[e+1]) belong to expert e; get_weights(e) returns
    (w_gate_e [H,H'], w_up_e [H,H'], w_down_e [H',H]) as bf16 bits. Experts with no
    rows are skipped. Returns (h_bits [M,H'], y_bits [M,H]).
    """
    M, H = x_perm_bits.shape
    h = np.zeros((M, Hp), dtype=np.uint16)
    y = np.zeros((M, H), dtype=np.uint16)
    E = len(cu_seqlens) - 1
    for e in range(E):
        r0, r1 = int(cu_seqlens[e]), int(cu_seqlens[e + 1])
        if r1 == r0:
            continue
        h[r0:r1], y[r0:r1] = expert_ffn_rows(x_perm_bits[r0:r1], *get_weights(e))
    return h, y


def expert_of_rows(cu_seqlens: np.ndarray, rows: np.ndarray) -> np.ndarray:
    """Expert owning each row: the e with cu[e] <= row < cu[e+1]."""
    return np.searchsorted(np.asarray(cu_seqlens), np.asarray(rows), side="right") - 1


# ----------------------------------------------------------------------------- combine


def unpermute_combine(y_bits: np.ndarray, row_id_map: np.ndarray, route_w: np.ndarray, S: int,
                      K: int) -> np.ndarray:
    """out[t] = bf16(sum over k ascending of w[t,k] * y[row_id_map[t*K+k]]), float64 sum.

    Scatter-add semantics: a token routed twice to the same expert gets both copies.
    """
    rmap = np.asarray(row_id_map, dtype=np.int64).reshape(S, K)
    w = np.asarray(route_w, dtype=np.float32).astype(np.float64).reshape(S, K)
    H = y_bits.shape[1]
    acc = np.zeros((S, H), dtype=np.float64)
    for k in range(K):
        acc += w[:, k:k + 1] * bf16_bits_to_f64(y_bits[rmap[:, k]])
    return f64_to_bf16_bits(acc)


def combine_token(y_rows_bits: np.ndarray, w_row: np.ndarray) -> np.ndarray:
    """One token: bf16(sum_k w[k] * y_k) with y_rows_bits [K,H] in slot order."""
    w = np.asarray(w_row, dtype=np.float32).astype(np.float64)
    acc = np.zeros(y_rows_bits.shape[1], dtype=np.float64)
    for k in range(len(w)):
        acc += w[k] * bf16_bits_to_f64(y_rows_bits[k])
    return f64_to_bf16_bits(acc)


# ----------------------------------------------------------------------------- backward
#
# MoonEP README, "dispatch bwd" (sum each token's K dispatched gradient copies back to
# token-major: a combine) and "combine bwd" (scatter the output gradient back to the
# expert-grouped order by re-dispatching with the saved plan). With the layer's combine
# out[t] = sum_k w[t,k] * y[r(t,k)], r = row_id_map, the gradients are
#   grad_y[r(t,k)] = w[t,k] * grad_out[t]          (combine bwd, a weighted re-dispatch)
#   grad_w[t,k]    = <grad_out[t], y[r(t,k)]>      (route-weight gradient)
#   grad_x[t]      = sum_k grad_x_perm[r(t,k)]     (dispatch bwd, an unweighted combine)


def combine_backward(grad_out_bits: np.ndarray, y_bits: np.ndarray, row_id_map: np.ndarray,
                     route_w: np.ndarray, S: int, K: int):
    """Returns (grad_y bits [M,H], grad_w float64 [S,K]); rows that no slot maps to stay 0."""
    rmap = np.asarray(row_id_map, dtype=np.int64).reshape(S, K)
    w = np.asarray(route_w, dtype=np.float32).astype(np.float64).reshape(S, K)
    g = bf16_bits_to_f64(grad_out_bits)
    M, H = y_bits.shape
    grad_y = np.zeros((M, H), dtype=np.uint16)
    grad_w = np.zeros((S, K), dtype=np.float64)
    for k in range(K):
        grad_y[rmap[:, k]] = f64_to_bf16_bits(w[:, k:k + 1] * g)
        grad_w[:, k] = np.sum(g * bf16_bits_to_f64(y_bits[rmap[:, k]]), axis=1)
    return grad_y, grad_w


def permute_backward(grad_x_perm_bits: np.ndarray, row_id_map: np.ndarray, S: int, K: int):
    """grad_x[t] = bf16(sum over k ascending of grad_x_perm[r(t,k)]), float64 sum."""
    rmap = np.asarray(row_id_map, dtype=np.int64).reshape(S, K)
    acc = np.zeros((S, grad_x_perm_bits.shape[1]), dtype=np.float64)
    for k in range(K):
        acc += bf16_bits_to_f64(grad_x_perm_bits[rmap[:, k]])
    return f64_to_bf16_bits(acc)


# ----------------------------------------------------------------------------- expert FFN backward
#
# The pages give the forward of an expert, Down(SwiGLU(Up x, Gate x)) ("Mixture of Kittens"
# digest, Step 1), and say that training keeps one fp32 gradient buffer per projection laid
# out like the weights (MoonEP README, "Gradient buffers"). The backward below is the chain
# rule of that forward. Readings: the training forward stores the gate and up
# pre-activations g = x Wg and u = x Wu as bf16 tensors (like every stored activation),
# and the backward starts from those; grad_h is not stored (it stays exact up to d_g and
# d_u); d_g, d_u and grad_x_perm are stored bf16; weight gradients are stored fp32.
# With s = sigmoid(g): silu(g) = g s, silu'(g) = s (1 + g (1 - s)), and for h = silu(g) u
#   grad_h = grad_y Wd^T
#   d_u    = grad_h * silu(g)              d_g = grad_h * u * silu'(g)
#   grad_x = d_g Wg^T + d_u Wu^T
#   dWg    = x^T d_g    dWu = x^T d_u    dWd = h^T grad_y     (sums over the expert's rows)


def expert_preact_rows(x_rows_bits: np.ndarray, w_gate_e: np.ndarray, w_up_e: np.ndarray):
    """Pre-activations saved by the training forward: (bf16(x Wg), bf16(x Wu)) bits."""
    x = bf16_bits_to_f64(x_rows_bits)
    return (f64_to_bf16_bits(x @ bf16_bits_to_f64(w_gate_e)),
            f64_to_bf16_bits(x @ bf16_bits_to_f64(w_up_e)))


def swiglu_backward(grad_h: np.ndarray, g_bits: np.ndarray, u_bits: np.ndarray):
    """(d_g bits, d_u bits) of h = silu(g) * u for a float64 grad_h and saved bf16 g, u."""
    g = bf16_bits_to_f64(g_bits)
    u = bf16_bits_to_f64(u_bits)
    s = 1.0 / (1.0 + np.exp(-g))
    return (f64_to_bf16_bits(grad_h * u * (s * (1.0 + g * (1.0 - s)))),
            f64_to_bf16_bits(grad_h * (g * s)))


def expert_down_backward_rows(grad_y_bits, g_bits, u_bits, w_down_e):
    """Down projection and SwiGLU backward of one expert's rows: (d_g bits, d_u bits)."""
    grad_h = bf16_bits_to_f64(grad_y_bits) @ bf16_bits_to_f64(w_down_e).T
    return swiglu_backward(grad_h, g_bits, u_bits)


def expert_up_gate_backward_rows(dg_bits, du_bits, w_gate_e, w_up_e):
    """Input-row gradient of one expert: bf16(d_g Wg^T + d_u Wu^T), one rounding."""
    return f64_to_bf16_bits(bf16_bits_to_f64(dg_bits) @ bf16_bits_to_f64(w_gate_e).T +
                            bf16_bits_to_f64(du_bits) @ bf16_bits_to_f64(w_up_e).T)


def expert_weight_grads_rows(x_rows_bits, h_bits, dg_bits, du_bits, grad_y_bits):
    """Weight gradients of one expert as float64 sums over its rows: (x^T d_g, x^T d_u,
    h^T grad_y)."""
    x = bf16_bits_to_f64(x_rows_bits)
    return (x.T @ bf16_bits_to_f64(dg_bits), x.T @ bf16_bits_to_f64(du_bits),
            bf16_bits_to_f64(h_bits).T @ bf16_bits_to_f64(grad_y_bits))


def expert_ffn_backward_rows(x_rows_bits, g_bits, u_bits, h_bits, grad_y_bits, w_gate_e, w_up_e,
                             w_down_e):
    """Backward of one expert on a block of rows: the three stages above in order.

    Returns (d_g bits, d_u bits, grad_x bits, dWg, dWu, dWd), the weight gradients as
    float64 sums of the block's rows (the caller stores them as fp32).
    """
    dg_bits, du_bits = expert_down_backward_rows(grad_y_bits, g_bits, u_bits, w_down_e)
    grad_x = expert_up_gate_backward_rows(dg_bits, du_bits, w_gate_e, w_up_e)
    return (dg_bits, du_bits, grad_x,
            *expert_weight_grads_rows(x_rows_bits, h_bits, dg_bits, du_bits, grad_y_bits))


def grouped_ffn_preact(x_perm_bits: np.ndarray, cu_seqlens: np.ndarray, get_weights, Hp: int):
    """Saved pre-activations of the whole grouped FFN: (g bits [M,H'], u bits [M,H'])."""
    M = x_perm_bits.shape[0]
    g = np.zeros((M, Hp), dtype=np.uint16)
    u = np.zeros((M, Hp), dtype=np.uint16)
    for e in range(len(cu_seqlens) - 1):
        r0, r1 = int(cu_seqlens[e]), int(cu_seqlens[e + 1])
        if r1 > r0:
            wg, wu, _ = get_weights(e)
            g[r0:r1], u[r0:r1] = expert_preact_rows(x_perm_bits[r0:r1], wg, wu)
    return g, u


def grouped_ffn_backward(x_perm_bits, g_bits, u_bits, h_bits, grad_y_bits, cu_seqlens,
                         get_weights, dw_prior=None):
    """Backward of the grouped FFN over expert-contiguous rows.

    Returns a dict: d_g, d_u, grad_x_perm (bf16 bits) and dWg [E,H,H'], dWu [E,H,H'],
    dWd [E,H',H] as float32. An expert with no rows gets zero weight gradients. With
    dw_prior = (Pg, Pu, Pd) the weight gradients are added to those fp32 buffers, each
    element rounded once (fp64 sum of the prior value and the exact product sum).
    """
    M, H = x_perm_bits.shape
    Hp = g_bits.shape[1]
    E = len(cu_seqlens) - 1
    out = dict(d_g=np.zeros((M, Hp), np.uint16), d_u=np.zeros((M, Hp), np.uint16),
               grad_x_perm=np.zeros((M, H), np.uint16))
    dw = [np.zeros((E, H, Hp)), np.zeros((E, H, Hp)), np.zeros((E, Hp, H))]
    if dw_prior is not None:
        dw = [np.asarray(p, dtype=np.float32).astype(np.float64) for p in dw_prior]
    for e in range(E):
        r0, r1 = int(cu_seqlens[e]), int(cu_seqlens[e + 1])
        if r1 == r0:
            continue
        res = expert_ffn_backward_rows(x_perm_bits[r0:r1], g_bits[r0:r1], u_bits[r0:r1],
                                       h_bits[r0:r1], grad_y_bits[r0:r1], *get_weights(e))
        out["d_g"][r0:r1], out["d_u"][r0:r1], out["grad_x_perm"][r0:r1] = res[:3]
        for i in range(3):
            dw[i][e] += res[3 + i]
    out["dWg"], out["dWu"], out["dWd"] = (d.astype(np.float32) for d in dw)
    return out


# ----------------------------------------------------------------------------- MXFP8
#
# "Mixture of Kittens" digest, Step 8 (MXFP8 Support): an MXFP8 mode with weights quantised
# once ahead of time and activation quantisation fused into dispatch, the GEMMs and SwiGLU;
# the shared expert stays in bf16. The pages do not spell the format out; these functions
# follow the public OCP Microscaling (MX) v1.0 definition of MXFP8: blocks of 32 consecutive
# elements along the reduction dimension share one power-of-two scale X = 2^(floor(log2
# amax) - 8) (8 = exponent of E4M3's largest normal), stored as E8M0 (exponent in
# [-127, 127]); each element is V / X rounded to nearest-even in FP8 E4M3 (3 mantissa bits,
# exponent bias 7, subnormal step 2^-9, largest finite 448, no infinities). Reading: values
# of V / X above 448 (possible since amax / X lies in [256, 512)) saturate to +-448.
# Products of two MXFP8 values are exact in float64; dot products here accumulate in float64.

MX_BLOCK = 32
E4M3_MAX = 448.0
E4M3_EMAX = 8


def e4m3_round(v: np.ndarray) -> np.ndarray:
    """Round float64 values to FP8 E4M3 (nearest, ties to even), saturating at +-448."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    _, fe = np.frexp(np.where(a > 0, a, 1.0))
    e = (fe - 1).astype(np.float64)  # floor(log2 a), exactly
    e = np.maximum(e, -6.0)  # below 2^-6 the spacing is the subnormal step 2^-9
    step = np.ldexp(1.0, (e - 3).astype(np.int64))
    q = np.minimum(np.rint(a / step) * step, E4M3_MAX)
    return np.copysign(q, v)


def mx_quantize(v: np.ndarray, axis: int = -1):
    """MXFP8 quantisation in blocks of 32 along `axis` (its length a multiple of 32).

    Returns (elements, scale exponents): elements are the E4M3 values as float64, with the
    shape of v; scale exponents are int64 with axis length / 32 blocks along `axis`."""
    v = np.moveaxis(np.asarray(v, dtype=np.float64), axis, -1)
    n = v.shape[-1]
    assert n % MX_BLOCK == 0
    blocks = v.reshape(v.shape[:-1] + (n // MX_BLOCK, MX_BLOCK))
    amax = np.abs(blocks).max(axis=-1)
    # floor(log2 amax) exactly: frexp gives amax = m * 2^e with m in [0.5, 1) (a rounded log2
    # would be one too large just below a power of two)
    _, e = np.frexp(np.where(amax > 0, amax, 1.0))
    sexp = np.where(amax > 0, (e - 1).astype(np.float64) - E4M3_EMAX, -127.0)
    sexp = np.clip(sexp, -127, 127).astype(np.int64)
    q = e4m3_round(blocks / np.ldexp(1.0, sexp)[..., None])
    return (np.moveaxis(q.reshape(v.shape), -1, axis),
            np.moveaxis(sexp, -1, axis))


def mx_dequantize(q: np.ndarray, sexp: np.ndarray, axis: int = -1) -> np.ndarray:
    """Elements times their block's scale (float64, exact)."""
    q = np.moveaxis(np.asarray(q, dtype=np.float64), axis, -1)
    s = np.moveaxis(np.asarray(sexp), axis, -1)
    out = q * np.repeat(np.ldexp(1.0, s), MX_BLOCK, axis=-1)
    return np.moveaxis(out, -1, axis)


def mx_weights(w_bits: np.ndarray):
    """Pre-quantised expert weights [.., k, n] (bf16 bits): blocks of 32 along k, the
    reduction dimension (axis -2). Returns (elements, scale exponents)."""
    return mx_quantize(bf16_bits_to_f64(w_bits), axis=-2)


def expert_ffn_rows_mxfp8(x_rows_bits, w_gate_q, w_up_q, w_down_q):
    """One expert in MXFP8: x quantised along H, h = silu(g) * u quantised along H' (fused in
    the SwiGLU epilogue), weights pre-quantised along their reduction dimension (mx_weights);
    products exact, sums in float64; y = bf16(deq(h_q) . deq(Wd_q)). Returns
    (h elements, h scale exponents, y bits)."""
    xq, xs = mx_quantize(bf16_bits_to_f64(x_rows_bits), axis=-1)
    x = mx_dequantize(xq, xs, axis=-1)
    g = x @ mx_dequantize(*w_gate_q, axis=-2)
    u = x @ mx_dequantize(*w_up_q, axis=-2)
    hq, hs = mx_quantize(silu(g) * u, axis=-1)
    y = mx_dequantize(hq, hs, axis=-1) @ mx_dequantize(*w_down_q, axis=-2)
    return hq, hs, f64_to_bf16_bits(y)


# ----------------------------------------------------------------------------- whole layer


def moe_layer(x_bits: np.ndarray, topk_ids: np.ndarray, route_w: np.ndarray, E: int, get_weights,
              Hp: int, identity_ffn: bool = False):
    """permute -> grouped FFN (or identity experts) -> weighted combine, plus maxvio.

    Returns a dict with counts, cu_seqlens, row_id_map, perm_src, maxvio, max_count,
    x_perm, h (None for identity experts), y and out.
    """
    S, K = np.asarray(topk_ids).shape
    counts, cu, rmap, psrc = permute_metadata(topk_ids, E)
    mv, mc = maxvio(counts, S, K)
    x_perm = permute_rows(x_bits, psrc, K)
    if identity_ffn:
        h, y = None, x_perm
    else:
        h, y = grouped_ffn(x_perm, cu, get_weights, Hp)
    out = unpermute_combine(y, rmap, route_w, S, K)
    return dict(counts=counts, cu_seqlens=cu, row_id_map=rmap, perm_src=psrc, maxvio=mv,
                max_count=mc, x_perm=x_perm, h=h, y=y, out=out)


def moe_layer_with_shared(x_bits: np.ndarray, topk_ids: np.ndarray, route_w: np.ndarray, E: int,
                          get_weights, Hp: int, shared_weights):
    """MoE(x) = SharedExpert(x) + sum over the top-k of router_weight_k * RoutedExpert_k(x)
    ("Mixture of Kittens" digest, Step 1, The Math). The shared expert is one SwiGLU FFN
    (shared_weights = (Wg_s [H,Hs], Wu_s [H,Hs], Wd_s [Hs,H]) bf16 bits) applied to every
    token; its output y_shared is a stored bf16 tensor like every expert output, and
    out[t] = bf16(y_shared[t] + sum_k w[t,k] * y[r(t,k)]) with one rounding.
    Returns moe_layer's dict with y_shared added and out replaced."""
    S, K = np.asarray(topk_ids).shape
    base = moe_layer(x_bits, topk_ids, route_w, E, get_weights, Hp)
    _, ys = expert_ffn_rows(x_bits, *shared_weights)
    rmap = np.asarray(base["row_id_map"], dtype=np.int64).reshape(S, K)
    w = np.asarray(route_w, dtype=np.float32).astype(np.float64).reshape(S, K)
    acc = bf16_bits_to_f64(ys).copy()
    for k in range(K):
        acc += w[:, k:k + 1] * bf16_bits_to_f64(base["y"][rmap[:, k]])
    return dict(base, y_shared=ys, out=f64_to_bf16_bits(acc))


def direct_expert_loop(x_bits: np.ndarray, topk_ids: np.ndarray, route_w: np.ndarray, get_weights):
    """The same layer without any permutation: for every token, run each of its K
    experts on the token's own row and add the weighted results ("Distributed expert parallelism", Exercises, item 3).
    Returns out bits [S,H]."""
    S, K = np.asarray(topk_ids).shape
    H = x_bits.shape[1]
    out = np.zeros((S, H), dtype=np.uint16)
    for t in range(S):
        ys = np.zeros((K, H), dtype=np.uint16)
        for k in range(K):
            e = int(topk_ids[t, k])
            _, ys[k] = expert_ffn_rows(x_bits[t:t + 1], *get_weights(e))
        out[t] = combine_token(ys, route_w[t])
    return out
