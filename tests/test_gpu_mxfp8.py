"""Parity of the MXFP8 path with the fp64 oracle's MXFP8 functions (OCP Microscaling v1.0
MXFP8, the precision mode of the "Mixture of Kittens" digest, Step 8).

* Quantisation of weights and of the permuted token rows decides integer codes from exact
  bf16 inputs on both sides: codes and scales must match bit for bit.
* h is quantised from the GPU's fp32 sums and from the oracle's exact sums, so a code may sit
  one E4M3 step (and, where the block maximum lies at a power of two, a scale may sit one
  binade) away where the exact value is next to a rounding boundary. Such elements must be
  within one step of the oracle's value and rare.
* y is checked twice: against the oracle's down projection of the GPU's own h (only the fp32
  accumulation differs: the bf16 acceptance bar), and end to end against the oracle chain.

Inputs are the seeded normal draws with every 32-element block along the reduction dimension
scaled by its own power of two 2^k, k in [-6, 6], so that each block has its own scale and a
scale read from the wrong place changes the result by powers of two; one block of x and one
of each weight are zero (scale byte 0).
"""
import numpy as np
import pytest
import torch

import grouped_ffn_moe_b200 as moe
import synth
from helpers import GUARD, assert_close_bf16, bits
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu

TAG_SHIFT = 64  # added to a tensor's tag for its block-exponent draws


# ----------------------------------------------------------------------------- inputs

def shift_exponent(b: np.ndarray, k: np.ndarray) -> np.ndarray:
    """bf16 bit patterns times 2^k (exact: only the exponent field moves); zeros stay zero."""
    b = b.astype(np.int64)
    e = (b >> 7) & 0xFF
    nz = e > 0
    e2 = e + k
    assert ((e2[nz] >= 1) & (e2[nz] <= 254)).all()
    return np.where(nz, (b & ~(0xFF << 7)) | (e2 << 7), b).astype(np.uint16)


def block_scaled_bits(seed: int, tag: int, shape, axis: int, sigma: float) -> np.ndarray:
    n = int(np.prod(shape))
    b = np.moveaxis(synth.normal_bf16_bits(seed, tag, n, sigma).reshape(shape), axis, -1)
    nblk = b.shape[:-1] + (b.shape[-1] // 32,)
    u = synth.uniform(seed, tag + TAG_SHIFT, int(np.prod(nblk))).reshape(nblk)
    k = np.repeat(np.floor(u * 13).astype(np.int64) - 6, 32, axis=-1)
    return np.ascontiguousarray(np.moveaxis(shift_exponent(b, k), -1, axis))


def to_dev(b: np.ndarray, dev) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).to(dev)


def decode_e4m3(u8: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(u8, dtype=np.uint8))
    return t.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def unpack_weight_scales(sf: np.ndarray, E: int, R: int, C: int) -> np.ndarray:
    """The chunked scale bytes of include/moe_b200.h -> scale exponents [E, R/32, C]."""
    a = np.asarray(sf, np.uint8)[: E * (R // 32) * C].reshape(E, C // 128, R // 128, 512)
    fl = np.arange(128)[:, None]
    kb = np.arange(4)[None, :]
    g = a[..., (fl % 32) * 16 + (fl // 32) * 4 + kb]          # [E, C/128, R/128, 128, 4]
    g = g.transpose(0, 2, 4, 1, 3).reshape(E, R // 32, C)     # (e, kt, kb, fb, fl)
    return g.astype(np.int64) - 127


def make_weights(seed: int, E: int, H: int, Hp: int):
    wg = block_scaled_bits(seed, synth.TAG_W_GATE, (E, H, Hp), 1, 0.05)
    wu = block_scaled_bits(seed, synth.TAG_W_UP, (E, H, Hp), 1, 0.05)
    wd = block_scaled_bits(seed, synth.TAG_W_DOWN, (E, Hp, H), 1, 0.05)
    wg[0, 32:64, 3] = 0
    wu[E - 1, :32, Hp - 1] = 0
    wd[0, 64:96, 7] = 0
    return wg, wu, wd


def check_h(hq_gpu: np.ndarray, hs_gpu: np.ndarray, hq_ref: np.ndarray, hs_ref: np.ndarray,
            what: str):
    """GPU h (E4M3 values, scale exponents) against the oracle's: differences only where the
    exact value lies at a rounding boundary, each within one step of the oracle's value."""
    deq_g = O.mx_dequantize(hq_gpu, hs_gpu, axis=-1)
    deq_r = O.mx_dequantize(hq_ref, hs_ref, axis=-1)
    # one step in the top binade of the oracle's block (the largest spacing in the block)
    step = np.repeat(np.ldexp(1.0, hs_ref + 5), O.MX_BLOCK, axis=-1)
    diff = np.abs(deq_g - deq_r)
    assert (diff <= step).all(), f"{what}: {(diff > step).sum()} h values beyond one step"
    n_code = int((diff > 0).sum())
    n_scale = int((hs_gpu != hs_ref).sum())
    stats = dict(code_mismatch=n_code / diff.size, scale_mismatch=n_scale / hs_ref.size)
    print(f"{what}: h {stats}")
    assert n_code <= 2e-3 * diff.size + 4, f"{what}: {n_code} h codes differ ({stats})"
    assert n_scale <= 2e-3 * hs_ref.size + 2, f"{what}: {n_scale} h scales differ ({stats})"
    return stats


# ----------------------------------------------------------------------------- quantisation

def test_mx_quantize_weights_bit_exact(cuda_device):
    E, R, C = 3, 256, 384
    w = block_scaled_bits(5, synth.TAG_W_GATE, (E, R, C), 1, 0.05)
    w[1, 32:64, 5] = 0
    w_q, w_sf = moe.mx_quantize_weights(to_dev(w, cuda_device))
    torch.cuda.synchronize()
    q_ref, s_ref = O.mx_weights(w)
    assert np.array_equal(decode_e4m3(w_q.cpu().numpy()), q_ref)
    assert np.array_equal(unpack_weight_scales(w_sf.cpu().numpy(), E, R, C), s_ref)
    assert s_ref[1, 1, 5] == -127  # the zero block


@pytest.mark.parametrize("S,H,K,E", [(300, 512, 4, 16), (64, 7168, 8, 384), (1, 128, 1, 1)])
def test_mx_permute_quantize_bit_exact(cuda_device, S, H, K, E):
    dev = cuda_device
    x = block_scaled_bits(7, synth.TAG_X, (S, H), 1, 1.0)
    x[0] = 0
    if S > 9:
        x[9, 64:96] = 0
    ids_np, _ = synth.route_es(7, S, K, E)
    ids = torch.from_numpy(ids_np.reshape(S, K)).to(dev)
    M = S * K
    i32 = torch.int32
    counts, cu = GUARD((E,), i32, dev), GUARD((E + 1,), i32, dev)
    rmap, psrc = GUARD((M,), i32, dev), GUARD((M,), i32, dev)
    moe.moe_permute(to_dev(x, dev), ids, E, None, counts, cu, rmap, psrc)
    x_q = GUARD.full((M, H), 0xEE, torch.uint8, dev)
    x_sf = GUARD.full((M, H // 32), 0xEE, torch.uint8, dev)
    moe.moe_mx_permute_quantize(to_dev(x, dev), rmap, K, x_q, x_sf)
    torch.cuda.synchronize()
    _, _, rmap_ref, psrc_ref = O.permute_metadata(ids_np.reshape(S, K), E)
    assert np.array_equal(rmap.cpu().numpy(), rmap_ref)
    q_ref, s_ref = O.mx_quantize(O.bf16_bits_to_f64(O.permute_rows(x, psrc_ref, K)), axis=-1)
    assert np.array_equal(decode_e4m3(x_q.cpu().numpy()), q_ref)
    assert np.array_equal(x_sf.cpu().numpy().astype(np.int64) - 127, s_ref)


# ----------------------------------------------------------------------------- grouped FFN

FFN_CASES = {
    # name: (E, H, Hp, rows per expert) -- empty experts, a single row, rows just above and
    # below a unit (224), several units, several 128-feature blocks
    "tiny": (4, 256, 256, [0, 17, 100, 250]),
    "ragged": (6, 384, 512, [1, 224, 225, 0, 31, 480]),
    "wide": (3, 1024, 768, [300, 64, 129]),
    # the largest expert count (full per-expert tables): mostly 0-3 rows, a hot expert last
    "many": (1024, 128, 256, [i % 4 for i in range(1023)] + [150]),
}


@pytest.mark.parametrize("case", list(FFN_CASES))
def test_mx_grouped_ffn_parity(cuda_device, case):
    dev = cuda_device
    E, H, Hp, rows = FFN_CASES[case]
    M = int(sum(rows))
    cu_np = np.concatenate([[0], np.cumsum(rows)]).astype(np.int32)
    x = block_scaled_bits(11, synth.TAG_X, (M, H), 1, 1.0)
    x[min(3, M - 1), 32:64] = 0
    wg, wu, wd = make_weights(13, E, H, Hp)
    mw = moe.MxWeights.from_bf16(to_dev(wg, dev), to_dev(wu, dev), to_dev(wd, dev))
    u8 = torch.uint8
    x_q, x_sf = GUARD((M, H), u8, dev), GUARD((M, H // 32), u8, dev)
    ident = torch.arange(M, dtype=torch.int32, device=dev)
    moe.moe_mx_permute_quantize(to_dev(x, dev), ident, 1, x_q, x_sf)
    cu = torch.from_numpy(cu_np).to(dev)
    h_q = GUARD.full((M, Hp), 0xEE, u8, dev)
    h_sf = GUARD.full((M, Hp // 32), 0xEE, u8, dev)
    y = GUARD.full((M, H), float("nan"), torch.bfloat16, dev)
    status = GUARD.zeros((1,), torch.int32, dev)
    moe.moe_grouped_ffn_mxfp8(x_q, x_sf, mw, cu, h_q, h_sf, y, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    hq_g = decode_e4m3(h_q.cpu().numpy())
    hs_g = h_sf.cpu().numpy().astype(np.int64) - 127
    y_g = bits(y)
    gq, gs = O.mx_weights(wg)
    uq, us = O.mx_weights(wu)
    dq, ds = O.mx_weights(wd)
    hq_r, hs_r = np.zeros((M, Hp)), np.zeros((M, Hp // 32), np.int64)
    y_r = np.zeros((M, H), np.uint16)
    y_from_gpu_h = np.zeros((M, H), np.uint16)
    for e in range(E):
        r0, r1 = int(cu_np[e]), int(cu_np[e + 1])
        if r1 == r0:
            continue
        hq_r[r0:r1], hs_r[r0:r1], y_r[r0:r1] = O.expert_ffn_rows_mxfp8(
            x[r0:r1], (gq[e], gs[e]), (uq[e], us[e]), (dq[e], ds[e]))
        h_deq = O.mx_dequantize(hq_g[r0:r1], hs_g[r0:r1], axis=-1)
        y_from_gpu_h[r0:r1] = O.f64_to_bf16_bits(h_deq @ O.mx_dequantize(dq[e], ds[e], axis=-2))
    check_h(hq_g, hs_g, hq_r, hs_r, f"{case} h")
    s1 = assert_close_bf16(y_g, y_from_gpu_h, f"{case} y (oracle down on the GPU's h)")
    s2 = assert_close_bf16(y_g, y_r, f"{case} y (oracle chain)")
    print(f"{case}: y vs oracle down {s1}; y vs oracle chain {s2}")


def test_mx_layer_end_to_end(cuda_device):
    """The MXFP8 layer (routing, permute-quantise, MXFP8 FFN, combine) against the oracle."""
    dev = cuda_device
    S, H, Hp, E, K = 256, 1024, 512, 8, 4
    x = block_scaled_bits(17, synth.TAG_X, (S, H), 1, 1.0)
    ids_np, _ = synth.route_es(17, S, K, E, hot_e=2, w_hot=6.0)
    ids_np = ids_np.reshape(S, K)
    rw = synth.route_weights(17, S, K)
    wg, wu, wd = make_weights(19, E, H, Hp)
    mw = moe.MxWeights.from_bf16(to_dev(wg, dev), to_dev(wu, dev), to_dev(wd, dev))
    buf = moe.LayerBuffers.allocate(S, H, Hp, E, K, dev, alloc=GUARD.for_device(dev))
    mxbuf = moe.MxBuffers.allocate(S, H, Hp, K, dev, alloc=GUARD.for_device(dev))
    ids = torch.from_numpy(ids_np).to(dev)
    route_w = torch.from_numpy(np.asarray(rw, np.float32).reshape(S, K)).to(dev)
    out = moe.moe_layer_forward_mxfp8(to_dev(x, dev), ids, route_w, mw, buf, mxbuf)
    torch.cuda.synchronize()
    assert int(buf.d_status.item()) == 0
    counts, cu, rmap, psrc = O.permute_metadata(ids_np, E)
    assert np.array_equal(buf.cu_seqlens.cpu().numpy(), cu)
    assert counts.max() > 224  # the hot expert spans several units
    x_perm = O.permute_rows(x, psrc, K)
    gq, gs = O.mx_weights(wg)
    uq, us = O.mx_weights(wu)
    dq, ds = O.mx_weights(wd)
    hq_r, hs_r = np.zeros((S * K, Hp)), np.zeros((S * K, Hp // 32), np.int64)
    y_r = np.zeros((S * K, H), np.uint16)
    for e in range(E):
        r0, r1 = int(cu[e]), int(cu[e + 1])
        if r1 > r0:
            hq_r[r0:r1], hs_r[r0:r1], y_r[r0:r1] = O.expert_ffn_rows_mxfp8(
                x_perm[r0:r1], (gq[e], gs[e]), (uq[e], us[e]), (dq[e], ds[e]))
    check_h(decode_e4m3(mxbuf.h_q.cpu().numpy()), mxbuf.h_sf.cpu().numpy().astype(np.int64) - 127,
            hq_r, hs_r, "layer h")
    assert_close_bf16(bits(buf.y), y_r, "layer y")
    out_r = O.unpermute_combine(y_r, rmap, np.asarray(rw, np.float32), S, K)
    st = assert_close_bf16(bits(out), out_r, "layer out")
    print(f"layer out {st}")


def test_mx_device_wait_timeout_reports_status(cuda_device):
    """Failure detection without a fault: with a 1 ns wait budget the MXFP8 passes' pipeline
    waits run out; they record MOE_ERR_DEVICE_TIMEOUT, drain their own copies (TMA, the scale
    warp's cp.async) and MMAs, free TMEM and return, and the CUDA context stays usable."""
    import os
    import subprocess
    import sys

    script = (
        "import torch, synth, grouped_ffn_moe_b200 as moe\n"
        "w = synth.WORKLOADS['tiny']\n"
        "dev = torch.device('cuda:0')\n"
        "inp = synth.make_layer_inputs(w, device='cuda:0')\n"
        "mw = moe.MxWeights.from_bf16(inp['w_gate'], inp['w_up'], inp['w_down'])\n"
        "buf = moe.LayerBuffers.allocate(w.S, w.H, w.Hp, w.E, w.K, dev)\n"
        "mxb = moe.MxBuffers.allocate(w.S, w.H, w.Hp, w.K, dev)\n"
        "moe.moe_layer_forward_mxfp8(inp['x'], inp['topk_ids'], inp['route_w'], mw, buf, mxb)\n"
        "torch.cuda.synchronize()\n"
        "st = int(buf.d_status.item())\n"
        "assert st & moe.MOE_ERR_DEVICE_TIMEOUT, st\n"
        "assert torch.arange(1000, device='cuda:0').sum().item() == 499500\n"
        "print('timeout status', st)\n")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, PYTHONPATH=root, MOE_WAIT_BUDGET_NS="1")
    r = subprocess.run([sys.executable, "-c", script], env=env, cwd=root, timeout=600,
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "timeout status" in r.stdout
