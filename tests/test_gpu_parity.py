"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle.

Integer outputs (counts, cu_seqlens, row_id_map, perm_src, max count, maxvio, x_perm) must
match bit for bit; bf16 outputs (h, y, out) must meet the acceptance bar in helpers.py.
Small workloads are compared element by element in full; the full-size workloads on
sampled rows and tokens that the oracle recomputes one by one.
"""
import json
import os
import zlib

import numpy as np
import pytest
import torch

import grouped_ffn_moe_b200 as moe
import synth
from helpers import GUARD, assert_close_bf16, bf16_ulp, bits, f64
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- helpers

def gpu_permute(x, ids, E, with_rows=True):
    S, K = ids.shape
    dev = ids.device
    H = x.shape[1]
    M = S * K
    i32 = torch.int32
    r = dict(
        x_perm=GUARD.full((M, H), float("nan"), torch.bfloat16, dev) if with_rows else None,
        counts=GUARD.full((E,), -7, i32, dev), cu=GUARD.full((E + 1,), -7, i32, dev),
        rmap=GUARD.full((M,), -7, i32, dev), psrc=GUARD.full((M,), -7, i32, dev),
        maxvio=GUARD.full((1,), -7.0, torch.float64, dev),
        max_count=GUARD.full((1,), -7, i32, dev), status=GUARD.zeros((1,), i32, dev))
    moe.moe_permute(x, ids, E, r["x_perm"], r["counts"], r["cu"], r["rmap"], r["psrc"], r["maxvio"],
                    r["max_count"], d_status=r["status"])
    torch.cuda.synchronize()
    return r


def check_permute_exact(r, ids_np, E, x_bits=None, sample_rows=None):
    S, K = ids_np.shape
    counts, cu, rmap, psrc = O.permute_metadata(ids_np, E)
    mv, mc = O.maxvio(counts, S, K)
    assert np.array_equal(r["counts"].cpu().numpy(), counts)
    assert np.array_equal(r["cu"].cpu().numpy(), cu)
    assert np.array_equal(r["rmap"].cpu().numpy(), rmap)
    assert np.array_equal(r["psrc"].cpu().numpy(), psrc)
    assert int(r["max_count"].item()) == mc
    assert r["maxvio"].item() == mv  # same IEEE expression: bit-exact
    assert int(r["status"].item()) == 0
    if x_bits is not None and r["x_perm"] is not None:
        if sample_rows is None:
            assert np.array_equal(bits(r["x_perm"]), O.permute_rows(x_bits, psrc, K))
        else:
            got = bits(r["x_perm"][torch.as_tensor(sample_rows, device=r["x_perm"].device)])
            assert np.array_equal(got, x_bits[psrc[sample_rows] // K])
    return counts, cu, rmap, psrc


def layer_inputs(w, dev):
    return synth.make_layer_inputs(w, device=str(dev))


def weights_getter(inp):
    cache = {}

    def get(e):
        if e not in cache:
            cache.clear()
            cache[e] = (bits(inp["w_gate"][e]), bits(inp["w_up"][e]), bits(inp["w_down"][e]))
        return cache[e]
    return get


def run_layer(inp, w, dev):
    buf = moe.LayerBuffers.allocate(w.S, w.H, w.Hp, w.E, w.K, dev, with_ffn=not w.identity_ffn,
                                    alloc=GUARD.for_device(dev))
    moe.moe_layer_forward(inp["x"], inp["topk_ids"], inp["route_w"], inp.get("w_gate"),
                          inp.get("w_up"), inp.get("w_down"), buf)
    torch.cuda.synchronize()
    assert int(buf.d_status.item()) == 0
    return buf


# ----------------------------------------------------------------------------- permute

def test_permute_four_rank_worked_example(cuda_device):
    g = json.load(open(os.path.join(GOLDEN, "four_rank_example.json")))
    ids = torch.tensor(g["topk_ids"], dtype=torch.int32, device=cuda_device)
    x = torch.arange(3 * 8, dtype=torch.float32, device=cuda_device).reshape(3, 8).to(torch.bfloat16)
    r = gpu_permute(x, ids, g["E"])
    assert r["counts"].tolist() == g["counts"]
    assert r["cu"].tolist() == g["cu_seqlens"]
    assert r["psrc"].tolist() == g["perm_src"]
    assert r["rmap"].tolist() == g["row_id_map"]
    assert r["max_count"].item() == g["max_count"]
    assert abs(r["maxvio"].item() - 5.0 / 3.0) <= 4e-16
    xp = r["x_perm"].float().cpu().numpy()
    for f, row in enumerate(g["row_id_map"]):
        assert np.array_equal(xp[row], x.float().cpu().numpy()[f // 2])


def _routing_case(name):
    rng = np.random.default_rng(zlib.crc32(name.encode()))
    if name == "one_expert_k1":
        return np.zeros((777, 1), np.int32), 5
    if name == "empty_experts":
        return rng.choice([1, 4, 9], size=(300, 2)).astype(np.int32), 12
    if name == "duplicates":
        return rng.integers(0, 6, size=(513, 4)).astype(np.int32), 6
    if name == "ragged":
        return rng.integers(0, 7, size=(1001, 3)).astype(np.int32), 7
    if name == "e_max":
        return rng.integers(0, 1024, size=(3000, 8)).astype(np.int32), 1024
    if name == "many_chunks":
        return rng.integers(0, 384, size=(20000, 8)).astype(np.int32), 384
    if name == "e4096":  # four expert windows of the cluster kernel
        return rng.integers(0, 4096, size=(3000, 8)).astype(np.int32), 4096
    if name == "e65535":  # the largest E: 64 windows, ids at both ends of the range
        ids = rng.integers(0, 65535, size=(4001, 6)).astype(np.int32)
        ids[:50, 0], ids[50:100, 1], ids[100:140, 2] = 0, 65534, 1023
        return ids, 65535
    if name == "e3000_hot":  # a hot expert in the last, partial window
        ids = rng.integers(0, 3000, size=(5000, 4)).astype(np.int32)
        ids[::3, 1] = 2999
        return ids, 3000
    if name == "cluster_max":  # exactly 2^17 slots: the cluster kernel's largest table
        return rng.integers(0, 384, size=(16384, 8)).astype(np.int32), 384
    if name == "coop_min":  # one slot more: the cooperative kernel
        return rng.integers(0, 384, size=(16385, 8)).astype(np.int32)[:, :8], 384
    if name == "coop_e64":  # the cooperative kernel and its workspace at 1.57 M slots
        return rng.integers(0, 64, size=(262147, 6)).astype(np.int32), 64
    if name == "coop_e1024":
        return rng.integers(0, 1024, size=(135001, 8)).astype(np.int32), 1024
    if name == "e4096_large":  # E > 1024 above 2^17 slots: still the cluster kernel
        return rng.integers(0, 4096, size=(40000, 4)).astype(np.int32), 4096
    raise KeyError(name)


@pytest.mark.parametrize("name", ["one_expert_k1", "empty_experts", "duplicates", "ragged", "e_max",
                                  "many_chunks", "e4096", "e65535", "e3000_hot", "cluster_max",
                                  "coop_min", "coop_e64", "coop_e1024", "e4096_large"])
def test_permute_edge_cases(cuda_device, name):
    """Metadata and rows bit-exact against the oracle: edge routings, E up to 65535 (the
    cluster kernel's expert windows), and tables on both sides of 2^17 slots (the cluster
    kernel without workspace, the cooperative kernel with one)."""
    ids_np, E = _routing_case(name)
    S, K = ids_np.shape
    H = 64
    xb = synth.normal_bf16_bits(11, synth.TAG_X, S * H).reshape(S, H)
    x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to(cuda_device)
    r = gpu_permute(x, torch.from_numpy(ids_np).to(cuda_device), E)
    check_permute_exact(r, ids_np, E, xb)


@pytest.mark.parametrize("wname", ["tiny", "medium", "large", "skew20", "skew20_last",
                                   "permute_combine_S65536_mv20"])
def test_permute_workloads(cuda_device, wname):
    w = synth.WORKLOADS[wname]
    ids_np, _ = synth.routing_for(w)
    x = synth.normal_bf16_into(torch.empty(w.S, w.H, dtype=torch.bfloat16, device=cuda_device),
                               w.seed, synth.TAG_X)
    with_rows = w.S * w.K * w.H * 2 < 8e9
    r = gpu_permute(x, torch.from_numpy(ids_np).to(cuda_device), w.E, with_rows=with_rows)
    M = w.S * w.K
    sample = None if M * w.H <= 64e6 else np.random.default_rng(0).choice(M, 4096, replace=False)
    xb = bits(x) if with_rows else None
    check_permute_exact(r, ids_np, w.E, xb, sample)


def test_permute_metadata_only_and_zero_tokens(cuda_device):
    ids_np, E = _routing_case("ragged")
    ids = torch.from_numpy(ids_np).to(cuda_device)
    x = torch.zeros(ids_np.shape[0], 64, dtype=torch.bfloat16, device=cuda_device)
    r = gpu_permute(x, ids, E, with_rows=False)
    check_permute_exact(r, ids_np, E)
    # S = 0: counts and offsets are zero, maxvio NaN (T_bar = 0)
    r0 = gpu_permute(x[:0], ids[:0], E, with_rows=False)
    assert r0["counts"].abs().sum().item() == 0 and r0["cu"].abs().sum().item() == 0
    assert np.isnan(r0["maxvio"].item())


@pytest.mark.parametrize("E,bad_id", [(4, 7), (3000, 3000), (3000, 70000)])
def test_bad_routing_is_flagged(cuda_device, E, bad_id):
    """Ids outside [0, E) set MOE_ERR_BAD_ROUTING, get row -1 and are not counted; with
    E = 3000 the valid ids fall in different expert windows of the cluster kernel."""
    ids_np = np.array([[0, 1], [2, bad_id], [3, -1], [1, E - 1]], dtype=np.int32)
    ids = torch.from_numpy(ids_np).to(cuda_device)
    x = torch.ones(4, 64, dtype=torch.bfloat16, device=cuda_device)
    r = gpu_permute(x, ids, E)
    assert int(r["status"].item()) & moe.MOE_ERR_BAD_ROUTING
    rmap = r["rmap"].cpu().numpy()
    assert rmap[3] == -1 and rmap[5] == -1
    good = ids_np.reshape(-1)[[0, 1, 2, 4, 6, 7]]
    assert r["counts"].tolist() == np.bincount(good, minlength=E).tolist()
    ok = np.sort(rmap[rmap >= 0])
    assert np.array_equal(ok, np.arange(6))  # the valid slots fill rows 0..5


def test_maxvio_entry_point(cuda_device):
    counts = torch.tensor([3584] + [161] * 383, dtype=torch.int32, device=cuda_device)
    mv = GUARD((1,), torch.float64, cuda_device)
    mc = GUARD((1,), torch.int32, cuda_device)
    moe.moe_maxvio(counts, 8192, 8, mv, mc)
    torch.cuda.synchronize()
    assert mc.item() == 3584
    assert mv.item() == O.maxvio(counts.cpu().numpy(), 8192, 8)[0] == 20.0
    # the largest E, hot expert last: 65535 experts, S*K = 65535 * 2 rows
    c = np.full(65535, 2, np.int32)
    c[0], c[-1] = 1, 3
    moe.moe_maxvio(torch.from_numpy(c).to(cuda_device), 65535, 2, mv, mc)
    torch.cuda.synchronize()
    assert mc.item() == 3 and mv.item() == O.maxvio(c, 65535, 2)[0] == 0.5


# ----------------------------------------------------------------------------- combine

IDENTITY_FULL = ["permute_combine_S1024_mv0", "permute_combine_S1024_mv1",
                 "permute_combine_S4096_mv1", "permute_combine_S4096_mv20",
                 "permute_combine_S16384_mv1"]
IDENTITY_SAMPLED = ["permute_combine_S65536_mv0", "permute_combine_S65536_mv1",
                    "permute_combine_S65536_mv20"]


@pytest.mark.parametrize("wname", IDENTITY_FULL + IDENTITY_SAMPLED)
def test_identity_expert_layer(cuda_device, wname):
    """The permute/combine workloads (identity experts, H = 7168, E = 384, K = 8) against the
    oracle's layer: metadata and maxvio exact; x_perm exact and out within the bar, in full
    up to S = 16384 (the oracle's combine taken 1024 tokens at a time) and on 2048 sampled
    tokens (with their K rows each) at S = 65536."""
    w = synth.WORKLOADS[wname]
    inp = layer_inputs(w, cuda_device)
    buf = run_layer(inp, w, cuda_device)
    ids_np = inp["topk_ids"].cpu().numpy()
    counts, cu, rmap, psrc = check_permute_exact(
        dict(counts=buf.counts, cu=buf.cu_seqlens, rmap=buf.row_id_map, psrc=buf.perm_src,
             maxvio=buf.maxvio, max_count=buf.max_count, status=buf.d_status, x_perm=None),
        ids_np, w.E)
    x_bits = bits(inp["x"])
    rw = inp["route_w"].cpu().numpy()
    S, K = w.S, w.K
    if wname in IDENTITY_FULL:
        x_perm_ref = O.permute_rows(x_bits, psrc, K)
        assert np.array_equal(bits(buf.x_perm), x_perm_ref)
        out_gpu = bits(buf.out)
        out_ref = np.zeros_like(out_gpu)
        for t0 in range(0, S, 1024):
            t1 = min(S, t0 + 1024)
            ys = x_perm_ref[rmap[t0 * K:t1 * K]]  # y = x_perm: the token's K rows, slot order
            out_ref[t0:t1] = O.unpermute_combine(ys, np.arange((t1 - t0) * K), rw[t0:t1],
                                                 t1 - t0, K)
        print(f"[{wname}] out: {assert_close_bf16(out_gpu, out_ref, 'out')}")
    else:
        rng = np.random.default_rng(7)
        toks = np.sort(rng.choice(S, 2048, replace=False))
        rows = rmap.reshape(S, K)[toks].reshape(-1)
        xp = bits(buf.x_perm[torch.as_tensor(rows, device=cuda_device)])
        assert np.array_equal(xp, x_bits[psrc[rows] // K])
        out_ref = np.stack([O.combine_token(x_bits[psrc[rmap[t * K:(t + 1) * K]] // K], rw[t])
                            for t in toks])
        out_gpu = bits(buf.out[torch.as_tensor(toks, device=cuda_device)])
        print(f"[{wname}] out (sampled): {assert_close_bf16(out_gpu, out_ref, 'out (sampled)')}")


@pytest.mark.parametrize("K", [33, 40])
def test_combine_and_its_backward_beyond_32_slots(cuda_device, K):
    """K > 32 route slots per token (the combine then reads its slots' rows and weights from
    memory instead of one lane each): permute, identity experts and combine against the
    oracle, and the combine / permutation backward on the same plan."""
    dev = cuda_device
    S, H, E = 300, 64, 64
    rng = np.random.default_rng(K)
    ids_np = rng.integers(0, E, size=(S, K)).astype(np.int32)  # duplicates included
    x_bits = O.f64_to_bf16_bits(rng.standard_normal((S, H)))
    rw_np = rng.random((S, K)).astype(np.float32)
    x = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).to(dev)
    ids, rw = torch.from_numpy(ids_np).to(dev), torch.from_numpy(rw_np).to(dev)
    buf = moe.LayerBuffers.allocate(S, H, 0, E, K, dev, with_ffn=False,
                                    alloc=GUARD.for_device(dev))
    moe.moe_layer_forward(x, ids, rw, None, None, None, buf)
    torch.cuda.synchronize()
    assert int(buf.d_status.item()) == 0
    counts, cu, rmap, psrc = O.permute_metadata(ids_np, E)
    assert np.array_equal(buf.row_id_map.cpu().numpy(), rmap)
    x_perm = O.permute_rows(x_bits, psrc, K)
    assert np.array_equal(bits(buf.x_perm), x_perm)
    out_ref = O.unpermute_combine(x_perm, rmap, rw_np, S, K)
    print(f"K={K} out: {assert_close_bf16(bits(buf.out), out_ref, 'out')}")
    # backward of the combine (y = x_perm) and of the permutation
    g_bits = O.f64_to_bf16_bits(rng.standard_normal((S, H)))
    g = torch.from_numpy(g_bits.view(np.int16)).view(torch.bfloat16).to(dev)
    grad_y = GUARD((S * K, H), torch.bfloat16, dev)
    grad_w = GUARD((S, K), torch.float32, dev)
    moe.moe_combine_backward(g, buf.x_perm, buf.row_id_map, rw, grad_y, grad_w)
    grad_x = GUARD((S, H), torch.bfloat16, dev)
    moe.moe_permute_backward(grad_y, buf.row_id_map, grad_x, K)
    torch.cuda.synchronize()
    gy_ref, gw_ref = O.combine_backward(g_bits, x_perm, rmap, rw_np, S, K)
    assert np.array_equal(bits(grad_y), gy_ref)
    gw = grad_w.cpu().numpy().astype(np.float64)
    assert np.abs(gw - gw_ref).max() <= 1e-4 * np.abs(gw_ref).max()
    gx_ref = O.permute_backward(gy_ref, rmap, S, K)
    print(f"K={K} grad_x: {assert_close_bf16(bits(grad_x), gx_ref, 'grad_x')}")


def test_combine_unit_weight_invariants(cuda_device):
    S, K, E, H = 2000, 4, 16, 256
    rng = np.random.default_rng(7)
    ids = torch.from_numpy(np.stack([rng.permutation(E)[:K] for _ in range(S)]).astype(np.int32))
    ids = ids.to(cuda_device)
    x = synth.normal_bf16_into(torch.empty(S, H, dtype=torch.bfloat16, device=cuda_device), 3,
                               synth.TAG_X)
    buf = moe.LayerBuffers.allocate(S, H, 0, E, K, cuda_device, with_ffn=False,
                                    alloc=GUARD.for_device(cuda_device))
    ones = torch.ones(S, K, dtype=torch.float32, device=cuda_device)
    moe.moe_layer_forward(x, ids, ones, None, None, None, buf)
    torch.cuda.synchronize()
    # unpermute o permute with identity experts and unit weights: exactly bf16(K * x)
    assert torch.equal(buf.out, (x.float() * K).to(torch.bfloat16))
    # K = 1, weight 1: exactly x
    buf1 = moe.LayerBuffers.allocate(S, H, 0, E, 1, cuda_device, with_ffn=False,
                                     alloc=GUARD.for_device(cuda_device))
    moe.moe_layer_forward(x, ids[:, :1].contiguous(), ones[:, :1].contiguous(), None, None, None, buf1)
    torch.cuda.synchronize()
    assert torch.equal(buf1.out, x)


# ----------------------------------------------------------------------------- grouped FFN

def _check_full_layer(inp, w, buf):
    ref = O.moe_layer(bits(inp["x"]), inp["topk_ids"].cpu().numpy(), inp["route_w"].cpu().numpy(),
                      w.E, weights_getter(inp), w.Hp)
    assert np.array_equal(buf.counts.cpu().numpy(), ref["counts"])
    assert np.array_equal(buf.cu_seqlens.cpu().numpy(), ref["cu_seqlens"])
    assert np.array_equal(buf.row_id_map.cpu().numpy(), ref["row_id_map"])
    assert np.array_equal(bits(buf.x_perm), ref["x_perm"])
    assert buf.maxvio.item() == ref["maxvio"]
    # end to end: the GPU chain against the oracle chain
    for name in ("h", "y"):
        stats = assert_close_bf16(bits(getattr(buf, name)), ref[name], name)
        print(f"[{w.name}] {name}: {stats}")
    rw = inp["route_w"].cpu().numpy().astype(np.float64)
    rmap = ref["row_id_map"].reshape(w.S, w.K)
    inherited = sum(np.abs(rw[:, k:k + 1]) * bf16_ulp(ref["y"][rmap[:, k]]) for k in range(w.K))
    stats = assert_close_bf16(bits(buf.out), ref["out"], "out", inherited=inherited)
    print(f"[{w.name}] out (end to end): {stats}")
    # stage by stage: each kernel against the oracle applied to the GPU's own inputs
    get = weights_getter(inp)
    h_gpu = bits(buf.h)
    y_stage = np.zeros_like(ref["y"])
    for e in range(w.E):
        a, b = int(ref["cu_seqlens"][e]), int(ref["cu_seqlens"][e + 1])
        if b > a:
            y_stage[a:b] = O.expert_down_rows(h_gpu[a:b], get(e)[2])
    print(f"[{w.name}] y (stage): {assert_close_bf16(bits(buf.y), y_stage, 'y stage')}")
    out_stage = O.unpermute_combine(bits(buf.y), ref["row_id_map"], inp["route_w"].cpu().numpy(),
                                    w.S, w.K)
    print(f"[{w.name}] out (stage): {assert_close_bf16(bits(buf.out), out_stage, 'out stage')}")


def test_layer_tiny_full(cuda_device):
    w = synth.WORKLOADS["tiny"]
    inp = layer_inputs(w, cuda_device)
    _check_full_layer(inp, w, run_layer(inp, w, cuda_device))


@pytest.mark.parametrize("H,Hp", [(256, 384), (384, 256)])
def test_layer_ragged_chunks_full(cuda_device, H, Hp):
    """Experts of 0, 1, 15, 16, 17, 255, 256, 257, 600 and 1100 rows: every chunking
    path of the tile scheduler (one chunk, balanced chunks, tails of 1 row); H = 384 leaves
    the down projection's last 256-feature pair half empty."""
    sizes = [0, 1, 15, 16, 17, 255, 256, 257, 600, 1100]
    E, K = len(sizes), 1
    ids_np = np.concatenate([np.full(n, e, np.int32) for e, n in enumerate(sizes)])
    ids_np = np.random.default_rng(9).permutation(ids_np).reshape(-1, 1)
    S = ids_np.shape[0]
    w = synth.Workload("ragged", S, H, Hp, E, K, 21)
    inp = {"topk_ids": torch.from_numpy(ids_np).to(cuda_device),
           "route_w": torch.ones(S, 1, dtype=torch.float32, device=cuda_device)}
    inp["x"] = synth.normal_bf16_into(torch.empty(S, H, dtype=torch.bfloat16, device=cuda_device),
                                      21, synth.TAG_X)
    for name, tag, shape in (("w_gate", synth.TAG_W_GATE, (E, H, Hp)),
                             ("w_up", synth.TAG_W_UP, (E, H, Hp)),
                             ("w_down", synth.TAG_W_DOWN, (E, Hp, H))):
        inp[name] = synth.normal_bf16_into(torch.empty(*shape, dtype=torch.bfloat16,
                                                       device=cuda_device), 21, tag,
                                           synth.weight_scale(w, name[2:]))
    _check_full_layer(inp, w, run_layer(inp, w, cuda_device))


@pytest.mark.parametrize("E", [1000, 1024])
def test_layer_many_experts_full(cuda_device, E):
    """The grouped FFN's largest expert count (its per-expert row and unit tables fill the
    shared memory they are sized for): 1000 or 1024 experts, most with 0-3 rows, a few
    larger, one hot expert in the last window of the table; whole layer against the oracle."""
    H, Hp, K = 128, 256, 4
    rng = np.random.default_rng(E)
    S = 700
    ids_np = np.stack([rng.choice(E, size=K, replace=False) for _ in range(S)]).astype(np.int32)
    ids_np[:150, 0] = E - 1  # a hot expert, last in the table
    w = synth.Workload("many_experts", S, H, Hp, E, K, 23)
    inp = {"topk_ids": torch.from_numpy(ids_np).to(cuda_device),
           "route_w": torch.from_numpy(rng.random((S, K)).astype(np.float32)).to(cuda_device)}
    inp["x"] = synth.normal_bf16_into(torch.empty(S, H, dtype=torch.bfloat16, device=cuda_device),
                                      23, synth.TAG_X)
    for name, tag, shape in (("w_gate", synth.TAG_W_GATE, (E, H, Hp)),
                             ("w_up", synth.TAG_W_UP, (E, H, Hp)),
                             ("w_down", synth.TAG_W_DOWN, (E, Hp, H))):
        inp[name] = synth.normal_bf16_into(torch.empty(*shape, dtype=torch.bfloat16,
                                                       device=cuda_device), 23, tag,
                                           synth.weight_scale(w, name[2:]))
    _check_full_layer(inp, w, run_layer(inp, w, cuda_device))


def test_layer_medium_full(cuda_device):
    w = synth.WORKLOADS["medium"]
    inp = layer_inputs(w, cuda_device)
    _check_full_layer(inp, w, run_layer(inp, w, cuda_device))


def _sampled_rows(cu, hot, rng, per=6):
    E = len(cu) - 1
    experts = sorted({0, E - 1, hot, *rng.choice(E, 5, replace=False).tolist()})
    rows = []
    for e in experts:
        a, b = int(cu[e]), int(cu[e + 1])
        if b > a:
            rows += sorted({a, b - 1, (a + b) // 2, *rng.integers(a, b, per).tolist()})
    return np.array(rows, dtype=np.int64)


@pytest.mark.parametrize("wname", ["large", "skew1", "skew10", "skew20", "skew20_last"])
def test_layer_full_size_sampled(cuda_device, wname):
    """Full-size layers (S = 8192, H = 7168, H' = 2048, E = 384, K = 8) on sampled rows, at
    maxvio 0.2 (large), 1, 10 and 20; skew20_last puts the hot expert (maxvio 20) last, so its
    units come at the end of the persistent schedule."""
    w = synth.WORKLOADS[wname]
    inp = layer_inputs(w, cuda_device)
    buf = run_layer(inp, w, cuda_device)
    ids_np = inp["topk_ids"].cpu().numpy()
    counts, cu, rmap, psrc = check_permute_exact(
        dict(counts=buf.counts, cu=buf.cu_seqlens, rmap=buf.row_id_map, psrc=buf.perm_src,
             maxvio=buf.maxvio, max_count=buf.max_count, status=buf.d_status, x_perm=None),
        ids_np, w.E)
    rng = np.random.default_rng(1)
    rows = _sampled_rows(cu, int(np.argmax(counts)), rng)
    x_bits = bits(inp["x"])
    get = weights_getter(inp)
    experts = O.expert_of_rows(cu, rows)
    h_ref = np.zeros((len(rows), w.Hp), np.uint16)
    y_ref = np.zeros((len(rows), w.H), np.uint16)
    for e in np.unique(experts):
        sel = np.nonzero(experts == e)[0]
        src = x_bits[psrc[rows[sel]] // w.K]
        h_ref[sel], y_ref[sel] = O.expert_ffn_rows(src, *get(int(e)))
    idx = torch.as_tensor(rows, device=cuda_device)
    assert np.array_equal(bits(buf.x_perm[idx]), x_bits[psrc[rows] // w.K])
    print(f"[{w.name}] h: {assert_close_bf16(bits(buf.h[idx]), h_ref, 'h (sampled rows)')}")
    print(f"[{w.name}] y: {assert_close_bf16(bits(buf.y[idx]), y_ref, 'y (sampled rows)')}")
    # whole-layer output for a few tokens, each through its K experts
    toks = rng.choice(w.S, 3, replace=False)
    rw = inp["route_w"].cpu().numpy()
    out_ref = np.zeros((len(toks), w.H), np.uint16)
    out_stage = np.zeros((len(toks), w.H), np.uint16)
    inherited = np.zeros((len(toks), w.H))
    for i, t in enumerate(toks):
        ys = np.zeros((w.K, w.H), np.uint16)
        for k in range(w.K):
            _, ys[k] = O.expert_ffn_rows(x_bits[t:t + 1], *get(int(ids_np[t, k])))
            inherited[i] += abs(float(rw[t, k])) * bf16_ulp(ys[k])
        out_ref[i] = O.combine_token(ys, rw[t])
        y_gpu = bits(buf.y[torch.as_tensor(rmap[t * w.K:(t + 1) * w.K], device=cuda_device)])
        out_stage[i] = O.combine_token(y_gpu, rw[t])
    out_gpu = bits(buf.out[torch.as_tensor(toks, device=cuda_device)])
    print(f"[{w.name}] out: {assert_close_bf16(out_gpu, out_ref, 'out (sampled)', inherited)}")
    print(f"[{w.name}] out (stage): {assert_close_bf16(out_gpu, out_stage, 'out stage (sampled)')}")


def test_empty_batch_layer(cuda_device):
    """S = 0 tokens ("Distributed expert parallelism", "Empty experts": every expert empty):
    the forward (copy and zero-copy), the training backward and the MXFP8 forward are legal
    no-ops on the data -- zero counts and offsets, d_status 0, nothing written outside the
    buffers."""
    dev = cuda_device
    S, H, Hp, E, K = 0, 256, 512, 8, 2
    gen = torch.Generator().manual_seed(5)
    # zero-row views inside guarded allocations (non-null pointers, as a caller's would be)
    x = GUARD((S, H), torch.bfloat16, dev)
    ids = GUARD((S, K), torch.int32, dev)
    rw = GUARD((S, K), torch.float32, dev)
    wg = (torch.randn(E, H, Hp, generator=gen) / 16).to(torch.bfloat16).to(dev)
    wu = (torch.randn(E, H, Hp, generator=gen) / 16).to(torch.bfloat16).to(dev)
    wd = (torch.randn(E, Hp, H, generator=gen) / 16).to(torch.bfloat16).to(dev)
    for zero_copy in (False, True):
        buf = moe.LayerBuffers.allocate(S, H, Hp, E, K, dev, train=True,
                                        alloc=GUARD.for_device(dev))
        moe.moe_layer_forward(x, ids, rw, wg, wu, wd, buf, zero_copy=zero_copy)
        grads = moe.LayerGrads.allocate(S, H, Hp, E, K, dev, alloc=GUARD.for_device(dev))
        moe.moe_layer_backward(GUARD((S, H), torch.bfloat16, dev), rw, wg, wu, wd, buf, grads)
        torch.cuda.synchronize()
        assert int(buf.d_status.item()) == 0
        assert buf.counts.cpu().tolist() == [0] * E
        assert buf.cu_seqlens.cpu().tolist() == [0] * (E + 1)
        assert int(buf.max_count.item()) == 0 and np.isnan(buf.maxvio.item())
        assert buf.out.shape == (0, H) and grads.grad_x.shape == (0, H)
        # no rows: every expert's weight gradient is written as zero
        for g in (grads.grad_w_gate, grads.grad_w_up, grads.grad_w_down):
            assert torch.count_nonzero(g).item() == 0
    mw = moe.MxWeights.from_bf16(wg, wu, wd)
    buf = moe.LayerBuffers.allocate(S, H, Hp, E, K, dev, alloc=GUARD.for_device(dev))
    mxb = moe.MxBuffers.allocate(S, H, Hp, K, dev, alloc=GUARD.for_device(dev))
    moe.moe_layer_forward_mxfp8(x, ids, rw, mw, buf, mxb)
    torch.cuda.synchronize()
    assert int(buf.d_status.item()) == 0 and buf.counts.cpu().tolist() == [0] * E


def test_layer_is_deterministic(cuda_device):
    w = synth.WORKLOADS["medium"]
    inp = layer_inputs(w, cuda_device)
    a = run_layer(inp, w, cuda_device)
    b = run_layer(inp, w, cuda_device)
    for name in ("x_perm", "h", "y", "out"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name


def test_generator_twin_matches_host(cuda_device):
    """The device twin of the input generator draws the same bf16 values as the host one."""
    n = 1 << 20
    for off in (0, 5_000_000_000):
        t = synth.normal_bf16_into(torch.empty(n, dtype=torch.bfloat16, device=cuda_device), 2,
                                   synth.TAG_W_GATE, 0.125, offset=off)
        host = synth.normal_bf16_bits(2, synth.TAG_W_GATE, n, 0.125, offset=off)
        assert (bits(t) != host).sum() <= 2


def test_device_wait_timeout_reports_status_and_keeps_context(cuda_device, tmp_path):
    """Failure detection without a fault: with a 1 ns wait budget every pipeline wait of the
    grouped FFN runs out; the kernels record MOE_ERR_DEVICE_TIMEOUT in d_status, drain their
    own copies and MMAs, free TMEM and return, and the CUDA context stays usable."""
    import subprocess
    import sys

    script = (
        "import torch, synth, grouped_ffn_moe_b200 as moe\n"
        "w = synth.WORKLOADS['tiny']\n"
        "inp = synth.make_layer_inputs(w, device='cuda:0')\n"
        "buf = moe.LayerBuffers.allocate(w.S, w.H, w.Hp, w.E, w.K, torch.device('cuda:0'))\n"
        "moe.moe_layer_forward(inp['x'], inp['topk_ids'], inp['route_w'], inp['w_gate'],"
        " inp['w_up'], inp['w_down'], buf)\n"
        "torch.cuda.synchronize()\n"
        "st = int(buf.d_status.item())\n"
        "assert st & moe.MOE_ERR_DEVICE_TIMEOUT, st\n"
        "z = torch.arange(1000, device='cuda:0').sum().item()\n"
        "assert z == 499500\n"
        "print('timeout status', st)\n")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, PYTHONPATH=root, MOE_WAIT_BUDGET_NS="1")
    r = subprocess.run([sys.executable, "-c", script], env=env, cwd=root, timeout=600,
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "timeout status" in r.stdout
    # this process (normal budget) still runs the layer correctly
    w = synth.WORKLOADS["tiny"]
    inp = layer_inputs(w, cuda_device)
    buf = run_layer(inp, w, cuda_device)
    assert int(buf.d_status.item()) == 0


# ----------------------------------------------------------------------------- backward

@pytest.mark.parametrize("wname,sample", [("medium", None), ("permute_combine_S65536_mv20", 4096)])
def test_combine_and_permute_backward(cuda_device, wname, sample):
    """moe_combine_backward (grad_y, grad_w) and moe_permute_backward (grad_x) against the
    oracle, on the forward's own routing and expert outputs. grad_y is one rounding of the
    exact product w * g on both sides and must match bit for bit."""
    w = synth.WORKLOADS[wname]
    inp = layer_inputs(w, cuda_device)
    buf = run_layer(inp, w, cuda_device)
    y = buf.y if buf.y is not None else buf.x_perm
    M = w.S * w.K
    g = synth.normal_bf16_into(torch.empty(w.S, w.H, dtype=torch.bfloat16, device=cuda_device),
                               w.seed, synth.TAG_GRAD)
    gxp = synth.normal_bf16_into(torch.empty(M, w.H, dtype=torch.bfloat16, device=cuda_device),
                                 w.seed + 100, synth.TAG_GRAD)
    grad_y = GUARD((M, w.H), torch.bfloat16, cuda_device)
    grad_w = GUARD((w.S, w.K), torch.float32, cuda_device)
    grad_x = GUARD((w.S, w.H), torch.bfloat16, cuda_device)
    moe.moe_combine_backward(g, y, buf.row_id_map, inp["route_w"], grad_y, grad_w)
    moe.moe_permute_backward(gxp, buf.row_id_map, grad_x, w.K)
    torch.cuda.synchronize()
    rmap = buf.row_id_map.cpu().numpy()
    rw = inp["route_w"].cpu().numpy()
    g_bits = bits(g)
    if sample is None:
        ref_gy, ref_gw = O.combine_backward(g_bits, bits(y), rmap, rw, w.S, w.K)
        print(f"[{wname}] grad_y: {assert_close_bf16(bits(grad_y), ref_gy, 'grad_y')}")
        # one rounding of an exact product on both sides: bit-exact
        np.testing.assert_array_equal(bits(grad_y), ref_gy)
        ref_gx = O.permute_backward(bits(gxp), rmap, w.S, w.K)
        print(f"[{wname}] grad_x: {assert_close_bf16(bits(grad_x), ref_gx, 'grad_x')}")
    else:
        toks = np.random.default_rng(2).choice(w.S, sample // w.K, replace=False)
        slots = (toks[:, None] * w.K + np.arange(w.K)[None, :]).reshape(-1)
        rows = rmap[slots]
        ref_rows = O.f64_to_bf16_bits(rw.reshape(-1)[slots, None].astype(np.float64) *
                                      O.bf16_bits_to_f64(g_bits[slots // w.K]))
        got_rows = bits(grad_y[torch.as_tensor(rows, device=cuda_device)])
        print(f"[{wname}] grad_y (sampled): {assert_close_bf16(got_rows, ref_rows, 'grad_y')}")
        np.testing.assert_array_equal(got_rows, ref_rows)
        _, ref_gw = O.combine_backward(g_bits, bits(y), rmap, rw, w.S, w.K)
        gxp_bits = bits(gxp)
        ref_gx = np.stack([O.combine_token(gxp_bits[rmap[t * w.K:(t + 1) * w.K]],
                                           np.ones(w.K, np.float32)) for t in toks])
        got_gx = bits(grad_x[torch.as_tensor(toks, device=cuda_device)])
        print(f"[{wname}] grad_x (sampled): {assert_close_bf16(got_gx, ref_gx, 'grad_x')}")
    gw = grad_w.cpu().numpy().astype(np.float64)
    scale = np.abs(ref_gw).max()
    err = np.abs(gw - ref_gw).max()
    print(f"[{wname}] grad_w max |err| / max |ref| = {err / scale:.2e}")
    assert err <= 1e-4 * scale


def test_backward_unit_weight_and_adjoint_exactness(cuda_device):
    """With unit route weights, grad_y rows are exact copies of grad_out; the permutation's
    backward of K identical copies is exactly bf16(K * x) (every partial sum is exact)."""
    S, K, E, H = 1500, 4, 16, 256
    rng = np.random.default_rng(31)
    ids = torch.from_numpy(np.stack([rng.permutation(E)[:K] for _ in range(S)]).astype(np.int32))
    ids = ids.to(cuda_device)
    x = synth.normal_bf16_into(torch.empty(S, H, dtype=torch.bfloat16, device=cuda_device), 4,
                               synth.TAG_X)
    buf = moe.LayerBuffers.allocate(S, H, 0, E, K, cuda_device, with_ffn=False,
                                    alloc=GUARD.for_device(cuda_device))
    ones = torch.ones(S, K, dtype=torch.float32, device=cuda_device)
    moe.moe_layer_forward(x, ids, ones, None, None, None, buf)
    grad_y = GUARD((S * K, H), torch.bfloat16, cuda_device)
    moe.moe_combine_backward(x, None, buf.row_id_map, ones, grad_y)
    grad_x = GUARD((S, H), torch.bfloat16, cuda_device)
    moe.moe_permute_backward(buf.x_perm, buf.row_id_map, grad_x, K)
    torch.cuda.synchronize()
    assert torch.equal(grad_y, buf.x_perm)  # w = 1: the backward re-dispatch is the permutation
    assert torch.equal(grad_x, (x.float() * K).to(torch.bfloat16))


# ----------------------------------------------------------------------------- zero copy

def _gather_vs_copy(inp, w, dev):
    ref = moe.LayerBuffers.allocate(w.S, w.H, w.Hp, w.E, w.K, dev, alloc=GUARD.for_device(dev))
    moe.moe_layer_forward(inp["x"], inp["topk_ids"], inp["route_w"], inp["w_gate"], inp["w_up"],
                          inp["w_down"], ref)
    zc = moe.LayerBuffers.allocate(w.S, w.H, w.Hp, w.E, w.K, dev, alloc=GUARD.for_device(dev))
    zc.x_perm.fill_(float("nan"))  # the zero-copy path must not read x_perm
    moe.moe_layer_forward(inp["x"], inp["topk_ids"], inp["route_w"], inp["w_gate"], inp["w_up"],
                          inp["w_down"], zc, zero_copy=True)
    torch.cuda.synchronize()
    assert int(ref.d_status.item()) == 0 and int(zc.d_status.item()) == 0
    assert torch.isnan(zc.x_perm.float()).all()  # metadata-only permute: no row copy
    for name in ("counts", "cu_seqlens", "row_id_map", "perm_src", "h", "y", "out"):
        assert torch.equal(getattr(zc, name), getattr(ref, name)), name
    return ref, zc


@pytest.mark.parametrize("wname", ["tiny", "medium", "large", "skew20"])
def test_zero_copy_gather_equals_copy_path(cuda_device, wname):
    """The SwiGLU pass gathering its token rows from x through perm_src (16-byte cp.async
    copies by four gather warps) gives h, y and out bit-identical to the path through x_perm, which is itself checked
    against the oracle above; the tiny layer is also checked against the oracle directly."""
    w = synth.WORKLOADS[wname]
    inp = layer_inputs(w, cuda_device)
    ref, zc = _gather_vs_copy(inp, w, cuda_device)
    if wname == "tiny":
        zc.x_perm.copy_(ref.x_perm)  # the oracle check also compares the (unused) x_perm
        _check_full_layer(inp, w, zc)


@pytest.mark.parametrize("H,Hp", [(256, 384), (384, 256)])
def test_zero_copy_gather_ragged(cuda_device, H, Hp):
    """Experts of 0 .. 1100 rows (every chunk and 16-row rounding path), K = 2 with
    duplicate experts inside tokens, against the copy path."""
    sizes = [0, 1, 15, 16, 17, 255, 256, 257, 600, 1100]
    E, K = len(sizes), 2
    ids_np = np.concatenate([np.full(n, e, np.int32) for e, n in enumerate(sizes)])
    ids_np = np.random.default_rng(12).permutation(ids_np)
    if len(ids_np) % 2:
        ids_np = ids_np[:-1]
    ids_np = ids_np.reshape(-1, K)
    S = ids_np.shape[0]
    w = synth.Workload("ragged_k2", S, H, Hp, E, K, 23)
    inp = {"topk_ids": torch.from_numpy(ids_np).to(cuda_device),
           "route_w": torch.full((S, K), 0.5, dtype=torch.float32, device=cuda_device)}
    inp["x"] = synth.normal_bf16_into(torch.empty(S, H, dtype=torch.bfloat16, device=cuda_device),
                                      23, synth.TAG_X)
    for name, tag, shape in (("w_gate", synth.TAG_W_GATE, (E, H, Hp)),
                             ("w_up", synth.TAG_W_UP, (E, H, Hp)),
                             ("w_down", synth.TAG_W_DOWN, (E, Hp, H))):
        inp[name] = synth.normal_bf16_into(torch.empty(*shape, dtype=torch.bfloat16,
                                                       device=cuda_device), 23, tag,
                                           synth.weight_scale(w, name[2:]))
    _gather_vs_copy(inp, w, cuda_device)


def test_zero_copy_gather_training_preactivations(cuda_device):
    """The gather pass stores the same pre-activations as the training forward on x_perm."""
    w = synth.WORKLOADS["medium"]
    inp = layer_inputs(w, cuda_device)
    buf = moe.LayerBuffers.allocate(w.S, w.H, w.Hp, w.E, w.K, cuda_device, train=True,
                                    alloc=GUARD.for_device(cuda_device))
    moe.moe_layer_forward(inp["x"], inp["topk_ids"], inp["route_w"], inp["w_gate"], inp["w_up"],
                          inp["w_down"], buf)
    h2 = GUARD(buf.h.shape, buf.h.dtype, cuda_device)
    g2 = GUARD(buf.gate_pre.shape, buf.gate_pre.dtype, cuda_device)
    u2 = GUARD(buf.up_pre.shape, buf.up_pre.dtype, cuda_device)
    moe.moe_grouped_ffn_up_gate_gather(inp["x"], buf.perm_src, w.K, inp["w_gate"], inp["w_up"],
                                       buf.cu_seqlens, h2, g2, u2, buf.d_status)
    torch.cuda.synchronize()
    assert int(buf.d_status.item()) == 0
    assert torch.equal(h2, buf.h) and torch.equal(g2, buf.gate_pre) and torch.equal(u2, buf.up_pre)


# ----------------------------------------------------------------------------- shared experts

@pytest.mark.parametrize("wname,n_shared", [("tiny", 1), ("tiny", 2), ("medium", 1), ("medium", 2)])
def test_shared_expert_layer(cuda_device, wname, n_shared):
    """MoE(x) = SharedExpert(x) + sum_k w_k RoutedExpert_k(x) with the shared expert appended
    to the routing (moe_append_shared) and run in the same launches; a shared expert of width
    n_shared * H' is n_shared column slices. Routing table exact; routed rows stage-wise
    within the bar; out end to end against the oracle's single shared FFN, allowing the
    slices' own roundings; the routed maxvio from moe_maxvio on the routed counts."""
    w = synth.WORKLOADS[wname]
    dev = cuda_device
    inp = synth.make_layer_inputs(w, device=str(dev), n_shared=n_shared)
    S, K, E = w.S, w.K, w.E
    K2, E2 = K + n_shared, E + n_shared
    ids2 = GUARD((S, K2), torch.int32, dev)
    w2 = GUARD((S, K2), torch.float32, dev)
    moe.moe_append_shared(inp["topk_ids"], inp["route_w"], E, n_shared, ids2, w2)
    buf = moe.LayerBuffers.allocate(S, w.H, w.Hp, E2, K2, dev, alloc=GUARD.for_device(dev))
    moe.moe_layer_forward(inp["x"], ids2, w2, inp["w_gate"], inp["w_up"], inp["w_down"], buf)
    mv = GUARD((1,), torch.float64, dev)
    mc = GUARD((1,), torch.int32, dev)
    moe.moe_maxvio(buf.counts[:E], S, K, mv, mc)
    torch.cuda.synchronize()
    assert int(buf.d_status.item()) == 0
    ids_np, rw = inp["topk_ids"].cpu().numpy(), inp["route_w"].cpu().numpy()
    assert np.array_equal(ids2[:, :K].cpu().numpy(), ids_np)
    assert np.array_equal(ids2[:, K:].cpu().numpy(), np.tile(np.arange(E, E2), (S, 1)))
    assert np.array_equal(w2[:, :K].cpu().numpy(), rw) and bool((w2[:, K:] == 1).all())
    counts, _, _, _ = O.permute_metadata(ids_np, E)
    assert (mv.item(), int(mc.item())) == O.maxvio(counts, S, K)
    # oracle: routed experts as usual, the shared expert as one FFN over the concatenated
    # slices
    wg_b, wu_b, wd_b = bits(inp["w_gate"]), bits(inp["w_up"]), bits(inp["w_down"])
    get = lambda e: (wg_b[e], wu_b[e], wd_b[e])
    shared = (np.concatenate([wg_b[E + j] for j in range(n_shared)], axis=1),
              np.concatenate([wu_b[E + j] for j in range(n_shared)], axis=1),
              np.concatenate([wd_b[E + j] for j in range(n_shared)], axis=0))
    ref = O.moe_layer_with_shared(bits(inp["x"]), ids_np, rw, E, get, w.Hp, shared)
    y = bits(buf.y)
    M = S * K
    stats = assert_close_bf16(y[:M], ref["y"], "routed y")
    print(f"[{wname}+{n_shared}] routed y: {stats}")
    rmap = ref["row_id_map"].reshape(S, K)
    slices = [y[M + j * S: M + (j + 1) * S] for j in range(n_shared)]  # shared rows in token order
    inherited = sum(np.abs(rw[:, k:k + 1]) * bf16_ulp(ref["y"][rmap[:, k]]) for k in range(K))
    inherited = inherited + sum(bf16_ulp(sl) for sl in slices) + bf16_ulp(ref["y_shared"])
    stats = assert_close_bf16(bits(buf.out), ref["out"], "out", inherited=inherited)
    print(f"[{wname}+{n_shared}] out (end to end): {stats}")
