"""Parity of the backward of the grouped expert FFN (CUDA path through the C ABI) with the
fp64 CPU oracle.

Stage by stage, each kernel is checked against the oracle applied to the GPU's own inputs:
  training forward:  gate_pre, up_pre (bf16 bar); h identical to the inference forward
  down backward:     d_gate, d_up from grad_y and the saved pre-activations (bf16 bar)
  up/gate backward:  grad_x_perm from d_gate, d_up (bf16 bar)
  weight gradients:  fp32, within the fp32 summation bound of helpers.py
  permutation bwd:   grad_x from grad_x_perm (bf16 bar)
and once end to end (oracle forward + backward from the same inputs) with a looser bar that
catches wiring mistakes, not rounding.
"""
import numpy as np
import pytest
import torch

import grouped_ffn_moe_b200 as moe
import synth
from helpers import GUARD, assert_close_bf16, assert_close_fp32_sums, bits
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


def _weights_getter(inp):
    cache = {}

    def get(e):
        if e not in cache:
            cache.clear()
            cache[e] = (bits(inp["w_gate"][e]), bits(inp["w_up"][e]), bits(inp["w_down"][e]))
        return cache[e]
    return get


def _ragged_inputs(dev, H, Hp, sizes, seed=21):
    E, K = len(sizes), 1
    ids_np = np.concatenate([np.full(n, e, np.int32) for e, n in enumerate(sizes)])
    ids_np = np.random.default_rng(seed).permutation(ids_np).reshape(-1, 1)
    S = ids_np.shape[0]
    w = synth.Workload("ragged", S, H, Hp, E, K, seed)
    inp = {"topk_ids": torch.from_numpy(ids_np).to(dev),
           "route_w": torch.rand(S, 1, generator=torch.Generator().manual_seed(seed)).to(dev)}
    inp["x"] = synth.normal_bf16_into(torch.empty(S, H, dtype=torch.bfloat16, device=dev), seed,
                                      synth.TAG_X)
    for name, tag, shape in (("w_gate", synth.TAG_W_GATE, (E, H, Hp)),
                             ("w_up", synth.TAG_W_UP, (E, H, Hp)),
                             ("w_down", synth.TAG_W_DOWN, (E, Hp, H))):
        inp[name] = synth.normal_bf16_into(torch.empty(*shape, dtype=torch.bfloat16, device=dev),
                                           seed, tag, synth.weight_scale(w, name[2:]))
    return w, inp


def _run_train(inp, w, dev, accumulate=False, prior=None):
    buf = moe.LayerBuffers.allocate(w.S, w.H, w.Hp, w.E, w.K, dev, train=True,
                                    alloc=GUARD.for_device(dev))
    moe.moe_layer_forward(inp["x"], inp["topk_ids"], inp["route_w"], inp["w_gate"], inp["w_up"],
                          inp["w_down"], buf)
    grads = moe.LayerGrads.allocate(w.S, w.H, w.Hp, w.E, w.K, dev, alloc=GUARD.for_device(dev))
    if prior is not None:
        for t, p in zip((grads.grad_w_gate, grads.grad_w_up, grads.grad_w_down), prior):
            t.copy_(p)
    grad_out = synth.normal_bf16_into(torch.empty(w.S, w.H, dtype=torch.bfloat16, device=dev),
                                      w.seed, synth.TAG_GRAD)
    moe.moe_layer_backward(grad_out, inp["route_w"], inp["w_gate"], inp["w_up"], inp["w_down"],
                           buf, grads, accumulate=accumulate)
    torch.cuda.synchronize()
    assert int(buf.d_status.item()) == 0
    return buf, grads, grad_out


def _abs_bits(b):
    return np.asarray(b, np.uint16) & np.uint16(0x7FFF)


def _check_stages(inp, w, buf, grads, prior=None, experts=None):
    """Every stage against the oracle on the GPU's own inputs, expert by expert (device
    slices, so the full-size layer needs only one expert's rows on the host). experts:
    subset to check (default all). Returns grad_x_perm bits when all experts are checked."""
    cu = buf.cu_seqlens.cpu().numpy()
    get = _weights_getter(inp)
    sel = range(w.E) if experts is None else experts
    names = ("g", "u", "dg", "du", "gx")
    got = {k: [] for k in names}
    refs = {k: [] for k in names}
    worst = {}
    for e in sel:
        a, b = int(cu[e]), int(cu[e + 1])
        dW = [t[e].cpu().numpy() for t in (grads.grad_w_gate, grads.grad_w_up, grads.grad_w_down)]
        pri = [np.zeros_like(t) if prior is None else prior[i][e].cpu().numpy()
               for i, t in enumerate(dW)]
        if b == a:
            for i in range(3):
                np.testing.assert_array_equal(dW[i], pri[i])  # zero, or left unchanged
            continue
        wg, wu, wd = get(e)
        x, h = bits(buf.x_perm[a:b]), bits(buf.h[a:b])
        gpre, upre = bits(buf.gate_pre[a:b]), bits(buf.up_pre[a:b])
        gy, dg, du = bits(grads.grad_y[a:b]), bits(grads.d_gate[a:b]), bits(grads.d_up[a:b])
        got["g"].append(gpre)
        got["u"].append(upre)
        got["dg"].append(dg)
        got["du"].append(du)
        got["gx"].append(bits(grads.grad_x_perm[a:b]))
        g_ref, u_ref = O.expert_preact_rows(x, wg, wu)
        dg_ref, du_ref = O.expert_down_backward_rows(gy, gpre, upre, wd)
        refs["g"].append(g_ref)
        refs["u"].append(u_ref)
        refs["dg"].append(dg_ref)
        refs["du"].append(du_ref)
        refs["gx"].append(O.expert_up_gate_backward_rows(dg, du, wg, wu))
        ref_w = O.expert_weight_grads_rows(x, h, dg, du, gy)
        abs_w = O.expert_weight_grads_rows(_abs_bits(x), _abs_bits(h), _abs_bits(dg),
                                           _abs_bits(du), _abs_bits(gy))
        for i, name in enumerate(("dW_gate", "dW_up", "dW_down")):
            st = assert_close_fp32_sums(dW[i], pri[i].astype(np.float64) + ref_w[i], abs_w[i],
                                        b - a, f"{name}[{e}]", added=prior is not None)
            worst[name] = max(worst.get(name, 0.0), st["max_err_over_bound"])
    for k in names:
        print(f"[{w.name}] {k}: "
              f"{assert_close_bf16(np.concatenate(got[k]), np.concatenate(refs[k]), k)}")
    print(f"[{w.name}] weight gradients, max error / bound: {worst}")
    return bits(grads.grad_x_perm) if experts is None else None


def test_ffn_backward_tiny_full(cuda_device):
    w = synth.WORKLOADS["tiny"]
    inp = synth.make_layer_inputs(w, device=str(cuda_device))
    buf, grads, grad_out = _run_train(inp, w, cuda_device)
    gxp = _check_stages(inp, w, buf, grads)
    # the training forward computes the same h as the inference forward
    ref = moe.LayerBuffers.allocate(w.S, w.H, w.Hp, w.E, w.K, cuda_device,
                                    alloc=GUARD.for_device(cuda_device))
    moe.moe_layer_forward(inp["x"], inp["topk_ids"], inp["route_w"], inp["w_gate"], inp["w_up"],
                          inp["w_down"], ref)
    torch.cuda.synchronize()
    assert torch.equal(ref.h, buf.h) and torch.equal(ref.out, buf.out)
    # permutation backward on the GPU's own grad_x_perm
    rmap = buf.row_id_map.cpu().numpy()
    gx_ref = O.permute_backward(gxp, rmap, w.S, w.K)
    print(f"[tiny] grad_x: {assert_close_bf16(bits(grads.grad_x), gx_ref, 'grad_x')}")


@pytest.mark.parametrize("H,Hp", [(256, 384), (384, 256)])
def test_ffn_backward_ragged_full(cuda_device, H, Hp):
    """Experts of 0, 1, 15, 16, 17, 63, 64, 65, 255, 256, 257, 600 rows: token tails of
    every length class in the weight gradient (cut at 16, a whole 64-block, one row), empty
    experts, and (Hp or H = 384) gradient column blocks of 128."""
    sizes = [0, 1, 15, 16, 17, 63, 64, 65, 255, 256, 257, 600]
    w, inp = _ragged_inputs(cuda_device, H, Hp, sizes)
    buf, grads, _ = _run_train(inp, w, cuda_device)
    _check_stages(inp, w, buf, grads)


def test_ffn_backward_many_experts_full(cuda_device):
    """1024 experts (the grouped FFN's largest count), most with 0-2 rows and a larger last
    one: every backward pass decodes units over full per-expert tables, and the weight
    gradients of the ~340 empty experts are written as zeros."""
    sizes = [i % 3 for i in range(1023)] + [40]
    w, inp = _ragged_inputs(cuda_device, 128, 128, sizes, seed=31)
    buf, grads, _ = _run_train(inp, w, cuda_device)
    _check_stages(inp, w, buf, grads)
    empty = [e for e, n in enumerate(sizes) if n == 0]
    for g in (grads.grad_w_gate, grads.grad_w_up, grads.grad_w_down):
        assert torch.count_nonzero(g[empty]).item() == 0


def test_ffn_backward_medium_full_accumulate(cuda_device):
    """Medium layer; the weight gradients are added into random prior fp32 buffers."""
    w = synth.WORKLOADS["medium"]
    inp = synth.make_layer_inputs(w, device=str(cuda_device))
    g = torch.Generator(device=cuda_device).manual_seed(5)
    prior = [torch.randn(w.E, w.H, w.Hp, device=cuda_device, generator=g),
             torch.randn(w.E, w.H, w.Hp, device=cuda_device, generator=g),
             torch.randn(w.E, w.Hp, w.H, device=cuda_device, generator=g)]
    buf, grads, _ = _run_train(inp, w, cuda_device, accumulate=True, prior=prior)
    _check_stages(inp, w, buf, grads, prior=prior)


def test_ffn_backward_large_sampled_experts(cuda_device):
    """Full-size layer (S=8192, H=7168, H'=2048, E=384, K=8); every stage checked in full on
    four experts (the first, the last, the largest and the smallest non-empty one)."""
    w = synth.WORKLOADS["large"]
    inp = synth.make_layer_inputs(w, device=str(cuda_device))
    buf, grads, _ = _run_train(inp, w, cuda_device)
    counts = buf.counts.cpu().numpy()
    nz = np.nonzero(counts)[0]
    experts = sorted({int(nz[0]), int(nz[-1]), int(np.argmax(counts)),
                      int(nz[np.argmin(counts[nz])])})
    _check_stages(inp, w, buf, grads, experts=experts)


def test_layer_backward_end_to_end_tiny(cuda_device):
    """The whole GPU chain against the whole oracle chain from the same inputs. One-step
    flips of intermediate bf16 tensors propagate, so the bar here is relative (1e-2): it
    catches a wrong operand, sign or transposition, not rounding."""
    w = synth.WORKLOADS["tiny"]
    inp = synth.make_layer_inputs(w, device=str(cuda_device))
    buf, grads, grad_out = _run_train(inp, w, cuda_device)
    get = _weights_getter(inp)
    ref = O.moe_layer(bits(inp["x"]), inp["topk_ids"].cpu().numpy(), inp["route_w"].cpu().numpy(),
                      w.E, get, w.Hp)
    rw = inp["route_w"].cpu().numpy()
    gy, gw = O.combine_backward(bits(grad_out), ref["y"], ref["row_id_map"], rw, w.S, w.K)
    g, u = O.grouped_ffn_preact(ref["x_perm"], ref["cu_seqlens"], get, w.Hp)
    fb = O.grouped_ffn_backward(ref["x_perm"], g, u, ref["h"], gy, ref["cu_seqlens"], get)
    gx = O.permute_backward(fb["grad_x_perm"], ref["row_id_map"], w.S, w.K)

    def rel(a, b):
        return float(np.linalg.norm(a - b) / np.linalg.norm(b))
    f = O.bf16_bits_to_f64
    checks = {"grad_x": rel(f(bits(grads.grad_x)), f(gx)),
              "grad_route_w": rel(grads.grad_route_w.cpu().numpy().astype(np.float64), gw),
              "dW_gate": rel(grads.grad_w_gate.cpu().numpy().astype(np.float64), fb["dWg"]),
              "dW_up": rel(grads.grad_w_up.cpu().numpy().astype(np.float64), fb["dWu"]),
              "dW_down": rel(grads.grad_w_down.cpu().numpy().astype(np.float64), fb["dWd"])}
    print(f"[tiny] end-to-end relative errors: {checks}")
    for k, v in checks.items():
        assert v <= 1e-2, (k, v)


def test_backward_wait_timeout_reports_status_and_keeps_context(cuda_device):
    """Failure detection of the backward GEMMs without a fault: with a 1 ns wait budget every
    pipeline wait of the dgrad and weight-gradient kernels runs out; they record
    MOE_ERR_DEVICE_TIMEOUT in d_status, drain their own copies and MMAs, free TMEM and
    return, and the CUDA context stays usable. (The forward, run first in the same child,
    times out as well; its status is cleared before the backward.)"""
    import os
    import subprocess
    import sys

    script = (
        "import torch, synth, grouped_ffn_moe_b200 as moe\n"
        "dev = torch.device('cuda:0')\n"
        "w = synth.WORKLOADS['tiny']\n"
        "inp = synth.make_layer_inputs(w, device='cuda:0')\n"
        "buf = moe.LayerBuffers.allocate(w.S, w.H, w.Hp, w.E, w.K, dev, train=True)\n"
        "moe.moe_layer_forward(inp['x'], inp['topk_ids'], inp['route_w'], inp['w_gate'],"
        " inp['w_up'], inp['w_down'], buf)\n"
        "torch.cuda.synchronize()\n"
        "buf.d_status.zero_()\n"
        "grads = moe.LayerGrads.allocate(w.S, w.H, w.Hp, w.E, w.K, dev)\n"
        "g = torch.ones(w.S, w.H, dtype=torch.bfloat16, device=dev)\n"
        "moe.moe_layer_backward(g, inp['route_w'], inp['w_gate'], inp['w_up'], inp['w_down'],"
        " buf, grads)\n"
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
    # this process (normal budget) still runs the training step correctly
    w, inp = _ragged_inputs(cuda_device, 256, 384, [3, 0, 17])
    buf, grads, _ = _run_train(inp, w, cuda_device)
    assert int(buf.d_status.item()) == 0
