"""CPU-side checks of the C ABI: the library loads, exports every declared symbol, and
rejects bad arguments on the host before touching the GPU."""
import ctypes
import os
import re

import pytest
import torch

import grouped_ffn_moe_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_four_calls():
    names = declared_functions()
    for n in ("moe_permute", "moe_grouped_ffn", "moe_unpermute_combine", "moe_maxvio",
              "moe_permute_workspace_bytes", "moe_status_string", "moe_abi_version"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = moe.lib()
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} not exported by {moe.LIB_PATH}"
        assert getattr(lib, n) is not None


def test_binding_names_match_abi():
    for n in ("moe_permute", "moe_grouped_ffn", "moe_unpermute_combine", "moe_maxvio",
              "moe_permute_workspace_bytes", "moe_status_string"):
        assert callable(getattr(moe, n))


def test_status_strings_and_version():
    assert moe.moe_status_string(0) == "ok"
    assert "argument" in moe.moe_status_string(moe.MOE_ERR_INVALID_ARGUMENT)
    assert "timed out" in moe.moe_status_string(moe.MOE_ERR_DEVICE_TIMEOUT)
    assert moe.lib().moe_abi_version() >> 16 == 1


def test_workspace_bytes():
    assert moe.moe_permute_workspace_bytes(0, 8, 384) == 0
    # up to 2^17 routed slots, or more than 1024 experts: one cluster, no workspace
    assert moe.moe_permute_workspace_bytes(16384, 8, 384) == 0
    assert moe.moe_permute_workspace_bytes(1 << 14, 8, 1024) == 0
    assert moe.moe_permute_workspace_bytes(1 << 18, 8, 4096) == 0
    # above: 65536 tokens x 8 slots = 1024 chunks of 512, times 384 experts, int32
    assert moe.moe_permute_workspace_bytes(65536, 8, 384) == 1024 * 384 * 4
    assert moe.moe_permute_workspace_bytes((1 << 14) + 1, 8, 100) % 256 == 0


P = ctypes.c_void_p


def fake(addr):
    return P(addr)


def test_host_validation_rejects_without_launch():
    L = moe.lib()
    a = fake(0x10000)  # never dereferenced: validation fails first
    null = P(0)
    # K > E
    assert L.moe_permute(a, a, 4, 64, 9, 8, a, a, a, a, null, null, null, a, 1 << 20, null, null) == 1
    # E beyond the supported maximum (65535)
    assert L.moe_permute(a, a, 4, 64, 2, 70000, a, a, a, a, null, null, null, a, 1 << 20, null,
                         null) == 2
    # missing outputs
    assert L.moe_permute(a, a, 4, 64, 2, 8, a, null, a, a, null, null, null, a, 1 << 20, null,
                         null) == 1
    # H not a multiple of 8 with a row copy
    assert L.moe_permute(a, a, 4, 60, 2, 8, a, a, a, a, null, null, null, a, 1 << 20, null, null) == 2
    # misaligned x_perm
    assert L.moe_permute(a, a, 4, 64, 2, 8, fake(0x10008), a, a, a, null, null, null, a, 1 << 20,
                         null, null) == 1
    # workspace too small (2^21 slots need one)
    assert L.moe_permute(a, a, 1 << 18, 64, 8, 384, a, a, a, a, null, null, null, a, 16, null,
                         null) == 1
    # grouped FFN: more experts than its shared-memory tables hold
    assert L.moe_grouped_ffn(a, a, a, a, a, 16, 256, 256, 1025, a, a, null, null) == 2
    # grouped FFN: H' not a multiple of 128, then a null weight
    assert L.moe_grouped_ffn(a, a, a, a, a, 16, 256, 200, 4, a, a, null, null) == 2
    assert L.moe_grouped_ffn(a, null, a, a, a, 16, 256, 256, 4, a, a, null, null) == 1
    assert L.moe_grouped_ffn(a, a, a, a, a, 0, 256, 256, 4, a, a, null, null) == 0  # M = 0: no-op
    # M = 0 with NULL row buffers (a zero-size tensor's data pointer): still a no-op; shapes
    # are still checked
    assert L.moe_grouped_ffn(null, a, a, a, a, 0, 256, 256, 4, null, null, null, null) == 0
    assert L.moe_grouped_ffn_up_gate_train(null, a, a, a, 0, 256, 256, 4, null, null, null,
                                           null, null) == 0
    assert L.moe_grouped_ffn_down_backward(null, a, null, null, a, 0, 256, 256, 4, null, null,
                                           null, null) == 0
    assert L.moe_grouped_ffn_up_gate_backward(null, null, a, a, a, 0, 256, 256, 4, null, null,
                                              null) == 0
    assert L.moe_grouped_ffn_gather(null, null, 0, 2, a, a, a, a, 256, 256, 4, null, null, null,
                                    null) == 0
    assert L.moe_grouped_ffn(null, a, a, a, a, 0, 256, 200, 4, null, null, null, null) == 2
    # combine: H % 8, K < 1
    assert L.moe_unpermute_combine(a, a, a, 4, 12, 2, a, null) == 2
    assert L.moe_unpermute_combine(a, a, a, 4, 16, 0, a, null) == 1
    assert L.moe_unpermute_combine(a, a, a, 0, 16, 2, a, null) == 0  # S = 0: no-op
    # maxvio: S*K must be positive
    assert L.moe_maxvio(a, 8, 0, 2, a, null, null) == 1


def test_host_validation_of_backward_gather_and_shared_calls():
    """The entry points of the backward, the zero-copy forward and the shared experts reject
    bad arguments on the host, before any launch (no GPU needed)."""
    L = moe.lib()
    a = fake(0x10000)
    mis = fake(0x10008)  # 8-byte aligned only
    null = P(0)
    # combine / permutation backward: H % 8, grad_w without y, S = 0 no-op
    assert L.moe_combine_backward(a, a, a, a, 4, 12, 2, a, null, null) == 2
    assert L.moe_combine_backward(a, null, a, a, 4, 16, 2, a, a, null) == 1
    assert L.moe_combine_backward(a, a, a, a, 0, 16, 2, a, a, null) == 0
    assert L.moe_permute_backward(a, a, 4, 16, 0, a, null) == 1
    assert L.moe_permute_backward(mis, a, 4, 16, 2, a, null) == 1
    # training forward: both pre-activation outputs required, 16-byte aligned
    assert L.moe_grouped_ffn_up_gate_train(a, a, a, a, 16, 256, 256, 4, a, null, a, null,
                                           null) == 1
    assert L.moe_grouped_ffn_up_gate_train(a, a, a, a, 16, 256, 256, 4, a, a, mis, null,
                                           null) == 1
    # FFN backward passes: H' % 128, missing d_up, the accumulate flag, misaligned buffers
    assert L.moe_grouped_ffn_down_backward(a, a, a, a, a, 16, 256, 200, 4, a, a, null, null) == 2
    assert L.moe_grouped_ffn_down_backward(a, a, a, a, a, 16, 256, 256, 4, a, null, null,
                                           null) == 1
    assert L.moe_grouped_ffn_up_gate_backward(a, a, a, null, a, 16, 256, 256, 4, a, null,
                                              null) == 1
    assert L.moe_grouped_ffn_weight_grad(a, a, a, a, a, a, 16, 256, 256, 4, a, a, a, 2, null,
                                         null) == 1
    assert L.moe_grouped_ffn_weight_grad(a, a, a, a, a, a, 16, 256, 256, 4, a, mis, a, 0, null,
                                         null) == 1
    assert L.moe_grouped_ffn_backward(a, a, a, a, a, a, a, a, 16, 256, 256, 4, a, a, a, null,
                                      a, a, a, 0, null, null) == 1
    assert L.moe_grouped_ffn_backward(a, a, a, a, a, a, a, a, 16, 256, 256, 4, a, a, a, a,
                                      a, a, a, 3, null, null) == 1
    # zero-copy forward: K < 1, misaligned x, one pre-activation output only, S = 0 no-op
    assert L.moe_grouped_ffn_gather(a, a, 4, 0, a, a, a, a, 256, 256, 4, a, a, null, null) == 1
    assert L.moe_grouped_ffn_gather(mis, a, 4, 2, a, a, a, a, 256, 256, 4, a, a, null, null) == 1
    assert L.moe_grouped_ffn_up_gate_gather(a, a, 4, 2, a, a, a, 256, 256, 4, a, a, null, null,
                                            null) == 1
    assert L.moe_grouped_ffn_gather(a, a, 0, 2, a, a, a, a, 256, 256, 4, a, a, null, null) == 0
    # shared experts: E + n beyond the maximum, n < 1, S = 0 no-op
    assert L.moe_append_shared(a, a, 4, 2, 65535, 1, a, a, null) == 2
    assert L.moe_append_shared(a, a, 4, 2, 8, 0, a, a, null) == 1
    assert L.moe_append_shared(a, a, 0, 2, 8, 1, a, a, null) == 0


def test_host_validation_of_mxfp8_calls():
    L = moe.lib()
    a = fake(0x10000)
    null = P(0)
    # scale bytes: E*R*C/32 for multiples of 128, else 0
    assert moe.moe_mx_weight_scale_bytes(2, 256, 384) == 2 * 8 * 384
    assert moe.moe_mx_weight_scale_bytes(2, 200, 384) == 0
    # weight quantisation: R or C not a multiple of 128; null or misaligned buffers
    assert L.moe_mx_quantize_weights(a, 2, 192, 256, a, a, null) == 2
    assert L.moe_mx_quantize_weights(a, 2, 256, 160, a, a, null) == 2
    assert L.moe_mx_quantize_weights(a, 0, 256, 256, a, a, null) == 1
    assert L.moe_mx_quantize_weights(a, 2, 256, 256, null, a, null) == 1
    assert L.moe_mx_quantize_weights(a, 2, 256, 256, a, fake(0x10004), null) == 1
    # permute-quantise: H % 128, missing row map, misaligned outputs; S == 0 is a no-op
    assert L.moe_mx_permute_quantize(a, a, 16, 96, 2, a, a, null) == 2
    assert L.moe_mx_permute_quantize(a, null, 16, 256, 2, a, a, null) == 1
    assert L.moe_mx_permute_quantize(a, a, 16, 256, 2, a, fake(0x10008), null) == 1
    assert L.moe_mx_permute_quantize(null, null, 0, 256, 2, null, null, null) == 0
    # FFN passes: shapes as moe_grouped_ffn; every operand required; M == 0 is a no-op
    args_ug = [a, a, a, a, a, a, a, 64, 256, 256, 4, a, a, null, null]
    bad = list(args_ug)
    bad[8] = 200  # H % 128
    assert L.moe_grouped_ffn_up_gate_mxfp8(*bad) == 2
    bad = list(args_ug)
    bad[1] = null  # x_sf
    assert L.moe_grouped_ffn_up_gate_mxfp8(*bad) == 1
    bad = list(args_ug)
    bad[12] = fake(0x10002)  # h_sf misaligned
    assert L.moe_grouped_ffn_up_gate_mxfp8(*bad) == 1
    zero = list(args_ug)
    zero[7] = 0
    assert L.moe_grouped_ffn_up_gate_mxfp8(*zero) == 0
    assert L.moe_grouped_ffn_down_mxfp8(a, null, a, a, a, 64, 256, 256, 4, a, null, null) == 1
    assert L.moe_grouped_ffn_down_mxfp8(a, a, a, a, a, 64, 256, 384 + 64, 4, a, null, null) == 2
    assert L.moe_grouped_ffn_down_mxfp8(a, a, a, a, a, 0, 256, 256, 4, a, null, null) == 0
    assert L.moe_grouped_ffn_mxfp8(a, a, a, a, a, a, a, null, a, 64, 256, 256, 4, a, a, a, null,
                                   null) == 1
    assert L.moe_grouped_ffn_mxfp8(a, a, a, a, a, a, a, a, a, 64, 256, 256, 0, a, a, a, null,
                                   null) == 1


@pytest.mark.parametrize("fn", ["moe_permute", "moe_permute_no_alloc"])
def test_permute_wrappers_refuse_short_buffers_before_any_launch(fn):
    """The C ABI cannot see buffer sizes: the Python wrappers of both permutation entry points
    refuse a buffer of the wrong size with ValueError (here on CPU tensors, so nothing could
    launch even if the check were missing)."""
    S, K, E, H = 16, 2, 4, 8
    i32 = dict(dtype=torch.int32)
    ok = dict(x=torch.zeros(S, H, dtype=torch.bfloat16), topk_ids=torch.zeros(S, K, **i32),
              x_perm=torch.zeros(S * K, H, dtype=torch.bfloat16), counts=torch.zeros(E, **i32),
              cu_seqlens=torch.zeros(E + 1, **i32), row_id_map=torch.zeros(S * K, **i32),
              perm_src=torch.zeros(S * K, **i32))
    call = getattr(moe, fn)
    bad = {"x_perm": torch.zeros(S * K - 1, H, dtype=torch.bfloat16),
           "counts": torch.zeros(E - 1, **i32), "cu_seqlens": torch.zeros(E, **i32),
           "row_id_map": torch.zeros(S * K - 1, **i32), "perm_src": torch.zeros(S, **i32),
           "x": torch.zeros(S + 1, H, dtype=torch.bfloat16)}
    for name, t in bad.items():
        args = dict(ok, **{name: t})
        with pytest.raises(ValueError, match=r"expected|sizes|rows"):
            call(args["x"], args["topk_ids"], E, args["x_perm"], args["counts"],
                 args["cu_seqlens"], args["row_id_map"], args["perm_src"])
    # right sizes: refused only because these are not CUDA tensors
    with pytest.raises(ValueError, match="CUDA"):
        call(ok["x"], ok["topk_ids"], E, ok["x_perm"], ok["counts"], ok["cu_seqlens"],
             ok["row_id_map"], ok["perm_src"])
