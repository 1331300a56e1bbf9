"""moe_permute_no_alloc: the permutation for callers that may not allocate device memory
(engine plugins with pre-planned memory, frameworks that own the device memory pool). It
takes its scratch from a fixed array inside the library instead of a caller workspace.

Checked through the C ABI against moe_permute (which takes a caller workspace) on two calls
in a row with different routings: the second call reuses the array the first one left
behind. Permutation outputs are integers and bit copies, so they must match exactly. This
file is collected last so that a failure here cannot hide the other tests' results."""
import ctypes

import numpy as np
import pytest
import torch

import grouped_ffn_moe_b200 as moe
import synth
from helpers import GUARD

pytestmark = pytest.mark.gpu


def _outputs(S, K, E, H, dev):
    i32 = torch.int32
    return dict(x_perm=GUARD.full((S * K, H), float("nan"), torch.bfloat16, dev),
                counts=GUARD.full((E,), -9, i32, dev), cu=GUARD.full((E + 1,), -9, i32, dev),
                rmap=GUARD.full((S * K,), -9, i32, dev), psrc=GUARD.full((S * K,), -9, i32, dev),
                maxvio=GUARD.full((1,), -9.0, torch.float64, dev),
                max_count=GUARD.full((1,), -9, i32, dev), status=GUARD.zeros((1,), i32, dev))


def _call(fn_name, x, ids, E, o, workspace=None):
    L = moe.lib()
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    S, K = ids.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    common = (P(x), P(ids), S, x.shape[1], K, E, P(o["x_perm"]), P(o["counts"]), P(o["cu"]),
              P(o["rmap"]), P(o["psrc"]), P(o["maxvio"]), P(o["max_count"]))
    if fn_name == "moe_permute":
        st = L.moe_permute(*common, P(workspace), workspace.numel(), P(o["status"]), stream)
    else:
        st = L.moe_permute_no_alloc(*common, P(o["status"]), stream)
    assert st == 0, moe.moe_status_string(st)


@pytest.mark.parametrize("S,K,E,H", [(262147, 6, 64, 64), (4096, 6, 64, 2048)])
def test_no_alloc_permute_matches_workspace_permute_twice(cuda_device, S, K, E, H):
    """Above 2^17 routed slots the permutation keeps per-chunk counts in its scratch (the
    library's array here, a caller workspace for moe_permute); up to 2^17 it needs none."""
    dev = cuda_device
    need = moe.moe_permute_workspace_bytes(S, K, E)
    assert (need > 0) == (S * K > (1 << 17)) and need <= moe.MOE_NO_ALLOC_SCRATCH_BYTES
    x = synth.normal_bf16_into(torch.empty(S, H, dtype=torch.bfloat16, device=dev), 1, synth.TAG_X)
    routings = [synth.route_es(1, S, K, E)[0],
                synth.route_es(5, S, K, E, hot_e=E - 1, w_hot=20.0)[0]]
    for ids_np in routings:  # two calls in a row; the second reuses the library's array
        ids = torch.from_numpy(ids_np).to(dev)
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
        ref, got = _outputs(S, K, E, H, dev), _outputs(S, K, E, H, dev)
        _call("moe_permute", x, ids, E, ref, ws)
        _call("moe_permute_no_alloc", x, ids, E, got)
        torch.cuda.synchronize()
        for name in ("counts", "cu", "rmap", "psrc", "max_count", "maxvio", "x_perm", "status"):
            a, b = ref[name], got[name]
            if a.dtype == torch.bfloat16:
                a, b = a.view(torch.int16), b.view(torch.int16)
            assert torch.equal(a, b), name
        assert int(got["status"].item()) == 0
        assert int(got["counts"].sum().item()) == S * K


def test_no_alloc_rejects_sizes_beyond_its_array(cuda_device):
    L = moe.lib()
    a = ctypes.c_void_p(0x10000)  # never dereferenced: the size check fails first
    null = ctypes.c_void_p(0)
    S, K, E = 1 << 20, 8, 1024  # needs 64 MiB of scratch, the array holds 4 MiB
    assert moe.moe_permute_workspace_bytes(S, K, E) > moe.MOE_NO_ALLOC_SCRATCH_BYTES
    st = L.moe_permute_no_alloc(a, a, S, 64, K, E, a, a, a, a, null, null, null, null, null)
    assert st == moe.MOE_ERR_UNSUPPORTED_SHAPE
