"""The plain C++ oracle (oracle/moe_oracle_ref.cpp) against the pages' worked example, against
torch's bf16 rounding, and against the numpy oracle that the GPU tests use: two independent
restatements of the same steps (loops in C++, array operations in numpy) must agree."""
import itertools
import json
import os

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from oracle import ref as R

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _bf16_of_f32(v):
    return torch.from_numpy(np.asarray(v, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_bf16_rounding_matches_torch_and_the_numpy_oracle():
    rng = np.random.default_rng(0)
    f32 = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(3.0),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),  # fp32 subnormals
        np.array([0.0, -0.0, 1.0, -1.0, 3.3895314e38, -3.3895314e38, 1e-45, 2 ** -133,
                  2 ** -134, 3 * 2 ** -135, 1.00390625, 1.01171875, 1.0078125], np.float32),
    ])
    # float32 inputs: torch's float32 -> bf16 cast is round-to-nearest-even
    assert np.array_equal(R.round_bf16(f32.astype(np.float64)), _bf16_of_f32(f32))
    # double inputs (one rounding, not two): the numpy oracle's routine
    d = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-40, 38, 20000),
                        np.array([1.0 + 2 ** -8 + 2 ** -40, 1.0 + 2 ** -8 - 2 ** -40, 2.0 ** 128,
                                  -(2.0 ** 128), 3.3961e38, 2.0 ** -134 + 2 ** -160])])
    assert np.array_equal(R.round_bf16(d), O.f64_to_bf16_bits(d))
    assert R.round_bf16([np.inf])[0] == 0x7F80 and R.round_bf16([-np.inf])[0] == 0xFF80
    assert (R.round_bf16([np.nan])[0] & 0x7F80) == 0x7F80 and (R.round_bf16([np.nan])[0] & 0x7F)


def test_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "four_rank_example.json")))
    counts, cu, rmap, psrc = R.permute(np.array(g["topk_ids"]), g["E"])
    assert counts.tolist() == g["counts"] and cu.tolist() == g["cu_seqlens"]
    assert rmap.tolist() == g["row_id_map"] and psrc.tolist() == g["perm_src"]
    mv, mc = R.maxvio(counts, g["S"], g["K"])
    assert mc == g["max_count"]
    assert abs(mv - g["maxvio_num"] / g["maxvio_den"]) <= 4 * np.finfo(float).eps
    assert (mv, mc) == O.maxvio(counts, g["S"], g["K"])  # the same evaluation order


@pytest.mark.parametrize("S,K,E", [(2, 2, 3), (3, 2, 2), (2, 3, 3)])
def test_permutation_every_tiny_routing(S, K, E):
    for combo in itertools.product(itertools.product(range(E), repeat=K), repeat=S):
        ids = np.array(combo, dtype=np.int32).reshape(S, K)
        for u, v in zip(R.permute(ids, E), O.permute_counting_sort(ids, E)):
            assert np.array_equal(u, v)


def test_permutation_maxvio_and_rows_on_random_routings():
    rng = np.random.default_rng(1)
    for S, K, E in [(1, 1, 1), (257, 3, 17), (1000, 8, 384), (64, 2, 3000)]:
        ids = rng.integers(0, E, size=(S, K)).astype(np.int32)
        got = R.permute(ids, E)
        for u, v in zip(got, O.permute_metadata(ids, E)):
            assert np.array_equal(u, v)
        assert R.maxvio(got[0], S, K) == O.maxvio(got[0], S, K)
        x = rng.integers(0, 1 << 16, size=(S, 24)).astype(np.uint16)
        assert np.array_equal(R.permute_rows(x, got[3], K), O.permute_rows(x, got[3], K))
    with pytest.raises(ValueError):
        R.permute(np.array([[0, 5]], np.int32), 5)


def test_combine_matches_bit_for_bit():
    rng = np.random.default_rng(2)
    S, K, E, H = 200, 4, 9, 48
    ids = rng.integers(0, E, size=(S, K)).astype(np.int32)
    _, _, rmap, _ = O.permute_metadata(ids, E)
    y = O.f64_to_bf16_bits(rng.standard_normal((S * K, H)))
    w = rng.random((S, K)).astype(np.float32)
    # the same double operations in the same order (multiply, then add, k ascending)
    assert np.array_equal(R.combine(y, rmap, w, S, K), O.unpermute_combine(y, rmap, w, S, K))


def test_grouped_ffn_agrees_with_the_numpy_oracle():
    """Both accumulate in double and round once; only the order of a dot product's additions
    differs (loops against BLAS), which can move a value lying next to a bf16 rounding
    boundary by one step."""
    rng = np.random.default_rng(3)
    E, H, Hp = 4, 64, 96
    counts = np.array([0, 7, 1, 20])
    cu = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    M = int(cu[-1])
    x = O.f64_to_bf16_bits(rng.standard_normal((M, H)))
    wg = O.f64_to_bf16_bits(rng.standard_normal((E, H, Hp)) / 8)
    wu = O.f64_to_bf16_bits(rng.standard_normal((E, H, Hp)) / 8)
    wd = O.f64_to_bf16_bits(rng.standard_normal((E, Hp, H)) / 10)
    h_c, y_c = R.grouped_ffn(x, cu, wg, wu, wd)
    h_n, y_n = O.grouped_ffn(x, cu, lambda e: (wg[e], wu[e], wd[e]), Hp)
    for a, b in ((h_c, h_n), (y_c, y_n)):
        diff = a.astype(np.int32) - b.astype(np.int32)
        assert np.count_nonzero(diff) <= max(2, a.size // 1000)
        assert np.abs(diff).max() <= 1  # one bf16 step (same sign: adjacent bit patterns)
    # dropping SiLU or swapping gate and up is visible
    h_swap, _ = R.grouped_ffn(x, cu, wu, wg, wd)
    assert np.count_nonzero(h_swap != h_c) > h_c.size // 2


def test_combine_and_permute_backward_match():
    rng = np.random.default_rng(4)
    S, K, E, H = 150, 5, 7, 40
    ids = rng.integers(0, E, size=(S, K)).astype(np.int32)
    _, _, rmap, _ = O.permute_metadata(ids, E)
    g = O.f64_to_bf16_bits(rng.standard_normal((S, H)))
    y = O.f64_to_bf16_bits(rng.standard_normal((S * K, H)))
    w = rng.random((S, K)).astype(np.float32)
    gy_c, gw_c = R.combine_backward(g, y, rmap, w, S, K)
    gy_n, gw_n = O.combine_backward(g, y, rmap, w, S, K)
    assert np.array_equal(gy_c, gy_n)  # one rounding of an exact product on both sides
    assert np.allclose(gw_c, gw_n, rtol=1e-12, atol=1e-12)  # double sums, orders differ
    gxp = O.f64_to_bf16_bits(rng.standard_normal((S * K, H)))
    assert np.array_equal(R.permute_backward(gxp, rmap, S, K), O.permute_backward(gxp, rmap, S, K))


def test_e4m3_and_mx_quantisation_match():
    rng = np.random.default_rng(5)
    # E4M3 rounding: torch's float8_e4m3fn cast inside the finite range, and the numpy oracle
    # (which saturates at 448) everywhere, ties and subnormals included
    v = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-4, 3, 20000),
                        np.array([0.0, -0.0, 448.0, 464.0, 480.0, 1e6, -1e6, 2 ** -9, 2 ** -10,
                                  3 * 2 ** -11, 1.0625, 1.1875, 17.0, 19.0])])
    got = R.e4m3_round(v)
    assert np.array_equal(got, O.e4m3_round(v))
    inside = np.abs(v) <= 448
    t = torch.from_numpy(v[inside]).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(got[inside], t)
    # MXFP8 blocks along rows: random magnitudes per block, zero blocks, exact powers of two
    x = rng.standard_normal((64, 256)) * np.repeat(2.0 ** rng.integers(-20, 20, (64, 8)), 32, axis=1)
    x[3, 32:64] = 0.0
    x[5, :32] = 2.0 ** 7
    q_c, s_c = R.mx_quantize_rows(x)
    q_n, s_n = O.mx_quantize(x, axis=-1)
    assert np.array_equal(q_c, q_n) and np.array_equal(s_c, s_n)
    assert s_c[3, 1] == -127 and s_c[5, 0] == -1


def _close_bits(a, b, max_diff=2):
    """Equal, except at most max_diff elements one bf16 step apart (a double sum taken in a
    different order can move a value next to a rounding boundary)."""
    d = np.abs(a.astype(np.int32) - b.astype(np.int32))
    assert np.count_nonzero(d) <= max_diff and d.max() <= 1


def test_expert_backward_matches():
    rng = np.random.default_rng(6)
    n, H, Hp = 20, 64, 96
    bf = O.f64_to_bf16_bits
    x = bf(rng.standard_normal((n, H)))
    wg, wu = bf(rng.standard_normal((H, Hp)) / 8), bf(rng.standard_normal((H, Hp)) / 8)
    wd = bf(rng.standard_normal((Hp, H)) / 10)
    g, u = O.expert_preact_rows(x, wg, wu)
    h = bf(O.silu(O.bf16_bits_to_f64(g)) * O.bf16_bits_to_f64(u))
    gy = bf(rng.standard_normal((n, H)))
    got = R.expert_backward(x, g, u, h, gy, wg, wu, wd)
    ref = O.expert_ffn_backward_rows(x, g, u, h, gy, wg, wu, wd)
    for a, b in zip(got[:3], ref[:3]):  # d_g, d_u, grad_x
        _close_bits(a, b)
    if np.array_equal(got[0], ref[0]) and np.array_equal(got[1], ref[1]):
        for a, b in zip(got[3:], ref[3:]):  # the weight gradients, double sums
            assert np.allclose(a, b, rtol=1e-12, atol=1e-12 * np.abs(b).max())


def test_mxfp8_expert_matches():
    rng = np.random.default_rng(7)
    n, H, Hp = 12, 128, 64
    bf = O.f64_to_bf16_bits
    x = bf(rng.standard_normal((n, H)))
    wg, wu = bf(rng.standard_normal((H, Hp)) / 8), bf(rng.standard_normal((H, Hp)) / 8)
    wd = bf(rng.standard_normal((Hp, H)) / 8)
    hq_c, hs_c, y_c = R.expert_ffn_mxfp8(x, wg, wu, wd)
    hq_n, hs_n, y_n = O.expert_ffn_rows_mxfp8(x, O.mx_weights(wg), O.mx_weights(wu),
                                              O.mx_weights(wd))
    assert np.array_equal(hs_c, hs_n)
    assert np.count_nonzero(hq_c != hq_n) <= 2
    _close_bits(y_c, y_n, max_diff=max(2, y_c.size // 1000))
