"""Pins of the CPU oracle to facts fixed by the pages and by mathematics, not by itself.

Every oracle function is checked here against something independent of its own code:
the pages' worked example, brute force over all tiny routings, invariants, closed
forms and library routines (torch CPU) on special cases that reduce to them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bits_of(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def torch_bf16_of(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


# ----------------------------------------------------------------------------- worked example

def test_four_rank_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "four_rank_example.json")))
    ids = np.array(g["topk_ids"], dtype=np.int32)
    for fn in (O.permute_counting_sort, O.permute_metadata):
        counts, cu, rmap, psrc = fn(ids, g["E"])
        assert counts.tolist() == g["counts"]
        assert cu.tolist() == g["cu_seqlens"]
        assert psrc.tolist() == g["perm_src"]
        assert rmap.tolist() == g["row_id_map"]
    # rank r owns experts [2r, 2r+2): copies sent to each rank
    per_rank = [int(counts[2 * r] + counts[2 * r + 1]) for r in range(g["ranks"])]
    assert per_rank == g["rank_send_splits"]
    mv, mc = O.maxvio(counts, g["S"], g["K"])
    assert mc == g["max_count"]
    assert abs(mv - g["maxvio_num"] / g["maxvio_den"]) <= 4 * np.finfo(float).eps


def test_four_rank_example_weighted_reconstruction():
    """Token A's output is w_A0*Expert1(A) + w_A1*Expert5(A) (the example's last
    sentence), with hand-computable experts Expert_e(x) = (e+1) * x * x elementwise.
    """
    H = 8
    x = np.full((3, H), 1.0)
    x[0] *= 2.0  # A
    x[1] *= 3.0  # B
    x[2] *= 4.0  # C
    x_bits = O.f64_to_bf16_bits(x)
    ids = np.array([[1, 5], [3, 5], [0, 6]], dtype=np.int32)
    w = np.array([[0.25, 0.75], [0.5, 0.5], [0.125, 0.875]], dtype=np.float32)

    def weights(e):
        # g = 64 x_j (>= 64, so silu(g) == g after bf16 rounding), u = x_j / 64,
        # h = g * u = x_j^2, y = (e+1) * h. Every value is an exact small integer.
        wg = O.f64_to_bf16_bits(64.0 * np.eye(H))
        wu = O.f64_to_bf16_bits(np.eye(H) / 64.0)
        wd = O.f64_to_bf16_bits((e + 1.0) * np.eye(H))
        return wg, wu, wd

    res = O.moe_layer(x_bits, ids, w, 8, weights, H)
    out = O.bf16_bits_to_f64(res["out"])
    # A (x=2, h=4):  0.25 * 2*4 + 0.75 * 6*4 = 2 + 18 = 20
    assert np.all(out[0] == 20.0)
    # B (x=3, h=9):  0.5 * 4*9 + 0.5 * 6*9 = 18 + 27 = 45
    assert np.all(out[1] == 45.0)
    # C (x=4, h=16): 0.125 * 1*16 + 0.875 * 7*16 = 2 + 98 = 100
    assert np.all(out[2] == 100.0)


# ----------------------------------------------------------------------------- brute force

def _all_routings(S, K, E):
    per_token = list(itertools.product(range(E), repeat=K))
    for combo in itertools.product(per_token, repeat=S):
        yield np.array(combo, dtype=np.int32).reshape(S, K)


@pytest.mark.parametrize("S,K,E", [(1, 1, 3), (2, 2, 3), (3, 2, 2), (3, 1, 4), (2, 2, 4)])
def test_permutation_brute_force(S, K, E):
    """Every routing of tiny shapes (duplicates within a token included)."""
    for ids in _all_routings(S, K, E):
        a = O.permute_counting_sort(ids, E)
        b = O.permute_metadata(ids, E)
        for u, v in zip(a, b):
            assert np.array_equal(u, v)
        counts, cu, rmap, psrc = b
        flat = ids.reshape(-1).tolist()
        # counts by direct enumeration
        assert counts.tolist() == [flat.count(e) for e in range(E)]
        assert cu[0] == 0 and cu[-1] == S * K
        assert all(cu[e + 1] - cu[e] == counts[e] for e in range(E))
        # bijection
        assert sorted(rmap.tolist()) == list(range(S * K))
        assert all(psrc[rmap[f]] == f for f in range(S * K))
        # expert-contiguous and stable: rows of expert e are its flat slots ascending
        for e in range(E):
            rows = psrc[cu[e]:cu[e + 1]].tolist()
            assert rows == [f for f in range(S * K) if flat[f] == e]


def test_permute_rows_and_identity_roundtrip():
    rng = np.random.default_rng(0)
    S, K, E, H = 5, 3, 4, 16
    ids = rng.integers(0, E, size=(S, K)).astype(np.int32)
    x = O.f64_to_bf16_bits(rng.standard_normal((S, H)))
    counts, cu, rmap, psrc = O.permute_metadata(ids, E)
    xp = O.permute_rows(x, psrc, K)
    for t in range(S):
        for k in range(K):
            assert np.array_equal(xp[rmap[t * K + k]], x[t])
    # identity experts, K copies with unit weight: out = bf16(K * x), exact sums
    out = O.unpermute_combine(xp, rmap, np.ones((S, K), np.float32), S, K)
    expect = bits_of((torch_bf16_of(x).to(torch.float32) * K).to(torch.bfloat16))
    assert np.array_equal(out, expect)


def test_k1_unit_weight_is_identity():
    rng = np.random.default_rng(1)
    S, E, H = 9, 3, 8
    ids = rng.integers(0, E, size=(S, 1)).astype(np.int32)
    x = O.f64_to_bf16_bits(rng.standard_normal((S, H)))
    res = O.moe_layer(x, ids, np.ones((S, 1), np.float32), E, None, 0, identity_ffn=True)
    assert np.array_equal(res["out"], x)


def test_duplicate_route_is_added_not_overwritten():
    """A token sent twice to the same expert gets both weighted copies."""
    H = 4
    x = O.f64_to_bf16_bits(np.array([[1.0, 2.0, 3.0, 4.0]]))
    ids = np.array([[2, 2]], dtype=np.int32)
    w = np.array([[0.5, 0.25]], dtype=np.float32)
    res = O.moe_layer(x, ids, w, 3, None, 0, identity_ffn=True)
    assert res["counts"].tolist() == [0, 0, 2]
    np.testing.assert_array_equal(O.bf16_bits_to_f64(res["out"]), 0.75 * np.array([[1, 2, 3, 4.0]]))


def test_empty_experts():
    ids = np.array([[0, 3], [3, 0]], dtype=np.int32)
    counts, cu, rmap, psrc = O.permute_metadata(ids, 6)
    assert counts.tolist() == [2, 0, 0, 2, 0, 0]
    assert cu.tolist() == [0, 2, 2, 2, 4, 4, 4]


def test_rejects_bad_routing():
    with pytest.raises(ValueError):
        O.permute_metadata(np.array([[0, 5]], np.int32), 5)
    with pytest.raises(ValueError):
        O.permute_counting_sort(np.array([[-1, 0]], np.int32), 5)


# ----------------------------------------------------------------------------- maxvio

def test_maxvio_closed_forms():
    S, K, E = 48, 4, 8  # E | S*K
    f = np.arange(S * K)
    ids = (f % E).astype(np.int32).reshape(S, K)
    counts, *_ = O.permute_metadata(ids, E)
    assert O.maxvio(counts, S, K) == (0.0, S * K // E)
    # all tokens on one expert with K=1: maxvio = E - 1 exactly
    ids1 = np.zeros((S, 1), np.int32)
    counts1, *_ = O.permute_metadata(ids1, E)
    assert O.maxvio(counts1, S, 1) == (float(E - 1), S)
    # large-geometry values: hot counts 204, 341, 1877, 3584 of 65536 rows over 384 experts
    for hot, expect in [(204, 0.1953125), (341, 0.998046875), (1877, 9.998046875), (3584, 20.0)]:
        c = np.zeros(384, np.int64)
        c[0] = hot
        assert O.maxvio(c, 8192, 8)[0] == expect


# ----------------------------------------------------------------------------- bf16 rounding

def test_bf16_round_matches_torch_on_float32_values():
    rng = np.random.default_rng(2)
    v = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
        rng.standard_normal(2000).astype(np.float32) * np.float32(1e-39),  # subnormals
    ]).astype(np.float32)
    ties = (np.arange(1, 2000, dtype=np.uint32) << 16 | 0x8000).view(np.float32)  # exact halves
    v = np.concatenate([v, ties, -ties, np.float32([0.0, -0.0, 3.3895e38])])
    ours = O.f64_to_bf16_bits(v.astype(np.float64))
    ref = bits_of(torch.from_numpy(v).to(torch.bfloat16))
    np.testing.assert_array_equal(ours, ref)


def test_bf16_round_single_rounding_from_double():
    # 1 + 2^-8 + 2^-30 is just above the tie between 1 and 1+2^-7: rounds up. Going
    # through float32 first would drop the 2^-30 and the tie would round to even (1.0).
    v = np.array([1.0 + 2.0 ** -8 + 2.0 ** -30, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8])
    assert O.bf16_bits_to_f64(O.f64_to_bf16_bits(v)).tolist() == [1.0 + 2.0 ** -7, 1.0, 1.0 + 2.0 ** -6]
    assert O.f64_to_bf16_bits(np.array([1e39]))[0] == 0x7F80  # overflow -> +inf


# ----------------------------------------------------------------------------- SiLU / FFN

def test_silu_identities_and_library():
    z = np.linspace(-40, 40, 2001)
    s = O.silu(z)
    np.testing.assert_allclose(s - O.silu(-z), z, rtol=0, atol=1e-12)  # silu(z) - silu(-z) = z
    assert O.silu(np.array([0.0]))[0] == 0.0
    ref = torch.nn.functional.silu(torch.from_numpy(z)).numpy()
    np.testing.assert_allclose(s, ref, rtol=1e-14, atol=1e-300)
    assert O.silu(np.array([-1000.0]))[0] == 0.0


def _weights_getter(wg, wu, wd):
    return lambda e: (wg[e], wu[e], wd[e])


def _rand_layer(rng, S, H, Hp, E, K):
    x = O.f64_to_bf16_bits(rng.standard_normal((S, H)))
    wg = O.f64_to_bf16_bits(rng.standard_normal((E, H, Hp)) / math.sqrt(H))
    wu = O.f64_to_bf16_bits(rng.standard_normal((E, H, Hp)) / math.sqrt(H))
    wd = O.f64_to_bf16_bits(rng.standard_normal((E, Hp, H)) / math.sqrt(Hp))
    ids = np.stack([rng.permutation(E)[:K] for _ in range(S)]).astype(np.int32)
    z = rng.standard_normal((S, K))
    w = (np.exp(z) / np.exp(z).sum(1, keepdims=True)).astype(np.float32)
    return x, wg, wu, wd, ids, w


def test_dense_special_case_against_torch():
    """K=1 with every token on expert 0 is a dense SwiGLU FFN: compare with torch CPU
    (matmul + F.silu in float64, rounded to bf16 by torch at the same points)."""
    rng = np.random.default_rng(3)
    S, H, Hp, E = 24, 32, 48, 3
    x, wg, wu, wd, _, _ = _rand_layer(rng, S, H, Hp, E, 1)
    ids = np.zeros((S, 1), np.int32)
    res = O.moe_layer(x, ids, np.ones((S, 1), np.float32), E, _weights_getter(wg, wu, wd), Hp)
    assert res["maxvio"] == float(E - 1)
    T = lambda b: torch_bf16_of(b).to(torch.float64)
    g, u = T(x) @ T(wg[0]), T(x) @ T(wu[0])
    h = (torch.nn.functional.silu(g) * u).to(torch.float32).to(torch.bfloat16)
    y = (h.to(torch.float64) @ T(wd[0])).to(torch.float32).to(torch.bfloat16)
    # torch rounds through float32 (double rounding); allow 1 bf16 ulp where that matters
    hd = np.abs(O.bf16_bits_to_f64(res["h"]) - h.to(torch.float64).numpy())
    assert np.all(hd <= 2.0 ** -7 * np.abs(h.to(torch.float64).numpy()) + 1e-30)
    assert (O.bf16_bits_to_f64(res["h"]) == h.to(torch.float64).numpy()).mean() > 0.999
    yd = np.abs(O.bf16_bits_to_f64(res["y"]) - y.to(torch.float64).numpy())
    assert np.all(yd <= 2.0 ** -6 * np.abs(y.to(torch.float64).numpy()) + 1e-6)
    # unit weight, K=1: out == y
    assert np.array_equal(res["out"], res["y"])


def test_layer_matches_direct_expert_loop():
    """Permute -> grouped FFN -> combine equals running each token's experts directly
    ("Distributed expert parallelism", Exercises, item 3)."""
    rng = np.random.default_rng(4)
    S, H, Hp, E, K = 13, 16, 24, 5, 2
    x, wg, wu, wd, ids, w = _rand_layer(rng, S, H, Hp, E, K)
    get = _weights_getter(wg, wu, wd)
    res = O.moe_layer(x, ids, w, E, get, Hp)
    direct = O.direct_expert_loop(x, ids, w, get)
    a, b = O.bf16_bits_to_f64(res["out"]), O.bf16_bits_to_f64(direct)
    # the only difference is BLAS summation order inside fp64 dot products
    assert (a == b).mean() > 0.99
    np.testing.assert_allclose(a, b, rtol=2 ** -7, atol=1e-6)


def test_hand_computable_ffn_values():
    """H = H' = 8 with a gate so large that silu(g) == g in bf16: the expert is then
    bilinear and every value below is an exact dyadic rational."""
    H = 8
    x = O.f64_to_bf16_bits(np.arange(1, 9, dtype=np.float64)[None, :] / 4.0)  # 0.25..2
    wg = O.f64_to_bf16_bits(128.0 * np.eye(H))  # g_j = 128 x_j >= 32
    wu = O.f64_to_bf16_bits(np.diag(np.full(H, 0.5)))  # u_j = x_j / 2
    wd = O.f64_to_bf16_bits(np.ones((H, H)) / 64.0)  # y_n = sum_j h_j / 64
    h, y = O.expert_ffn_rows(x, wg, wu, wd)
    xv = np.arange(1, 9) / 4.0
    np.testing.assert_array_equal(O.bf16_bits_to_f64(h)[0], 64.0 * xv * xv)  # 128 x * x/2
    np.testing.assert_array_equal(O.bf16_bits_to_f64(y)[0], np.full(H, (64.0 * xv * xv).sum() / 64.0))
    # a large negative gate drives h to (almost) zero: silu(-128 x) * u
    h2, _ = O.expert_ffn_rows(x, O.f64_to_bf16_bits(-128.0 * np.eye(H)), wu, wd)
    assert np.all(np.abs(O.bf16_bits_to_f64(h2)) < 1e-10)


def test_swiglu_roles_gate_vs_up():
    """silu applies to the Gate branch only: swapping Gate and Up changes the result."""
    H = 8
    x = O.f64_to_bf16_bits(np.full((1, H), 1.0))
    a = O.f64_to_bf16_bits(np.eye(H))  # projection giving 1
    b = O.f64_to_bf16_bits(-np.eye(H))  # projection giving -1
    wd = O.f64_to_bf16_bits(np.eye(H))
    h_ab, _ = O.expert_ffn_rows(x, a, b, wd)  # silu(1) * (-1)
    h_ba, _ = O.expert_ffn_rows(x, b, a, wd)  # silu(-1) * 1
    s1 = 1.0 / (1.0 + math.exp(-1.0))
    assert O.bf16_bits_to_f64(h_ab)[0, 0] == O.bf16_bits_to_f64(O.f64_to_bf16_bits(np.array([-s1])))[0]
    assert O.bf16_bits_to_f64(h_ba)[0, 0] == O.bf16_bits_to_f64(O.f64_to_bf16_bits(np.array([-(1 - s1)])))[0]


def test_mis_addressed_expert_is_visible():
    """Distinct weights per expert: routing a row to the wrong expert changes y a lot."""
    rng = np.random.default_rng(5)
    S, H, Hp, E, K = 8, 16, 16, 4, 1
    x, wg, wu, wd, ids, w = _rand_layer(rng, S, H, Hp, E, K)
    get = _weights_getter(wg, wu, wd)
    good = O.moe_layer(x, ids, w, E, get, Hp)
    bad = O.moe_layer(x, (ids + 1) % E, w, E, get, Hp)
    a, b = O.bf16_bits_to_f64(good["out"]), O.bf16_bits_to_f64(bad["out"])
    assert np.linalg.norm(a - b) > 0.3 * np.linalg.norm(a)


# ----------------------------------------------------------------------------- acceptance bar

def test_acceptance_bar_accepts_one_step_flips_only():
    """The bf16 bar: rel-Frobenius and max-abs, where an element beyond the max-abs bar must
    be exactly one bf16 step from the reference (a rounding-boundary flip)."""
    from helpers import assert_close_bf16

    rng = np.random.default_rng(12)
    ref = O.f64_to_bf16_bits(rng.standard_normal(100000))
    ref[7] = O.f64_to_bf16_bits(np.array([13.0]))[0]  # an outlier at ~13 rms
    got = ref.copy()
    got[7] += 1  # one step: 13.0 -> 13.0625, above 3e-2 * rms
    stats = assert_close_bf16(got, ref, "flip")
    assert stats["one_step_flips_over_bar"] == 1
    bad = ref.copy()
    bad[7] += 2  # two steps: rejected
    with pytest.raises(AssertionError):
        assert_close_bf16(bad, ref, "two steps")
    wrong_row = ref.copy()
    wrong_row[:100] = ref[100:200]  # mis-addressed rows: rejected
    with pytest.raises(AssertionError):
        assert_close_bf16(wrong_row, ref, "wrong rows")


def test_expert_down_rows_against_torch():
    """The stage-wise down projection (used to check the down kernel on its own inputs)
    equals torch's fp64 matmul rounded to bf16 (torch rounds via float32: allow 1 step)."""
    rng = np.random.default_rng(13)
    h = O.f64_to_bf16_bits(rng.standard_normal((40, 24)))
    wd = O.f64_to_bf16_bits(rng.standard_normal((24, 16)) / math.sqrt(24))
    got = O.bf16_bits_to_f64(O.expert_down_rows(h, wd))
    T = lambda b: torch_bf16_of(b).to(torch.float64)
    ref = (T(h) @ T(wd)).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    assert (got == ref).mean() > 0.99
    np.testing.assert_allclose(got, ref, rtol=2.0 ** -7, atol=1e-30)


# ----------------------------------------------------------------------------- backward

def _autograd_combine(g, y, rmap, w, S, K):
    """torch fp64 autograd of out[t] = sum_k w[t,k] * y[rmap[t,k]]."""
    yt = torch.tensor(y, dtype=torch.float64, requires_grad=True)
    wt = torch.tensor(w, dtype=torch.float64, requires_grad=True)
    idx = torch.tensor(rmap.reshape(S, K), dtype=torch.long)
    out = (wt.unsqueeze(-1) * yt[idx]).sum(dim=1)
    out.backward(torch.tensor(g, dtype=torch.float64))
    return yt.grad.numpy(), wt.grad.numpy()


def test_combine_backward_against_autograd():
    rng = np.random.default_rng(21)
    S, K, E, H = 37, 3, 5, 24
    ids = rng.integers(0, E, size=(S, K)).astype(np.int32)  # duplicates included
    counts, cu, rmap, psrc = O.permute_metadata(ids, E)
    y = O.f64_to_bf16_bits(rng.standard_normal((S * K, H)))
    g = O.f64_to_bf16_bits(rng.standard_normal((S, H)))
    w = rng.random((S, K)).astype(np.float32)
    gy, gw = O.combine_backward(g, y, rmap, w, S, K)
    ref_gy, ref_gw = _autograd_combine(O.bf16_bits_to_f64(g), O.bf16_bits_to_f64(y), rmap,
                                       w.astype(np.float64), S, K)
    # grad_y: every row is hit by exactly one slot, so the gradient is w * g rounded once
    np.testing.assert_array_equal(gy, O.f64_to_bf16_bits(ref_gy))
    np.testing.assert_allclose(gw, ref_gw, rtol=1e-12, atol=1e-12)


def test_permute_backward_against_autograd():
    rng = np.random.default_rng(22)
    S, K, E, H = 29, 4, 6, 16
    ids = rng.integers(0, E, size=(S, K)).astype(np.int32)
    counts, cu, rmap, psrc = O.permute_metadata(ids, E)
    gxp = O.f64_to_bf16_bits(rng.standard_normal((S * K, H)))
    got = O.permute_backward(gxp, rmap, S, K)
    xt = torch.zeros((S, H), dtype=torch.float64, requires_grad=True)
    xperm = xt[torch.tensor(psrc.astype(np.int64) // K)]  # the permutation's forward gather
    xperm.backward(torch.tensor(O.bf16_bits_to_f64(gxp)))
    np.testing.assert_array_equal(got, O.f64_to_bf16_bits(xt.grad.numpy()))


def test_backward_adjoint_identity():
    """<grad_out, combine(y)> = <grad_y, y> (before rounding): the combine's backward is its
    transpose; checked with exact small-integer data where every value is representable."""
    rng = np.random.default_rng(23)
    S, K, E, H = 11, 2, 3, 8
    ids = rng.integers(0, E, size=(S, K)).astype(np.int32)
    counts, cu, rmap, psrc = O.permute_metadata(ids, E)
    y = O.f64_to_bf16_bits(rng.integers(-4, 5, size=(S * K, H)).astype(np.float64))
    g = O.f64_to_bf16_bits(rng.integers(-4, 5, size=(S, H)).astype(np.float64))
    w = (rng.integers(1, 5, size=(S, K)) / 4.0).astype(np.float32)
    out = O.bf16_bits_to_f64(O.unpermute_combine(y, rmap, w, S, K))
    gy, gw = O.combine_backward(g, y, rmap, w, S, K)
    lhs = np.sum(O.bf16_bits_to_f64(g) * out)
    rhs = np.sum(O.bf16_bits_to_f64(gy) * O.bf16_bits_to_f64(y))
    assert lhs == rhs
    assert np.sum(gw * w) == lhs  # sum_k w * <g, y_k> = <g, out>


# ----------------------------------------------------------------------------- FFN backward


def _ffn_bwd_case(seed, rows_per_expert, H, Hp):
    rng = np.random.default_rng(seed)
    E = len(rows_per_expert)
    cu = np.concatenate([[0], np.cumsum(rows_per_expert)]).astype(np.int32)
    M = int(cu[-1])
    x = O.f64_to_bf16_bits(rng.standard_normal((M, H)))
    wg = O.f64_to_bf16_bits(rng.standard_normal((E, H, Hp)) / math.sqrt(H))
    wu = O.f64_to_bf16_bits(rng.standard_normal((E, H, Hp)) / math.sqrt(H))
    wd = O.f64_to_bf16_bits(rng.standard_normal((E, Hp, H)) / math.sqrt(Hp))
    get = _weights_getter(wg, wu, wd)
    h, _ = O.grouped_ffn(x, cu, get, Hp)
    g, u = O.grouped_ffn_preact(x, cu, get, Hp)
    gy = O.f64_to_bf16_bits(rng.standard_normal((M, H)))
    return dict(E=E, cu=cu, M=M, x=x, wg=wg, wu=wu, wd=wd, get=get, h=h, g=g, u=u, gy=gy)


def _within_one_bf16_step(got_bits, ref_f64, min_exact=0.99):
    ref_bits = O.f64_to_bf16_bits(ref_f64)
    diff = np.abs(got_bits.astype(np.int32) - ref_bits.astype(np.int32))
    assert diff.max() <= 1, diff.max()
    assert np.mean(diff == 0) >= min_exact


def test_ffn_backward_against_autograd():
    """Each stage of the oracle's backward against torch autograd (float64) of the forward
    definition, evaluated at the oracle's own stored tensors."""
    c = _ffn_bwd_case(41, [5, 0, 9, 3], H=16, Hp=24)
    res = O.grouped_ffn_backward(c["x"], c["g"], c["u"], c["h"], c["gy"], c["cu"], c["get"])
    f = lambda b: torch.tensor(O.bf16_bits_to_f64(b))
    for e in range(c["E"]):
        r0, r1 = int(c["cu"][e]), int(c["cu"][e + 1])
        if r1 == r0:
            for k in ("dWg", "dWu", "dWd"):
                assert not res[k][e].any()
            continue
        sl = slice(r0, r1)
        # down projection: grad_h and dWd
        hl = f(c["h"][sl]).requires_grad_()
        wd = f(c["wd"][e]).requires_grad_()
        (hl @ wd).backward(f(c["gy"][sl]))
        np.testing.assert_allclose(res["dWd"][e], wd.grad.numpy().astype(np.float32), rtol=1e-6,
                                   atol=1e-6)
        # SwiGLU at the saved pre-activations
        G = f(c["g"][sl]).requires_grad_()
        U = f(c["u"][sl]).requires_grad_()
        (torch.nn.functional.silu(G) * U).backward(hl.grad)
        _within_one_bf16_step(res["d_g"][sl], G.grad.numpy())
        _within_one_bf16_step(res["d_u"][sl], U.grad.numpy())
        # up and gate projections, driven by the stored d_g, d_u
        xl = f(c["x"][sl]).requires_grad_()
        wg = f(c["wg"][e]).requires_grad_()
        wu = f(c["wu"][e]).requires_grad_()
        torch.autograd.backward([xl @ wg, xl @ wu], [f(res["d_g"][sl]), f(res["d_u"][sl])])
        _within_one_bf16_step(res["grad_x_perm"][sl], xl.grad.numpy())
        np.testing.assert_allclose(res["dWg"][e], wg.grad.numpy().astype(np.float32), rtol=1e-6,
                                   atol=1e-6)
        np.testing.assert_allclose(res["dWu"][e], wu.grad.numpy().astype(np.float32), rtol=1e-6,
                                   atol=1e-6)


def test_ffn_backward_brute_force_rows():
    """Row by row with scalar loops: each row uses its own expert's weights, weight
    gradients are sums of per-row outer products, empty experts get zeros."""
    c = _ffn_bwd_case(42, [2, 3, 0, 1], H=4, Hp=6)
    res = O.grouped_ffn_backward(c["x"], c["g"], c["u"], c["h"], c["gy"], c["cu"], c["get"])
    f = O.bf16_bits_to_f64
    H, Hp, E = 4, 6, c["E"]
    dWg = np.zeros((E, H, Hp)); dWu = np.zeros((E, H, Hp)); dWd = np.zeros((E, Hp, H))
    for r in range(c["M"]):
        e = int(np.searchsorted(c["cu"], r, side="right") - 1)
        wg, wu, wd = f(c["wg"][e]), f(c["wu"][e]), f(c["wd"][e])
        gy, x, hrow = f(c["gy"][r]), f(c["x"][r]), f(c["h"][r])
        dg = np.zeros(Hp); du = np.zeros(Hp)
        for j in range(Hp):
            gh = sum(gy[n] * wd[j, n] for n in range(H))
            gj, uj = f(c["g"][r, j]), f(c["u"][r, j])
            sg = 1.0 / (1.0 + math.exp(-gj))
            dg[j] = f(O.f64_to_bf16_bits(np.array(gh * uj * sg * (1 + gj * (1 - sg)))))
            du[j] = f(O.f64_to_bf16_bits(np.array(gh * gj * sg)))
        assert np.array_equal(f(res["d_g"][r]), dg) and np.array_equal(f(res["d_u"][r]), du)
        gx = [sum(dg[j] * wg[n, j] + du[j] * wu[n, j] for j in range(Hp)) for n in range(H)]
        assert np.array_equal(res["grad_x_perm"][r], O.f64_to_bf16_bits(np.array(gx)))
        dWg[e] += np.outer(x, dg); dWu[e] += np.outer(x, du); dWd[e] += np.outer(hrow, gy)
    np.testing.assert_allclose(res["dWg"], dWg.astype(np.float32), rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(res["dWu"], dWu.astype(np.float32), rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(res["dWd"], dWd.astype(np.float32), rtol=1e-6, atol=1e-7)
    assert not res["dWg"][2].any() and not res["dWd"][2].any()


def test_swiglu_backward_closed_forms():
    gh = np.array([[1.5, -2.0, 0.75, 3.0]])
    u_bits = O.f64_to_bf16_bits(np.array([[2.0, 0.5, -1.25, 4.0]]))
    u = O.bf16_bits_to_f64(u_bits)
    # g = 0: silu(0) = 0, silu'(0) = 1/2
    dg, du = O.swiglu_backward(gh, O.f64_to_bf16_bits(np.zeros((1, 4))), u_bits)
    assert not O.bf16_bits_to_f64(du).any()
    np.testing.assert_array_equal(dg, O.f64_to_bf16_bits(gh * u / 2))
    # g = +-128: sigmoid is 1 or below bf16's range, so silu(g) -> g or 0 and
    # silu'(g) -> 1 or 0 after rounding (compared as values: the zeros carry a sign)
    for gv, sil, dsil in ((128.0, 128.0, 1.0), (-128.0, 0.0, 0.0)):
        dg, du = O.swiglu_backward(gh, O.f64_to_bf16_bits(np.full((1, 4), gv)), u_bits)
        np.testing.assert_array_equal(O.bf16_bits_to_f64(du), gh * sil)
        np.testing.assert_array_equal(O.bf16_bits_to_f64(dg),
                                      O.bf16_bits_to_f64(O.f64_to_bf16_bits(gh * u * dsil)))
    # silu'(g) against a central difference of silu
    gs = O.f64_to_bf16_bits(np.linspace(-6, 6, 25)[None, :])
    gv = O.bf16_bits_to_f64(gs)
    ones = O.f64_to_bf16_bits(np.ones_like(gv))
    dg, _ = O.swiglu_backward(np.ones_like(gv), gs, ones)
    eps = 1e-6
    fd = (O.silu(gv + eps) - O.silu(gv - eps)) / (2 * eps)
    _within_one_bf16_step(dg, fd, min_exact=0.9)


def test_ffn_backward_accumulates_into_fp32_buffers():
    c = _ffn_bwd_case(43, [4, 2], H=8, Hp=8)
    fresh = O.grouped_ffn_backward(c["x"], c["g"], c["u"], c["h"], c["gy"], c["cu"], c["get"])
    rng = np.random.default_rng(44)
    prior = [rng.standard_normal(fresh[k].shape).astype(np.float32) for k in ("dWg", "dWu", "dWd")]
    acc = O.grouped_ffn_backward(c["x"], c["g"], c["u"], c["h"], c["gy"], c["cu"], c["get"],
                                 dw_prior=prior)
    for k, p in zip(("dWg", "dWu", "dWd"), prior):
        e1 = fresh[k].astype(np.float64)  # fresh is already fp32-rounded: allow that step
        np.testing.assert_allclose(acc[k], p.astype(np.float64) + e1, rtol=1e-6, atol=1e-6)
    np.testing.assert_array_equal(acc["d_g"], fresh["d_g"])


def test_preactivations_against_torch():
    rng = np.random.default_rng(45)
    x = O.f64_to_bf16_bits(rng.standard_normal((7, 16)))
    wg = O.f64_to_bf16_bits(rng.standard_normal((16, 8)))
    wu = O.f64_to_bf16_bits(rng.standard_normal((16, 8)))
    g, u = O.expert_preact_rows(x, wg, wu)
    tx = torch_bf16_of(x).double()
    np.testing.assert_array_equal(g, bits_of((tx @ torch_bf16_of(wg).double()).to(torch.bfloat16)))
    np.testing.assert_array_equal(u, bits_of((tx @ torch_bf16_of(wu).double()).to(torch.bfloat16)))


# ----------------------------------------------------------------------------- shared expert


def test_shared_expert_layer_against_direct_loop_and_dense_ffn():
    """The layer with a shared expert equals a per-token loop that runs the shared FFN and the
    token's K experts on its own row and sums them in one rounding; with zero route weights
    it is the dense SwiGLU FFN of the shared weights (torch float64)."""
    rng = np.random.default_rng(51)
    S, H, Hp, Hs, E, K = 9, 16, 24, 40, 4, 2
    x, wg, wu, wd, ids, w = _rand_layer(rng, S, H, Hp, E, K)
    get = _weights_getter(wg, wu, wd)
    sh = (O.f64_to_bf16_bits(rng.standard_normal((H, Hs)) / 4),
          O.f64_to_bf16_bits(rng.standard_normal((H, Hs)) / 4),
          O.f64_to_bf16_bits(rng.standard_normal((Hs, H)) / 6))
    res = O.moe_layer_with_shared(x, ids, w, E, get, Hp, sh)
    f = O.bf16_bits_to_f64
    for t in range(S):
        acc = f(O.expert_ffn_rows(x[t:t + 1], *sh)[1])[0].copy()
        for k in range(K):
            acc += float(w[t, k]) * f(O.expert_ffn_rows(x[t:t + 1], *get(int(ids[t, k])))[1])[0]
        np.testing.assert_array_equal(res["out"][t], O.f64_to_bf16_bits(acc))
    zero = O.moe_layer_with_shared(x, ids, np.zeros_like(w), E, get, Hp, sh)
    tx = torch.tensor(f(x))
    g = tx @ torch.tensor(f(sh[0]))
    u = tx @ torch.tensor(f(sh[1]))
    hh = torch.tensor(f(O.f64_to_bf16_bits((torch.nn.functional.silu(g) * u).numpy())))
    dense = (hh @ torch.tensor(f(sh[2]))).numpy()
    np.testing.assert_array_equal(zero["out"], O.f64_to_bf16_bits(dense))


# ----------------------------------------------------------------------------- MXFP8


def test_e4m3_round_against_torch_and_saturation():
    rng = np.random.default_rng(61)
    v = np.concatenate([rng.standard_normal(4000) * s for s in (1e-3, 0.1, 1.0, 30.0, 200.0)])
    v = np.concatenate([v, [0.0, 2 ** -9, 2 ** -10, 3 * 2 ** -11, 2 ** -6, 1.0625, 1.1875,
                            440.0, 448.0, 460.0, 464.0, -463.9]])
    v = v[np.abs(v) <= 464.0]  # torch's cast gives NaN above 464; the oracle saturates there
    ref = torch.tensor(v, dtype=torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.e4m3_round(v.astype(np.float32).astype(np.float64))
    np.testing.assert_array_equal(got, ref)
    np.testing.assert_array_equal(O.e4m3_round(np.array([465.0, 511.9, -1e9])),
                                  [448.0, 448.0, -448.0])


def test_mx_quantize_block_values_by_hand():
    """A block holding 1..32: amax 32 gives scale 2^(5-8) = 1/8, so v*8 is rounded in E4M3.
    8k is exact up to k = 16; above, the binade [128, 256) has step 16: 136 -> 128 (tie to
    even), 152 -> 160 (tie to even), 200 -> 192 (nearest), 256 exact."""
    v = np.arange(1, 33, dtype=np.float64)[None, :]
    q, s = O.mx_quantize(v)
    assert s.shape == (1, 1) and s[0, 0] == -3
    np.testing.assert_array_equal(q[0, :16], 8.0 * np.arange(1, 17))
    assert (q[0, 16], q[0, 18], q[0, 24], q[0, 31]) == (128.0, 160.0, 192.0, 256.0)
    deq = O.mx_dequantize(q, s)
    assert (deq[0, 16], deq[0, 31]) == (16.0, 32.0)


def test_mx_quantize_invariants():
    rng = np.random.default_rng(62)
    v = rng.standard_normal((7, 96)) * np.exp(rng.uniform(-8, 8, (7, 1)))
    v[3, 32:64] = 0.0  # an all-zero block
    q, s = O.mx_quantize(v, axis=-1)
    assert s.shape == (7, 3) and s[3, 1] == -127 and not q[3, 32:64].any()
    blocks = np.abs(q).reshape(7, 3, 32).max(-1)
    nz = np.abs(v).reshape(7, 3, 32).max(-1) > 0
    assert np.all((blocks[nz] >= 256) & (blocks[nz] <= 448))
    # within half an E4M3 step of the scaled value (or saturated), never more
    scaled = v / np.repeat(np.ldexp(1.0, s), 32, axis=-1)
    a = np.abs(scaled)
    half = np.ldexp(1.0, (np.maximum(np.floor(np.log2(np.where(a > 0, a, 1))), -6) - 4).astype(int))
    assert np.all((np.abs(q - scaled) <= half) | (np.abs(q) == 448.0))
    # values already on the grid come back exactly; quantising along another axis agrees
    q2, s2 = O.mx_quantize(O.mx_dequantize(q, s))
    np.testing.assert_array_equal(q2, q)
    qt, st = O.mx_quantize(v.T.copy(), axis=0)
    np.testing.assert_array_equal(qt.T, q)
    np.testing.assert_array_equal(st.T, s)


def test_mxfp8_dot_block_factorisation():
    """An MXFP8 dot product is a sum over blocks of 2^(sa + sb) * sum of element products;
    dequantise-then-multiply (as the FFN oracle does) must equal that form exactly."""
    rng = np.random.default_rng(63)
    a = rng.standard_normal((5, 128))
    b = rng.standard_normal((128, 6)) * 10
    qa, sa = O.mx_quantize(a, axis=-1)
    qb, sb = O.mx_quantize(b, axis=0)
    ref = np.zeros((5, 6))
    for blk in range(4):
        sl = slice(32 * blk, 32 * blk + 32)
        ref += np.ldexp(1.0, sa[:, blk:blk + 1] + sb[blk:blk + 1, :]) * (qa[:, sl] @ qb[sl, :])
    got = O.mx_dequantize(qa, sa, axis=-1) @ O.mx_dequantize(qb, sb, axis=0)
    np.testing.assert_array_equal(got, ref)


def test_mxfp8_expert_ffn_close_to_bf16_expert():
    """The MXFP8 expert against the bf16 expert on the same inputs. E4M3 keeps 3 mantissa
    bits: an element's rounding error is at most 2^-4 and about 3.6% RMS, a product of two
    quantised values about 5%, and the three quantised GEMMs plus the quantised h add in
    quadrature to about 9% (measured 9.3%). A dropped scale, a wrong axis or a wrong
    rounding mode shows as an O(1) error, beyond the 20% bar."""
    rng = np.random.default_rng(64)
    H, Hp, n = 128, 96, 10
    x = O.f64_to_bf16_bits(rng.standard_normal((n, H)))
    wg = O.f64_to_bf16_bits(rng.standard_normal((H, Hp)) / math.sqrt(H))
    wu = O.f64_to_bf16_bits(rng.standard_normal((H, Hp)) / math.sqrt(H))
    wd = O.f64_to_bf16_bits(rng.standard_normal((Hp, H)) / math.sqrt(Hp))
    _, y_bf16 = O.expert_ffn_rows(x, wg, wu, wd)
    hq, hs, y_mx = O.expert_ffn_rows_mxfp8(x, O.mx_weights(wg), O.mx_weights(wu), O.mx_weights(wd))
    assert hs.shape == (n, Hp // 32)
    r = O.bf16_bits_to_f64(y_bf16)
    rel = np.linalg.norm(O.bf16_bits_to_f64(y_mx) - r) / np.linalg.norm(r)
    assert 1e-2 < rel < 0.2, rel
    # the band alone would also pass an expert that skips the quantisation of h or of x;
    # on these inputs both variants give outputs that differ from the oracle's
    xq = O.mx_dequantize(*O.mx_quantize(O.bf16_bits_to_f64(x)))
    wgd, wud, wdd = (O.mx_dequantize(*O.mx_weights(w), axis=-2) for w in (wg, wu, wd))
    y_no_h = O.f64_to_bf16_bits((O.silu(xq @ wgd) * (xq @ wud)) @ wdd)
    xr = O.bf16_bits_to_f64(x)
    h_no_x = O.mx_dequantize(*O.mx_quantize(O.silu(xr @ wgd) * (xr @ wud)))
    y_no_x = O.f64_to_bf16_bits(h_no_x @ wdd)
    for variant in (y_no_h, y_no_x):
        assert (variant != y_mx).mean() > 0.5


def test_mxfp8_expert_exact_hand_case():
    """One token, H = H' = 32 (one MXFP8 block per row and column), every value worked out by
    hand. Each quantisation step of the MXFP8 expert changes at least one output, so dropping
    any of them (x, the up/gate weights, h, the down weights) or quantising a weight along the
    wrong axis fails this pin.

    x = [2, 1.0625, 0, ...]: amax 2 gives scale 2^(1-8); x*128 = [256, 136] and 136 is a tie
    in the [128, 256) binade (step 16), so x dequantises to [2, 1].
    W_gate[0, :] = 64 (on the grid) gives g = 128 for every feature, where
    1 + e^-128 == 1 in float64, so silu(g) = g exactly and h_j = 128 * u_j.
    W_up rows 0 and 1 hold (a_j, b_j), on the grid of their column's block except a_9 = 1.0625
    (amax 1.0625, scale 2^-8: 272 is a tie, kept 256, so a_9 becomes 1.0); u_j = 2 a_j + b_j.
    h = 128 u = [448, 264, 272, 304, 288, 144, 136, 68, 2.5 * 2^-9, 264] has amax 448, so
    scale 1 and E4M3 codes [448 (max), 256 (nearest), 256 (tie, even below), 320 (tie, even
    above), 288, 144, 128 (tie), 64 (tie), 2^-8 (subnormal tie), 256].
    W_down is the identity on features 0..9, so y_j is h's code; column 31 holds 2 at row 10
    (h_10 = 0) and 1.25 * 2^-15 at row 0: its block's scale is 2^(1-8), the entry scales to
    2.5 * 2^-9, a subnormal tie rounded to 2 * 2^-9, so y_31 = 448 * 2^-15.
    """
    H = Hp = 32
    x = np.zeros((1, H))
    x[0, :2] = (2.0, 1.0625)
    wg = np.zeros((H, Hp))
    wg[0, :] = 64.0
    a = [1.5, 1.0, 0.5625, 1.125, 1.0, 0.5, 0.5, 0.25, 1.25 * 2 ** -16, 1.0625]
    b = [0.5, 0.0625, 1.0, 0.125, 0.25, 0.125, 0.0625, 0.03125, 0.0, 0.0625]
    wu = np.zeros((H, Hp))
    wu[0, :10], wu[1, :10] = a, b
    wd = np.zeros((Hp, H))
    wd[np.arange(10), np.arange(10)] = 1.0
    wd[0, 31], wd[10, 31] = 1.25 * 2 ** -15, 2.0
    bits = {k: O.f64_to_bf16_bits(v) for k, v in (("x", x), ("wg", wg), ("wu", wu), ("wd", wd))}
    for k, v in (("x", x), ("wg", wg), ("wu", wu), ("wd", wd)):
        np.testing.assert_array_equal(O.bf16_bits_to_f64(bits[k]), v)  # inputs are bf16 values

    codes = np.zeros(Hp)
    codes[:10] = [448, 256, 256, 320, 288, 144, 128, 64, 2.0 ** -8, 256]
    y_want = np.zeros(H)
    y_want[:10] = codes[:10]
    y_want[31] = 448 * 2.0 ** -15

    xq, xs = O.mx_quantize(O.bf16_bits_to_f64(bits["x"]))
    np.testing.assert_array_equal(xq[0, :3], [256.0, 128.0, 0.0])
    assert xs[0, 0] == -7
    hq, hs, y = O.expert_ffn_rows_mxfp8(bits["x"], O.mx_weights(bits["wg"]),
                                        O.mx_weights(bits["wu"]), O.mx_weights(bits["wd"]))
    np.testing.assert_array_equal(hq[0], codes)
    assert hs.shape == (1, 1) and hs[0, 0] == 0
    np.testing.assert_array_equal(O.bf16_bits_to_f64(y)[0], y_want)

    # what each dropped step would give instead (worked out by hand from the values above)
    no_x_quant = 128 * (2 * 0.5625 + 1.0625 * 1.0)       # h_2 = 280 -> code 288, not 256
    no_h_quant = 264.0                                     # y_1 = bf16(264) = 264, not 256
    no_up_weight_quant = 128 * (2 * 1.0625 + 0.0625)      # h_9 = 280 -> code 288, not 256
    no_down_weight_quant = 448 * 1.25 * 2.0 ** -15        # also the row-wise (wrong axis) value
    assert O.e4m3_round(np.array([no_x_quant]))[0] == 288 != y_want[2]
    assert no_h_quant != y_want[1]
    assert O.e4m3_round(np.array([no_up_weight_quant]))[0] == 288 != y_want[9]
    assert no_down_weight_quant != y_want[31]
    row_wise = O.mx_quantize(O.bf16_bits_to_f64(bits["wd"]), axis=-1)  # wrong axis for Down
    assert O.mx_dequantize(*row_wise, axis=-1)[0, 31] == 1.25 * 2 ** -15


def test_mx_scale_exponent_just_below_a_power_of_two():
    """The block scale is 2^(floor(log2 amax) - 8) with the floor taken exactly (OCP MX v1.0,
    MXFP8): a block maximum one double ulp below 2^8 has floor(log2 amax) = 7, so its scale
    exponent is -1; the scaled maximum (256 - ulp) * 2 then lies above 448 and saturates to
    448, and an element 1.0 becomes 2.0. A maximum of exactly 2^8 gives exponent 0."""
    x = np.zeros((1, 32))
    x[0, 0] = np.nextafter(256.0, 0.0)
    x[0, 1] = 1.0
    q, s = O.mx_quantize(x, axis=-1)
    assert s[0, 0] == -1
    assert q[0, 0] == 448.0 and q[0, 1] == 2.0
    # exactly 2^8 gives exponent 0 and the element 256
    x[0, 0] = 256.0
    q, s = O.mx_quantize(x, axis=-1)
    assert s[0, 0] == 0 and q[0, 0] == 256.0
