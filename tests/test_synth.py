"""The seeded input generator (host side, no GPU): its draws are deterministic and
counter-based, its distributions are what the measurement recipe states, and each workload's
routing reaches the imbalance it is named for (measured with the oracle's maxvio)."""
import numpy as np
import pytest

import synth
from oracle import moe_oracle as O


def test_draws_are_counter_based_and_deterministic():
    a = synth.uniform(3, 7, 1000)
    assert np.array_equal(a, synth.uniform(3, 7, 1000))
    # draw i does not depend on how many draws precede it in the call
    assert np.array_equal(synth.uniform(3, 7, 500, offset=500), a[500:])
    assert not np.array_equal(a, synth.uniform(3, 8, 1000))  # another tag, another stream
    assert not np.array_equal(a, synth.uniform(4, 7, 1000))  # another seed
    assert (a > 0).all() and (a < 1).all()


def test_normals_and_bf16_rounding():
    z = synth.normal_f64(1, 2, 200000)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1.0) < 0.01
    b = synth.normal_bf16_bits(1, 2, 200000, scale=0.5)
    # the recipe: scaled in double, rounded to float (nearest), then to bf16 (nearest even)
    f32 = (z * 0.5).astype(np.float32).astype(np.float64)
    assert np.array_equal(b, O.f64_to_bf16_bits(f32))


def test_route_weights_are_a_softmax_per_token():
    w = synth.route_weights(5, 1000, 8)
    assert w.dtype == np.float32 and (w > 0).all()
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-6)


@pytest.mark.parametrize("name,target", [("large", 0.1953125), ("skew1", 0.998046875),
                                         ("skew10", 9.998046875), ("skew20", 20.0),
                                         ("skew20_last", 20.0)])
def test_capped_routings_reach_their_maxvio(name, target):
    w = synth.WORKLOADS[name]
    ids, rw = synth.routing_for(w)
    assert ids.shape == (w.S, w.K) and rw.shape == (w.S, w.K)
    assert ids.min() >= 0 and ids.max() < w.E
    # a token's K experts are distinct (top-K keys without replacement)
    s = np.sort(ids, axis=1)
    assert (s[:, 1:] != s[:, :-1]).all()
    counts = np.bincount(ids.reshape(-1), minlength=w.E)
    mv, mc = O.maxvio(counts, w.S, w.K)
    assert mv == target
    hot = w.hot_e
    assert counts[hot] == mc  # the hot expert is the one at the cap
    assert np.array_equal(ids, synth.routing_for(w)[0])  # deterministic


def test_balanced_routing_is_as_even_as_possible():
    w = synth.WORKLOADS["permute_combine_S1024_mv0"]
    ids, _ = synth.routing_for(w)
    counts = np.bincount(ids.reshape(-1), minlength=w.E)
    assert counts.max() - counts.min() <= 1
    s = np.sort(ids, axis=1)
    assert (s[:, 1:] != s[:, :-1]).all()  # K <= E keeps a token's experts distinct
