"""Routing-generator unit tests (Mooncake RFC "CI Strategy": unit tests for
routing distribution generation; "Validation": routing-load distribution).

The counting below uses numpy directly; it tests the generator, not the
method."""

import numpy as np
import pytest

from workloads import CONFIGS, RoutingSpec, make_routing, make_weights, make_workload, seed_streams


def _rng(seed=0):
    return np.random.Generator(np.random.PCG64(seed))


@pytest.mark.parametrize("name", list(CONFIGS))
def test_ids_distinct_in_range_and_seeded(name):
    w = CONFIGS[name].scaled(min(CONFIGS[name].T, 2048))
    ids1, wt1, _, _ = make_workload(w, with_x=False, with_y=False)
    ids2, wt2, _, _ = make_workload(w, with_x=False, with_y=False)
    assert ids1.dtype == np.int32 and ids1.shape == (w.T, w.k)
    assert ids1.min() >= 0 and ids1.max() < w.E
    srt = np.sort(ids1, axis=1)
    assert (np.diff(srt, axis=1) > 0).all(), "experts must be distinct within a token"
    np.testing.assert_array_equal(ids1, ids2)
    np.testing.assert_array_equal(wt1, wt2)
    assert wt1.dtype == np.float32
    assert np.allclose(wt1.sum(axis=1), 1.0, atol=1e-6)
    assert (wt1 > 0).all()


def test_uniform_marginal_is_flat():
    T, E, k = 20000, 64, 4
    ids = make_routing(T, E, k, RoutingSpec("uniform"), _rng(1))
    c = np.bincount(ids.ravel(), minlength=E)
    expect = T * k / E
    # 6 sigma band of a binomial count
    assert np.abs(c - expect).max() < 6 * np.sqrt(expect)


def test_khot_fraction():
    T, E, k, h = 20000, 256, 8, 8
    ids = make_routing(T, E, k, RoutingSpec("khot", hot_experts=h, hot_fraction=0.9), _rng(2))
    hot = ids < h
    # Every slot draws hot with probability 0.9 and the hot pool never runs
    # dry while k <= h, so the per-slot hot fraction is 0.9.
    frac = hot.mean(axis=0)
    assert np.all(np.abs(frac - 0.9) < 0.01), frac
    assert set(np.unique(ids[hot]).tolist()) == set(range(h))


def test_khot_pool_exhaustion_draws_from_other_pool():
    # hot set of 2 and k = 4: at least 2 slots per token must be cold.
    ids = make_routing(5000, 16, 4, RoutingSpec("khot", hot_experts=2, hot_fraction=1.0), _rng(3))
    assert ((ids < 2).sum(axis=1) == 2).all()
    assert (np.diff(np.sort(ids, axis=1), axis=1) > 0).all()


def test_zipf_rank_frequency_slope():
    # With k = 1 the marginal is the Zipf law itself: log count vs log rank
    # has slope -s.
    T, E, s = 200000, 64, 1.2
    ids = make_routing(T, E, 1, RoutingSpec("zipf", zipf_s=s), _rng(4))
    c = np.sort(np.bincount(ids.ravel(), minlength=E))[::-1].astype(np.float64)
    r = np.arange(1, E + 1)
    top = c > 200
    slope = np.polyfit(np.log(r[top]), np.log(c[top]), 1)[0]
    assert abs(slope + s) < 0.1, slope


def test_zipf_popularity_follows_seeded_permutation():
    w = CONFIGS["zipf_fp8_t16384_h4096_e288_k8"].scaled(4096)
    ids, _, _, _ = make_workload(w, with_x=False, with_y=False)
    s_ids = seed_streams(w.seed)[0]
    perm = np.random.Generator(np.random.PCG64(s_ids)).permutation(w.E)
    c = np.bincount(ids.ravel(), minlength=w.E)
    # the most popular expert is rank 1 of the permutation
    assert c.argmax() == perm[0]


def test_weights_softmax_of_chosen_logits():
    w = make_weights(100, 6, _rng(5))
    logits = _rng(5).standard_normal(size=(100, 6))
    ref = np.exp(logits) / np.exp(logits).sum(axis=1, keepdims=True)
    np.testing.assert_allclose(w, ref, rtol=1e-6)


def test_activations_are_seeded_and_rounded():
    import torch
    w = CONFIGS["tiny_t32_h4096_e256_k8"]
    _, _, x1, y1 = make_workload(w)
    _, _, x2, y2 = make_workload(w)
    assert x1.dtype == torch.bfloat16 and x1.shape == (w.T, w.H)
    assert y1.shape == (w.S, w.H)
    assert torch.equal(x1, x2) and torch.equal(y1, y2)
    assert abs(float(x1.float().std()) - 1.0) < 0.05
