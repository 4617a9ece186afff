"""Pins for the oracle's router step (softmax + top-k).

Megatron MoE page, MoELayer.router_and_preprocess: the router yields probs
and a top-k routing map; Megatron MORI page, router.py: padding tokens are
masked out of routing. Reading: softmax over all E experts (no
renormalisation), descending order, equal logits to the lower id.
"""

import math

import numpy as np
import pytest
import scipy.special

from synthetic import get_workload, make_inputs

pytestmark = []


def _rand_logits(seed, N, E, integer=False):
    rng = np.random.default_rng(seed)
    if integer:  # many exact ties
        return rng.integers(-3, 4, size=(N, E)).astype(np.float32)
    return rng.standard_normal((N, E)).astype(np.float32)


@pytest.mark.parametrize("E,k", [(8, 2), (16, 4), (64, 8), (256, 8), (5, 5)])
@pytest.mark.parametrize("integer", [False, True])
def test_ids_match_full_sort(oracle_lib, E, k, integer):
    logits = _rand_logits(E * 31 + k, 64, E, integer)
    idx, _ = oracle_lib.route_topk(logits, k)
    for t in range(logits.shape[0]):
        # a different method: a full stable sort on (-logit, id)
        expect = sorted(range(E), key=lambda e: (-float(logits[t, e]), e))[:k]
        assert idx[t].tolist() == expect


@pytest.mark.parametrize("E,k", [(8, 2), (64, 8), (256, 8)])
def test_probs_match_library_softmax(oracle_lib, E, k):
    logits = _rand_logits(E + k, 128, E) * 3.0
    idx, probs = oracle_lib.route_topk(logits, k)
    ref = scipy.special.softmax(logits.astype(np.float64), axis=1)
    picked = np.take_along_axis(ref, idx.astype(np.int64), axis=1)
    # the oracle rounds the double softmax once to float32: within one float32 ulp
    assert np.all(np.abs(probs.astype(np.float64) - picked) <= 2.0 ** -23 * picked + 1e-45)


def test_two_expert_logistic_closed_form(oracle_lib):
    rng = np.random.default_rng(7)
    logits = rng.uniform(-8, 8, size=(200, 2)).astype(np.float32)
    idx, probs = oracle_lib.route_topk(logits, 2)
    for t in range(200):
        l0, l1 = float(logits[t, 0]), float(logits[t, 1])
        p0 = 1.0 / (1.0 + math.exp(l1 - l0))
        got = dict(zip(idx[t].tolist(), probs[t].tolist()))
        assert abs(got[0] - p0) <= 2.0 ** -23 * p0
        assert abs(got[1] - (1.0 - p0)) <= 2.0 ** -23 * (1.0 - p0) + 1e-12


def test_uniform_logits_give_exact_reciprocal(oracle_lib):
    for E in (2, 8, 64, 256):
        logits = np.full((3, E), 0.75, np.float32)
        idx, probs = oracle_lib.route_topk(logits, min(8, E))
        assert np.all(probs == np.float32(1.0 / E))
        assert idx[0].tolist() == list(range(min(8, E)))  # all tied: ascending ids


def test_full_k_sums_to_one_and_is_sorted(oracle_lib):
    logits = _rand_logits(3, 50, 32)
    idx, probs = oracle_lib.route_topk(logits, 32)
    assert np.all(np.abs(probs.astype(np.float64).sum(1) - 1.0) <= 32 * 2.0 ** -24)
    assert np.all(np.diff(probs, axis=1) <= 0)
    assert all(sorted(r) == list(range(32)) for r in idx.tolist())


def test_shift_invariance(oracle_lib):
    logits = _rand_logits(11, 40, 64)
    i0, p0 = oracle_lib.route_topk(logits, 8)
    i1, p1 = oracle_lib.route_topk(logits + np.float32(16.0), 8)
    assert np.array_equal(i0, i1)
    assert np.allclose(p0, p1, rtol=1e-5, atol=0)


def test_masked_tokens(oracle_lib):
    logits = _rand_logits(5, 10, 16)
    mask = np.array([0, 1, 0, 0, 1, 1, 0, 0, 0, 1], np.uint8)
    idx, probs = oracle_lib.route_topk(logits, 4, token_mask=mask)
    idx0, probs0 = oracle_lib.route_topk(logits, 4)
    for t in range(10):
        if mask[t]:
            assert idx[t].tolist() == [-1] * 4 and probs[t].tolist() == [0.0] * 4
        else:
            assert np.array_equal(idx[t], idx0[t]) and np.array_equal(probs[t], probs0[t])


def test_workload_route_is_distinct_and_skewed(oracle_lib):
    w = get_workload("tiny")
    d = make_inputs(w, hidden=False)
    idx, probs = oracle_lib.route_topk(d["logits"], w.k)
    assert all(len(set(r)) == w.k for r in idx.tolist())
    assert np.all((probs > 0) & (probs <= 1))
