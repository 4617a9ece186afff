"""Pins for the oracle's permute, combine and their backward passes.

Permute is a byte copy (Megatron MoE page, dispatch_postprocess; Megatron MORI
page, fused permute, tails masked with 0). Combine is the prob-weighted
gather-reduce added back one top-k slot at a time in ascending order (DeepSpeed
EP page, restore_combined), with fp32 accumulation and one rounding to bf16.

Pins used: numpy fancy indexing for the copy; the identity-expert round trip;
hand-built cases whose bf16 result flips if the slot order, the single final
rounding or the fused multiply-add were different; an fp64 sum within the
standard summation error bound; the adjoint identity <combine(Y), G> =
<Y, combine_backward(G)>; closed forms k*h for the permute backward.
"""

import numpy as np
import pytest

from synthetic import bf16_bits_from_f32, f32_from_bf16_bits, get_workload, make_inputs


def _rand_problem(oracle_lib, seed, N=64, H=24, k=4, E=8, R=2, C=0, neg=0.0):
    rng = np.random.default_rng(seed)
    idx = (rng.zipf(1.5, size=(N, k)) % E).astype(np.int32)
    idx[rng.random((N, k)) < neg] = -1
    probs = rng.random((N, k)).astype(np.float32)
    hidden = bf16_bits_from_f32(rng.standard_normal((N, H)).astype(np.float32))
    L = oracle_lib.layout(idx, probs, E_log=E, R=R, C=C)
    return idx, probs, hidden, L


@pytest.mark.parametrize("C,neg", [(0, 0.0), (0, 0.2), (20, 0.0), (9, 0.1)])
def test_permute_is_row_copy_with_zero_pads(oracle_lib, C, neg):
    idx, probs, hidden, L = _rand_problem(oracle_lib, C + int(neg * 10), C=C, neg=neg)
    send = oracle_lib.permute(hidden, L["dest_row"], L["rows_max"])
    dest = L["dest_row"]
    t, j = np.nonzero(dest >= 0)
    assert np.array_equal(send[dest[t, j]], hidden[t])
    assert np.all(send[L["pad_mask"].astype(bool)] == 0)
    # and the inverse map says the same thing
    rows = np.nonzero(L["row_token"] >= 0)[0]
    assert np.array_equal(send[rows], hidden[L["row_token"][rows]])


@pytest.mark.parametrize("k", [2, 8])
def test_identity_round_trip_with_reciprocal_probs(oracle_lib, k):
    rng = np.random.default_rng(k)
    N, H, E = 50, 40, 16
    idx = np.stack([rng.permutation(E)[:k] for _ in range(N)]).astype(np.int32)
    probs = np.full((N, k), 1.0 / k, np.float32)
    hidden = bf16_bits_from_f32(rng.standard_normal((N, H)).astype(np.float32))
    L = oracle_lib.layout(idx, probs, E_log=E, R=4)
    send = oracle_lib.permute(hidden, L["dest_row"], L["rows_max"])
    out = oracle_lib.combine(send, L["dest_row"], probs)
    assert np.array_equal(out, hidden)


def test_identity_round_trip_one_hot(oracle_lib):
    idx, probs, hidden, L = _rand_problem(oracle_lib, 3)
    one_hot = np.zeros_like(probs)
    one_hot[:, 0] = 1.0
    send = oracle_lib.permute(hidden, L["dest_row"], L["rows_max"])
    out = oracle_lib.combine(send, L["dest_row"], one_hot)
    assert np.array_equal(out, hidden)


def test_drops_scale_by_kept_fraction(oracle_lib):
    rng = np.random.default_rng(5)
    N, H, E, k, C = 200, 16, 4, 8, 150
    idx = np.stack([rng.integers(0, E, size=k) for _ in range(N)]).astype(np.int32)
    probs = np.full((N, k), 0.125, np.float32)
    hidden = bf16_bits_from_f32(rng.standard_normal((N, H)).astype(np.float32))
    L = oracle_lib.layout(idx, probs, E_log=E, R=2, C=C)
    assert L["counters"][2] > 0
    send = oracle_lib.permute(hidden, L["dest_row"], L["rows_max"])
    out = oracle_lib.combine(send, L["dest_row"], probs)
    kept = (L["dest_row"] >= 0).sum(1)
    exact = kept[:, None] / 8.0 * f32_from_bf16_bits(hidden).astype(np.float64)  # exact in double and float
    exact = exact + 0.0  # the accumulator starts at +0, so a token with no kept slot gives +0, never -0
    assert np.array_equal(out, bf16_bits_from_f32(exact.astype(np.float32)))


def _bits(x):
    return int(bf16_bits_from_f32(np.array([x], np.float32))[0])


def test_slot_order_and_single_rounding_are_pinned(oracle_lib):
    # y = 1 in three rows; p = [1 + 2^-8, 2^-24, 2^-24].
    # Ascending slots in fp32: 1+2^-8, then +2^-24 twice rounds back (ties to even) -> 1+2^-8,
    # which is a bf16 tie and rounds to 1.0. Descending order (or an fp64 sum) reaches
    # 1 + 2^-8 + 2^-23, which rounds up to 1 + 2^-7.
    one = _bits(1.0)
    y = np.array([[one], [one], [one]], np.uint16)
    dest = np.array([[0, 1, 2]], np.int32)
    p = np.array([[1 + 2.0 ** -8, 2.0 ** -24, 2.0 ** -24]], np.float32)
    out = oracle_lib.combine(y, dest, p)
    assert out[0, 0] == _bits(1.0)
    assert out[0, 0] != _bits(1 + 2.0 ** -7)
    out_rev = oracle_lib.combine(y[::-1].copy(), dest, p[:, ::-1].copy())
    assert out_rev[0, 0] == _bits(1 + 2.0 ** -7)


def test_fused_multiply_add_is_pinned(oracle_lib):
    # slot 0: -1 * (1 + 2^-7); slot 1: (1 + 2^-23) * (1 + 2^-7).
    # With one rounding per fma the result is 2^-23 + 2^-30 = 2^-23 (1 + 2^-7), exact in bf16;
    # a separately rounded product would lose 2^-30 and give 2^-23.
    yv = _bits(1 + 2.0 ** -7)
    y = np.array([[yv], [yv]], np.uint16)
    dest = np.array([[0, 1]], np.int32)
    p = np.array([[-1.0, 1 + 2.0 ** -23]], np.float32)
    out = oracle_lib.combine(y, dest, p)
    assert out[0, 0] == _bits(2.0 ** -23 * (1 + 2.0 ** -7))
    assert out[0, 0] != _bits(2.0 ** -23)


@pytest.mark.parametrize("seed", range(3))
def test_combine_within_fp64_error_bound(oracle_lib, seed):
    idx, probs, hidden, L = _rand_problem(oracle_lib, 10 + seed, N=128, H=64, k=8, E=16, neg=0.05)
    rng = np.random.default_rng(seed)
    Y = bf16_bits_from_f32(rng.standard_normal((L["rows_max"], 64)).astype(np.float32))
    out = f32_from_bf16_bits(oracle_lib.combine(Y, L["dest_row"], probs)).astype(np.float64)
    Yf = f32_from_bf16_bits(Y).astype(np.float64)
    dest = L["dest_row"]
    w = np.where(dest >= 0, probs, 0.0).astype(np.float64)
    g = Yf[np.maximum(dest, 0)]  # [N,k,H]
    exact = np.einsum("nk,nkh->nh", w, g)
    S = np.einsum("nk,nkh->nh", np.abs(w), np.abs(g))
    u = 2.0 ** -24
    gamma = 8 * u / (1 - 8 * u)
    bound = gamma * S + 2.0 ** -8 * (np.abs(exact) + gamma * S) + 1e-38
    assert np.all(np.abs(out - exact) <= bound)


def test_prob_scaling_by_two_is_exact(oracle_lib):
    idx, probs, hidden, L = _rand_problem(oracle_lib, 21, N=40, H=32)
    send = oracle_lib.permute(hidden, L["dest_row"], L["rows_max"])
    o1 = f32_from_bf16_bits(oracle_lib.combine(send, L["dest_row"], probs))
    o2 = f32_from_bf16_bits(oracle_lib.combine(send, L["dest_row"], probs * np.float32(2.0)))
    assert np.array_equal(o2, o1 * 2)


def test_unit_weights_equal_permute_backward(oracle_lib):
    idx, probs, hidden, L = _rand_problem(oracle_lib, 8, N=70, H=16, C=30, neg=0.1)
    rng = np.random.default_rng(0)
    G = bf16_bits_from_f32(rng.standard_normal((L["rows_max"], 16)).astype(np.float32))
    assert np.array_equal(oracle_lib.combine(G, L["dest_row"], None), oracle_lib.permute_backward(G, L["dest_row"]))


@pytest.mark.parametrize("k,C", [(8, 0), (2, 0), (3, 0), (8, 40)])
def test_permute_backward_closed_form(oracle_lib, k, C):
    rng = np.random.default_rng(k + C)
    N, H, E = 60, 32, 8
    idx = np.stack([rng.integers(0, E, size=k) for _ in range(N)]).astype(np.int32)
    hidden = bf16_bits_from_f32(rng.standard_normal((N, H)).astype(np.float32))
    L = oracle_lib.layout(idx, None, E_log=E, R=2, C=C)
    send = oracle_lib.permute(hidden, L["dest_row"], L["rows_max"])
    gh = oracle_lib.permute_backward(send, L["dest_row"])
    kept = (L["dest_row"] >= 0).sum(1).astype(np.float64)
    exact = kept[:, None] * f32_from_bf16_bits(hidden).astype(np.float64) + 0.0  # m*h is exact in fp32 for m <= 8
    assert np.array_equal(gh, bf16_bits_from_f32(exact.astype(np.float32)))


@pytest.mark.parametrize("C,neg", [(0, 0.0), (12, 0.1)])
def test_combine_backward_adjoint(oracle_lib, C, neg):
    rng = np.random.default_rng(99 + C)
    N, H, k, E = 48, 32, 4, 8
    idx = (rng.zipf(1.5, size=(N, k)) % E).astype(np.int32)
    idx[rng.random((N, k)) < neg] = -1
    probs = (2.0 ** -rng.integers(0, 4, size=(N, k))).astype(np.float32)  # powers of two: d_Y exact
    L = oracle_lib.layout(idx, probs, E_log=E, R=2, C=C)
    RM = L["rows_max"]
    Y = bf16_bits_from_f32(rng.standard_normal((RM, H)).astype(np.float32))
    G = bf16_bits_from_f32(rng.standard_normal((N, H)).astype(np.float32))
    gY, gp = oracle_lib.combine_backward(G, Y, L["dest_row"], L["row_token"], L["row_prob"])
    Yf = f32_from_bf16_bits(Y).astype(np.float64)
    Gf = f32_from_bf16_bits(G).astype(np.float64)
    dest = L["dest_row"]
    w = np.where(dest >= 0, probs, 0.0).astype(np.float64)
    comb = np.einsum("nk,nkh->nh", w, Yf[np.maximum(dest, 0)])
    lhs = float((comb * Gf).sum())
    rhs = float((Yf * f32_from_bf16_bits(gY).astype(np.float64)).sum())
    assert abs(lhs - rhs) <= 1e-9 * (np.abs(comb * Gf).sum() + 1)
    assert np.all(gY[L["pad_mask"].astype(bool)] == 0)
    # grad_probs: a different summation (numpy einsum) within the double-sum bound
    ref = np.einsum("nh,nkh->nk", Gf, Yf[np.maximum(dest, 0)])
    ref = np.where(dest >= 0, ref, 0.0)
    S = np.einsum("nh,nkh->nk", np.abs(Gf), np.abs(Yf[np.maximum(dest, 0)]))
    assert np.all(np.abs(gp.astype(np.float64) - ref) <= H * 2.0 ** -52 * S + 2.0 ** -24 * np.abs(ref) + 1e-38)
    assert np.all(gp[dest < 0] == 0)


def test_combine_backward_dY_single_rounding(oracle_lib):
    # p = 1/3 (fp32) times g = 1.5: the fp32 product rounds once, then bf16 rounds once.
    p = np.float32(1.0 / 3.0)
    G = bf16_bits_from_f32(np.array([[1.5]], np.float32))
    Y = np.zeros((1, 1), np.uint16)
    gY, _ = oracle_lib.combine_backward(G, Y, np.array([[0]], np.int32), np.array([0], np.int32),
                                        np.array([p], np.float32))
    prod32 = np.float32(p) * np.float32(1.5)
    assert gY[0, 0] == bf16_bits_from_f32(np.array([prod32], np.float32))[0]


def test_workload_tiny_full_path(oracle_lib):
    w = get_workload("tiny")
    d = make_inputs(w)
    idx, probs = oracle_lib.route_topk(d["logits"], w.k)
    L = oracle_lib.layout(idx, probs, E_log=w.E_log, R=w.R)
    send = oracle_lib.permute(d["hidden"], L["dest_row"], L["rows_max"])
    out = oracle_lib.combine(send, L["dest_row"], probs)
    # every token keeps both slots, so out = bf16(p0*h + p1*h) within the bound of two terms
    h = f32_from_bf16_bits(d["hidden"]).astype(np.float64)
    exact = probs.astype(np.float64).sum(1)[:, None] * h
    got = f32_from_bf16_bits(out).astype(np.float64)
    assert np.all(np.abs(got - exact) <= 2.0 ** -8 * np.abs(exact) * 1.001 + 1e-38)
