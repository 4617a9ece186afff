"""Pins for the oracle's DeepEP-style token-dedup view and two-level combine.

Megatron MORI page: the dispatcher follows the DeepEP contract (each token sent
once per destination rank; receiver-side local top-k ids with -1 sentinels and
receiver-side weights; _indices_to_multihot makes a [tokens, local experts]
routing map with probs). Pinned against: a hand-worked example; numpy counts;
the main layout's per-rank local view (a different computation of the same
ids); the multihot definition; the two-stage dispatch reproducing the
one-stage permute; a closed form of the two-level combine; and R = 1, where it
must equal the one-level combine.
"""

import numpy as np
import pytest

from synthetic import bf16_bits_from_f32, f32_from_bf16_bits


def _case(seed, N=257, k=4, E=16, R=4, C=0, neg=0.05):
    rng = np.random.default_rng(seed)
    idx = (rng.zipf(1.3, size=(N, k)) % E).astype(np.int32)
    idx[rng.random((N, k)) < neg] = -1
    probs = rng.random((N, k)).astype(np.float32)
    hidden = bf16_bits_from_f32(rng.standard_normal((N, 32)).astype(np.float32))
    return idx, probs, hidden


def test_dedup_worked_by_hand(oracle_lib):
    # experts 0,1 on rank 0 and 2,3 on rank 1; every token has one slot on each rank
    idx = np.array([[3, 0], [0, 2], [3, 1]], np.int32)
    w = np.array([[0.5, 0.25], [0.125, 1.0], [2.0, 4.0]], np.float32)
    L = oracle_lib.layout(idx, w, E_log=4, R=2)
    D = oracle_lib.dedup_layout(L, w, E_log=4, R=2)
    assert D["num_tokens_per_rank"].tolist() == [3, 3]
    assert D["token_rank_row"].tolist() == [[0, 3], [1, 4], [2, 5]]
    assert D["recv_src_token"].tolist() == [0, 1, 2, 0, 1, 2]
    assert D["recv_topk_idx"].tolist() == [[-1, 0], [0, -1], [-1, 1], [1, -1], [-1, 0], [1, -1]]
    assert D["recv_topk_weights"].tolist() == [[0, 0.25], [0.125, 0], [0, 4.0], [0.5, 0], [0, 1.0], [2.0, 0]]
    assert D["recv_routing_map"].tolist() == [[1, 0], [1, 0], [0, 1], [0, 1], [1, 0], [0, 1]]
    assert D["recv_probs"].tolist() == [[0.25, 0], [0.125, 0], [0, 4.0], [0, 0.5], [1.0, 0], [0, 2.0]]


@pytest.mark.parametrize("R,C,reps", [(4, 0, 0), (2, 20, 0), (8, 0, 8), (1, 0, 0)])
def test_dedup_invariants(oracle_lib, R, C, reps):
    E = 16
    idx, probs, hidden = _case(R * 7 + C, R=R, C=C)
    L = oracle_lib.layout(idx, probs, E_log=E, R=R, C=C, num_replicas=reps)
    D = oracle_lib.dedup_layout(L, probs, E_log=E, R=R, num_replicas=reps)
    N, k = idx.shape
    E_loc = (E + reps) // R
    kept = L["dest_row"] >= 0
    rank = np.where(kept, L["phys_idx"] // E_loc, -1)
    in_rank = np.stack([(rank == r).any(1) for r in range(R)], 1)
    assert np.array_equal(D["is_token_in_rank"].astype(bool), in_rank)
    assert np.array_equal(D["num_tokens_per_rank"], in_rank.sum(0))
    assert D["recv_max"] == N * min(k, R)
    rows = D["token_rank_row"]
    for r in range(R):
        t_r = np.nonzero(in_rank[:, r])[0]
        # rank-major, token-ascending rows
        assert np.array_equal(rows[t_r, r], D["recv_rank_offsets"][r] + np.arange(len(t_r)))
        assert np.array_equal(D["recv_src_token"][rows[t_r, r]], t_r)
        # the main layout's per-rank local view gives the same local ids
        assert np.array_equal(D["recv_topk_idx"][rows[t_r, r]], L["local_topk"][r][t_r])
    assert np.all(rows[~in_rank] == -1)
    real = np.zeros(D["recv_max"], bool)
    real[: D["num_recv"][0]] = True
    assert np.array_equal(D["recv_pad_mask"].astype(bool), ~real)
    # _indices_to_multihot
    ids = D["recv_topk_idx"]
    mh = np.zeros((D["recv_max"], E_loc), np.uint8)
    pr = np.zeros((D["recv_max"], E_loc), np.float32)
    for j in range(k):
        m = ids[:, j] >= 0
        mh[np.nonzero(m)[0], ids[m, j]] = 1
        pr[np.nonzero(m)[0], ids[m, j]] = D["recv_topk_weights"][m, j]
    assert np.array_equal(D["recv_routing_map"], mh)
    assert np.array_equal(D["recv_probs"], pr)
    assert np.all(D["recv_topk_weights"][ids < 0] == 0)
    # two-stage dispatch (token once per rank, then the local permute) = the one-stage permute
    recv_x = oracle_lib.permute(hidden, rows, D["recv_max"])
    send = oracle_lib.permute(hidden, L["dest_row"], L["rows_max"])
    t, j = np.nonzero(kept)
    assert np.array_equal(recv_x[rows[t, rank[t, j]]], send[L["dest_row"][t, j]])


@pytest.mark.parametrize("R", [2, 4, 8])
def test_two_level_combine_closed_form(oracle_lib, R):
    E = 16
    rng = np.random.default_rng(R)
    N, k = 200, 8
    idx = np.stack([rng.permutation(E)[:k] for _ in range(N)]).astype(np.int32)
    probs = np.full((N, k), 0.125, np.float32)
    hidden = bf16_bits_from_f32(rng.standard_normal((N, 32)).astype(np.float32))
    L = oracle_lib.layout(idx, probs, E_log=E, R=R)
    D = oracle_lib.dedup_layout(L, probs, E_log=E, R=R)
    send = oracle_lib.permute(hidden, L["dest_row"], L["rows_max"])
    partial = oracle_lib.dedup_combine_local(send, L, D, probs, R)
    out = oracle_lib.combine(partial, D["token_rank_row"], None)
    # closed form: out = bf16( sum_r bf16( m_r / 8 * h ) ), m_r = slots of t on rank r;
    # every fp32 sum here is exact (equal h, <= 8 terms within 3 binades)
    E_loc = E // R
    m = np.stack([((L["phys_idx"] // E_loc) == r).sum(1) for r in range(R)], 1)
    h = f32_from_bf16_bits(hidden).astype(np.float64)
    parts = [f32_from_bf16_bits(bf16_bits_from_f32((m[:, r:r + 1] / 8.0 * h).astype(np.float32))).astype(np.float64)
             for r in range(R)]
    expect = bf16_bits_from_f32((sum(parts) + 0.0).astype(np.float32))
    assert np.array_equal(out, expect)


def test_single_rank_dedup_equals_combine(oracle_lib):
    idx, probs, hidden = _case(3, R=1)
    L = oracle_lib.layout(idx, probs, E_log=16, R=1)
    D = oracle_lib.dedup_layout(L, probs, E_log=16, R=1)
    send = oracle_lib.permute(hidden, L["dest_row"], L["rows_max"])
    partial = oracle_lib.dedup_combine_local(send, L, D, probs, 1)
    out = oracle_lib.combine(partial, D["token_rank_row"], None)
    assert np.array_equal(out, oracle_lib.combine(send, L["dest_row"], probs))
