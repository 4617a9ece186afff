"""Pins for the oracle's dispatch layout.

What fixes the answers, independent of the oracle's own running-count code:
* DeepSpeed EP page, assignment_ordinals_by_expert: ordinals are position
  minus the running maximum of segment starts over the expert-sorted
  assignments — restated below as a different computation (stable sort + cummax);
* brute force O(n^2) over every id pattern of a tiny problem;
* closed forms: sum(tokens_per_expert) = N*k - (#-1 ids) - drops,
  drops = sum(max(c_e - C, 0)), splits summing to the row count;
* DeepSpeed EP page, _debug_validate_restore_coverage: the rows of the send
  buffer are exactly the active assignments, none missing, none twice;
* Megatron MORI page: local ids with -1 sentinels (DeepEP contract), tails
  masked with 0 / -1 / 0.
"""

import itertools

import numpy as np
import pytest

from synthetic import get_workload, make_inputs


def page_ordinals(expert_ids_flat):
    """Ordinals by the page's method: stable-sort by expert, then position minus
    the running max of segment starts, scattered back to flattened order."""
    ids = np.asarray(expert_ids_flat, dtype=np.int64)
    valid = np.nonzero(ids >= 0)[0]
    order = valid[np.argsort(ids[valid], kind="stable")]
    sorted_ids = ids[order]
    n = len(order)
    out = np.full(len(ids), -1, dtype=np.int64)
    if n == 0:
        return out
    pos = np.arange(n)
    seg_start = np.zeros(n, dtype=bool)
    seg_start[0] = True
    seg_start[1:] = sorted_ids[1:] != sorted_ids[:-1]
    starts = np.maximum.accumulate(np.where(seg_start, pos, 0))
    out[order] = pos - starts
    return out


def check_invariants(L, idx, probs, E_log, R, C, num_replicas=0, align=0):
    N, k = idx.shape
    E = E_log + num_replicas
    A = max(align, 1)
    E_loc = E // R
    NK = N * k
    flat = idx.reshape(-1)
    valid = (flat >= 0) & (flat < E_log)
    phys = L["phys_idx"].reshape(-1)
    ordn = L["ordinal"].reshape(-1)
    dest = L["dest_row"].reshape(-1)
    drop = L["drop_mask"].reshape(-1).astype(bool)
    rows_max = L["rows_max"]
    assert rows_max == (E * C if C > 0 else NK + E * (A - 1))

    # per expert: ordinals are exactly 0..c-1, strictly increasing in flattened order
    for e in range(E):
        a = np.nonzero(phys == e)[0]
        assert L["counts_raw"][e] == len(a)
        assert ordn[a].tolist() == list(range(len(a)))
    assert np.all(phys[~valid] == -1) and np.all(ordn[~valid] == -1)

    # capacity: first come, first kept
    drops_closed = sum(max(int(c) - C, 0) for c in L["counts_raw"]) if C > 0 else 0
    assert int(drop.sum()) == drops_closed
    assert np.array_equal(drop, valid & (C > 0) & (ordn >= C))
    tpe = L["tokens_per_expert"]
    assert np.array_equal(tpe, np.minimum(L["counts_raw"], C) if C > 0 else L["counts_raw"])
    assert int(tpe.sum()) == NK - int((~valid).sum()) - drops_closed

    # scan and splits
    off = L["expert_offsets"]
    if C > 0:
        assert off.tolist() == [e * C for e in range(E + 1)]
    else:
        assert off[0] == 0 and np.array_equal(np.diff(off), -(-tpe // A) * A)
    assert L["num_rows"][0] == off[E]
    sp = L["input_splits"]
    assert int(sp.sum()) == off[E]
    assert np.array_equal(sp, L["output_splits"])
    for r in range(R):
        assert sp[r] == off[(r + 1) * E_loc] - off[r * E_loc]
        assert L["rank_offsets"][r] == off[r * E_loc]
    assert L["rank_offsets"][R] == off[E]

    # row maps: a bijection between kept assignments and non-pad rows
    kept = valid & ~drop
    assert np.all(dest[~kept] == -1)
    kd = dest[kept]
    assert len(np.unique(kd)) == len(kd) and (len(kd) == 0 or (kd.min() >= 0 and kd.max() < rows_max))
    a_kept = np.nonzero(kept)[0]
    assert np.array_equal(L["row_token"][kd], a_kept // k)
    assert np.array_equal(L["row_slot"][kd], a_kept % k)
    assert np.array_equal(kd, off[phys[kept]] + ordn[kept])
    if probs is not None:
        assert np.array_equal(L["row_prob"][kd], probs.reshape(-1)[kept])
    assert np.array_equal(L["row_local_expert"][kd], phys[kept] % E_loc)
    pad = np.ones(rows_max, bool)
    pad[kd] = False
    assert np.array_equal(L["pad_mask"].astype(bool), pad)
    assert np.all(L["row_token"][pad] == -1) and np.all(L["row_slot"][pad] == -1)
    assert np.all(L["row_local_expert"][pad] == -1) and np.all(L["row_prob"][pad] == 0)
    # rows are expert-major (hence rank-major), ordinal-minor
    row_expert = np.full(rows_max, -1)
    row_expert[kd] = phys[kept]
    assert np.all(np.diff(row_expert[kd][np.argsort(kd)]) >= 0)

    # DeepEP-contract local view: exactly one rank sees each kept assignment
    if "local_topk" in L:
        lt = L["local_topk"].reshape(R, NK)
        seen = (lt >= 0).sum(0)
        assert np.array_equal(seen, kept.astype(int))
        r_of = phys[kept] // E_loc
        assert np.array_equal(lt[r_of, a_kept], phys[kept] - r_of * E_loc)
        assert np.all(lt[(lt >= 0) == False] == -1)

    c = L["counters"]
    assert c[0] == int(valid.sum()) and c[1] == int(kept.sum()) and c[2] == int(drop.sum())
    assert c[3] == rows_max - int(kept.sum())
    assert c[4] == c[5] == int(sp.sum()) and c[6] == L["num_rows"][0]


@pytest.mark.parametrize("seed", range(6))
def test_ordinals_match_page_segment_method(oracle_lib, seed):
    rng = np.random.default_rng(seed)
    N, k, E = 97, 3, 11
    idx = rng.integers(-1, E, size=(N, k)).astype(np.int32)
    L = oracle_lib.layout(idx, None, E_log=E, R=1)
    assert np.array_equal(L["ordinal"].reshape(-1), page_ordinals(idx.reshape(-1)))


def _brute(idx_flat, E, C):
    n = len(idx_flat)
    ordn = [sum(1 for b in range(a) if idx_flat[b] == idx_flat[a]) if idx_flat[a] >= 0 else -1 for a in range(n)]
    counts = [sum(1 for x in idx_flat if x == e) for e in range(E)]
    kept = [idx_flat[a] >= 0 and (C == 0 or ordn[a] < C) for a in range(n)]
    tpe = [sum(1 for a in range(n) if kept[a] and idx_flat[a] == e) for e in range(E)]
    off = [0]
    for e in range(E):
        off.append(off[-1] + (C if C > 0 else tpe[e]))
    dest = [off[idx_flat[a]] + ordn[a] if kept[a] else -1 for a in range(n)]
    return ordn, counts, tpe, off, dest


@pytest.mark.parametrize("C,R", [(0, 1), (0, 3), (1, 1), (2, 3)])
def test_exhaustive_tiny(oracle_lib, C, R):
    N, k, E = 3, 2, 3
    for combo in itertools.product(range(-1, E), repeat=N * k):
        idx = np.array(combo, np.int32).reshape(N, k)
        L = oracle_lib.layout(idx, None, E_log=E, R=R, C=C)
        ordn, counts, tpe, off, dest = _brute(list(combo), E, C)
        assert L["ordinal"].reshape(-1).tolist() == ordn
        assert L["counts_raw"].tolist() == counts
        assert L["tokens_per_expert"].tolist() == tpe
        assert L["expert_offsets"].tolist() == off
        assert L["dest_row"].reshape(-1).tolist() == dest


@pytest.mark.parametrize(
    "N,k,E,R,C,neg",
    [(128, 2, 8, 2, 0, 0.0), (300, 4, 16, 4, 0, 0.1), (512, 2, 8, 2, 100, 0.0), (257, 3, 12, 3, 40, 0.05),
     (64, 8, 32, 8, 8, 0.2), (1, 1, 1, 1, 0, 0.0), (5, 2, 4, 2, 1, 0.0)],
)
def test_invariants_random(oracle_lib, N, k, E, R, C, neg):
    rng = np.random.default_rng(N * 7 + k)
    # skewed ids so that capacity actually drops
    w = rng.zipf(1.6, size=(N, k)) % E
    idx = w.astype(np.int32)
    idx[rng.random((N, k)) < neg] = -1
    probs = rng.random((N, k)).astype(np.float32)
    L = oracle_lib.layout(idx, probs, E_log=E, R=R, C=C)
    check_invariants(L, idx, probs, E, R, C)


def test_workload_invariants(oracle_lib):
    for name in ("tiny", "capacity"):
        w = get_workload(name)
        if name == "capacity":
            w = w.scaled(2048)
        d = make_inputs(w, hidden=False)
        idx, probs = oracle_lib.route_topk(d["logits"], w.k)
        C = w.capacity
        L = oracle_lib.layout(idx, probs, E_log=w.E_log, R=w.R, C=C)
        check_invariants(L, idx, probs, w.E_log, w.R, C)
        if name == "capacity":
            assert L["counters"][2] > 0 and L["counters"][3] > 0  # Zipf(1.5) overflows some experts


def test_capacity_shape_matches_spec():
    w = get_workload("capacity")
    # ceil(1.25 * 16384 * 2 / 64) = 640 slots per expert, 64 * 640 rows
    assert w.capacity == 640
    assert w.E * w.capacity == 40960


def test_out_of_range_ids_flag_and_skip(oracle_lib):
    idx = np.array([[0, 5], [9, -1], [-7, 2]], np.int32)
    L = oracle_lib.layout(idx, None, E_log=4, R=2)
    assert L["counters"][7] == 1
    assert L["phys_idx"].tolist() == [[0, -1], [-1, -1], [-1, 2]]
    assert L["counters"][0] == 2


def test_empty_and_all_masked(oracle_lib):
    idx = np.zeros((0, 4), np.int32)
    L = oracle_lib.layout(idx, None, E_log=8, R=2)
    assert L["rows_max"] == 0 and L["num_rows"][0] == 0 and L["tokens_per_expert"].sum() == 0
    L = oracle_lib.layout(idx, None, E_log=8, R=2, C=3)
    assert L["rows_max"] == 24 and L["pad_mask"].all() and L["counters"][3] == 24
    idx = np.full((10, 2), -1, np.int32)
    L = oracle_lib.layout(idx, None, E_log=4, R=1)
    assert L["num_rows"][0] == 0 and L["pad_mask"].all() and np.all(L["dest_row"] == -1)


def test_rank_major_example_by_hand(oracle_lib):
    # 3 tokens, top-2, 4 experts on 2 ranks; worked by hand from the definitions.
    idx = np.array([[3, 0], [0, 2], [3, 1]], np.int32)
    L = oracle_lib.layout(idx, None, E_log=4, R=2)
    # counts e0:2 e1:1 e2:1 e3:2 -> offsets 0,2,3,4,6; rank0 = experts 0,1 -> 3 rows
    assert L["expert_offsets"].tolist() == [0, 2, 3, 4, 6]
    assert L["input_splits"].tolist() == [3, 3]
    assert L["ordinal"].tolist() == [[0, 0], [1, 0], [1, 0]]
    assert L["dest_row"].tolist() == [[4, 0], [1, 3], [5, 2]]
    assert L["row_token"].tolist() == [0, 1, 2, 1, 0, 2]
    assert L["row_slot"].tolist() == [1, 0, 1, 1, 0, 0]
    assert L["row_local_expert"].tolist() == [0, 0, 1, 0, 1, 1]
    assert L["local_topk"][0].tolist() == [[-1, 0], [0, -1], [-1, 1]]
    assert L["local_topk"][1].tolist() == [[1, -1], [-1, 0], [1, -1]]


@pytest.mark.parametrize("A", [2, 16, 128])
@pytest.mark.parametrize("C", [0, 256])
def test_row_alignment_closed_forms(oracle_lib, A, C):
    """Megatron MORI page: routing maps padded for FP8 / grouped GEMMs. Every expert's rows
    round up to a multiple of A; kept rows keep their order and move down by the pad rows of
    the experts before them; the pads are exactly the tail of each expert's segment."""
    if C % A:
        pytest.skip("capacity must be a multiple of the alignment")
    rng = np.random.default_rng(A + C)
    N, k, E, R = 500, 4, 24, 4
    idx = (rng.zipf(1.4, size=(N, k)) % E).astype(np.int32)
    idx[rng.random((N, k)) < 0.05] = -1
    probs = rng.random((N, k)).astype(np.float32)
    L1 = oracle_lib.layout(idx, probs, E_log=E, R=R, C=C)
    LA = oracle_lib.layout(idx, probs, E_log=E, R=R, C=C, align=A)
    check_invariants(LA, idx, probs, E, R, C, align=A)
    t = LA["tokens_per_expert"]
    assert np.array_equal(t, L1["tokens_per_expert"])
    rows = np.diff(LA["expert_offsets"])
    assert np.all(rows % A == 0) and np.all(rows >= t) and np.all(rows - t < A if C == 0 else rows == C)
    # kept rows move down by the pads of earlier experts
    pads_before = np.concatenate([[0], np.cumsum(rows - np.diff(L1["expert_offsets"]))])
    phys = LA["phys_idx"]
    kept = LA["dest_row"] >= 0
    assert np.array_equal(LA["dest_row"][kept], L1["dest_row"][kept] + pads_before[phys[kept]])
    pad = np.ones(LA["rows_max"], bool)
    for e in range(E):
        pad[LA["expert_offsets"][e]: LA["expert_offsets"][e] + t[e]] = False
    assert np.array_equal(LA["pad_mask"].astype(bool), pad)
    assert LA["counters"][3] == LA["rows_max"] - LA["counters"][1]


def test_row_alignment_rejects_capacity_not_multiple(oracle_lib):
    with pytest.raises(ValueError):
        oracle_lib.layout(np.zeros((4, 2), np.int32), None, E_log=4, R=2, C=10, align=4)
