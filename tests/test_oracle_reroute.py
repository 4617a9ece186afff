"""Pins for the UltraEP logical->physical reroute in the oracle.

UltraEP page (background and "UltraEP runtime" list): hot experts get replicas
built from the current layer's actual load, part of their tokens go to the
replica slot, and the router keeps logical semantics. The pages give no
placement or split rule; the reading pinned here: the num_replicas largest
logical counts (ties to the lower id) are hot; each takes the free replica slot
of the least-loaded other rank; a hot expert's logical ordinal o goes to the
master when o is even and to the replica when odd.
"""

import dataclasses

import numpy as np
import pytest

from synthetic import get_workload, make_inputs
from test_oracle_layout import check_invariants


def _ids_with_counts(counts, k, seed=0):
    """A [N, k] id array (N*k = sum(counts)) with the given per-expert counts, shuffled."""
    flat = np.repeat(np.arange(len(counts)), counts)
    rng = np.random.default_rng(seed)
    rng.shuffle(flat)
    assert len(flat) % k == 0
    return flat.reshape(-1, k).astype(np.int32)


def test_placement_worked_by_hand(oracle_lib):
    # 4 logical experts on 2 ranks (M=2), 2 replica slots (one per rank), E_loc = 3.
    # counts: e0=10, e1=2, e2=7, e3=3 -> hot = [e0, e2]; loads: rank0 = 12, rank1 = 10.
    # e0 (home 0) -> rank 1's slot (phys 1*3+2 = 5); moves 5: loads 7 / 15.
    # e2 (home 1) -> rank 0's slot (phys 0*3+2 = 2); moves 3: loads 10 / 12.
    idx = _ids_with_counts([10, 2, 7, 3], k=2)
    L = oracle_lib.layout(idx, None, E_log=4, R=2, num_replicas=2)
    assert L["placement"].tolist() == [5, -1, 2, -1]
    # physical numbering: e0->0, e1->1, replica slot 2; e2->3, e3->4, replica slot 5
    assert L["counts_raw"].tolist() == [5, 2, 3, 4, 3, 5]


def test_least_loaded_other_rank_wins(oracle_lib):
    # 8 logical experts on 4 ranks (M=2), 4 replica slots (S=1 per rank).
    # counts (by expert): [20,0, 0,0, 1,0, 2,0] -> loads 20, 0, 1, 2.
    # hot order by count then id: e0(20), e6(2), e4(1), e1(0).
    # e0 home 0 -> least loaded other rank is 1 (load 0) -> moves 10 -> loads 10,10,1,2
    # e6 home 3 -> others with free slot: 0 (10), 2 (1) -> rank 2 -> moves 1 -> 10,10,2,1
    # e4 home 2 -> others with free slot: 0 (10), 3 (1) -> rank 3 -> moves 0
    # e1 home 0 -> others free: none (1,2,3 used) -> its own rank 0
    idx = _ids_with_counts([20, 0, 0, 0, 1, 0, 2, 0], k=1)
    L = oracle_lib.layout(idx, None, E_log=8, R=4, num_replicas=4)
    E_loc = 3
    assert L["placement"].tolist() == [1 * E_loc + 2, 0 * E_loc + 2, -1, -1, 3 * E_loc + 2, -1, 2 * E_loc + 2, -1]


@pytest.mark.parametrize("seed", range(4))
def test_reroute_closed_forms(oracle_lib, seed):
    rng = np.random.default_rng(seed)
    E_log, R, nrep, k, N = 16, 4, 4, 4, 300
    idx = (rng.zipf(1.4, size=(N, k)) % E_log).astype(np.int32)
    idx[rng.random((N, k)) < 0.05] = -1
    L = oracle_lib.layout(idx, rng.random((N, k)).astype(np.float32), E_log=E_log, R=R, num_replicas=nrep)
    M, S = E_log // R, nrep // R
    E_loc = M + S
    c = np.array([(idx == e).sum() for e in range(E_log)])
    assert np.array_equal(L["counts_logical"], c)
    hot = sorted(range(E_log), key=lambda e: (-c[e], e))[:nrep]
    pl = L["placement"]
    assert sorted(np.nonzero(pl >= 0)[0].tolist()) == sorted(hot)
    assert len(set(pl[pl >= 0].tolist())) == nrep
    assert all((q % E_loc) >= M for q in pl[pl >= 0])
    phys = L["phys_idx"].reshape(-1)
    flat = idx.reshape(-1)
    lo = L["logical_ordinal"].reshape(-1)
    for e in range(E_log):
        master = (e // M) * E_loc + e % M
        if pl[e] >= 0:
            assert L["counts_raw"][master] == (c[e] + 1) // 2
            assert L["counts_raw"][pl[e]] == c[e] // 2
            a = np.nonzero(flat == e)[0]
            assert np.array_equal(phys[a], np.where(lo[a] % 2 == 1, pl[e], master))
            assert np.array_equal(L["ordinal"].reshape(-1)[a], lo[a] // 2)
        else:
            assert L["counts_raw"][master] == c[e]
    # physical -> logical gives back the router's ids
    logical_of = {}
    for e in range(E_log):
        logical_of[(e // M) * E_loc + e % M] = e
        if pl[e] >= 0:
            logical_of[int(pl[e])] = e
    back = np.array([logical_of[q] if q >= 0 else -1 for q in phys])
    assert np.array_equal(back, flat)
    L2 = dict(L)
    check_invariants(L2, idx, None, E_log, R, 0, num_replicas=nrep)


def test_reroute_leaves_combine_unchanged(oracle_lib):
    # With identity experts the combined output must not depend on where a token went.
    w = get_workload("ultraep").scaled(96)
    w = dataclasses.replace(w, H=64)
    d = make_inputs(w)
    idx, probs = oracle_lib.route_topk(d["logits"], w.k)
    L0 = oracle_lib.layout(idx, probs, E_log=w.E_log, R=w.R)
    L1 = oracle_lib.layout(idx, probs, E_log=w.E_log, R=w.R, num_replicas=w.num_replicas)
    assert not np.array_equal(L0["dest_row"], L1["dest_row"])
    s0 = oracle_lib.permute(d["hidden"], L0["dest_row"], L0["rows_max"])
    s1 = oracle_lib.permute(d["hidden"], L1["dest_row"], L1["rows_max"])
    o0 = oracle_lib.combine(s0, L0["dest_row"], probs)
    o1 = oracle_lib.combine(s1, L1["dest_row"], probs)
    assert np.array_equal(o0, o1)
    check_invariants(L1, idx, probs, w.E_log, w.R, 0, num_replicas=w.num_replicas)


def test_ultraep_workload_balances_load(oracle_lib):
    w = get_workload("ultraep").scaled(1024)
    d = make_inputs(w, hidden=False)
    idx, probs = oracle_lib.route_topk(d["logits"], w.k)
    L0 = oracle_lib.layout(idx, probs, E_log=w.E_log, R=w.R)
    L1 = oracle_lib.layout(idx, probs, E_log=w.E_log, R=w.R, num_replicas=w.num_replicas)
    # the busiest rank gets lighter (the point of replicas)
    assert L1["input_splits"].max() <= L0["input_splits"].max()
    assert L1["input_splits"].sum() == L0["input_splits"].sum() == w.N * w.k
