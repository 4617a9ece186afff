"""Pins for TP folding in the oracle (DeepSpeed EP page, partition_assignments and
restore_combined).

Reading: the "assignment index" a peer filters on is the stable per-expert
ordinal of the active (valid, not dropped) assignments, computed as on that page
(assignment_ordinals_by_expert); peer r keeps the ones with index % tp_size == r.
Pinned against: that page's own ordinal method (restated in test_oracle_layout);
closed forms for the peer's local ordinal (o // T) and counts; and the restore
over all peers, which must equal the unfolded combine bit for bit.
"""

import numpy as np
import pytest

from synthetic import bf16_bits_from_f32
from test_oracle_layout import page_ordinals


def _case(seed, N=300, k=4, E=16, neg=0.05, zipf=1.4):
    rng = np.random.default_rng(seed)
    idx = (rng.zipf(zipf, size=(N, k)) % E).astype(np.int32)
    idx[rng.random((N, k)) < neg] = -1
    probs = rng.random((N, k)).astype(np.float32)
    hidden = bf16_bits_from_f32(rng.standard_normal((N, 24)).astype(np.float32))
    return idx, probs, hidden


@pytest.mark.parametrize("T", [2, 3, 4])
@pytest.mark.parametrize("C", [0, 60])
def test_partition_by_page_ordinals(oracle_lib, T, C):
    idx, probs, _ = _case(T * 10 + C)
    N, k = idx.shape
    E, R = 16, 4
    full = oracle_lib.layout(idx, probs, E_log=E, R=R, C=C)
    active = full["dest_row"].reshape(-1) >= 0
    # the page's method: ordinals of the expert-sorted active assignments
    ids = np.where(active, full["phys_idx"].reshape(-1), -1)
    index = page_ordinals(ids)
    owners = np.zeros(N * k, int)
    total_kept = 0
    for r in range(T):
        L = oracle_lib.layout(idx, probs, E_log=E, R=R, C=C, tp_size=T, tp_rank=r)
        mine = L["dest_row"].reshape(-1) >= 0
        assert np.array_equal(mine, active & (index % T == r))
        owners += mine
        o = full["ordinal"].reshape(-1)
        q = full["phys_idx"].reshape(-1)
        # local ordinal o // T, rows from the peer's own offsets
        assert np.array_equal(L["dest_row"].reshape(-1)[mine], L["expert_offsets"][q[mine]] + o[mine] // T)
        t = full["tokens_per_expert"]
        assert np.array_equal(L["tokens_per_expert"], np.where(t > r, (t - r + T - 1) // T, 0))
        assert L["num_rows"][0] <= L["rows_max"]
        assert L["counters"][1] == int(mine.sum())
        assert L["counters"][2] == full["counters"][2]  # capacity drops are global
        if C > 0:
            assert np.all(np.diff(L["expert_offsets"]) == -(-C // T))
        total_kept += int(mine.sum())
    assert np.all(owners[active] == 1) and np.all(owners[~active] == 0)
    assert total_kept == int(active.sum())


@pytest.mark.parametrize("T", [2, 4])
@pytest.mark.parametrize("C,align", [(0, 0), (64, 8), (0, 16)])
def test_restore_over_peers_equals_unfolded_combine(oracle_lib, T, C, align):
    idx, probs, hidden = _case(100 + T + C + align)
    E, R = 16, 4
    full = oracle_lib.layout(idx, probs, E_log=E, R=R, C=C, align=align)
    send = oracle_lib.permute(hidden, full["dest_row"], full["rows_max"])
    expect = oracle_lib.combine(send, full["dest_row"], probs)
    sends, dests = [], []
    for r in range(T):
        L = oracle_lib.layout(idx, probs, E_log=E, R=R, C=C, align=align, tp_size=T, tp_rank=r)
        sends.append(oracle_lib.permute(hidden, L["dest_row"], L["rows_max"]))
        dests.append(L["dest_row"])
    assert np.array_equal(oracle_lib.restore_combined(sends, dests, probs), expect)
    # restore coverage (DeepSpeed EP, _debug_validate_restore_coverage): each kept
    # (token, slot) has exactly one row across the peers, none appears twice
    owners = sum((d >= 0).astype(int) for d in dests)
    assert np.array_equal(owners, (full["dest_row"] >= 0).astype(int))


def test_tp_rows_max_bound(oracle_lib):
    # each peer holds at most ceil(c_e / T) of expert e: sum <= (N*k + E*(T-1)) // T
    for T in (2, 3, 5):
        assert oracle_lib.rows_max(100, 3, 8, 2, tp_size=T) == (300 + 8 * (T - 1)) // T
    assert oracle_lib.rows_max(100, 3, 8, 2, C=10, tp_size=3) == 8 * 4
    with pytest.raises(ValueError):
        oracle_lib.layout(np.zeros((2, 2), np.int32), None, E_log=4, R=2, tp_size=2, tp_rank=2)
    with pytest.raises(ValueError):  # ceil(10 / 3) = 4 is not a multiple of the alignment 8
        oracle_lib.layout(np.zeros((2, 2), np.int32), None, E_log=4, R=2, C=10, align=8, tp_size=3)
