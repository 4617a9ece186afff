"""Pins for the expert-parallel exchange in the oracle (Megatron MoE page, the
all-to-all token dispatcher: every rank's rows go to the rank owning their
expert, which orders what it received by local expert; Megatron MORI page,
dispatch into the receivers' buffers and a combine that reads them back).

Reading: a receiver orders its rows by its local experts ascending, and within
one expert by source rank ascending, each source's rows in the order of its own
send buffer (stable ordinal order, padding rows last).

Pinned against what the exchange must preserve, found by scanning the routing
itself: every kept assignment of every source arrives exactly once, at the rank
owning its expert, in the block of that expert; the blocks are in the reading's
order; padding rows are zero and sit after their source's tokens; row counts add
up to the senders' splits; a combine over the received rows returns every
source's own combine bit for bit.
"""

import numpy as np
import pytest

from synthetic import bf16_bits_from_f32


def _sources(seed, S, N, k, E_log, C, reps, neg=0.05):
    """S source ranks with their own routings; hidden row t of source s holds (s, t) exactly."""
    rng = np.random.default_rng(seed)
    out = []
    for s in range(S):
        idx = (rng.zipf(1.3, size=(N, k)) % E_log).astype(np.int32)
        for t in range(N):  # distinct experts per token
            row = rng.permutation(E_log)[:k] if E_log >= k else np.arange(k) % E_log
            idx[t] = np.where(idx[t] >= 0, row, -1)
        idx[rng.random((N, k)) < neg] = -1
        probs = rng.random((N, k)).astype(np.float32)
        H = 16
        h = np.zeros((N, H), np.float32)
        h[:, 0] = s + 1  # small integers are exact in bf16
        h[:, 1] = np.arange(N) % 256
        h[:, 2] = np.arange(N) // 256
        h[:, 3:] = rng.standard_normal((N, H - 3))
        out.append((idx, probs, bf16_bits_from_f32(h)))
    return out


def _decode(rows):
    """(source, token) of received rows (-1 for an all-zero padding row)."""
    f = (rows.astype(np.uint32) << 16).view(np.float32)
    src = f[:, 0].astype(np.int64) - 1
    tok = (f[:, 1] + 256 * f[:, 2]).astype(np.int64)
    pad = ~rows.any(axis=1)
    return np.where(pad, -1, src), np.where(pad, -1, tok)


CASES = [
    # S=R, N, k, E_log, C, replicas
    (2, 50, 2, 8, 0, 0),
    (4, 80, 3, 16, 0, 0),
    (4, 120, 4, 16, 20, 0),  # capacity: drops and padding rows
    (4, 200, 4, 16, 0, 4),  # reroute (one replica slot per rank)
    (3, 60, 2, 9, 12, 0),
]


@pytest.mark.parametrize("case", CASES, ids=[f"R{c[0]}_N{c[1]}_k{c[2]}_E{c[3]}_C{c[4]}_rep{c[5]}" for c in CASES])
def test_exchange_delivers_every_kept_assignment_once(oracle_lib, case):
    R, N, k, E_log, C, reps = case
    srcs = _sources(sum(case), R, N, k, E_log, C, reps)
    layouts, sends = [], []
    for idx, probs, hidden in srcs:
        L = oracle_lib.layout(idx, probs, E_log=E_log, R=R, C=C, num_replicas=reps)
        layouts.append(L)
        sends.append(oracle_lib.permute(hidden, L["dest_row"], L["rows_max"]))
    recv, recv_off, base = oracle_lib.ep_exchange(layouts, sends, R)
    E = len(layouts[0]["expert_offsets"]) - 1
    E_loc = E // R
    for r in range(R):
        # row count: what the senders' splits say rank r receives
        assert len(recv[r]) == sum(int(L["input_splits"][r]) for L in layouts)
        assert recv_off[r][0] == 0 and recv_off[r][-1] == len(recv[r])
        src, tok = _decode(recv[r])
        for l in range(E_loc):
            q = r * E_loc + l
            lo, hi = recv_off[r][l], recv_off[r][l + 1]
            # the assignments for expert q, by scanning every source's routing
            want = [(s, t) for s, L in enumerate(layouts) for t in range(N)
                    if np.any((L["phys_idx"][t] == q) & (L["dest_row"][t] >= 0))]
            got_s, got_t = src[lo:hi], tok[lo:hi]
            real = got_s >= 0
            assert sorted(zip(got_s[real].tolist(), got_t[real].tolist())) == sorted(want)
            # order: sources ascending; a source's tokens ascending, then its padding rows
            ranks_seen = []
            for s in range(R):
                n_rows = int(layouts[s]["expert_offsets"][q + 1] - layouts[s]["expert_offsets"][q])
                n_tok = int(layouts[s]["tokens_per_expert"][q])
                part_s = got_s[:n_rows]
                part_t = got_t[:n_rows]
                assert np.all(part_s[:n_tok] == s) and np.all(np.diff(part_t[:n_tok]) > 0)
                assert np.all(part_s[n_tok:] == -1)  # padding rows are zero
                got_s, got_t = got_s[n_rows:], got_t[n_rows:]
                ranks_seen.append(n_rows)
            assert len(got_s) == 0 and sum(ranks_seen) == hi - lo
    # every source's rows are found where base says, and the combine over the received
    # rows gives the source's own combine (identity experts)
    for s, (L, (idx, probs, hidden)) in enumerate(zip(layouts, srcs)):
        y = np.zeros_like(sends[s])
        for q in range(E):
            lo, hi = int(L["expert_offsets"][q]), int(L["expert_offsets"][q + 1])
            y[lo:hi] = recv[q // E_loc][base[s][q]:base[s][q] + hi - lo]
        assert np.array_equal(y, sends[s])
        assert np.array_equal(oracle_lib.combine(y, L["dest_row"], probs), oracle_lib.combine(sends[s], L["dest_row"], probs))
