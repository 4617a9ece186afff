"""Host model of the dispatch layout count kernel's decomposition, against the oracle (CPU).

The count kernel splits the flattened [N, k] assignments over G blocks of 16 warps;
warp w of the block with ticket b owns the slice [(16 b + w) sub, (16 b + w + 1) sub)
and takes it 32 items at a time in ascending order. An assignment's logical ordinal is
then  (same-id items of earlier blocks) + (same-id items of earlier warps of its
block) + (same-id items earlier in its own slice).  With replicas, the physical
expert and ordinal follow in closed form from the logical ordinal o: the master
for even o and the replica for odd o, physical ordinal o / 2. The model rebuilds
both from the grid the host computes and checks them against the oracle's
running counts, which follow the definition directly.
"""

import numpy as np
import pytest

LAYOUT_THREADS = 512
LAYOUT_WARPS = 16
LAYOUT_MAX_BLOCKS = 128
LAYOUT_TARGET_BLOCKS = 32
LAYOUT_MAX_IPL = 8


def layout_grid(NK):
    """The host's grid rule: the fewest ids per lane (1, 2, 4, 8) that keep the grid at
    32 blocks or fewer; else 8 per lane on up to 128 blocks; else longer slices."""
    ipl = 1
    while ipl < LAYOUT_MAX_IPL and -(-NK // (LAYOUT_THREADS * ipl)) > LAYOUT_TARGET_BLOCKS:
        ipl <<= 1
    G = -(-NK // (LAYOUT_THREADS * ipl))
    kind, sub = ipl, 32 * ipl
    if G > LAYOUT_MAX_BLOCKS:
        kind = 0
        per_warp = -(-NK // (LAYOUT_MAX_BLOCKS * LAYOUT_WARPS))
        sub = -(-per_warp // 32) * 32
        G = -(-NK // (LAYOUT_WARPS * sub))
    return max(G, 1), sub, kind


def model_logical_ordinals(ids, E_log):
    """Ordinals composed the kernel's way: block prefix + warp prefix + rank in the warp's slice."""
    NK = len(ids)
    G, sub, _ = layout_grid(NK)
    assert 1 <= G <= LAYOUT_MAX_BLOCKS and sub % 32 == 0
    nslices = G * LAYOUT_WARPS
    assert nslices * sub >= NK  # every item has a slice
    pad = np.full(nslices * sub, -1, np.int64)
    pad[:NK] = ids
    sl = pad.reshape(G, LAYOUT_WARPS, sub)
    # per-slice counts per id, then exclusive prefixes over warps and over blocks
    onehot_counts = np.zeros((G, LAYOUT_WARPS, E_log), np.int64)
    rank_in_slice = np.full((G, LAYOUT_WARPS, sub), -1, np.int64)
    for b in range(G):
        for w in range(LAYOUT_WARPS):
            seen = np.zeros(E_log, np.int64)
            for i in range(0, sub, 32):  # 32 items per round, lanes in ascending order
                for lane in range(32):
                    e = sl[b, w, i + lane]
                    if e >= 0:
                        rank_in_slice[b, w, i + lane] = seen[e]
                        seen[e] += 1
            onehot_counts[b, w] = seen
    warp_pre = np.cumsum(onehot_counts, axis=1) - onehot_counts
    block_tot = onehot_counts.sum(axis=1)
    block_pre = np.cumsum(block_tot, axis=0) - block_tot
    out = np.full(nslices * sub, -1, np.int64)
    for b in range(G):
        for w in range(LAYOUT_WARPS):
            for i in range(sub):
                e = sl[b, w, i]
                if e >= 0:
                    out[(b * LAYOUT_WARPS + w) * sub + i] = block_pre[b, e] + warp_pre[b, w, e] + rank_in_slice[b, w, i]
    return out[:NK]


def test_grid_shapes():
    for NK in [0, 1, 511, 512, 513, 16384, 16385, 32768, 65535, 65536, 65537, 288000, 524288, 524289,
               600000, 2 ** 22, 2 ** 31 - 1]:
        G, sub, kind = layout_grid(NK)
        assert 1 <= G <= LAYOUT_MAX_BLOCKS and G * LAYOUT_WARPS * sub >= NK
        assert kind in (0, 1, 2, 4, 8) and (kind == 0 or sub == 32 * kind)
        assert sub % 32 == 0 and sub < 2 ** 31
        if NK:  # no block is left without items
            assert (G - 1) * LAYOUT_WARPS * sub < NK
        if NK <= LAYOUT_TARGET_BLOCKS * LAYOUT_THREADS * LAYOUT_MAX_IPL:  # the look-back ends in one round
            assert G <= LAYOUT_TARGET_BLOCKS
    # the surveyed shapes: 4096 x 8 and 8192 x 8 assignments take 32 blocks
    assert layout_grid(32768)[:1] == (32,) and layout_grid(65536)[:1] == (32,)


@pytest.mark.parametrize("N,k,E_log,reps,R,seed", [
    (3, 2, 3, 0, 1, 1),
    (700, 3, 8, 0, 2, 2),  # a ragged last block
    (4100, 8, 64, 8, 8, 3),  # 32800 assignments: several blocks, replicas
    (9000, 8, 32, 4, 4, 4),  # two assignments per lane
    (40000, 8, 16, 0, 4, 5),  # 320000 assignments: eight per lane
])
def test_model_ordinals_and_reroute_closed_form_match_the_oracle(oracle_lib, N, k, E_log, reps, R, seed):
    rng = np.random.default_rng(seed)
    idx = (rng.zipf(1.4, size=(N, k)) % E_log).astype(np.int32)
    idx[rng.random((N, k)) < 0.05] = -1
    L = oracle_lib.layout(idx, None, E_log=E_log, R=R, num_replicas=reps)
    lo = model_logical_ordinals(idx.reshape(-1).astype(np.int64), E_log)
    flat = idx.reshape(-1)
    # logical ordinals: the running count of earlier same-id assignments (the definition)
    running = np.zeros(E_log, np.int64)
    want = np.full(len(flat), -1, np.int64)
    for a, e in enumerate(flat):
        if e >= 0:
            want[a] = running[e]
            running[e] += 1
    assert np.array_equal(lo, want)
    # physical expert and ordinal in closed form against the oracle's running physical counts
    M = E_log // R
    E_loc = (E_log + reps) // R
    placement = np.asarray(L["placement"])
    master = np.where(flat >= 0, (flat // M) * E_loc + flat % M, -1)
    repl = np.where(flat >= 0, placement[np.maximum(flat, 0)], -1)
    odd = (lo % 2) == 1
    q = np.where(flat < 0, -1, np.where((repl >= 0) & odd, repl, master))
    ordn = np.where(flat < 0, -1, np.where(repl >= 0, lo // 2, lo))
    assert np.array_equal(q, np.asarray(L["phys_idx"]).reshape(-1))
    assert np.array_equal(ordn, np.asarray(L["ordinal"]).reshape(-1))
