"""Host model of the short-row combine's work split (index arithmetic only).

For k <= 2 and V = H / 8 in {128, 256, 512, 1024} 16-byte chunks per row, the
combine runs CTAs of 256 threads; a token's row is covered by tpt = V / 4
threads (whole warps), thread l of a token owns chunks l, l + tpt, l + 2 tpt,
l + 3 tpt, and a CTA holds 256 / tpt tokens; the grid has ceil(N / (256 / tpt))
CTAs and tokens may be taken last first. The model replays that split and
checks that every output chunk of every token is written exactly once, that
every source-row read stays inside its row, that the threads of a warp always
share one token (so the early exit past the last token and the slot shuffles
are warp-uniform), and that the other (V, k) pairs are left to the general
kernel.
"""

import pytest

THREADS = 256
CPT = 4


def _eligible(k, V):
    return k in (1, 2) and V in (128, 256, 512, 1024)


def _split(N, V, last_first):
    tpt = V // CPT
    per_cta = THREADS // tpt
    blocks = -(-N // per_cta)
    writes = {}
    warp_tokens = {}
    for b in range(blocks):
        for tid in range(THREADS):
            u, l = divmod(tid, tpt)
            tb = b * per_cta + u
            warp_tokens.setdefault((b, tid // 32), set()).add(tb)
            if tb >= N:
                continue
            t = N - 1 - tb if last_first else tb
            for i in range(CPT):
                c = l + i * tpt
                assert 0 <= c < V  # the read of row d is d * V + c: inside the row
                writes[(t, c)] = writes.get((t, c), 0) + 1
    return writes, warp_tokens


@pytest.mark.parametrize("V", [128, 256, 512, 1024])
@pytest.mark.parametrize("N", [1, 2, 7, 8, 9, 33, 1001])
@pytest.mark.parametrize("last_first", [False, True])
def test_every_chunk_written_once(V, N, last_first):
    writes, warp_tokens = _split(N, V, last_first)
    assert len(writes) == N * V
    assert set(writes.values()) == {1}
    assert all(len(ts) == 1 for ts in warp_tokens.values())


def test_selection_covers_only_whole_warp_splits():
    for V in range(1, 2049):
        for k in range(1, 9):
            if _eligible(k, V):
                assert V % (CPT * 32) == 0 and THREADS % (V // CPT) == 0
    assert not _eligible(8, 256) and not _eligible(2, 896) and not _eligible(2, 32)
