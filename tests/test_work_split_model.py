"""Host model of how the permute and the combine split their work (index arithmetic only).

Permute: a row of V 16-byte chunks is copied by a group of 32, 64 or 128 threads
(the smallest that covers 8 chunks per thread, else 128 with the row cut into
pieces of 128 x 8 chunks); thread gt of a group copies chunks c0 + c * group,
c < 8, c0 = piece * group * 8 + gt, those below V. A CTA of 128 threads holds
128 / group (token, piece) units; the leading CTAs instead zero the pad rows: one
warp per worker, worker w checking rows w + lane * W + 32 * W * pass (W workers).

Combine: CTAs of 32..256 threads, the widest that divides the row's chunk count
rounded up to 32; nchunks CTAs per token, thread v = c * threads + tid owning one
chunk when v < V.

The model replays both splits for many row lengths and checks that every chunk of
every token is handled exactly once and that every row is zeroed by exactly one
worker.
"""

import pytest

SMS = 148
PERMUTE_THREADS = 128
PERMUTE_CHUNKS = 8


def permute_split(V):
    group = 32 if V <= 32 * PERMUTE_CHUNKS else (64 if V <= 64 * PERMUTE_CHUNKS else PERMUTE_THREADS)
    pieces = -(-V // (group * PERMUTE_CHUNKS))
    return group, pieces


@pytest.mark.parametrize("V", [1, 3, 16, 33, 130, 256, 257, 512, 513, 896, 1024, 1025, 2500])
@pytest.mark.parametrize("N", [1, 5, 33])
def test_permute_copies_every_chunk_once(V, N):
    group, pieces = permute_split(V)
    groups = PERMUTE_THREADS // group
    blocks = -(-N * pieces // groups)
    seen = {}
    for b in range(blocks):
        for tid in range(PERMUTE_THREADS):
            g, gt = divmod(tid, group)
            unit = b * groups + g
            if unit >= N * pieces:
                continue
            t, piece = divmod(unit, pieces)
            c0 = piece * group * PERMUTE_CHUNKS + gt
            for c in range(PERMUTE_CHUNKS):
                idx = c0 + c * group
                if idx < V:
                    seen[(t, idx)] = seen.get((t, idx), 0) + 1
    assert len(seen) == N * V and set(seen.values()) == {1}


@pytest.mark.parametrize("rows_max", [1, 31, 127, 128, 129, 4097, 40960, 100000, 300001])
def test_pad_rows_zeroed_once(rows_max):
    zb = min(-(-rows_max // PERMUTE_THREADS), 4 * SMS)
    W = zb * (PERMUTE_THREADS // 32)
    seen = [0] * rows_max
    for w in range(W):
        r0 = w
        while r0 < rows_max:
            for lane in range(32):
                r = r0 + lane * W
                if r < rows_max:
                    seen[r] += 1
            r0 += 32 * W
    assert seen == [1] * rows_max


def combine_split(V):
    v32 = -(-V // 32) * 32
    threads = 256 if v32 % 256 == 0 else (128 if v32 % 128 == 0 else (64 if v32 % 64 == 0 else 32))
    return threads, -(-V // threads)


@pytest.mark.parametrize("V", [1, 3, 16, 33, 130, 256, 257, 512, 896, 1025, 2500])
@pytest.mark.parametrize("last_first", [False, True])
def test_combine_covers_every_chunk_once(V, last_first):
    N = 7
    threads, nchunks = combine_split(V)
    assert threads in (32, 64, 128, 256)
    seen = {}
    for b in range(N * nchunks):
        tb, c = divmod(b, nchunks)
        t = N - 1 - tb if last_first else tb
        for tid in range(threads):
            v = c * threads + tid
            if v < V:
                seen[(t, v)] = seen.get((t, v), 0) + 1
    assert len(seen) == N * V and set(seen.values()) == {1}
    # the split wastes less than one warp per CTA on average
    assert N * nchunks * threads - N * V < N * nchunks * 32 or threads == 32
