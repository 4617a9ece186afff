"""Host model of the dispatch layout's decoupled look-back (the arithmetic and indexing only).

The count kernel's blocks take tickets v = 0..G-1 from one 64-bit word (low half: tickets
taken, high half: launch epoch); the block drawing ticket G-1 rolls the word over to
(epoch + 1, 0). Each block publishes, per expert column, a 64-bit word [epoch | status |
error bit | count]: AGG (its own count) first, INCL (count of every block up to it) once its
look-back is done. The look-back of block v splits its predecessors into P parts per round,
part p reading blocks hi - p W, hi - p W - 1, ... (W = 16 per part, nearest first, stopping
after the first INCL); the parts of a column are merged in order up to the first one that
closed the prefix (met an INCL or ran past block 0), and the next round starts at
hi - P W. A word from another epoch reads as not yet published.

The model replays the kernel's index arithmetic on random snapshots of which predecessors
have published what, and checks the prefixes, the error bit and the epoch handling; it also
replays ticket draws across launches of different grid sizes.
"""

import random

LB_AGG, LB_INCL = 1, 2
W = 16
LAYOUT_THREADS = 512
EPOCH_MASK = (1 << 30) - 1


def parts(E_log):
    return 1 if E_log >= LAYOUT_THREADS else min(32, LAYOUT_THREADS // E_log)


def word(epoch, status, value, err):
    assert 0 <= value < 2 ** 31
    return ((epoch & EPOCH_MASK) << 34) | (status << 32) | (int(err) << 31) | value


def ready(w, epoch):
    return (w >> 32) & 3 != 0 and (w >> 34) == (epoch & EPOCH_MASK)


def scan_chunk(flags, col, top, epoch, resolve):
    """lb_scan_chunk: `resolve(j)` plays the later polls of a word that was not ready."""
    s, err = 0, False
    for i in range(W):
        j = top - i
        if j < 0:
            return s, err, True
        w = flags[j][col]
        if not ready(w, epoch):
            w = resolve(j, col)
        s += w & 0x7FFFFFFF
        err |= bool((w >> 31) & 1)
        if (w >> 32) & 3 == LB_INCL:
            return s, err, True
    return s, err, False


def lookback(flags, vb, E_log, epoch, resolve):
    """The count kernel's rounds for block vb: exclusive prefix and error bit per column."""
    P = parts(E_log)
    excl = [0] * E_log
    done = [False] * E_log
    errs = [False] * E_log
    hi = vb - 1
    rounds = 0
    while True:
        rounds += 1
        psum, pflag = {}, {}
        for item in range(P * E_log):
            e, p = item % E_log, item // E_log
            if done[e]:
                continue
            psum[item], perr, closed = scan_chunk(flags, e, hi - p * W, epoch, resolve)
            pflag[item] = (closed, perr)
        more = False
        for e in range(E_log):
            if done[e]:
                continue
            for p in range(P):
                closed, perr = pflag[p * E_log + e]
                excl[e] += psum[p * E_log + e]
                errs[e] |= perr
                if closed:
                    done[e] = True
                    break
            more |= not done[e]
        hi -= P * W
        if not more:
            return excl, errs, rounds


def _launch(rng, G, E_log, epoch, stale_epoch):
    agg = [[rng.randrange(0, 50) for _ in range(E_log)] for _ in range(G)]
    berr = [rng.random() < 0.1 for _ in range(G)]
    incl = [[sum(agg[i][e] for i in range(j + 1)) for e in range(E_log)] for j in range(G)]
    ierr = [any(berr[: j + 1]) for j in range(G)]
    return agg, berr, incl, ierr


def test_prefixes_for_every_snapshot_of_published_words():
    rng = random.Random(7)
    for trial in range(60):
        E_log = rng.choice([1, 3, 8, 64, 100, 256, 600])
        G = rng.choice([1, 2, 5, 17, 32, 33, 70, 128])
        epoch = rng.randrange(0, 2 ** 32)
        agg, berr, incl, ierr = _launch(rng, G, E_log, epoch, None)
        for vb in sorted({0, G - 1, rng.randrange(G), min(G - 1, 16), min(G - 1, 32)}):
            # snapshot: each predecessor's word is INCL, AGG, or not published (a word of an
            # older epoch or zero); block 0 publishes INCL directly
            flags = []
            for j in range(G):
                row = []
                for e in range(E_log):
                    r = rng.random()
                    if j == 0 or r < 0.3:
                        row.append(word(epoch, LB_INCL, incl[j][e], ierr[j]))
                    elif r < 0.7:
                        row.append(word(epoch, LB_AGG, agg[j][e], berr[j]))
                    elif r < 0.85:
                        row.append(word(epoch - 1, LB_INCL, rng.randrange(2 ** 31), True))  # stale
                    else:
                        row.append(0)
                flags.append(row)

            def resolve(j, e):  # a later poll finds the word published (either kind)
                if rng.random() < 0.5:
                    return word(epoch, LB_INCL, incl[j][e], ierr[j])
                return word(epoch, LB_AGG, agg[j][e], berr[j])

            excl, errs, rounds = lookback(flags, vb, E_log, epoch, resolve)
            for e in range(E_log):
                assert excl[e] == sum(agg[i][e] for i in range(vb)), (trial, vb, e)
                assert errs[e] == any(berr[:vb])
            # all-AGG worst case bounds the rounds: one round reaches P * W blocks back
            assert rounds <= max(1, -(-vb // (parts(E_log) * W)) + 1)


def test_one_round_up_to_the_target_grid():
    """Every block of a grid of at most 32 blocks finishes its look-back in one round,
    even when no predecessor has published an inclusive prefix yet (for E_log < 512)."""
    for E_log in (8, 64, 128, 256):
        G = 32
        epoch = 5
        flags = [[word(epoch, LB_INCL if j == 0 else LB_AGG, 1, False) for _ in range(E_log)] for j in range(G)]
        for vb in range(G):
            excl, _, rounds = lookback(flags, vb, E_log, epoch, lambda j, e: None)
            assert rounds == 1 and excl == [vb] * E_log


def test_ticket_word_rolls_over_between_launches():
    """Tickets are 0..G-1 in draw order within a launch whatever G is; the epoch advances by
    one per launch, so the look-back words of the previous launch read as not published."""
    rng = random.Random(3)
    tw = 0
    for launch in range(500):
        G = rng.choice([1, 2, 7, 32, 128])
        seen = []
        for _ in range(G):  # draws in any interleaving are serialised by the atomic
            old = tw
            tw = (tw + 1) & (2 ** 64 - 1)
            vb, ep = old & 0xFFFFFFFF, old >> 32
            if vb == G - 1:
                tw = (tw + (1 << 32) - G) & (2 ** 64 - 1)
            seen.append((vb, ep))
        assert [v for v, _ in seen] == list(range(G))
        assert {ep for _, ep in seen} == {launch}
        assert tw == (launch + 1) << 32
        w_old = word(launch, LB_INCL, 5, False)
        assert ready(w_old, launch) and not ready(w_old, launch + 1)


def test_epoch_wraps_modulo_2_30():
    w = word(EPOCH_MASK, LB_AGG, 3, False)
    assert ready(w, EPOCH_MASK) and ready(w, 2 * EPOCH_MASK + 1) and not ready(w, 0)
    assert not ready(0, 0)  # zero-filled scratch reads as not published in the first epoch
