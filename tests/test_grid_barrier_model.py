"""Host model of the dedup layout's single-word grid barrier (the arithmetic only).

Each launch of G blocks adds exactly 2^20 to one 32-bit word: block 0 adds
2^20 - (G - 1) - extra, every other block 1. A block computes its target from the
value it saw, (old & ~(2^20 - 1)) + 2^20, and waits until the word, compared
modulo 2^32, reaches it. The model replays arrivals in random orders, across the
2^32 wrap, and checks that every block's target is the launch's final value, that
no partial sum reaches a target early, and that extra > 0 (the timeout test hook)
never completes.
"""

import random

SPAN = 1 << 20
MASK = 0xFFFFFFFF


def _reached(word, target):
    d = (word - target) & MASK
    return d < (1 << 31)  # (int32)(word - target) >= 0


def _launch(word, G, order, extra=0):
    targets, sums = [], []
    for b in order:
        inc = SPAN - (G - 1) - extra if b == 0 else 1
        old = word
        word = (word + inc) & MASK
        targets.append((old & ~(SPAN - 1) & MASK) + SPAN & MASK)
        sums.append(word)
    return word, targets, sums


def test_every_target_is_the_launch_end_across_the_wrap():
    rng = random.Random(5)
    word = 0
    for launch in range(4096 * 2 + 7):  # wraps twice
        G = rng.choice([1, 2, 3, 16, 64, 128])
        order = list(range(G))
        rng.shuffle(order)
        start = word
        word, targets, sums = _launch(word, G, order)
        assert word == (start + SPAN) & MASK
        assert all(t == word for t in targets)
        # no partial sum reaches the target before the last arrival
        assert not any(_reached(s, word) for s in sums[:-1])
        assert _reached(sums[-1], word)


def test_extra_arrival_never_completes():
    rng = random.Random(6)
    for start in (0, SPAN * 4095, (1 << 32) - SPAN, 12345 * SPAN & MASK):
        G = 16
        order = list(range(G))
        rng.shuffle(order)
        word, targets, sums = _launch(start, G, order, extra=1)
        assert all(t == (start + SPAN) & MASK for t in targets)
        assert not any(_reached(s, targets[0]) for s in sums)
