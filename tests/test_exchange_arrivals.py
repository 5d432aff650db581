"""The arrival count of the in-kernel merge, as host arithmetic (no GPU).

Every split of a (sequence, KV head) that publishes its (m, l) adds to one 64-bit word:
split 0 adds STEP - (n - 1), every other split adds 1, so one launch adds exactly STEP
whatever n is.  A split that read v before its own add waits until the word reaches
(v // STEP + 1) * STEP.  These tests replay that scheme for every arrival order they draw:
when the word starts a launch at a multiple of STEP (a zeroed workspace, or any number of
completed launches before), every split derives the same target, the word reaches it
exactly when the last split arrives, and never earlier.  (The count is only a hint in the
kernel: the merge warp still checks the launch tag of every exchange entry, so a word left
at another value by a different request's data costs a bounded wait, not a wrong result.)
"""
import random

import pytest

STEP = 1 << 16  # kArriveStep in the device code: larger than any number of splits
MAX_SPLITS = 4096  # KVQ_MAX_SPLITS


def replay(start, n, order):
    word = start
    targets = []
    reached_at = None
    for k, split in enumerate(order):
        add = STEP - (n - 1) if split == 0 else 1
        old = word
        word += add
        targets.append((old // STEP + 1) * STEP)
        if reached_at is None and word >= targets[0]:
            reached_at = k
    return word, targets, reached_at


@pytest.mark.parametrize("n", [1, 2, 3, 37, 128, 1000, MAX_SPLITS])
def test_every_split_derives_the_same_target_in_any_order(n):
    rng = random.Random(n)
    assert n - 1 < STEP
    for launches_before in (0, 1, 5, 12345):
        start = launches_before * STEP
        for _ in range(20):
            order = list(range(n))
            rng.shuffle(order)
            word, targets, reached_at = replay(start, n, order)
            assert word == start + STEP
            assert set(targets) == {start + STEP}
            # the word reaches the target with the last arrival and not before
            assert reached_at == n - 1


def test_split_zero_first_or_last():
    n = 37
    for order in (list(range(n)), list(range(n))[::-1]):
        word, targets, reached_at = replay(0, n, order)
        assert word == STEP and set(targets) == {STEP} and reached_at == n - 1


def test_consecutive_launches_with_different_split_counts():
    # the same (sequence, KV head) word across launches whose sequences have grown
    word = 0
    rng = random.Random(7)
    for n in (1, 5, 36, 37, 37, 200, 3):
        order = list(range(n))
        rng.shuffle(order)
        word, targets, reached_at = replay(word, n, order)
        assert word % STEP == 0 and len(set(targets)) == 1 and reached_at == n - 1
