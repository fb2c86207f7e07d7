"""CPU model of the exponential-turn protocol of the forward kernel.

The two softmax warpgroups of a CTA take turns on the exponential unit.  A
turn is handed on through one mbarrier whose waits test a single phase-parity
bit: a wait for the completion of turn m - 1 passes as soon as the barrier's
count of completed phases has the parity of m.  That is only correct if a
waiter is never two or more phases short.  The kernel's rule: for the key
blocks j < min(n0, n1) that both query blocks of a pair visit, block 0 takes
turn 2(K + j) and block 1 turn 2(K + j) + 1, where K counts such rounds over
all earlier pairs of the CTA; blocks past that run without a turn.

This model runs both warpgroups' turn operations under many random
interleavings and random pair sequences (square causal, bottom-right causal,
odd tails, split-KV items where one block sees no key) and checks that every
wait that passes has really seen its turn complete, and that no run ends
with a warpgroup stuck.  An earlier rule that numbered every block's
exponential phase in one global sequence (so a causal second block took two
turns in a row) is kept as a planted mistake that the model must catch.
"""
from __future__ import annotations

import random

import pytest


def ops_strict(pairs, wg):
    """The kernel's rule: (wait_for, arrive) turn numbers of warpgroup wg."""
    ops, rounds = [], 0
    for n0, n1 in pairs:
        n = (n0, n1)[wg]
        n_turns = min(n0, n1)
        for j in range(n):
            if j < n_turns:
                m = 2 * (rounds + j) + wg
                ops.append((m - 1 if m > 0 else None, m))
        rounds += n_turns
    return ops


def ops_window(pairs, wg):
    """The kernel's rule for windowed pairs (n0, st1, n1): block 1 visits
    iterations st1 .. st1 + n1 - 1 of the pair's stream, block 0 iterations
    0 .. n0 - 1; turns alternate over the iterations both visit."""
    ops, rounds = [], 0
    for n0, st1, n1 in pairs:
        cb, ce = st1, min(n0, st1 + n1)
        n_turns = max(0, ce - cb)
        t0, n = (0, n0) if wg == 0 else (st1, n1)
        for j in range(n):
            tc = t0 + j - cb
            if 0 <= tc < n_turns:
                m = 2 * (rounds + tc) + wg
                ops.append((m - 1 if m > 0 else None, m))
        rounds += n_turns
    return ops


def random_window_pairs(rng, n_pairs):
    """(n0, st1, n1) as the windowed cursor produces them: block 1's window
    starts st1 >= 0 key blocks later and ends at or after block 0's."""
    pairs = []
    for _ in range(n_pairs):
        n0 = rng.randint(1, 6)
        st1 = rng.randint(0, n0 + 1)
        end1 = max(n0, st1 + 1) + rng.randint(0, 1)
        n1 = 0 if rng.randrange(6) == 0 else end1 - st1
        pairs.append((n0, st1, n1))
    return pairs


def ops_global_sequence(pairs, wg):
    """The planted mistake: every exponential phase of either block takes the
    next number of one global sequence (block 0 first at each key step)."""
    ops, t = [], 0
    for n0, n1 in pairs:
        for j in range(max(n0, n1)):
            for w, n in enumerate((n0, n1)):
                if j < n:
                    if w == wg:
                        ops.append((t - 1 if t > 0 else None, t))
                    t += 1
    return ops


def simulate(ops0, ops1, rng):
    """Random interleaving of the two warpgroups.  The turn barrier counts
    completed phases; a wait for turn w passes when the count's parity equals
    (w + 1) mod 2.  Returns 'early' if a passing wait had not really seen
    turn w complete, 'stuck' if neither can move, else 'ok'."""
    ops = (ops0, ops1)
    pos = [0, 0]
    completed = 0
    arrived = set()
    while pos[0] < len(ops0) or pos[1] < len(ops1):
        ready = []
        for w in (0, 1):
            if pos[w] >= len(ops[w]):
                continue
            wait_for, _ = ops[w][pos[w]]
            if wait_for is None or (completed & 1) == ((wait_for + 1) & 1):
                ready.append(w)
        if not ready:
            return "stuck"
        w = rng.choice(ready)
        wait_for, arrive = ops[w][pos[w]]
        if wait_for is not None and wait_for not in arrived:
            return "early"
        # The exponential phase, then the arrival that completes this turn.
        # Arrivals happen in turn order when the protocol is correct.
        if arrive != completed:
            return "early"
        arrived.add(arrive)
        completed += 1
        pos[w] += 1
    return "ok"


def random_pairs(rng, n_pairs):
    """(n0, n1) per pair as the persistent cursor produces them."""
    pairs = []
    for _ in range(n_pairs):
        kind = rng.randrange(5)
        if kind == 0:      # non-causal
            n = rng.randint(1, 6)
            pairs.append((n, n))
        elif kind == 1:    # square causal: the second block has one more key block
            p = rng.randint(0, 4)
            pairs.append((2 * p + 1, 2 * p + 2))
        elif kind == 2:    # bottom-right causal or ragged: second block >= first
            a = rng.randint(1, 6)
            pairs.append((a, a + rng.randint(0, 2)))
        elif kind == 3:    # odd block count: the last pair's second block is empty
            pairs.append((rng.randint(1, 6), 0))
        else:              # split-KV item that the first block cannot see
            pairs.append((0, rng.randint(1, 3)))
    return pairs


def run_model(ops_fn, n_sequences=400, n_interleavings=20, seed=0):
    rng = random.Random(seed)
    outcomes = {"ok": 0, "early": 0, "stuck": 0}
    for _ in range(n_sequences):
        pairs = random_pairs(rng, rng.randint(1, 8))
        o0, o1 = ops_fn(pairs, 0), ops_fn(pairs, 1)
        for _ in range(n_interleavings):
            outcomes[simulate(o0, o1, rng)] += 1
    return outcomes


def test_kernel_turn_rule_is_safe_under_every_interleaving():
    out = run_model(ops_strict)
    assert out["early"] == 0 and out["stuck"] == 0, out


def test_strict_rule_alternates_turns():
    # Turn numbers are 0, 1, 2, ... with block 0 even and block 1 odd.
    pairs = [(1, 2), (3, 4), (2, 0), (0, 2), (5, 5)]
    a0 = [a for _, a in ops_strict(pairs, 0)]
    a1 = [a for _, a in ops_strict(pairs, 1)]
    assert sorted(a0 + a1) == list(range(len(a0) + len(a1)))
    assert all(a % 2 == 0 for a in a0) and all(a % 2 == 1 for a in a1)


def test_model_catches_the_global_sequence_rule():
    # Planted mistake: two turns in a row for one warpgroup lets the other
    # fall two phases behind, so one of its parity waits passes early.
    out = run_model(ops_global_sequence)
    assert out["early"] > 0, out


@pytest.mark.parametrize("pairs", [[(1, 2), (1, 2)], [(3, 4), (5, 6)]])
def test_global_sequence_rule_fails_on_causal_pairs(pairs):
    rng = random.Random(1)
    o0, o1 = ops_global_sequence(pairs, 0), ops_global_sequence(pairs, 1)
    results = {simulate(o0, o1, rng) for _ in range(200)}
    assert "early" in results or "stuck" in results


def test_window_turn_rule_is_safe_under_every_interleaving():
    rng = random.Random(7)
    for _ in range(400):
        pairs = random_window_pairs(rng, rng.randint(1, 8))
        o0, o1 = ops_window(pairs, 0), ops_window(pairs, 1)
        for _ in range(20):
            assert simulate(o0, o1, rng) == "ok", pairs


def test_window_rule_reduces_to_the_unwindowed_rule():
    rng = random.Random(8)
    for _ in range(200):
        pairs = random_pairs(rng, rng.randint(1, 8))
        pairs = [(n0, 0, n1) for n0, n1 in pairs if n0 > 0]
        for wg in (0, 1):
            assert ops_window(pairs, wg) == ops_strict([(a, c) for a, _, c in pairs], wg)
