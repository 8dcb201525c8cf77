"""A model check of the in-kernel split merge's counter protocol, on the CPU.

The protocol (as the decode kernel runs it), per sequence n cut into S > 1
splits owned by CTAs c0..c1 (the plan of `plan_model`):
  - each of the S split CTAs, once all its work is done, adds 1 to
    seq_cnt[n] (an arrival; a CTA has at most two split sequences, the first
    and the last of its range);
  - the CTAs whose range ends in n (c0..c1-1, and c1 when n is its last
    sequence: G of them) wait until seq_cnt[n] >= S, then add 1 (a
    departure) and merge their share of the rows; the one whose add sees
    S + G - 1 returns the counter to zero for the next launch.  (The count
    guards only the wait: the partials a member reads after leaving it stay
    in place until the next launch, which starts after this one completes.)
CTAs interleave arbitrarily within a launch; launches follow each other.

The model draws lengths and grid sizes, derives the splits and groups from
the plan statement, runs every action (arrival, poll, departure) atomically
in random order over several launches, and checks: a member passes its wait
only after all S arrivals; every row range is merged exactly once per
launch; no deadlock; every counter is zero between launches.  Planted
mistakes -- a reset one departure early, a wait for S - 1 arrivals -- must be
caught.
"""
import random

import pytest

from tests import plan_model

P, MAXP = 64, 4096


def structure(seqlens, ctas):
    """Per sequence: its split CTAs; per CTA: its split sequences (in range
    order) and the sequence it merges (or None)."""
    own = plan_model.owners(seqlens, P, MAXP, ctas)
    splits = {}
    last_seq = {}
    for n, _, c in own:
        splits.setdefault(n, [])
        if c not in splits[n]:
            splits[n].append(c)
        last_seq[c] = n
    multi = {n: cs for n, cs in splits.items() if len(cs) > 1}
    arrivals = {c: [] for c in range(ctas)}
    for n, cs in multi.items():
        for c in cs:
            arrivals[c].append(n)
    merges = {c: (last_seq[c] if last_seq.get(c) in multi else None) for c in range(ctas)}
    groups = {n: [c for c in range(ctas) if merges[c] == n] for n in multi}
    return multi, arrivals, merges, groups


def run(seqlens_per_launch, ctas, seed, reset_at=0, wait_for=0, abort_launch=None,
        clear_after_abort=True):
    """reset_at / wait_for: offsets planted into the reset threshold and the
    wait target (0 = the protocol).  abort_launch: index of a launch in which
    some CTAs give up (a bounded wait that expired): each stops at a random
    point of its program, and every wait that can then never be satisfied
    expires too.  That launch's results are reported as a timeout and not
    checked; with clear_after_abort the host then clears the counters (what
    mlra_read_device_error does when it reports the timeout, and what the
    static-scratch entry does before every call)."""
    rng = random.Random(seed)
    cnt = {}
    for li, seqlens in enumerate(seqlens_per_launch):
        aborting = li == abort_launch
        multi, arrivals, merges, groups = structure(seqlens, ctas)
        arrived = {n: 0 for n in multi}
        merged = {n: [] for n in multi}
        # per CTA: remaining actions of this launch, in program order
        todo = {c: [("arrive", n) for n in arrivals[c]] for c in range(ctas)}
        for c in range(ctas):
            if merges[c] is not None:
                todo[c] += [("wait", merges[c]), ("depart", merges[c])]
        if aborting:
            for c in rng.sample(range(ctas), max(1, ctas // 4)):
                todo[c] = todo[c][:rng.randrange(len(todo[c]) + 1)]
        while any(todo.values()):
            live = []
            for c, acts in todo.items():
                if not acts:
                    continue
                kind, n = acts[0]
                if kind == "wait" and cnt.get(n, 0) < len(multi[n]) + wait_for:
                    continue
                live.append(c)
            if not live:
                if aborting:
                    break  # the remaining waits expire: those CTAs stop
                return "deadlock"
            c = rng.choice(live)
            kind, n = todo[c].pop(0)
            S, G = len(multi[n]), len(groups[n])
            if kind == "arrive":
                cnt[n] = cnt.get(n, 0) + 1
                arrived[n] += 1
            elif kind == "wait":
                if arrived[n] != S:
                    return "merged early"
                merged[n].append(groups[n].index(c))
            else:
                old = cnt.get(n, 0)
                cnt[n] = old + 1
                if old == S + G - 1 + reset_at:
                    cnt[n] = 0
        if aborting:
            if clear_after_abort:
                cnt = {}
            continue
        for n in multi:
            if sorted(merged[n]) != list(range(len(groups[n]))):
                return "rows not merged once"
        if any(v != 0 for v in cnt.values()):
            return "counter left set"
    return "ok"


def _launches(rng, ctas):
    shapes = []
    for _ in range(3):
        kind = rng.randrange(3)
        if kind == 0:
            shapes.append([rng.choice([0, 1, 128, 129, 4000, 20000]) for _ in range(rng.randint(1, 12))])
        elif kind == 1:
            shapes.append([8192] * rng.randint(1, 20))
        else:
            shapes.append([rng.randint(1, 40000) for _ in range(rng.randint(1, 30))])
    return shapes


@pytest.mark.parametrize("ctas", [3, 7, 16, 148])
def test_no_cta_has_more_than_two_split_sequences(ctas):
    """The kernel keeps two pending arrivals per CTA (its range's first and
    last sequence); a third would lose an arrival and stall that merge."""
    rng = random.Random(100 + ctas)
    for _ in range(200):
        for seqlens in _launches(rng, ctas):
            _, arrivals, _, _ = structure(seqlens, ctas)
            assert max(len(v) for v in arrivals.values()) <= 2, seqlens


@pytest.mark.parametrize("ctas", [3, 7, 16, 148])
def test_merge_counters_are_exact_and_reset_between_launches(ctas):
    rng = random.Random(ctas)
    for seed in range(60):
        assert run(_launches(rng, ctas), ctas, seed) == "ok", seed


@pytest.mark.parametrize("ctas", [7, 16, 148])
def test_a_launch_after_an_aborted_one_is_exact_once_counters_are_cleared(ctas):
    """An aborted launch (some CTAs give up mid-protocol) followed by clean
    ones: with the host-side clear that reporting the timeout performs, the
    next launches merge exactly and leave every counter at zero; without it,
    the stale counts let a later merge start early or stay set."""
    rng = random.Random(500 + ctas)
    uncleared = set()
    for seed in range(60):
        shapes = [[8192] * 16] + _launches(rng, ctas)
        assert run(shapes, ctas, seed, abort_launch=0) == "ok", seed
        uncleared.add(run(shapes, ctas, seed, abort_launch=0, clear_after_abort=False))
    assert uncleared - {"ok"}, uncleared


def test_planted_protocol_mistakes_are_caught():
    shapes = [[8192] * 16, [8192] * 16, [20000, 3, 9000, 40000]]
    early_reset = {run(shapes, 148, s, reset_at=-1) for s in range(40)}
    assert early_reset - {"ok"}, early_reset
    short_wait = {run(shapes, 148, s, wait_for=-1) for s in range(40)}
    assert short_wait - {"ok"}, short_wait
