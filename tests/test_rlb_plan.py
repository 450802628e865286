"""Head-to-rank plans of Runtime Load Balancing, on the CPU (host code of the
C ABI, no GPU).

fvattn_rlb_plan follows the pages' rule -- the most loaded rank moves one
of its heads to a lightly loaded rank, each rank sending and receiving at
most one head -- and fvattn_lpt_assign places heads from scratch. Both are
checked against brute force over every admissible plan on tiny head sets.
"""
import itertools
import random
from fractions import Fraction

import pytest


@pytest.fixture(scope="module")
def fa():
    from block_sparse_attention_fvattn_b200 import build
    build.build()
    from block_sparse_attention_fvattn_b200 import fvattn
    return fvattn


def static_owner(H, W):
    return [r for r in range(W) for _ in range(r * H // W, (r + 1) * H // W)]


def loads(costs, owner, W):
    out = [0] * W
    for h, c in enumerate(costs):
        out[owner[h]] += c
    return out


def single_move_plans(costs, W):
    own = static_owner(len(costs), W)
    yield list(own)
    for h in range(len(costs)):
        for d in range(W):
            if d != own[h]:
                o = list(own)
                o[h] = d
                yield o


def one_per_rank_plans(costs, W):
    """Every plan in which each rank sends at most one of its own heads and
    receives at most one."""
    H = len(costs)
    own = static_owner(H, W)
    opts = [[None] + [(h, d) for h in range(H) if own[h] == r for d in range(W) if d != r] for r in range(W)]
    for plan in itertools.product(*opts):
        dsts = [p[1] for p in plan if p]
        if len(dsts) != len(set(dsts)):
            continue
        o = list(own)
        for p in plan:
            if p:
                o[p[0]] = p[1]
        yield o


def random_cases(seed, n, W_range=(2, 4)):
    rng = random.Random(seed)
    for _ in range(n):
        W = rng.randint(*W_range)
        H = rng.randint(W, 2 * W + 2)
        yield [rng.choice([rng.randint(1, 10), rng.randint(10, 100)]) for _ in range(H)], W


def test_rlb_respects_the_move_limit_and_never_hurts(fa):
    for costs, W in random_cases(1, 200, (2, 8)):
        own = static_owner(len(costs), W)
        owner, load = fa.rlb_plan(costs, W)
        assert load == loads(costs, owner, W)
        sent = [0] * W
        recv = [0] * W
        for h in range(len(costs)):
            if owner[h] != own[h]:
                sent[own[h]] += 1
                recv[owner[h]] += 1
        assert max(sent) <= 1 and max(recv) <= 1
        assert max(load) <= max(loads(costs, own, W))
        assert fa.rlb_plan(costs, W) == (owner, load)      # deterministic


def test_rlb_beats_every_single_move_and_no_plan_beats_it_by_much(fa):
    # the first move is the best single move, so no single-move plan is
    # better; against every admissible plan (one send and one receive per
    # rank, enumerated) the greedy is never better than the optimum and on
    # these seeded cases at most 4/3 of it
    matched = total = 0
    for costs, W in random_cases(2, 150):
        owner, load = fa.rlb_plan(costs, W)
        best_single = min(max(loads(costs, o, W)) for o in single_move_plans(costs, W))
        best = min(max(loads(costs, o, W)) for o in one_per_rank_plans(costs, W))
        assert max(load) <= best_single
        assert best <= max(load) <= Fraction(4, 3) * best
        matched += max(load) == best
        total += 1
    assert matched >= 0.8 * total


def test_rlb_zero_moves_and_one_rank(fa):
    costs = [5, 1, 9, 2]
    assert fa.rlb_plan(costs, 2, max_moves=0)[0] == static_owner(4, 2)
    assert fa.rlb_plan(costs, 1) == ([0, 0, 0, 0], [17])


def test_lpt_within_graham_bound_of_the_optimum(fa):
    # LPT's largest load is at most (4/3 - 1/(3m)) times the optimum over all
    # m^H assignments (Graham 1969), checked by enumeration
    for costs, W in random_cases(3, 120, (2, 3)):
        H = len(costs)
        if W ** H > 200000:
            continue
        owner, load = fa.lpt_assign(costs, W)
        assert load == loads(costs, owner, W)
        opt = min(max(loads(costs, o, W)) for o in itertools.product(range(W), repeat=H))
        assert opt <= max(load) <= (Fraction(4, 3) - Fraction(1, 3 * W)) * opt
