"""Pins of the oracle's fig. 9 solver ("BASE Layers: Simplifying Training of
Large, Sparse Models", wikillm.com summary: "Solver", the fig. 9 listing in
which experts bid for tokens and prices are per token; "Paper vs code":
eps = range / 50, retained winners at the largest score, the update rule
after the iteration cap).  Each case below is worked out by hand in its
docstring; the expected values are copied from that working."""
import numpy as np
import pytest


def case_conflict():
    """T=4, E=2, C=2, cap 100.  q = [[5,4],[4,0],[3,0],[0,1]].
    S0 = (5,4,3,0), S1 = (4,0,0,1); range 5: eps = max(1, 5 // 50) = 1;
    RETAIN = 5 + 1 = 6.

    Round 0 (no retention yet).  e0's three largest: t0 5, t1 4, t2 3: bids
    t0 5-3+1 = 3, t1 4-3+1 = 2.  e1's: t0 4, t3 1, t1 0 (t1 before t2 at 0):
    bids t0 4-0+1 = 5, t3 1-0+1 = 2.  t0 goes to e1 (5 > 3), t1 to e0, t3 to
    e1; t2 got no bid.  price = (5, 2, 0, 2).  adjusted = S - price, winners
    at 6 in their holder's row: e0 = (0, 6, 3, -2), e1 = (6, -2, 0, 6).

    Round 1 (t2 not won).  e0's three largest: t1 6, t2 3, t0 0: bid t2
    3-0+1 = 4 (t1 is e0's: bid eps = 1).  e1's: t0 6, t3 6, t2 0: t0 and t3
    are e1's: eps each.  Every token has a bid: t0 1 (e1), t1 1 (e0), t2 4
    (e0), t3 1 (e1); price = (6, 3, 4, 3).  All won: stop after 2 rounds.
    Lists: e0 (t1, t2), e1 (t0, t3): assign = (1, 0, 0, 1), objective
    4 + 4 + 3 + 1 = 12 (the optimum).
    """
    q = [[5, 4], [4, 0], [3, 0], [0, 1]]
    return q, 100, dict(assign=[1, 0, 0, 1], price=[6, 3, 4, 3], rounds=2, eps=1, objective=12)


def case_after_the_cap():
    """The same q with the iteration cap at 1.  Round 0 as above (winners at
    RETAIN = 6 since 0 < 1).  Round 1 is past the cap: no retention bids.
    e0's three largest: t1 6, t2 3, t0 0: bids t1 6-0+1 = 7, t2 3-0+1 = 4.
    e1's: t0 6, t3 6, t2 0: bids t0 7, t3 7.  price += (7, 7, 4, 7) =
    (12, 9, 4, 9).  All won after 2 rounds; assign = (1, 0, 0, 1).
    """
    q = [[5, 4], [4, 0], [3, 0], [0, 1]]
    return q, 1, dict(assign=[1, 0, 0, 1], price=[12, 9, 4, 9], rounds=2, eps=1, objective=12)


def case_equal_bids_lowest_expert():
    """T=4, E=2, cap 100.  q = [[3,3],[0,0],[3,0],[0,3]].  S0 = (3,0,3,0),
    S1 = (3,0,0,3); range 3: eps = 1; RETAIN = 4.

    Round 0.  e0's three largest: t0 3, t2 3, t1 0: bids t0 3-0+1 = 4, t2 4.
    e1's: t0 3, t3 3, t1 0: bids t0 4, t3 4.  t0 has two bids of 4: the
    smaller expert, e0, wins it.  t1: no bid.  price = (4, 0, 4, 4).
    adjusted = S - price with winners at 4: e0 = (4, 0, 4, -4),
    e1 = (-1, 0, -4, 4).

    Round 1.  e0's: t0 4, t2 4, t1 0: both its own, eps each.  e1's: t3 4,
    t1 0, t0 -1: t3 eps; t1 0-(-1)+1 = 2.  Bids: t0 1 (e0), t1 2 (e1), t2 1
    (e0), t3 1 (e1); price = (5, 2, 5, 5); all won after 2 rounds.
    assign = (0, 1, 0, 1), objective 3 + 0 + 3 + 3 = 9.
    """
    q = [[3, 3], [0, 0], [3, 0], [0, 3]]
    return q, 100, dict(assign=[0, 1, 0, 1], price=[5, 2, 5, 5], rounds=2, eps=1, objective=9)


CASES = [case_conflict, case_after_the_cap, case_equal_bids_lowest_expert]


def fig9_hand_cases():
    out = []
    for fn in CASES:
        q, cap, exp = fn()
        out.append((fn.__name__, np.asarray(q, dtype=np.int32), cap, exp))
    return out


def check_fig9(exp, assign, price, stats):
    assert int(stats["status"]) == 0
    assert list(map(int, assign)) == exp["assign"]
    assert list(map(int, price)) == exp["price"]
    for k in ("rounds", "eps", "objective"):
        assert int(stats[k]) == exp[k], k


@pytest.mark.parametrize("fn", CASES, ids=[f.__name__ for f in CASES])
def test_fig9_follows_hand_worked_rounds(orc, fn):
    q, cap, exp = fn()
    a, p, st = orc.fig9_auction(np.asarray(q, dtype=np.int32), max_iterations=cap)
    check_fig9(exp, a, p, st)


def test_fig9_result_is_balanced_and_never_above_the_optimum(orc):
    rng = np.random.default_rng(12)
    for i in range(300):
        T, E = [(8, 2), (12, 3), (12, 4)][i % 3]
        q = (rng.integers(0, 4, size=(T, E)) if i % 2 else
             rng.integers(-1000, 1000, size=(T, E))).astype(np.int32)
        a, p, st = orc.fig9_auction(q)
        assert st["status"] == 0
        assert np.all(np.bincount(a, minlength=E) == T // E)
        assert st["objective"] == int(q[np.arange(T), a].sum())
        assert st["objective"] <= orc.bruteforce(q)[0]


def test_fig9_bad_arguments(orc):
    q = np.zeros((10, 3), dtype=np.int32)
    assert orc.fig9_auction(q)[2]["status"] == 1  # T % E != 0
