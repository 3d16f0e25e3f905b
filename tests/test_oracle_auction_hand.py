"""Hand-worked auction trajectories: the tie rules, the price rule and the
phase rules of the balanced assignment, pinned by values derived on paper.

The optimum of eq. 2 ("BASE Layers: Simplifying Training of Large, Sparse
Models", wikillm.com summary, Method / "Training assignment") is pinned
elsewhere by brute force and the Hungarian method.  Those pins cannot tell
WHICH optimum the auction returns, or along which trajectory: with equal
scores several assignments are optimal.  The rules that decide it are the
auction's own spec -- lowest expert index on equal values, lowest token index
on equal bids, the price of a full expert is the lowest bid it holds and an
expert that is not full keeps its price, prices carry over between phases and
held sets do not.  Each case below is small enough to run by hand; its
docstring works through every round, and the expected values are copied from
that working, not from any program.

Notation of the spec: A[t][e] = q[t][e] (T+1); eps0 = max(1, floor((max q -
min q)(T+1)/50)); a bidder t computes v_e = A[t][e] - p_e, its best expert
e* = argmax v_e (lowest e on ties), v2 = max over e != e* of v_e, and bids
b = A[t][e*] - v2 + eps; an expert keeps its C = T/E best of held + new by
(bid desc, token asc); once it holds C its price becomes its lowest held bid.

`test_mutations_are_caught` plants each rule's plausible mistake in a copy of
the oracle's C source (on the CPU) and checks that some case here fails.
"""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

# ---------------------------------------------------------------------------
# the cases: (name, q, expected)
# ---------------------------------------------------------------------------


def case_equal_bids_lowest_token_wins():
    """T=4, E=2, C=2.  q = [[10,0],[5,0],[5,0],[0,0]].

    R = 10, T+1 = 5: eps = max(1, floor(50/50)) = 1, one phase.
    A = [[50,0],[25,0],[25,0],[0,0]].

    Round 1, p = (0, 0), bidders {0,1,2,3}:
      t0: v = (50, 0)  -> e0, v2 = 0,  b = 50 - 0 + 1 = 51
      t1: v = (25, 0)  -> e0, v2 = 0,  b = 26
      t2: v = (25, 0)  -> e0, v2 = 0,  b = 26
      t3: v = (0, 0)   -> e0 (equal values: lowest expert), v2 = 0, b = 1
      e0 candidates (51,t0) (26,t1) (26,t2) (1,t3): keeps (51,t0) and
      (26,t1) -- t1 and t2 bid the same, the lower token wins -- and rejects
      t2, t3; it is full, p0 = 26.  e1 got nothing: p1 stays 0.
    Round 2, p = (26, 0), bidders {2,3}:
      t2: v = (25-26, 0) = (-1, 0) -> e1, v2 = -1, b = 0 + 1 + 1 = 2
      t3: v = (-26, 0)            -> e1, v2 = -26, b = 0 + 26 + 1 = 27
      e1 keeps both (C = 2), full, p1 = min(27, 2) = 2.
    Nobody is unassigned and eps = 1: stop.

    assign = [0,0,1,1], price = [26,2], 1 phase, 2 rounds, 4 + 2 = 6 bids,
    objective 10 + 5 + 0 + 0 = 15.  [0,1,0,1] is an optimum too (t1 and t2
    have equal rows): the token tie rule picks [0,0,1,1].
    """
    q = [[10, 0], [5, 0], [5, 0], [0, 0]]
    exp = dict(assign=[0, 0, 1, 1], price=[26, 2], phases=1, rounds=2, bids=6,
               final_eps=1, objective=15, trace=[4, 2])
    return q, exp


def case_equal_values_lowest_expert_wins():
    """T=2, E=2, C=1.  q = [[3,3],[0,0]].

    R = 3, T+1 = 3: eps = max(1, floor(9/50)) = 1, one phase.
    A = [[9,9],[0,0]].

    Round 1, p = (0, 0), bidders {0,1}:
      t0: v = (9, 9) -> e0 (equal values: lowest expert), v1 = 9, v2 = 9,
          b = 9 - 9 + 1 = 1
      t1: v = (0, 0) -> e0, v2 = 0, b = 1
      e0 candidates (1,t0) (1,t1): keeps t0 (lower token), rejects t1;
      full, p0 = 1.
    Round 2, p = (1, 0), bidder {1}:
      t1: v = (-1, 0) -> e1, v2 = -1, b = 0 + 1 + 1 = 2; e1 keeps it, p1 = 2.

    assign = [0,1], price = [1,2], 1 phase, 2 rounds, 3 bids, objective 3.
    [1,0] is also optimal (objective 3): the expert tie rule picks [0,1].
    """
    q = [[3, 3], [0, 0]]
    exp = dict(assign=[0, 1], price=[1, 2], phases=1, rounds=2, bids=3,
               final_eps=1, objective=3, trace=[2, 1])
    return q, exp


def case_expert_short_of_capacity_keeps_its_price():
    """T=4, E=2, C=2.  q = [[8,0],[8,0],[8,0],[0,2]].

    R = 8, T+1 = 5: eps = max(1, floor(40/50)) = 1, one phase.
    A = [[40,0],[40,0],[40,0],[0,10]].

    Round 1, p = (0, 0), bidders {0,1,2,3}:
      t0, t1, t2: v = (40, 0) -> e0, v2 = 0, b = 41
      t3: v = (0, 10) -> e1, v2 = 0, b = 10 - 0 + 1 = 11
      e0 candidates (41,t0) (41,t1) (41,t2): keeps t0, t1, rejects t2;
      full, p0 = 41.
      e1 holds only (11,t3): 1 < C, so its price stays 0 (it does NOT
      become 11).
    Round 2, p = (41, 0), bidder {2}:
      t2: v = (40-41, 0-0) = (-1, 0) -> e1, v2 = -1, b = 0 + 1 + 1 = 2
      e1 keeps (11,t3) (2,t2), full, p1 = 2.

    assign = [0,0,1,1], price = [41,2], 1 phase, 2 rounds, 5 bids,
    objective 8 + 8 + 0 + 2 = 18.
    """
    q = [[8, 0], [8, 0], [8, 0], [0, 2]]
    exp = dict(assign=[0, 0, 1, 1], price=[41, 2], phases=1, rounds=2, bids=5,
               final_eps=1, objective=18, trace=[4, 1])
    return q, exp


def case_two_phases_prices_carry_over():
    """T=4, E=2, C=2.  q = [[20,0],[10,5],[10,0],[0,0]].

    R = 20, T+1 = 5: eps0 = max(1, floor(100/50)) = 2.
    A = [[100,0],[50,25],[50,0],[0,0]].

    Phase 1, eps = 2, p = (0, 0).
    Round 1, bidders {0,1,2,3}:
      t0: v = (100, 0) -> e0, v2 = 0,  b = 100 - 0 + 2 = 102
      t1: v = (50, 25) -> e0, v2 = 25, b = 50 - 25 + 2 = 27
      t2: v = (50, 0)  -> e0, v2 = 0,  b = 52
      t3: v = (0, 0)   -> e0, v2 = 0,  b = 2
      e0 keeps (102,t0) (52,t2), rejects t1, t3; p0 = 52.
    Round 2, p = (52, 0), bidders {1,3}:
      t1: v = (-2, 25)  -> e1, v2 = -2,  b = 25 + 2 + 2 = 29
      t3: v = (-52, 0)  -> e1, v2 = -52, b = 0 + 52 + 2 = 54
      e1 keeps both, p1 = 29.
    eps = max(1, floor(2/8)) = 1.
    Phase 2, eps = 1: every token unassigned again, prices kept (52, 29).
    Round 3, bidders {0,1,2,3}:
      t0: v = (48, -29)  -> e0, v2 = -29, b = 100 + 29 + 1 = 130
      t1: v = (-2, -4)   -> e0, v2 = -4,  b = 50 + 4 + 1 = 55
      t2: v = (-2, -29)  -> e0, v2 = -29, b = 50 + 29 + 1 = 80
      t3: v = (-52, -29) -> e1, v2 = -52, b = 0 + 52 + 1 = 53
      e0 keeps (130,t0) (80,t2), rejects t1; p0 = 80.
      e1 holds (53,t3) only: p1 stays 29.
    Round 4, p = (80, 29), bidder {1}:
      t1: v = (-30, -4) -> e1, v2 = -30, b = 25 + 30 + 1 = 56
      e1 keeps (56,t1) (53,t3), full, p1 = 53.
    eps = 1: stop.

    assign = [0,1,0,1], price = [80,53], 2 phases, 4 rounds,
    4 + 2 + 4 + 1 = 11 bids, objective 20 + 5 + 10 + 0 = 35 (the optimum:
    t0 and t2 have the largest q0 - q1).
    """
    q = [[20, 0], [10, 5], [10, 0], [0, 0]]
    exp = dict(assign=[0, 1, 0, 1], price=[80, 53], phases=2, rounds=4, bids=11,
               final_eps=1, objective=35, trace=[4, 2, 4, 1])
    return q, exp


CASES = [case_equal_bids_lowest_token_wins, case_equal_values_lowest_expert_wins,
         case_expert_short_of_capacity_keeps_its_price, case_two_phases_prices_carry_over]


def hand_cases():
    """(name, q int32 array, expected dict) for every hand-worked case."""
    out = []
    for fn in CASES:
        q, exp = fn()
        out.append((fn.__name__, np.asarray(q, dtype=np.int32), exp))
    return out


def check_result(exp, assign, price, stats, trace=None):
    """Compares one auction result with a hand-worked expectation."""
    assert list(map(int, assign)) == exp["assign"]
    assert list(map(int, price)) == exp["price"]
    for k in ("phases", "rounds", "bids", "final_eps", "objective"):
        assert int(stats[k]) == exp[k], k
    assert int(stats["status"]) == 0
    if trace is not None:
        assert list(map(int, trace)) == exp["trace"]


# ---------------------------------------------------------------------------
# the oracle against the hand-worked values
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("fn", CASES, ids=[f.__name__ for f in CASES])
def test_oracle_follows_hand_worked_trajectory(orc, fn):
    q, exp = fn()
    q = np.asarray(q, dtype=np.int32)
    a, p, st, tr = orc.auction(q, trace=True)
    check_result(exp, a, p, st, tr)
    # the hand-worked optimum is the optimum
    assert orc.bruteforce(q)[0] == exp["objective"]
    assert orc.certificate(q, a, p)["ok"]


# ---------------------------------------------------------------------------
# planted mistakes in a copy of the oracle must be caught by these cases
# ---------------------------------------------------------------------------

_SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "oracle", "base_oracle.c")

# (what the mistake is, text in base_oracle.c, replacement)
MUTATIONS = [
    ("equal bids: the larger token wins",
     "if (a->tok != b->tok) return (a->tok < b->tok) ? -1 : 1;",
     "if (a->tok != b->tok) return (a->tok > b->tok) ? -1 : 1;"),
    ("equal values: the highest expert wins",
     "if (v > v1) { v1 = v; best = e; }",
     "if (v >= v1) { v1 = v; best = e; }"),
    ("price of a full expert: its second-lowest held bid",
     "if (keep == C) price[e] = c[C - 1].bid;",
     "if (keep == C) price[e] = c[C > 1 ? C - 2 : 0].bid;"),
    ("price set although the expert is not full",
     "if (keep == C) price[e] = c[C - 1].bid;",
     "if (keep > 0) price[e] = c[keep - 1].bid;"),
    ("prices reset at every phase",
     "for (int e = 0; e < E; ++e) held_cnt[e] = 0;",
     "for (int e = 0; e < E; ++e) { held_cnt[e] = 0; price[e] = 0; }"),
]


def _run_auction(L, q, max_rounds=10000):
    T, E = q.shape
    i32p = ctypes.POINTER(ctypes.c_int32)
    i64p = ctypes.POINTER(ctypes.c_int64)
    assign = np.full(T, -1, dtype=np.int32)
    price = np.zeros(E, dtype=np.int64)
    st = np.zeros(6, dtype=np.int64)
    tr = np.zeros(max_rounds, dtype=np.int32)
    L.orc_auction(q.ctypes.data_as(i32p), T, E, max_rounds, assign.ctypes.data_as(i32p),
                  price.ctypes.data_as(i64p), st.ctypes.data_as(i64p), tr.ctypes.data_as(i32p),
                  max_rounds)
    stats = dict(status=st[0], phases=st[1], rounds=st[2], final_eps=st[3], objective=st[4],
                 bids=st[5])
    return assign, price, stats, tr[:min(int(st[2]), max_rounds)]


def _compile(src_text, tmpdir, name):
    c = os.path.join(tmpdir, name + ".c")
    so = os.path.join(tmpdir, name + ".so")
    with open(c, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-shared", "-fPIC", "-o", so, c])
    L = ctypes.CDLL(so)
    L.orc_auction.restype = ctypes.c_int
    L.orc_auction.argtypes = [ctypes.POINTER(ctypes.c_int32), ctypes.c_int, ctypes.c_int,
                              ctypes.c_int64, ctypes.POINTER(ctypes.c_int32),
                              ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64),
                              ctypes.POINTER(ctypes.c_int32), ctypes.c_int64]
    return L


def _passes_all(L):
    for _, q, exp in hand_cases():
        try:
            check_result(exp, *_run_auction(L, q))
        except AssertionError:
            return False
    return True


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_mutations_are_caught(tmp_path):
    with open(_SRC) as f:
        src = f.read()
    # the unmodified source passes (the harness itself is sound)
    assert _passes_all(_compile(src, str(tmp_path), "unmodified"))
    for i, (what, old, new) in enumerate(MUTATIONS):
        assert src.count(old) == 1, "mutation target moved: " + what
        L = _compile(src.replace(old, new), str(tmp_path), "mut%d" % i)
        assert not _passes_all(L), "no hand-worked case catches: " + what
