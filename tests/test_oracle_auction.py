"""Pins of the oracle's balanced assignment (eq. 2 of "BASE Layers:
Simplifying Training of Large, Sparse Models", Method / "Training
assignment") against things other than itself: exhaustive enumeration, the
Hungarian method the page names as the alternative solver, the LP-duality
certificate, and invariances of eq. 2."""
import math

import numpy as np
import pytest

from balanced_token_expert_b200 import synth


def _rand_q(rng, T, E, small):
    if small:
        return rng.integers(0, 4, size=(T, E)).astype(np.int32)   # many ties
    return rng.integers(-300000, 300000, size=(T, E)).astype(np.int32)


def test_bruteforce_counts_every_balanced_assignment(orc):
    # the number of balanced assignments is the multinomial T! / (C!)^E
    q = np.zeros((8, 2), dtype=np.int32)
    _, _, n_assign, n_opt = orc.bruteforce(q)
    assert n_assign == math.factorial(8) // math.factorial(4) ** 2 == 70
    assert n_opt == 70  # all-zero scores: every assignment is optimal
    q = np.zeros((12, 3), dtype=np.int32)
    assert orc.bruteforce(q)[2] == math.factorial(12) // math.factorial(4) ** 3 == 34650


@pytest.mark.parametrize("T,E", [(8, 2), (12, 3)])
def test_auction_matches_bruteforce(orc, T, E):
    rng = np.random.default_rng(1234 + T)
    for seed in range(1000):
        q = _rand_q(rng, T, E, small=(seed % 2 == 1))
        a, p, st = orc.auction(q)
        best, _, _, _ = orc.bruteforce(q)
        assert st["status"] == 0
        assert st["objective"] == best, (seed, q.tolist())
        assert st["final_eps"] == 1
        assert np.all(np.bincount(a, minlength=E) == T // E)
        assert orc.certificate(q, a, p)["ok"]


def test_hungarian_matches_bruteforce(orc):
    rng = np.random.default_rng(7)
    for seed in range(200):
        for T, E in ((8, 2), (12, 3), (12, 4), (6, 6)):
            q = _rand_q(rng, T, E, small=(seed % 3 == 0))
            hv, ha = orc.hungarian(q)
            assert hv == orc.bruteforce(q)[0]
            assert np.all(np.bincount(ha, minlength=E) == T // E)
            assert int(q[np.arange(T), ha].sum()) == hv


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_auction_matches_hungarian_routing_ref(orc, seed):
    inp = synth.make_inputs(synth.WORKLOADS["routing_ref"], seed)
    q = orc.quantize(orc.scores(inp.h, inp.w))
    a, p, st = orc.auction(q)
    hv, _ = orc.hungarian(q)
    assert st["status"] == 0 and st["objective"] == hv
    assert orc.certificate(q, a, p)["ok"]


@pytest.mark.parametrize("T,E", [(256, 4), (300, 3), (384, 16), (128, 2), (64, 64), (512, 512)])
def test_auction_matches_hungarian_random(orc, T, E):
    rng = np.random.default_rng(T * 31 + E)
    for small in (False, True):
        q = _rand_q(rng, T, E, small)
        a, p, st = orc.auction(q)
        hv, _ = orc.hungarian(q)
        assert st["objective"] == hv
        assert orc.certificate(q, a, p)["ok"]


def test_auction_reduces_to_assignment_when_one_token_per_expert(orc):
    # E == T (C = 1) is the ordinary assignment problem
    rng = np.random.default_rng(5)
    q = rng.integers(-1000, 1000, size=(40, 40)).astype(np.int32)
    a, p, st = orc.auction(q)
    assert sorted(a.tolist()) == list(range(40))
    assert st["objective"] == orc.hungarian(q)[0]


def test_auction_equals_greedy_when_greedy_is_balanced(orc):
    # every token's favourite expert is t % E with a margin: greedy is balanced
    rng = np.random.default_rng(9)
    T, E = 96, 8
    q = rng.integers(0, 1000, size=(T, E)).astype(np.int32)
    q[np.arange(T), np.arange(T) % E] += 5000
    ga, gc = orc.greedy(q)
    assert np.all(gc == T // E)
    a, p, st = orc.auction(q)
    assert st["objective"] == int(q[np.arange(T), ga].sum())


def test_expert_and_token_offsets(orc):
    # eq. 2's constraint fixes how many tokens each expert takes, so adding d_e
    # to column e shifts every feasible objective by C sum d_e, and adding c_t
    # to row t shifts it by sum c_t: the optimum moves by exactly that much.
    rng = np.random.default_rng(11)
    T, E = 192, 6
    C = T // E
    q = rng.integers(-50000, 50000, size=(T, E)).astype(np.int32)
    base = orc.auction(q)[2]["objective"]
    d = rng.integers(-20000, 20000, size=E).astype(np.int32)
    c = rng.integers(-20000, 20000, size=T).astype(np.int32)
    a1, _, st1 = orc.auction(q + d[None, :])
    assert st1["objective"] == base + C * int(d.sum())
    assert int(q[np.arange(T), a1].sum()) == base
    st2 = orc.auction(q + c[:, None])[2]
    assert st2["objective"] == base + int(c.sum())


@pytest.mark.parametrize("name", ["routing_ref", "layer_fwd", "skewed", "large_routing",
                                  "layer_fwd_bwd"])
def test_certificate_on_every_workload(orc, name):
    inp = synth.make_inputs(synth.WORKLOADS[name], 0, with_weights=False, with_dout=False)
    q = orc.quantize(orc.scores(inp.h, inp.w))
    if inp.bump_tokens is not None:
        q[inp.bump_tokens.numpy(), 0] += int(round(inp.bump_value * orc.QSCALE))
    a, p, st = orc.auction(q)
    cert = orc.certificate(q, a, p)
    assert st["status"] == 0 and st["final_eps"] == 1
    assert cert["ok"], cert
    assert cert["objective"] == st["objective"]
    assert st["bids"] >= st["phases"] * q.shape[0]


def test_certificate_rejects_planted_mistakes(orc):
    # the checks have teeth: a swap that loses objective, an unbalanced
    # assignment and a shifted price vector must each fail
    rng = np.random.default_rng(3)
    T, E = 64, 4
    q = rng.integers(-100000, 100000, size=(T, E)).astype(np.int32)
    a, p, st = orc.auction(q)
    assert orc.certificate(q, a, p)["ok"]
    worst = None
    for i in range(T):
        for j in range(T):
            if a[i] != a[j]:
                delta = (int(q[i, a[j]]) + int(q[j, a[i]])) - (int(q[i, a[i]]) + int(q[j, a[j]]))
                if worst is None or delta < worst[0]:
                    worst = (delta, i, j)
    delta, i, j = worst
    assert delta < 0
    b = a.copy()
    b[i], b[j] = a[j], a[i]
    assert not orc.certificate(q, b, p)["ok"]
    c = a.copy()
    c[0] = (c[0] + 1) % E
    assert not orc.certificate(q, c, p)["balanced"]
    p2 = p.copy()
    p2[0] += 10 * (T + 1) * 100000
    assert not orc.certificate(q, a, p2)["ok"]


def test_round_cap_and_bad_arguments(orc):
    rng = np.random.default_rng(0)
    q = rng.integers(-1000, 1000, size=(64, 4)).astype(np.int32)
    st = orc.auction(q, max_rounds=1)[2]
    assert st["status"] == 3  # not converged
    assert orc.auction(q[:63])[2]["status"] == 1  # T % E != 0
    assert orc.auction(q[:, :1])[2]["status"] == 1  # E < 2


def test_epsilon_schedule(orc):
    # phases = 1 + number of divisions by 8 from eps0 = R (T+1) / 50 down to 1
    rng = np.random.default_rng(21)
    T, E = 128, 4
    q = rng.integers(-65536, 65536, size=(T, E)).astype(np.int32)
    R = int(q.max()) - int(q.min())
    eps = max(1, R * (T + 1) // 50)
    phases = 1
    while eps > 1:
        eps = max(1, eps // 8)
        phases += 1
    st = orc.auction(q)[2]
    assert st["phases"] == phases
    # equal scores: range 0 gives eps = 1 and a single phase
    st0 = orc.auction(np.zeros((T, E), dtype=np.int32))[2]
    assert st0["phases"] == 1 and st0["objective"] == 0
