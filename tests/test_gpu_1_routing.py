"""GPU parity of the routing steps (scores, greedy, balanced auction,
permute, combine) against the CPU oracle, through the C ABI."""
import numpy as np
import pytest
import torch

from _util import close_scores, dev, to_np
from balanced_token_expert_b200 import binding as B
from balanced_token_expert_b200 import buffers, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def no_device_error():
    B.base_device_error(clear=True)
    yield
    torch.cuda.synchronize()
    assert B.base_device_error(clear=True) == 0


def gpu_auction(q_np, max_rounds=None, trace=False):
    T, E = q_np.shape
    q = dev(q_np)
    assign = torch.full((T,), -1, dtype=torch.int32, device="cuda")
    price = torch.zeros(E, dtype=torch.int64, device="cuda")
    st = buffers.stats()
    ws = buffers.workspace(T, E)
    u = torch.full((200000,), -1, dtype=torch.int32, device="cuda") if trace else None
    if max_rounds is None and not trace:
        B.base_assign_balanced(q, assign, price, st, ws)
    else:
        B.base_assign_balanced_ex(q, assign, price, st, ws, max_rounds or 1000000, u_trace=u)
    torch.cuda.synchronize()
    out = (to_np(assign), to_np(price), buffers.stats_dict(st))
    if trace:
        out = out + (to_np(u)[: out[2]["rounds"]],)
    return out


def oracle_q(orc, wl, seed=0):
    inp = synth.make_inputs(wl, seed, with_weights=False, with_dout=False)
    s = orc.scores(inp.h, inp.w)
    q = orc.quantize(s)
    if inp.bump_tokens is not None:
        q[inp.bump_tokens.numpy(), 0] += int(round(inp.bump_value * orc.QSCALE))
    return inp, s, q


# ------------------------------------------------------------------ scores
def test_scores_fp32_routing_reference(orc):
    for seed in (0, 1, 2):
        inp = synth.make_inputs(synth.WORKLOADS["routing_ref"], seed)
        T, E = 512, 8
        s = torch.empty(T, E, device="cuda")
        q = torch.empty(T, E, dtype=torch.int32, device="cuda")
        B.base_scores(dev(inp.h), dev(inp.w), s, q)
        torch.cuda.synchronize()
        so = orc.scores(inp.h, inp.w)
        ok, worst = close_scores(to_np(s), so, 1e-5)
        assert ok, worst
        sg, qg = to_np(s), to_np(q)
        # q is the kernel's own fp32 s rounded half-to-even after scaling by 2^16
        assert np.array_equal(qg, np.rint(sg.astype(np.float32) * np.float32(65536)).astype(np.int32))
        qo = orc.quantize(so)
        assert np.abs(qg.astype(np.int64) - qo).max() <= 1


# token tails (T not a multiple of the 128-row tile), column tails (D not a
# multiple of the 64-column k-block) and E from 2 to 300 (the 16- to 256-wide
# N tiles)
@pytest.mark.parametrize("T,E,D", [(1000, 16, 200), (333, 40, 64), (256, 8, 128), (640, 300, 96),
                                   (129, 128, 1024), (1001, 3, 72), (31, 2, 8), (4099, 16, 1032),
                                   (32767, 16, 256), (40000, 16, 64)])
def test_scores_bf16_shapes(orc, T, E, D):
    wl = synth.WORKLOADS["layer_fwd"].scaled(T=T, E=E, D=D, F=0)
    inp = synth.make_inputs(wl, 7)
    s = torch.empty(T, E, device="cuda")
    q = torch.empty(T, E, dtype=torch.int32, device="cuda")
    B.base_scores(dev(inp.h), dev(inp.w), s, q)
    torch.cuda.synchronize()
    ok, worst = close_scores(to_np(s), orc.scores(inp.h, inp.w), 1e-5)
    assert ok, worst
    sg = to_np(s)
    assert np.array_equal(to_np(q), np.rint(sg * np.float32(65536)).astype(np.int32))


@pytest.mark.parametrize("name", ["layer_fwd", "skewed", "large_routing"])
def test_scores_bf16_full_workloads(orc, name):
    wl = synth.WORKLOADS[name]
    inp = synth.make_inputs(wl, 0, with_weights=False, with_dout=False)
    s = torch.empty(wl.T, wl.E, device="cuda")
    q = torch.empty(wl.T, wl.E, dtype=torch.int32, device="cuda")
    B.base_scores(dev(inp.h), dev(inp.w), s, q)
    torch.cuda.synchronize()
    rows = np.random.default_rng(0).choice(wl.T, size=min(wl.T, 4096), replace=False)
    so = orc.scores(inp.h[rows], inp.w)
    sg = to_np(s)
    ok, worst = close_scores(sg[rows], so, 1e-5)
    assert ok, worst
    assert np.array_equal(to_np(q), np.rint(sg * np.float32(65536)).astype(np.int32))


# ------------------------------------------------------------------ greedy
@pytest.mark.parametrize("T,E,small", [(512, 8, False), (1000, 5, True), (4096, 16, False),
                                       (3000, 33, True), (8192, 128, False), (777, 1000, True),
                                       (64, 2, True)])
def test_greedy_bit_exact(orc, T, E, small):
    rng = np.random.default_rng(T + E)
    q = (rng.integers(0, 3, size=(T, E)) if small else
         rng.integers(-300000, 300000, size=(T, E))).astype(np.int32)
    a = torch.empty(T, dtype=torch.int32, device="cuda")
    c = torch.empty(E, dtype=torch.int32, device="cuda")
    B.base_assign_greedy(dev(q), a, c)
    torch.cuda.synchronize()
    ao, co = orc.greedy(q)
    assert np.array_equal(to_np(a), ao)
    assert np.array_equal(to_np(c), co)


def test_greedy_large_routing(orc):
    _, _, q = oracle_q(orc, synth.WORKLOADS["large_routing"])
    T, E = q.shape
    a = torch.empty(T, dtype=torch.int32, device="cuda")
    c = torch.empty(E, dtype=torch.int32, device="cuda")
    B.base_assign_greedy(dev(q), a, c)
    torch.cuda.synchronize()
    ao, co = orc.greedy(q)
    assert np.array_equal(to_np(a), ao) and np.array_equal(to_np(c), co)


# ------------------------------------------------------------------ auction
def _check_auction(orc, q):
    a, p, st = gpu_auction(q)
    ao, po, so = orc.auction(q)
    assert st == so, (st, so)
    assert np.array_equal(a, ao)
    assert np.array_equal(p, po)
    assert orc.certificate(q, a, p)["ok"]
    return st


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_auction_routing_reference_is_optimal_and_bit_exact(orc, seed):
    _, _, q = oracle_q(orc, synth.WORKLOADS["routing_ref"], seed)
    st = _check_auction(orc, q)
    assert st["objective"] == orc.hungarian(q)[0]


# C = T/E >= ~3000 (the last three) leaves no room for the sorted held sets in
# shared memory: the wide rounds then resolve with the radix select and the
# fringe merges instead
@pytest.mark.parametrize("T,E,small", [(8, 2, False), (12, 3, True), (64, 64, False),
                                       (100, 4, True), (1000, 8, False), (2048, 2, False),
                                       (4096, 1024, False), (6000, 3, True), (8192, 16, True),
                                       (30000, 40, False), (16384, 2, False), (24000, 3, True),
                                       (65536, 8, False)])
def test_auction_shapes_bit_exact(orc, T, E, small):
    rng = np.random.default_rng(T * 7 + E)
    q = (rng.integers(0, 4, size=(T, E)) if small else
         rng.integers(-300000, 300000, size=(T, E))).astype(np.int32)
    _check_auction(orc, q)


def test_auction_many_tiny_problems(orc):
    rng = np.random.default_rng(99)
    for i in range(60):
        T, E = [(8, 2), (12, 3), (12, 4), (16, 8)][i % 4]
        q = (rng.integers(0, 4, size=(T, E)) if i % 2 else
             rng.integers(-1000, 1000, size=(T, E))).astype(np.int32)
        a, p, st = gpu_auction(q)
        ao, po, so = orc.auction(q)
        assert st == so and np.array_equal(a, ao) and np.array_equal(p, po)
        assert st["objective"] == orc.bruteforce(q)[0] if T <= 12 else True


@pytest.mark.parametrize("name", ["layer_fwd", "skewed", "large_routing", "layer_fwd_bwd"])
def test_auction_full_workloads(orc, name):
    _, _, q = oracle_q(orc, synth.WORKLOADS[name])
    _check_auction(orc, q)


@pytest.mark.parametrize("name", ["routing_ref", "layer_fwd", "skewed"])
def test_auction_trajectory_matches_round_by_round(orc, name):
    # the number of bidders of every round, not only the totals
    _, _, q = oracle_q(orc, synth.WORKLOADS[name])
    a, p, st, u = gpu_auction(q, trace=True)
    ao, po, so, uo = orc.auction(q, trace=True)
    assert st == so
    assert np.array_equal(u, uo)


def test_auction_hand_worked_cases():
    # the tie, price and phase rules on the cases worked through by hand in
    # test_oracle_auction_hand.py: the GPU must reproduce the paper working
    from test_oracle_auction_hand import check_result, hand_cases
    for name, q, exp in hand_cases():
        a, p, st, u = gpu_auction(q, trace=True)
        check_result(exp, a, p, st, u)


@pytest.mark.parametrize("name", ["skewed", "large_routing"])
def test_auction_is_deterministic(name):
    # bidders of a wide round reserve bucket space with atomics, in whatever
    # order the SMs get there; the result must not depend on that order: five
    # runs on the same q, reusing the workspace, give the same bits
    wl = synth.WORKLOADS[name]
    inp = synth.make_inputs(wl, 1, with_weights=False, with_dout=False)
    q = torch.empty(wl.T, wl.E, dtype=torch.int32, device="cuda")
    B.base_scores(dev(inp.h), dev(inp.w), None, q)
    if inp.bump_tokens is not None:
        q[inp.bump_tokens.cuda(), 0] += int(round(inp.bump_value * 65536))
    ws = buffers.workspace(wl.T, wl.E)
    runs = []
    for _ in range(5):
        assign = torch.full((wl.T,), -1, dtype=torch.int32, device="cuda")
        price = torch.full((wl.E,), -7, dtype=torch.int64, device="cuda")
        st = buffers.stats()
        u = torch.full((100000,), -1, dtype=torch.int32, device="cuda")
        B.base_assign_balanced_ex(q, assign, price, st, ws, 1000000, u_trace=u)
        torch.cuda.synchronize()
        runs.append((to_np(assign), to_np(price), buffers.stats_dict(st), to_np(u)))
    a0, p0, s0, u0 = runs[0]
    assert s0["status"] == 0
    for a, p, s, u in runs[1:]:
        assert s == s0
        assert np.array_equal(a, a0) and np.array_equal(p, p0) and np.array_equal(u, u0)


def test_auction_equal_scores_single_phase(orc):
    q = np.zeros((256, 8), dtype=np.int32)
    _check_auction(orc, q)


def test_auction_round_cap_reports_not_converged(orc):
    _, _, q = oracle_q(orc, synth.WORKLOADS["routing_ref"], 0)
    a, p, st = gpu_auction(q, max_rounds=5)
    assert st["status"] == 3 and st["rounds"] == 5
    so = orc.auction(q, max_rounds=5)[2]
    assert so["status"] == 3 and so["rounds"] == 5 and so["bids"] == st["bids"]


@pytest.mark.parametrize("name", ["layer_fwd", "skewed"])
def test_auction_round_cap_in_the_last_rounds_of_a_phase(orc, name):
    # caps that fall in the tails of phases (few bidders, one warp) and in
    # the middle of the run: the same stopping point as the oracle
    _, _, q = oracle_q(orc, synth.WORKLOADS[name])
    R = orc.auction(q)[2]["rounds"]
    for cap in sorted({R - 1, R - 2, R - 3, R - 6, R - 11, R // 2, R // 3 + 1}):
        a, p, st = gpu_auction(q, max_rounds=cap)
        so = orc.auction(q, max_rounds=cap)[2]
        assert st == so, (cap, st, so)


# ------------------------------------------------------------------ permute / combine
# the sort by expert splits the tokens into up to 128 slices of 512..8192
# consecutive tokens: one slice (T <= 512), a ragged last slice, the 8192-token
# cap, and the three full workload shapes (balanced counts, shuffled experts)
@pytest.mark.parametrize("T,E,D,kind", [(1536, 4, 64, "balanced"), (1000, 5, 200, "ragged"),
                                        (4096, 128, 128, "ragged"), (333, 7, 8, "ragged"),
                                        (2048, 2, 1024, "empty-expert"), (16384, 1024, 8, "ragged"),
                                        (16385, 3, 16, "ragged"), (40000, 64, 64, "ragged"),
                                        (20000, 5, 8, "empty-expert"),
                                        (8192, 16, 1024, "shuffled-balanced"),
                                        (32768, 32, 2048, "shuffled-balanced"),
                                        (131072, 128, 2048, "shuffled-balanced")])
def test_permute_and_combine_bit_exact(orc, T, E, D, kind):
    rng = np.random.default_rng(T + D)
    if kind == "balanced":
        q = rng.integers(-100000, 100000, size=(T, E)).astype(np.int32)
        assign = orc.auction(q)[0]
    elif kind == "shuffled-balanced":
        assign = rng.permutation(np.repeat(np.arange(E, dtype=np.int32), T // E))
    elif kind == "empty-expert":
        assign = np.zeros(T, dtype=np.int32)
    else:
        assign = rng.integers(0, E, size=T).astype(np.int32)
    h = torch.randn(T, D, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    s = rng.standard_normal((T, E)).astype(np.float32)
    perm = torch.empty(T, dtype=torch.int32, device="cuda")
    inv = torch.empty_like(perm)
    offs = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    xp = torch.empty(T, D, dtype=torch.bfloat16, device="cuda")
    gate = torch.empty(T, dtype=torch.float32, device="cuda")
    ws = buffers.workspace(T, E, D)
    B.base_permute(dev(h), dev(assign), E, perm, inv, offs, xp, dev(s), gate, ws)
    out = torch.empty_like(xp)
    B.base_combine(xp, perm, out)
    torch.cuda.synchronize()
    po, io, oo = orc.permutation(assign, E)
    assert np.array_equal(to_np(perm), po)
    assert np.array_equal(to_np(inv), io)
    assert np.array_equal(to_np(offs), oo)
    assert torch.equal(xp.cpu(), h[torch.from_numpy(po.astype(np.int64))])
    assert np.array_equal(to_np(gate), s[po, assign[po]])
    assert torch.equal(out.cpu(), h)  # combine undoes the permutation exactly


def test_out_of_range_entries_are_recorded_not_followed():
    # the kernels' own range checks: an expert index outside [0, E) in the
    # assignment (2001) and a row index outside [0, T) in the permutation
    # (2002) are recorded in the device error word and skipped
    T, E, D = 1000, 5, 64
    B.base_device_error(clear=True)
    assign = torch.randint(0, E, (T,), dtype=torch.int32, generator=torch.Generator().manual_seed(1))
    assign[17] = E
    perm = torch.empty(T, dtype=torch.int32, device="cuda")
    inv = torch.empty_like(perm)
    offs = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    B.base_permute(None, assign.cuda(), E, perm, inv, offs, None, ws=buffers.workspace(T, E, D))
    torch.cuda.synchronize()
    assert B.base_device_error(clear=True) == 2001
    assert int(offs[E].item()) == T - 1  # the bad token is left out
    y = torch.randn(T, D).to(torch.bfloat16).cuda()
    bad = torch.arange(T, dtype=torch.int32, device="cuda")
    bad[3] = T
    out = torch.zeros(T, D, dtype=torch.bfloat16, device="cuda")
    B.base_combine(y, bad, out)
    torch.cuda.synchronize()
    assert B.base_device_error(clear=True) == 2002
    keep = torch.ones(T, dtype=torch.bool)
    keep[3] = False
    assert torch.equal(out.cpu()[keep], y.cpu()[keep])


# ------------------------------------------------------------------ non-finite scores
def test_sanitize_scores_bit_exact(orc):
    rng = np.random.default_rng(8)
    T, E = 1000, 7
    s = rng.standard_normal((T, E)).astype(np.float32)
    bad = rng.choice(T * E, size=40, replace=False)
    s.flat[bad] = [(np.nan, np.inf, -np.inf)[i % 3] for i in range(40)]
    ws = buffers.workspace(T, E)
    sg = dev(s)
    q = torch.zeros(T, E, dtype=torch.int32, device="cuda")
    B.base_sanitize_scores(sg, q, ws)
    torch.cuda.synchronize()
    so = orc.sanitize_scores(s)
    assert np.array_equal(to_np(sg), so)
    qn = to_np(q)
    assert np.array_equal(qn.flat[bad], orc.quantize(so).flat[bad])
    keep = np.ones(T * E, dtype=bool)
    keep[bad] = False
    assert np.all(qn.flat[keep] == 0)  # only the replaced entries are written
    # all finite: nothing changes; nothing finite: zeros
    f = rng.standard_normal((T, E)).astype(np.float32)
    fg = dev(f)
    B.base_sanitize_scores(fg, None, ws)
    n = dev(np.full((64, 4), np.nan, dtype=np.float32))
    nq = torch.full((64, 4), 5, dtype=torch.int32, device="cuda")
    B.base_sanitize_scores(n, nq, ws)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(fg), f)
    assert np.all(to_np(n) == 0.0) and np.all(to_np(nq) == 0)


def test_layer_fwd_sanitizes_non_finite_scores(orc):
    # tokens whose features hold NaN or Inf have non-finite affinities; with
    # BASE_ROUTE_SANITIZE the layer gives them the smallest finite score and
    # routes every token exactly as the oracle's auction does on those scores
    from _util import close_rel_rms
    wl = synth.WORKLOADS["layer_fwd"].scaled(T=2048, E=8, D=256, F=512)
    inp = synth.make_inputs(wl, 5)
    h = inp.h.clone()
    h[3] = float("nan")
    h[100, 7] = float("inf")
    h[2047, :5] = float("-inf")
    badrows = [3, 100, 2047]
    T, E, D, F = wl.T, wl.E, wl.D, wl.F
    sv = buffers.layer_saved(T, E, D, F, for_backward=False)
    out = torch.empty(T, D, dtype=torch.bfloat16, device="cuda")
    ws = buffers.workspace(T, E, D, F)
    B.base_layer_fwd(dev(h), dev(inp.w), dev(inp.W1), dev(inp.W2), B.BASE_RELU,
                     B.BASE_ROUTE_BALANCED | B.BASE_ROUTE_SANITIZE, out, sv, ws)
    torch.cuda.synchronize()
    s_g, q_g = to_np(sv["s"]), to_np(sv["q"])
    assert np.all(np.isfinite(s_g))
    assert np.all(s_g[badrows] == s_g.min())
    good = np.setdiff1d(np.arange(T), badrows)
    ok, worst = close_scores(s_g[good], orc.scores(h[good], inp.w), 1e-5)
    assert ok, worst
    assert np.array_equal(q_g, np.rint(s_g * np.float32(65536)).astype(np.int32))
    a_g = to_np(sv["assign"])
    ao, po, so = orc.auction(q_g)
    assert buffers.stats_dict(sv["stats"]) == so
    assert np.array_equal(a_g, ao) and np.array_equal(to_np(sv["price"]), po)
    fw = orc.layer_forward(h, inp.w, inp.W1, inp.W2, "relu", a_g)
    ok, worst = close_rel_rms(to_np(out)[good], fw["out"][good], 2e-2)
    assert ok, worst


# ------------------------------------------------------------------ fig. 9 solver
def gpu_fig9(q_np, max_iterations=100):
    T, E = q_np.shape
    assign = torch.full((T,), -1, dtype=torch.int32, device="cuda")
    price = torch.zeros(T, dtype=torch.int64, device="cuda")
    st = torch.zeros(4, dtype=torch.int64, device="cuda")
    B.base_assign_fig9(dev(q_np), assign, price, st, buffers.workspace_fig9(T, E), max_iterations)
    torch.cuda.synchronize()
    s = st.tolist()
    return to_np(assign), to_np(price), dict(status=s[0], rounds=s[1], eps=s[2], objective=s[3])


def test_fig9_hand_worked_cases():
    from test_oracle_fig9 import check_fig9, fig9_hand_cases
    for name, q, cap, exp in fig9_hand_cases():
        check_fig9(exp, *gpu_fig9(q, cap))


@pytest.mark.parametrize("T,E,small,cap", [(12, 3, True, 100), (512, 8, False, 100),
                                           (1000, 8, True, 100), (4096, 16, False, 2),
                                           (2048, 64, False, 100), (1536, 1536 // 16, True, 100)])
def test_fig9_bit_exact(orc, T, E, small, cap):
    rng = np.random.default_rng(T + 3 * E)
    q = (rng.integers(0, 4, size=(T, E)) if small else
         rng.integers(-300000, 300000, size=(T, E))).astype(np.int32)
    a, p, st = gpu_fig9(q, cap)
    ao, po, so = orc.fig9_auction(q, max_iterations=cap)
    assert st == so, (st, so)
    assert np.array_equal(a, ao) and np.array_equal(p, po)


@pytest.mark.parametrize("name", ["routing_ref", "layer_fwd"])
def test_fig9_workloads_bit_exact(orc, name):
    _, _, q = oracle_q(orc, synth.WORKLOADS[name])
    a, p, st = gpu_fig9(q)
    ao, po, so = orc.fig9_auction(q)
    assert st == so and np.array_equal(a, ao) and np.array_equal(p, po)
    assert st["objective"] <= orc.auction(q)[2]["objective"]  # never above the optimum


# ------------------------------------------------------------------ scores + greedy in one pass
@pytest.mark.parametrize("T,E,D", [(1000, 16, 200), (4099, 32, 256), (777, 100, 64),
                                   (8192, 128, 512), (640, 256, 128), (513, 300, 64),
                                   (2048, 2, 64), (1001, 7, 72), (32767, 16, 64), (40000, 16, 64)])
def test_scores_greedy_fused(orc, T, E, D):
    wl = synth.WORKLOADS["layer_fwd"].scaled(T=T, E=E, D=D, F=0)
    inp = synth.make_inputs(wl, 11)
    s = torch.empty(T, E, device="cuda")
    q = torch.empty(T, E, dtype=torch.int32, device="cuda")
    a = torch.full((T,), -1, dtype=torch.int32, device="cuda")
    c = torch.full((E,), 123, dtype=torch.int32, device="cuda")
    B.base_scores_greedy(dev(inp.h), dev(inp.w), s, q, a, c)
    torch.cuda.synchronize()
    sg, qg = to_np(s), to_np(q)
    ok, worst = close_scores(sg, orc.scores(inp.h, inp.w), 1e-5)
    assert ok, worst
    assert np.array_equal(qg, np.rint(sg * np.float32(65536)).astype(np.int32))
    ao, co = orc.greedy(qg)
    assert np.array_equal(to_np(a), ao)
    assert np.array_equal(to_np(c), co)


def test_scores_greedy_fused_with_ties_few_experts(orc):
    # E = 16 (the 16-wide N tile): the lowest expert wins ties, also between
    # columns the two epilogue warps of a lane quadrant scan (3 and 12)
    T, E, D = 1002, 16, 64
    h = torch.zeros(T, D)
    h[:, 0] = 1.0
    w = torch.zeros(E, D)
    w[[3, 12, 15], 0] = 0.5
    h[::3, 1] = 1.0
    w[12, 1] = 0.25           # every third row prefers expert 12
    hb, wb = h.to(torch.bfloat16), w.to(torch.bfloat16)
    q = torch.empty(T, E, dtype=torch.int32, device="cuda")
    a = torch.empty(T, dtype=torch.int32, device="cuda")
    c = torch.empty(E, dtype=torch.int32, device="cuda")
    B.base_scores_greedy(dev(hb), dev(wb), None, q, a, c)
    torch.cuda.synchronize()
    ao, co = orc.greedy(to_np(q))
    assert np.array_equal(to_np(a), ao) and np.array_equal(to_np(c), co)
    rows = np.arange(T)
    assert set(to_np(a)[rows % 3 != 0].tolist()) == {3} and set(to_np(a)[::3].tolist()) == {12}


def test_scores_greedy_fused_with_ties(orc):
    # equal scores in a row: the lowest expert wins, across the two column
    # halves of the epilogue too (E = 64: columns 0-31 and 32-63)
    T, E, D = 512, 64, 64
    h = torch.zeros(T, D)
    h[:, 0] = 1.0
    w = torch.zeros(E, D)
    w[[5, 40, 63], 0] = 0.5   # three experts tie on every row
    h[::2, 1] = 1.0
    w[40, 1] = 0.25            # even rows prefer expert 40
    hb, wb = h.to(torch.bfloat16), w.to(torch.bfloat16)
    q = torch.empty(T, E, dtype=torch.int32, device="cuda")
    a = torch.empty(T, dtype=torch.int32, device="cuda")
    B.base_scores_greedy(dev(hb), dev(wb), None, q, a)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(a), orc.greedy(to_np(q))[0])
    assert set(to_np(a)[1::2].tolist()) == {5} and set(to_np(a)[::2].tolist()) == {40}
