"""The expert-parallel exchange kernels (base_ep_dispatch, base_ep_combine)
with every worker's buffers on one GPU ("BASE Layers", wikillm.com summary,
Method: Sharding; fig. 2's forward pass).

With balanced routing every expert gets C = T/E of each worker's tokens, so
the expert-parallel layer on G workers computes, for each worker's tokens,
what the single-GPU layer with all E experts computes: the grouped GEMM's
result for a row does not depend on which other rows share its tile.  The
tests check the exchange maps element by element, the whole forward against
the single-GPU layer bit for bit (and against the oracle within the forward
tolerance), and that one call per worker gives what one call over all
workers gives."""
import pytest
import torch

from _util import close_rel_rms, dev, to_np
from balanced_token_expert_b200 import binding as B
from balanced_token_expert_b200 import buffers, synth
from balanced_token_expert_b200 import expert_parallel as ep

pytestmark = pytest.mark.gpu

FWD_TOL = 2e-2  # the forward's tolerance against the fp64 oracle (bf16 storage)


def _batches(G, T, E, D, F, seed):
    wl = synth.WORKLOADS["layer_fwd"].scaled(T=T, E=E, D=D, F=F)
    base = synth.make_inputs(wl, seed)
    hs = [dev(synth.make_inputs(wl, seed + 1 + g, with_weights=False).h) for g in range(G)]
    return wl, base, hs


def _route(h, w, E, ws):
    """scores, balanced assignment and the slot order of one worker"""
    T = h.shape[0]
    s = torch.empty(T, E, device="cuda")
    q = torch.empty(T, E, dtype=torch.int32, device="cuda")
    B.base_scores(h, w, s, q)
    a = torch.empty(T, dtype=torch.int32, device="cuda")
    B.base_assign_balanced(q, a, torch.empty(E, dtype=torch.int64, device="cuda"),
                           buffers.stats(), ws)
    perm = torch.empty(T, dtype=torch.int32, device="cuda")
    inv = torch.empty_like(perm)
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    gate = torch.empty(T, device="cuda")
    B.base_permute(None, a, E, perm, inv, off, None, s, gate, ws)
    return a, perm, gate


@pytest.mark.parametrize("G,T,E,D", [(2, 1024, 8, 256), (4, 2048, 16, 128), (8, 512, 8, 64)])
def test_ep_exchange_maps(G, T, E, D):
    wl, base, hs = _batches(G, T, E, D, 0, 3)
    w = dev(base.w)
    ws = buffers.workspace(T, E)
    C, El = T // E, E // G
    perms, gates = [], []
    for g in range(G):
        _, perm, gate = _route(hs[g], w, E, ws)
        perms.append(perm)
        gates.append(gate)
    recv = [torch.full((T, D), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(G)]
    rgate = [torch.full((T,), float("nan"), device="cuda") for _ in range(G)]
    B.base_ep_dispatch(hs, perms, gates, recv, rgate, 0, E)
    torch.cuda.synchronize()
    # recv_r[(j G + g) C + c] = h_g[perm_g[(r El + j) C + c]], the gate alike
    c = torch.arange(C, device="cuda")
    for r in range(G):
        for j in range(El):
            for g in range(G):
                rows = (j * G + g) * C + c
                slots = (r * El + j) * C + c
                assert torch.equal(recv[r][rows], hs[g][perms[g][slots].long()])
                assert torch.equal(rgate[r][rows], gates[g][slots])
    # back: out_g[perm_g[(r El + j) C + c]] = y_r[(j G + g) C + c]; y = recv
    # makes the round trip the identity
    outs = [torch.zeros(T, D, dtype=torch.bfloat16, device="cuda") for _ in range(G)]
    B.base_ep_combine(recv, perms, outs, 0, E)
    torch.cuda.synchronize()
    for g in range(G):
        assert torch.equal(outs[g], hs[g])
    assert B.base_device_error(clear=True) == 0


@pytest.mark.parametrize("G,T,E,D,F", [(2, 1024, 8, 256, 512), (4, 2048, 16, 128, 256)])
def test_ep_layer_matches_the_single_gpu_layer(orc, G, T, E, D, F):
    wl, base, hs = _batches(G, T, E, D, F, 5)
    w, W1, W2 = dev(base.w), dev(base.W1), dev(base.W2)
    El = E // G
    plan = ep.EPPlan(T=T, E=E, G=G)
    outs = ep.ep_layer_fwd_fused(hs, w, [W1[r * El:(r + 1) * El] for r in range(G)],
                                 [W2[r * El:(r + 1) * El] for r in range(G)], B.BASE_RELU, plan)
    torch.cuda.synchronize()
    ws = buffers.workspace(T, E, D, F)
    for g in range(G):
        sv = buffers.layer_saved(T, E, D, F, for_backward=False)
        ref = torch.empty(T, D, dtype=torch.bfloat16, device="cuda")
        B.base_layer_fwd(hs[g], w, W1, W2, B.BASE_RELU, B.BASE_ROUTE_BALANCED, ref, sv, ws)
        torch.cuda.synchronize()
        assert torch.equal(outs[g], ref)
        if g == 0:  # and the oracle, with the GPU's assignment
            expect = orc.layer_forward(hs[g].cpu(), base.w, base.W1, base.W2, "relu",
                                       to_np(sv["assign"]))["out"]
            ok, worst = close_rel_rms(to_np(outs[g]), expect, FWD_TOL)
            assert ok, worst
    assert B.base_device_error(clear=True) == 0


@pytest.mark.parametrize("G,T,E,D,F", [(2, 1024, 8, 256, 512), (4, 2048, 16, 128, 256)])
def test_ep_layer_with_shuffle(G, T, E, D, F):
    # the four exchanges of fig. 2 as fused kernels: the shuffle and the
    # unshuffle are the same exchange with one block of T/G rows per worker
    wl, base, hs = _batches(G, T, E, D, F, 11)
    w, W1, W2 = dev(base.w), dev(base.W1), dev(base.W2)
    El = E // G
    seeds = [100 + g for g in range(G)]
    plan = ep.EPPlan(T=T, E=E, G=G)
    outs = ep.ep_layer_fwd_fused(hs, w, [W1[r * El:(r + 1) * El] for r in range(G)],
                                 [W2[r * El:(r + 1) * El] for r in range(G)], B.BASE_RELU, plan,
                                 seeds=seeds)
    torch.cuda.synchronize()
    # reference: each worker's shuffled batch through the single-GPU layer,
    # every row then put back where it came from
    n = T // G
    sp = [ep.shuffle_permutation(T, sd).cuda() for sd in seeds]
    expect = [torch.empty(T, D, dtype=torch.bfloat16, device="cuda") for _ in range(G)]
    ws = buffers.workspace(T, E, D, F)
    for r in range(G):
        sh = torch.cat([hs[g][sp[g][r * n:(r + 1) * n]] for g in range(G)])
        sv = buffers.layer_saved(T, E, D, F, for_backward=False)
        y = torch.empty(T, D, dtype=torch.bfloat16, device="cuda")
        B.base_layer_fwd(sh, w, W1, W2, B.BASE_RELU, B.BASE_ROUTE_BALANCED, y, sv, ws)
        for g in range(G):
            expect[g][sp[g][r * n:(r + 1) * n]] = y[g * n:(g + 1) * n]
    torch.cuda.synchronize()
    for g in range(G):
        assert torch.equal(outs[g], expect[g])
    assert B.base_device_error(clear=True) == 0


def test_ep_one_call_per_worker_equals_one_call_for_all():
    G, T, E, D = 4, 1024, 8, 128
    wl, base, hs = _batches(G, T, E, D, 0, 7)
    w = dev(base.w)
    ws = buffers.workspace(T, E)
    perms, gates = [], []
    for g in range(G):
        _, perm, gate = _route(hs[g], w, E, ws)
        perms.append(perm)
        gates.append(gate)
    mk = lambda: [torch.zeros(T, D, dtype=torch.bfloat16, device="cuda") for _ in range(G)]  # noqa: E731
    mkg = lambda: [torch.zeros(T, device="cuda") for _ in range(G)]  # noqa: E731
    r_all, g_all, r_one, g_one = mk(), mkg(), mk(), mkg()
    B.base_ep_dispatch(hs, perms, gates, r_all, g_all, 0, E)
    for g in range(G):  # each source its own call, as a worker would
        B.base_ep_dispatch([hs[g]], [perms[g]], [gates[g]], r_one, g_one, g, E)
    torch.cuda.synchronize()
    for r in range(G):
        assert torch.equal(r_all[r], r_one[r]) and torch.equal(g_all[r], g_one[r])
    o_all, o_one = mk(), mk()
    B.base_ep_combine(r_all, perms, o_all, 0, E)
    for r in range(G):  # each receiver its own call
        B.base_ep_combine([r_all[r]], perms, o_one, r, E)
    torch.cuda.synchronize()
    for g in range(G):
        assert torch.equal(o_all[g], o_one[g]) and torch.equal(o_all[g], hs[g])


def test_ep_rejects_bad_shapes():
    T, E, D = 1024, 8, 64
    h = [torch.zeros(T, D, dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    p = [torch.zeros(T, dtype=torch.int32, device="cuda") for _ in range(3)]
    with pytest.raises(B.BaseError):  # 3 workers do not divide 8 experts
        B.base_ep_dispatch(h, p, None, h, None, 0, E)
    with pytest.raises(B.BaseError):  # gate without recv_gate
        B.base_ep_dispatch(h[:2], p[:2], [torch.zeros(T, device="cuda")] * 2, h[:2], None, 0, E)
    with pytest.raises(B.BaseError):  # sources past the last worker
        B.base_ep_dispatch(h[:2], p[:2], None, h[:2], None, 1, E)
