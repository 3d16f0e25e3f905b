"""GPU parity of the expert FFN (a6+a7), the fused layer forward and the
backward (a9) against the float64 CPU oracle, through the C ABI."""
import numpy as np
import pytest
import torch

from _util import close_rel_rms, close_scores, dev, to_np
from balanced_token_expert_b200 import binding as B
from balanced_token_expert_b200 import buffers, synth

pytestmark = pytest.mark.gpu

FWD_TOL = 2e-2
GRAD_TOL = 3e-2
ACT = {"relu": B.BASE_RELU, "gelu": B.BASE_GELU}


@pytest.fixture(autouse=True)
def no_device_error():
    B.base_device_error(clear=True)
    yield
    torch.cuda.synchronize()
    assert B.base_device_error(clear=True) == 0


def _assign(orc, q, routing):
    return orc.auction(q)[0] if routing == "balanced" else orc.greedy(q)[0]


def _ffn_case(orc, wl, seed, routing, experts=None):
    """Oracle-side inputs of the FFN step: permuted tokens, offsets, gate."""
    inp = synth.make_inputs(wl, seed)
    s = orc.scores(inp.h, inp.w)
    q = orc.quantize(s)
    assign = _assign(orc, q, routing)
    perm, inv, offsets = orc.permutation(assign, wl.E)
    x_perm = inp.h[torch.from_numpy(perm.astype(np.int64))]
    gate = s[perm, assign[perm]].astype(np.float32)
    return inp, s, assign, perm, inv, offsets, x_perm, gate


def _run_ffn(wl, inp, offsets, x_perm, gate):
    T, D, F = wl.T, wl.D, wl.F
    bf = torch.bfloat16
    y = torch.empty(T, D, dtype=bf, device="cuda")
    h1 = torch.empty(T, F, dtype=bf, device="cuda")
    a1 = torch.empty(T, F, dtype=bf, device="cuda")
    f = torch.empty(T, D, dtype=bf, device="cuda")
    ws = buffers.workspace(T, wl.E, D, F)
    B.base_expert_ffn(dev(x_perm), dev(offsets), dev(inp.W1), dev(inp.W2), ACT[wl.act], dev(gate),
                      y, h1, a1, f, ws)
    torch.cuda.synchronize()
    return y, h1, a1, f


@pytest.mark.parametrize("T,E,D,F,act,routing", [
    (1536, 4, 256, 512, "relu", "balanced"),
    (1000, 5, 200, 328, "gelu", "greedy"),
    (640, 2, 64, 256, "gelu", "balanced"),
    (2048, 16, 128, 384, "relu", "greedy"),
])
def test_expert_ffn_matches_oracle(orc, T, E, D, F, act, routing):
    wl = synth.WORKLOADS["layer_fwd"].scaled(T=T, E=E, D=D, F=F, act=act)
    inp, s, assign, perm, inv, offsets, x_perm, gate = _ffn_case(orc, wl, 1, routing)
    y, h1, a1, f = _run_ffn(wl, inp, offsets, x_perm, gate)
    r = orc.expert_ffn(x_perm, offsets, inp.W1, inp.W2, act, gate_s=gate)
    for name, g, o in (("y", y, r["y"]), ("a1", a1, r["a1"]), ("h1", h1, r["h1"]), ("f", f, r["f"])):
        ok, worst = close_rel_rms(to_np(g), o, FWD_TOL)
        assert ok, (name, worst)


def test_expert_ffn_full_layer_fwd_workload(orc):
    # the benchmarked shape (T=8192, E=16, D=1024, F=4096, ReLU); the oracle
    # recomputes two experts' slot segments in float64
    wl = synth.WORKLOADS["layer_fwd"]
    inp, s, assign, perm, inv, offsets, x_perm, gate = _ffn_case(orc, wl, 0, "balanced")
    y, h1, a1, f = _run_ffn(wl, inp, offsets, x_perm, gate)
    experts = [0, wl.E - 1]
    r = orc.expert_ffn(x_perm, offsets, inp.W1, inp.W2, wl.act, gate_s=gate, experts=experts)
    rows = np.concatenate([np.arange(offsets[e], offsets[e + 1]) for e in experts])
    for name, g, o in (("y", y, r["y"]), ("h1", h1, r["h1"]), ("f", f, r["f"])):
        ok, worst = close_rel_rms(to_np(g)[rows], o[rows], FWD_TOL)
        assert ok, (name, worst)


def _run_layer_fwd(wl, inp, routing, for_backward=False):
    T, E, D, F = wl.T, wl.E, wl.D, wl.F
    sv = buffers.layer_saved(T, E, D, F, for_backward=for_backward)
    out = torch.empty(T, D, dtype=torch.bfloat16, device="cuda")
    ws = buffers.workspace(T, E, D, F)
    B.base_layer_fwd(dev(inp.h), dev(inp.w), dev(inp.W1), dev(inp.W2), ACT[wl.act],
                     B.BASE_ROUTE_BALANCED if routing == "balanced" else B.BASE_ROUTE_GREEDY,
                     out, sv, ws)
    torch.cuda.synchronize()
    return out, sv, ws


def _check_routing_of_fwd(orc, inp, sv, routing):
    """The fused forward's routing against the oracle, step by step: the fp32
    scores within 1e-5, q the kernel's own s rounded, and the assignment (with
    prices and statistics for the auction) bit-exact with the oracle run on
    the GPU's q -- the one place where floating point decides an integer is
    the rounding of s, and both sides then take the same integer problem."""
    s_o = orc.scores(inp.h, inp.w)
    s_g, q_g = to_np(sv["s"]), to_np(sv["q"])
    ok, worst = close_scores(s_g, s_o, 1e-5)
    assert ok, worst
    assert np.array_equal(q_g, np.rint(s_g * np.float32(65536)).astype(np.int32))
    assert np.abs(q_g.astype(np.int64) - orc.quantize(s_o)).max() <= 1
    a_g = to_np(sv["assign"])
    if routing == "balanced":
        st = buffers.stats_dict(sv["stats"])
        ao, po, so = orc.auction(q_g)
        assert st == so, (st, so)
        assert np.array_equal(a_g, ao)
        assert np.array_equal(to_np(sv["price"]), po)
        assert orc.certificate(q_g, a_g, po)["ok"]
    else:
        assert np.array_equal(a_g, orc.greedy(q_g)[0])
    # the slot order is the oracle's permutation of that assignment
    po_, io_, oo_ = orc.permutation(a_g, q_g.shape[1])
    assert np.array_equal(to_np(sv["perm"]), po_)
    assert np.array_equal(to_np(sv["inv"]), io_)
    assert np.array_equal(to_np(sv["offsets"]), oo_)
    return a_g


def _layer_fwd_check(orc, wl, seed, routing, experts=None):
    inp = synth.make_inputs(wl, seed)
    out, sv, _ = _run_layer_fwd(wl, inp, routing)
    a_g = _check_routing_of_fwd(orc, inp, sv, routing)
    # outputs: the oracle's forward with the same assignment, token by token
    fw = orc.layer_forward(inp.h, inp.w, inp.W1, inp.W2, wl.act, a_g, experts=experts)
    keep = np.ones(wl.T, dtype=bool) if experts is None else np.isin(a_g, experts)
    ok, worst = close_rel_rms(to_np(out)[keep], fw["out"][keep], FWD_TOL)
    assert ok, worst


@pytest.mark.parametrize("routing", ["balanced", "greedy"])
@pytest.mark.parametrize("act", ["relu", "gelu"])
def test_layer_fwd_small(orc, routing, act):
    wl = synth.WORKLOADS["layer_fwd"].scaled(T=2048, E=8, D=256, F=512, act=act)
    _layer_fwd_check(orc, wl, 3, routing)


def test_layer_fwd_full_workload_sampled(orc):
    wl = synth.WORKLOADS["layer_fwd"]
    _layer_fwd_check(orc, wl, 0, "balanced", experts=[0, 7, 15])


def _bwd_case(orc, wl, seed, experts=None):
    """Everything the backward reads comes from the oracle's forward (rounded
    to bf16 where the layer stores bf16)."""
    inp = synth.make_inputs(wl, seed, with_dout=True)
    s = orc.scores(inp.h, inp.w)
    assign = orc.auction(orc.quantize(s))[0]
    fw = orc.layer_forward(inp.h, inp.w, inp.W1, inp.W2, wl.act, assign, experts=experts)
    g = orc.layer_backward(fw, inp.h, inp.w, inp.W1, inp.W2, wl.act, inp.dout, experts=experts)
    bf = torch.bfloat16
    T, E, D, F = wl.T, wl.E, wl.D, wl.F
    sv = buffers.layer_saved(T, E, D, F)
    sv["assign"].copy_(dev(assign))
    sv["perm"].copy_(dev(fw["perm"]))
    sv["inv"].copy_(dev(fw["inv"]))
    sv["offsets"].copy_(dev(fw["offsets"]))
    sv["gate"].copy_(dev(fw["gate_s"].astype(np.float32)))
    sv["x_perm"].copy_(dev(fw["x_perm"], bf))
    if experts is not None:
        # rows of the experts the oracle skipped are NaN; only the listed
        # experts are compared, so the others are fed zeros
        for k in ("a1", "f"):
            fw[k] = np.nan_to_num(fw[k])
    sv["a1"].copy_(dev(fw["a1"], bf))
    sv["h1"].copy_(dev(orc.act(fw["a1"], wl.act), bf))
    sv["f"].copy_(dev(fw["f"], bf))
    dh = torch.empty(T, D, dtype=bf, device="cuda")
    dw = torch.empty(E, D, dtype=torch.float32, device="cuda")
    dW1 = torch.empty(E, F, D, dtype=torch.float32, device="cuda")
    dW2 = torch.empty(E, D, F, dtype=torch.float32, device="cuda")
    ws = buffers.workspace(T, E, D, F)
    B.base_layer_bwd(dev(inp.h), dev(inp.w), dev(inp.W1), dev(inp.W2), ACT[wl.act], sv,
                     dev(inp.dout), dh, dw, dW1, dW2, ws)
    torch.cuda.synchronize()
    return fw, g, dict(dh=to_np(dh), dw=to_np(dw), dW1=to_np(dW1), dW2=to_np(dW2))


@pytest.mark.parametrize("act", ["relu", "gelu"])
@pytest.mark.parametrize("T,E,D,F", [(1024, 4, 256, 512), (2048, 8, 192, 320)])
def test_layer_bwd_matches_oracle(orc, T, E, D, F, act):
    wl = synth.WORKLOADS["layer_fwd_bwd"].scaled(T=T, E=E, D=D, F=F, act=act)
    fw, g, gg = _bwd_case(orc, wl, 5)
    for k in ("dh", "dw", "dW1", "dW2"):
        ok, worst = close_rel_rms(gg[k], g[k], GRAD_TOL)
        assert ok, (k, worst)


def test_layer_bwd_full_workload_sampled(orc):
    # the forward+backward workload (T=32768, E=32, D=2048, F=8192, GELU);
    # the oracle recomputes two experts in float64
    wl = synth.WORKLOADS["layer_fwd_bwd"]
    experts = [0, 31]
    fw, g, gg = _bwd_case(orc, wl, 0, experts=experts)
    offs = fw["offsets"]
    rows = np.concatenate([np.arange(offs[e], offs[e + 1]) for e in experts])
    toks = fw["perm"][rows]
    for k in ("dW1", "dW2"):
        for e in experts:
            ok, worst = close_rel_rms(gg[k][e], g[k][e], GRAD_TOL)
            assert ok, (k, e, worst)
    ok, worst = close_rel_rms(gg["dw"][experts], g["dw"][experts], GRAD_TOL)
    assert ok, ("dw", worst)
    ok, worst = close_rel_rms(gg["dh"][toks], g["dh"][toks], GRAD_TOL)
    assert ok, ("dh", worst)


def _training_step_check(orc, wl, seed, experts=None):
    """base_layer_fwd then base_layer_bwd on the GPU's own saved buffers, as
    the timed training step runs them.  The oracle runs its float64 forward
    with the GPU's assignment (itself checked bit-exact) and its backward on
    that forward; every stored activation and every gradient is compared."""
    inp = synth.make_inputs(wl, seed, with_dout=True)
    T, E, D, F = wl.T, wl.E, wl.D, wl.F
    out, sv, ws = _run_layer_fwd(wl, inp, "balanced", for_backward=True)
    a_g = _check_routing_of_fwd(orc, inp, sv, "balanced")
    bf = torch.bfloat16
    dh = torch.empty(T, D, dtype=bf, device="cuda")
    dw = torch.empty(E, D, dtype=torch.float32, device="cuda")
    dW1 = torch.empty(E, F, D, dtype=torch.float32, device="cuda")
    dW2 = torch.empty(E, D, F, dtype=torch.float32, device="cuda")
    B.base_layer_bwd(dev(inp.h), dev(inp.w), dev(inp.W1), dev(inp.W2), ACT[wl.act], sv,
                     dev(inp.dout), dh, dw, dW1, dW2, ws)
    torch.cuda.synchronize()
    fw = orc.layer_forward(inp.h, inp.w, inp.W1, inp.W2, wl.act, a_g, experts=experts)
    ex = list(range(E)) if experts is None else list(experts)
    offs = fw["offsets"]
    rows = np.concatenate([np.arange(offs[e], offs[e + 1]) for e in ex])
    toks = fw["perm"][rows]
    rows_t = torch.from_numpy(rows.astype(np.int64)).cuda()
    toks_t = torch.from_numpy(toks.astype(np.int64)).cuda()
    # the permuted tokens are the inputs' rows exactly; the gate is s[t, a_t]
    assert torch.equal(sv["x_perm"][rows_t].cpu(), inp.h[torch.from_numpy(toks.astype(np.int64))])
    ok, worst = close_scores(to_np(sv["gate"][rows_t]), fw["gate_s"][rows], 1e-5)
    assert ok, ("gate", worst)
    fwd = (("out", out[toks_t], fw["out"][toks]), ("a1", sv["a1"][rows_t], fw["a1"][rows]),
           ("h1", sv["h1"][rows_t], orc.act(fw["a1"][rows], wl.act)),
           ("f", sv["f"][rows_t], fw["f"][rows]), ("y_perm", sv["y_perm"][rows_t], fw["y_perm"][rows]))
    for name, g, o in fwd:
        ok, worst = close_rel_rms(to_np(g), o, FWD_TOL)
        assert ok, (name, worst)
    g = orc.layer_backward(fw, inp.h, inp.w, inp.W1, inp.W2, wl.act, inp.dout, experts=experts)
    for e in ex:
        for name, gg in (("dW1", dW1), ("dW2", dW2)):
            ok, worst = close_rel_rms(to_np(gg[e]), g[name][e], GRAD_TOL)
            assert ok, (name, e, worst)
    ok, worst = close_rel_rms(to_np(dw)[ex], g["dw"][ex], GRAD_TOL)
    assert ok, ("dw", worst)
    ok, worst = close_rel_rms(to_np(dh[toks_t]), g["dh"][toks], GRAD_TOL)
    assert ok, ("dh", worst)


@pytest.mark.parametrize("act", ["relu", "gelu"])
def test_training_step_small(orc, act):
    wl = synth.WORKLOADS["layer_fwd_bwd"].scaled(T=2048, E=8, D=256, F=512, act=act)
    _training_step_check(orc, wl, 4)


def test_training_step_full_workload_sampled(orc):
    # the forward+backward workload (T=32768, E=32, D=2048, F=8192, GELU) as
    # the benchmark times it; the oracle recomputes three experts in float64
    _training_step_check(orc, synth.WORKLOADS["layer_fwd_bwd"], 0, experts=[0, 17, 31])


def test_layer_bwd_rejects_unbalanced_shapes():
    wl = synth.WORKLOADS["layer_fwd_bwd"].scaled(T=96, E=4, D=64, F=64)
    T, E, D, F = wl.T, wl.E, wl.D, wl.F
    sv = buffers.layer_saved(T, E, D, F)
    z = torch.zeros
    with pytest.raises(B.BaseError) as ei:
        B.base_layer_bwd(z(T, D, dtype=torch.bfloat16, device="cuda"),
                         z(E, D, dtype=torch.bfloat16, device="cuda"),
                         z(E, F, D, dtype=torch.bfloat16, device="cuda"),
                         z(E, D, F, dtype=torch.bfloat16, device="cuda"), B.BASE_RELU, sv,
                         z(T, D, dtype=torch.bfloat16, device="cuda"),
                         z(T, D, dtype=torch.bfloat16, device="cuda"),
                         z(E, D, device="cuda"), z(E, F, D, device="cuda"),
                         z(E, D, F, device="cuda"), buffers.workspace(T, E, D, F))
    assert ei.value.status == 6  # C = 24 is not a multiple of 64


# ------------------------------------------------------------------ the released code's variant
def _blend_inputs(wl, S, seed):
    """The workload's inputs plus S sublayers of weights per expert (the
    first sublayer's are the workload's own W1 / W2) and layer-norm gains and
    biases near (1, 0)."""
    inp = synth.make_inputs(wl, seed)
    extra = synth.make_stack_params(wl, S, seed)
    W1 = torch.cat([inp.W1[:, None], extra["W1"]], dim=1) if S > 1 else inp.W1[:, None]
    W2 = torch.cat([inp.W2[:, None], extra["W2"]], dim=1) if S > 1 else inp.W2[:, None]
    return inp, W1.contiguous(), W2.contiguous(), extra["gamma"], extra["beta"]


def _blend_check(orc, wl, S, seed, routing, experts=None):
    inp, W1, W2, gam, bet = _blend_inputs(wl, S, seed)
    T, E, D, F = wl.T, wl.E, wl.D, wl.F
    sv = buffers.layer_saved(T, E, D, F, for_backward=False)
    out = torch.empty(T, D, dtype=torch.bfloat16, device="cuda")
    ws = buffers.workspace_blend(T, E, D, F)
    B.base_layer_fwd_blend(dev(inp.h), dev(inp.w), dev(W1), dev(W2), dev(gam), dev(bet),
                           ACT[wl.act],
                           B.BASE_ROUTE_BALANCED if routing == "balanced" else B.BASE_ROUTE_GREEDY,
                           out, sv, ws)
    torch.cuda.synchronize()
    a_g = _check_routing_of_fwd(orc, inp, sv, routing)
    r = orc.layer_forward_blend(inp.h, inp.w, W1, W2, gam, bet, wl.act, a_g, experts=experts)
    keep = np.ones(T, dtype=bool) if experts is None else np.isin(a_g, experts)
    ok, worst = close_rel_rms(to_np(out)[keep], r["out"][keep], FWD_TOL)
    assert ok, worst


@pytest.mark.parametrize("S,routing,act", [(1, "balanced", "relu"), (2, "balanced", "relu"),
                                           (3, "greedy", "gelu")])
def test_blend_variant_small(orc, S, routing, act):
    wl = synth.WORKLOADS["layer_fwd"].scaled(T=1536, E=6, D=256, F=1024, act=act)
    _blend_check(orc, wl, S, 6, routing)


def test_blend_variant_full_layer_fwd_workload_sampled(orc):
    # the benchmarked shape (T=8192, E=16, D=1024, F=4096) with two sublayers
    _blend_check(orc, synth.WORKLOADS["layer_fwd"], 2, 0, "balanced", experts=[0, 9])


# ------------------------------------------------------------------ expert parallelism, one worker
def test_expert_parallel_layer_one_worker(orc):
    # one worker holds every expert: the shuffle, the layer on the shuffled
    # tokens with the library's kernels and the undoing of the shuffle
    from balanced_token_expert_b200 import expert_parallel as ep
    wl = synth.WORKLOADS["layer_fwd"].scaled(T=2048, E=8, D=256, F=512)
    inp = synth.make_inputs(wl, 9)
    T, E, D, F = wl.T, wl.E, wl.D, wl.F
    plan = ep.EPPlan(T=T, E=E, G=1)
    be = ep.CudaBackend(T, E, D, F)
    y, shuffled, assign = ep.ep_layer_fwd(dev(inp.h), dev(inp.w), dev(inp.W1), dev(inp.W2),
                                          B.BASE_RELU, plan, seed=77, backend=be,
                                          return_route=True)
    torch.cuda.synchronize()
    perm = ep.shuffle_permutation(T, 77)
    assert torch.equal(shuffled.cpu(), inp.h[perm])
    q = torch.empty(T, E, dtype=torch.int32, device="cuda")
    B.base_scores(shuffled, dev(inp.w), None, q)
    torch.cuda.synchronize()
    a_g = to_np(assign)
    assert np.array_equal(a_g, orc.auction(to_np(q))[0])
    ysh = orc.layer_forward(inp.h[perm], inp.w, inp.W1, inp.W2, "relu", a_g)["out"]
    expect = np.empty_like(ysh)
    expect[perm.numpy()] = ysh
    ok, worst = close_rel_rms(to_np(y), expect, FWD_TOL)
    assert ok, worst


def test_training_step_is_deterministic():
    # the forward and the backward three times on the same inputs: every
    # output, saved activation and gradient the same bits each time (no
    # floating-point atomics: the centroid gradient sums in a fixed order)
    wl = synth.WORKLOADS["layer_fwd_bwd"].scaled(T=4096, E=16, D=512, F=1024)
    inp = synth.make_inputs(wl, 21, with_dout=True)
    T, E, D, F = wl.T, wl.E, wl.D, wl.F
    runs = []
    for _ in range(3):
        out, sv, ws = _run_layer_fwd(wl, inp, "balanced", for_backward=True)
        dh = torch.empty(T, D, dtype=torch.bfloat16, device="cuda")
        dw = torch.empty(E, D, dtype=torch.float32, device="cuda")
        dW1 = torch.empty(E, F, D, dtype=torch.float32, device="cuda")
        dW2 = torch.empty(E, D, F, dtype=torch.float32, device="cuda")
        B.base_layer_bwd(dev(inp.h), dev(inp.w), dev(inp.W1), dev(inp.W2), ACT[wl.act], sv,
                         dev(inp.dout), dh, dw, dW1, dW2, ws)
        torch.cuda.synchronize()
        runs.append(dict(out=out, dh=dh, dw=dw, dW1=dW1, dW2=dW2, **{
            k: sv[k] for k in ("s", "q", "assign", "price", "perm", "a1", "h1", "f", "y_perm")}))
    for k, v in runs[0].items():
        for other in runs[1:]:
            assert torch.equal(v, other[k]), k
