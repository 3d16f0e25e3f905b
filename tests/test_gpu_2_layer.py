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


def _layer_fwd_check(orc, wl, seed, routing, experts=None):
    inp = synth.make_inputs(wl, seed)
    T, E, D, F = wl.T, wl.E, wl.D, wl.F
    sv = buffers.layer_saved(T, E, D, F)
    out = torch.empty(T, D, dtype=torch.bfloat16, device="cuda")
    ws = buffers.workspace(T, E, D, F)
    B.base_layer_fwd(dev(inp.h), dev(inp.w), dev(inp.W1), dev(inp.W2), ACT[wl.act],
                     B.BASE_ROUTE_BALANCED if routing == "balanced" else B.BASE_ROUTE_GREEDY,
                     out, sv, ws)
    torch.cuda.synchronize()
    s_o = orc.scores(inp.h, inp.w)
    s_g, q_g = to_np(sv["s"]), to_np(sv["q"])
    ok, worst = close_scores(s_g, s_o, 1e-5)
    assert ok, worst
    assert np.array_equal(q_g, np.rint(s_g * np.float32(65536)).astype(np.int32))
    a_g = to_np(sv["assign"])
    q_o = orc.quantize(s_o)
    a_o = _assign(orc, q_o, routing)
    if routing == "balanced":
        st = buffers.stats_dict(sv["stats"])
        assert st["status"] == 0
        # the GPU's q differs from the oracle's only where fp32 accumulation
        # crosses a rounding boundary; its assignment must be optimal for its q
        cert = orc.certificate(q_g, a_g, to_np(sv["price"]))
        assert cert["ok"]
        assert np.abs(q_g.astype(np.int64) - q_o).max() <= 1
        opt_o = orc.auction(q_o)[2]["objective"]
        assert int(q_o[np.arange(T), a_g].astype(np.int64).sum()) >= opt_o - 2 * T
        if np.array_equal(q_g, q_o):
            assert np.array_equal(a_g, a_o)
    else:
        assert np.array_equal(a_g, orc.greedy(q_g)[0])
    diff = np.nonzero(a_g != a_o)[0]
    assert diff.size <= max(2, T // 100), diff.size
    # outputs: the oracle's forward with its own assignment, token by token;
    # tokens the GPU routed elsewhere (score rounding ties) are recomputed by
    # the oracle for the expert the GPU chose
    fw = orc.layer_forward(inp.h, inp.w, inp.W1, inp.W2, wl.act, a_o, experts=experts)
    out_g = to_np(out)
    keep = np.ones(T, dtype=bool)
    keep[diff] = False
    if experts is not None:
        keep &= np.isin(a_o, experts)
    ok, worst = close_rel_rms(out_g[keep], fw["out"][keep], FWD_TOL)
    assert ok, worst
    if diff.size:
        alt = orc.layer_forward(inp.h, inp.w, inp.W1, inp.W2, wl.act, a_g,
                                experts=sorted(set(a_g[diff].tolist())))
        ok, worst = close_rel_rms(out_g[diff], alt["out"][diff], FWD_TOL)
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
