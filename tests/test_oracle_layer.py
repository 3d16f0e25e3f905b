"""Pins of the oracle's dense parts: scores, quantisation, greedy routing,
permutation, expert FFN, the eq. 1 combine and the backward (page "BASE
Layers: Simplifying Training of Large, Sparse Models": Method eq. 1, fig. 2,
"Test time", "Placement and shape", "Paper vs code" on gradients)."""
import math

import numpy as np
import pytest
import torch

from balanced_token_expert_b200 import synth


def test_scores_are_the_textbook_product(orc):
    rng = np.random.default_rng(0)
    h = rng.standard_normal((5, 7))
    w = rng.standard_normal((3, 7))
    s = orc.scores(h, w)
    for t in range(5):
        for e in range(3):
            acc = 0.0
            for d in range(7):
                acc += h[t, d] * w[e, d]
            assert abs(s[t, e] - acc) < 1e-12


def test_scores_accept_bf16_tensors_exactly(orc):
    inp = synth.make_inputs(synth.WORKLOADS["layer_fwd"].scaled(T=16, E=4, D=32, F=0), 0)
    assert inp.h.dtype == torch.bfloat16
    s = orc.scores(inp.h, inp.w)
    ref = inp.h.double().numpy() @ inp.w.double().numpy().T
    assert np.array_equal(s, ref)


def test_quantize_rounds_half_to_even_and_saturates(orc):
    u = 1.0 / 65536.0
    s = np.array([[0.5 * u, 1.5 * u, 2.5 * u, -0.5 * u, -1.5 * u, 3.49 * u, 1e6, -1e6, 0.0]])
    q = orc.quantize(s)
    assert q.tolist() == [[0, 2, 2, 0, -2, 3, 2147483647, -2147483647, 0]]
    assert q.dtype == np.int32


def test_quantize_decides_in_fp32(orc):
    # s = 1 + 2^-24 is not representable in fp32 and rounds to 1.0 first
    s = np.array([[1.0 + 2.0 ** -24, 1.0 + 2.0 ** -22]])
    q = orc.quantize(s)
    assert q[0, 0] == 65536
    assert q[0, 1] == 65536  # 2^-22 * 2^16 = 2^-6, rounds to 0 above 65536


def test_greedy_lowest_index_on_ties(orc):
    q = np.array([[3, 5, 5, 1], [7, 7, 7, 7], [-1, -2, -3, -1], [0, 0, 9, 9]], dtype=np.int32)
    a, c = orc.greedy(q)
    assert a.tolist() == [1, 0, 0, 2]
    assert c.tolist() == [2, 1, 1, 0]
    rng = np.random.default_rng(1)
    q = rng.integers(0, 3, size=(50, 6)).astype(np.int32)
    a, _ = orc.greedy(q)
    for t in range(50):
        best = 0
        for e in range(1, 6):
            if q[t, e] > q[t, best]:
                best = e
        assert a[t] == best


def test_permutation_is_a_stable_counting_sort(orc):
    rng = np.random.default_rng(2)
    T, E = 100, 7
    assign = rng.integers(0, E, size=T).astype(np.int32)
    perm, inv, offsets = orc.permutation(assign, E)
    slots = []
    for e in range(E):
        for t in range(T):
            if assign[t] == e:
                slots.append(t)
    assert perm.tolist() == slots
    assert np.array_equal(perm[inv], np.arange(T))
    counts = [int((assign == e).sum()) for e in range(E)]
    assert offsets.tolist() == [0] + list(np.cumsum(counts))
    x = rng.standard_normal((T, 3))
    assert np.array_equal(orc.scatter_rows(orc.gather_rows(x, perm), perm), x)


def test_activations(orc):
    assert orc.sigmoid(0.0) == 0.5
    x = np.linspace(-6, 6, 49)
    g = orc.act(x, "gelu")
    assert orc.act(np.array([0.0]), "gelu")[0] == 0.0
    assert np.allclose(g - orc.act(-x, "gelu"), x, atol=1e-14)  # x Phi(x) - (-x Phi(-x)) = x
    assert np.allclose(g, [v * 0.5 * (1 + math.erf(v / math.sqrt(2))) for v in x], atol=1e-15)
    assert np.array_equal(orc.act(x, "relu"), np.maximum(x, 0))
    for kind in ("relu", "gelu"):
        xs = x[np.abs(x) > 1e-3]
        fd = (orc.act(xs + 1e-6, kind) - orc.act(xs - 1e-6, kind)) / 2e-6
        assert np.allclose(orc.act_grad(xs, kind), fd, atol=1e-7)


def _tiny(kind, seed=0, T=8, E=2, D=8, F=16):
    rng = np.random.default_rng(seed)
    h = rng.standard_normal((T, D))
    w = rng.standard_normal((E, D)) / math.sqrt(D)
    W1 = rng.standard_normal((E, F, D)) * 0.3
    W2 = rng.standard_normal((E, D, F)) * 0.3
    dout = rng.standard_normal((T, D))
    assign = np.array([t % E for t in range(T)], dtype=np.int32)
    rng.shuffle(assign)
    return h, w, W1, W2, dout, assign


@pytest.mark.parametrize("kind", ["relu", "gelu"])
def test_layer_forward_matches_eq1_token_by_token(orc, kind):
    h, w, W1, W2, _, assign = _tiny(kind)
    fw = orc.layer_forward(h, w, W1, W2, kind, assign)
    for t in range(h.shape[0]):
        e = assign[t]
        g = 1.0 / (1.0 + math.exp(-float(h[t] @ w[e])))
        f = W2[e] @ orc.act(W1[e] @ h[t], kind)
        assert np.allclose(fw["out"][t], g * f + h[t], atol=1e-13)


def test_zero_expert_weights_leave_the_residual(orc):
    h, w, W1, W2, _, assign = _tiny("relu")
    fw = orc.layer_forward(h, w, W1, np.zeros_like(W2), "relu", assign)
    assert np.array_equal(fw["out"], h)
    fw = orc.layer_forward(h, w, np.zeros_like(W1), W2, "relu", assign)
    assert np.array_equal(fw["out"], h)


@pytest.mark.parametrize("kind", ["relu", "gelu"])
def test_backward_matches_finite_differences(orc, kind):
    h, w, W1, W2, dout, assign = _tiny(kind, seed=4)

    def loss(h_, w_, W1_, W2_):
        return float((orc.layer_forward(h_, w_, W1_, W2_, kind, assign)["out"] * dout).sum())

    fw = orc.layer_forward(h, w, W1, W2, kind, assign)
    g = orc.layer_backward(fw, h, w, W1, W2, kind, dout)
    step = 1e-6
    rng = np.random.default_rng(8)
    for name, arr, grad in (("h", h, g["dh"]), ("w", w, g["dw"]), ("W1", W1, g["dW1"]),
                            ("W2", W2, g["dW2"])):
        flat = arr.reshape(-1)
        for idx in rng.choice(flat.size, size=min(flat.size, 24), replace=False):
            old = flat[idx]
            flat[idx] = old + step
            lp = loss(h, w, W1, W2)
            flat[idx] = old - step
            lm = loss(h, w, W1, W2)
            flat[idx] = old
            fd = (lp - lm) / (2 * step)
            assert abs(grad.reshape(-1)[idx] - fd) < 1e-6 * (1 + abs(fd)), (name, idx)


def test_backward_of_zero_dout_is_zero(orc):
    h, w, W1, W2, dout, assign = _tiny("gelu", seed=2)
    fw = orc.layer_forward(h, w, W1, W2, "gelu", assign)
    g = orc.layer_backward(fw, h, w, W1, W2, "gelu", np.zeros_like(dout))
    for k in ("dh", "dw", "dW1", "dW2"):
        assert not np.any(g[k])


def test_synth_is_deterministic_and_shaped():
    wl = synth.WORKLOADS["skewed"].scaled(T=256, E=8, D=32)
    a = synth.make_inputs(wl, 3)
    b = synth.make_inputs(wl, 3)
    assert torch.equal(a.h, b.h) and torch.equal(a.w, b.w)
    assert a.h.shape == (256, 32) and a.w.shape == (8, 32)
    assert a.bump_tokens.numel() == 128 and a.bump_value == 3.0
    c = synth.make_inputs(wl, 4)
    assert not torch.equal(a.h, c.h)
    f = synth.make_inputs(synth.WORKLOADS["layer_fwd"].scaled(T=64, E=4, D=16, F=32), 0)
    assert f.W1.shape == (4, 32, 16) and f.W2.shape == (4, 16, 32)
    assert f.W1.dtype == torch.bfloat16


def test_sanitize_replaces_non_finite_scores_by_the_smallest_finite_one(orc):
    # "Paper vs code", Non-finite scores: NaN and +-Inf become the minimum finite score
    s = np.array([[0.5, np.nan, -2.0], [np.inf, 3.0, -np.inf], [1.0, 0.25, -1.5]], dtype=np.float32)
    out = orc.sanitize_scores(s)
    assert out.tolist() == [[0.5, -2.0, -2.0], [-2.0, 3.0, -2.0], [1.0, 0.25, -1.5]]
    assert np.isnan(s[0, 1])  # the input is left alone
    # finite scores pass unchanged; no finite score at all gives zeros (a reading)
    f = np.arange(6, dtype=np.float32).reshape(2, 3)
    assert np.array_equal(orc.sanitize_scores(f), f)
    assert orc.sanitize_scores(np.full((2, 2), np.nan, dtype=np.float32)).tolist() == [[0, 0], [0, 0]]
    # sanitised, the quantised scores are those of the minimum: every
    # replaced entry quantises to the smallest quantised finite entry
    q = orc.quantize(out)
    assert q[0, 1] == q[1, 0] == q[1, 2] == q[0, 2] == orc.quantize(np.array([[-2.0]]))[0, 0]
