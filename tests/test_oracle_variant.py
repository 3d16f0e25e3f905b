"""Pins of the oracle's released-code layer variant ("BASE Layers:
Simplifying Training of Large, Sparse Models", wikillm.com summary: "Paper vs
code", Mixing equation -- a convex blend alpha f + (1 - alpha) h instead of
eq. 1's residual form; "Placement and shape" -- each expert a stack of
sublayers with layer norm, projection up, ReLU, projection back and a
residual connection)."""
import numpy as np
import torch


def test_layer_norm_of_a_hand_worked_row(orc):
    # x = (1, 2, 3, 4): mean 2.5, biased variance (2.25 + 0.25 + 0.25 + 2.25)/4
    # = 1.25; sqrt(1.25 + 1e-5) = 1.1180384...; 1.5 / 1.1180384 = 1.3416354,
    # 0.5 / 1.1180384 = 0.4472118
    y = orc.layer_norm(np.array([[1.0, 2.0, 3.0, 4.0]]), np.ones(4), np.zeros(4))
    assert np.allclose(y[0], [-1.3416354, -0.4472118, 0.4472118, 1.3416354], atol=2e-7)
    # gain and bias act per column after the normalisation
    y2 = orc.layer_norm(np.array([[1.0, 2.0, 3.0, 4.0]]), np.array([2.0, 1.0, 0.0, -1.0]),
                        np.array([0.5, 0.0, 7.0, 0.0]))
    assert np.allclose(y2[0], [-2.6832708 + 0.5, -0.4472118, 7.0, -1.3416354], atol=4e-7)
    # a constant row has no deviation: the output is the bias
    y3 = orc.layer_norm(np.full((1, 8), 3.25), np.full(8, 5.0), np.arange(8.0))
    assert np.array_equal(y3[0], np.arange(8.0))


def test_layer_norm_rows_have_zero_mean_and_unit_variance(orc):
    x = np.random.default_rng(0).standard_normal((6, 256)) * 3.0 + 1.5
    y = orc.layer_norm(x, np.ones(256), np.zeros(256))
    assert np.allclose(y.mean(axis=1), 0.0, atol=1e-12)
    var = x.var(axis=1)
    assert np.allclose(y.var(axis=1), var / (var + 1e-5), atol=1e-12)


def test_expert_stack_special_cases(orc):
    rng = np.random.default_rng(1)
    S, D, F = 3, 16, 40
    x = rng.standard_normal((5, D))
    W1 = rng.standard_normal((S, F, D)) * 0.1
    g = rng.standard_normal((S, D))
    b = rng.standard_normal((S, D))
    # zero output projections: every sublayer adds nothing
    assert np.array_equal(orc.expert_stack(x, W1, np.zeros((S, D, F)), g, b), x)
    # zero gains: the layer norm returns its bias for every row, so one
    # sublayer adds the same vector W2 relu(W1 b) to every row
    W2 = rng.standard_normal((1, D, F)) * 0.1
    out = orc.expert_stack(x, W1[:1], W2, np.zeros((1, D)), b[:1])
    add = np.maximum(W1[0] @ b[0], 0.0) @ W2[0].T
    assert np.allclose(out, x + add[None, :], atol=1e-12)


def test_blend_mixes_token_by_token(orc):
    rng = np.random.default_rng(2)
    T, E, S, D, F = 12, 3, 2, 8, 16
    h = rng.standard_normal((T, D))
    w = rng.standard_normal((E, D))
    W1 = rng.standard_normal((E, S, F, D)) * 0.2
    W2 = rng.standard_normal((E, S, D, F)) * 0.2
    g = 1.0 + 0.1 * rng.standard_normal((E, S, D))
    b = 0.1 * rng.standard_normal((E, S, D))
    assign = np.repeat(np.arange(E), T // E)
    rng.shuffle(assign)
    r = orc.layer_forward_blend(h, w, W1, W2, g, b, "relu", assign)
    for t in range(T):
        e = assign[t]
        a = 1.0 / (1.0 + np.exp(-sum(h[t, d] * w[e, d] for d in range(D))))
        f = orc.expert_stack(h[t:t + 1], W1[e], W2[e], g[e], b[e])[0]
        assert np.allclose(r["out"][t], a * f + (1.0 - a) * h[t], atol=1e-12)


def test_blend_at_zero_affinity_is_the_midpoint(orc):
    # h . w_a = 0 gives alpha = 1/2: the output is the mean of the expert's
    # output and the input (eq. 1's residual form would give f/2 + h instead)
    rng = np.random.default_rng(3)
    T, E, D, F = 4, 2, 8, 8
    h = rng.standard_normal((T, D))
    w = np.zeros((E, D))
    W1 = rng.standard_normal((E, 1, F, D))
    W2 = rng.standard_normal((E, 1, D, F))
    g = np.ones((E, 1, D))
    b = np.zeros((E, 1, D))
    assign = np.array([0, 1, 0, 1])
    r = orc.layer_forward_blend(h, w, W1, W2, g, b, "relu", assign)
    for t in range(T):
        f = orc.expert_stack(h[t:t + 1], W1[assign[t]], W2[assign[t]], g[assign[t]], b[assign[t]])
        assert np.allclose(r["out"][t], 0.5 * (f[0] + h[t]), atol=1e-12)


def test_blend_accepts_bf16_tensors(orc):
    T, E, S, D, F = 8, 2, 1, 16, 32
    g = torch.Generator().manual_seed(4)
    h = torch.randn(T, D, generator=g).to(torch.bfloat16)
    w = torch.randn(E, D, generator=g).to(torch.bfloat16)
    W1 = (torch.randn(E, S, F, D, generator=g) * 0.1).to(torch.bfloat16)
    W2 = (torch.randn(E, S, D, F, generator=g) * 0.1).to(torch.bfloat16)
    gam = torch.ones(E, S, D)
    bet = torch.zeros(E, S, D)
    assign = np.array([0, 1] * 4)
    r = orc.layer_forward_blend(h, w, W1, W2, gam, bet, "relu", assign)
    assert r["out"].shape == (T, D) and np.all(np.isfinite(r["out"]))
