"""CPU oracle for the BASE-layer hot path.

TEST INFRASTRUCTURE ONLY.  The test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference legs are the only callers.  The oracle
shares no code with the CUDA library and never imports it.

Everything follows the page "BASE Layers: Simplifying Training of Large,
Sparse Models" (wikillm.com summary; section names below are that page's):

* scores ``s[t,e] = h_t . w_e`` -- Method, fig. 2 listing (affinities =
  features @ centroids^T), in float64.
* quantisation ``q = rint(fp32(s) * 2^16)`` -- not on the pages; the scale is
  the workload definition's.  The rounding decision is taken in fp32, the
  precision the kernel takes it in.
* greedy routing ``a_t = argmax_e q[t,e]`` (lowest e on ties) -- Method,
  "Test time".
* balanced assignment -- Method, "Training assignment", eq. 2, solved by the
  integer Jacobi auction in ``base_oracle.c`` (pinned there by the Hungarian
  method and brute force).
* permutation -- fig. 2 ``sort_by_expert`` / ``inverse_sort``; the order
  inside an expert is ascending token index.
* expert FFN ``f_e(x) = W2_e act(W1_e x)`` -- Placement and shape (projection
  to the FFN width, activation, projection back; no bias, no norm).
* combine ``sigma(h_t . w_{a_t}) f_{a_t}(h_t) + h_t`` -- eq. 1.
* backward with the assignment held fixed -- "Paper vs code", gradient into
  routing: affinities for assignment carry no gradient, centroids get
  gradient only through the gate.
* the released code's layer variant -- "Paper vs code", Mixing equation (a
  convex blend ``alpha f + (1 - alpha) h``) and "Placement and shape" (each
  expert a stack of sublayers: layer norm, projection up, ReLU, projection
  back, residual).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

__all__ = [
    "QSCALE", "EPS_DIVISOR", "EPS_FACTOR", "MAX_ROUNDS", "lib", "build",
    "scores", "quantize", "greedy", "auction", "hungarian", "bruteforce",
    "certificate", "permutation", "gather_rows", "scatter_rows", "act",
    "act_grad", "sigmoid", "expert_ffn", "layer_forward", "layer_backward",
    "LN_EPS", "layer_norm", "expert_stack", "layer_forward_blend", "sanitize_scores",
    "fig9_auction", "FIG9_MAX_ITERATIONS",
]

# Spec constants, restated independently of the CUDA library.
QSCALE = 65536.0          # quantised score = rint(s * 2^16)
EPS_DIVISOR = 50          # eps0 = (max q - min q) * (T+1) / 50
EPS_FACTOR = 8            # eps <- eps / 8 between phases
MAX_ROUNDS = 1_000_000    # hang guard on the total number of rounds

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``base_oracle.c`` into ``liboracle.so`` (gcc, OpenMP)."""
    src = os.path.join(_HERE, "base_oracle.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        tmp = _SO + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC",
                               "-o", tmp, src])
        os.replace(tmp, _SO)
    return _SO


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        i32p = ctypes.POINTER(ctypes.c_int32)
        i64p = ctypes.POINTER(ctypes.c_int64)
        L.orc_auction.restype = ctypes.c_int
        L.orc_auction.argtypes = [i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int64, i32p, i64p,
                                  i64p, i32p, ctypes.c_int64]
        L.orc_hungarian.restype = ctypes.c_int64
        L.orc_hungarian.argtypes = [i32p, ctypes.c_int, ctypes.c_int, i32p]
        L.orc_fig9.restype = ctypes.c_int
        L.orc_fig9.argtypes = [i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                               i32p, i64p, i64p]
        L.orc_bruteforce.restype = ctypes.c_int64
        L.orc_bruteforce.argtypes = [i32p, ctypes.c_int, ctypes.c_int, i32p, i64p, i64p]
        _lib = L
    return _lib


def _p32(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def _p64(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))


def _f64(x) -> np.ndarray:
    """float64 copy of a numpy array or torch tensor (bf16 values are exact)."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch
        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------
# scores, quantisation, greedy routing
# --------------------------------------------------------------------------
def scores(h, w) -> np.ndarray:
    """``s = h w^T`` in float64 (fig. 2: affinities = features @ centroids.T)."""
    return _f64(h) @ _f64(w).T


def quantize(s) -> np.ndarray:
    """``q = rint(fp32(s) * 2^16)``, half-to-even, clamped to +-(2^31 - 1)."""
    s32 = np.asarray(s, dtype=np.float64).astype(np.float32)
    x = np.rint(s32 * np.float32(QSCALE)).astype(np.float64)
    return np.clip(x, -2147483647.0, 2147483647.0).astype(np.int32)


def sanitize_scores(s) -> np.ndarray:
    """Non-finite affinities replaced by the smallest finite one ("Paper vs
    code", Non-finite scores: the released code does this before solving).
    When no score is finite the pages leave the value open; this reading uses
    0.  Returns a float32 copy (the scores are fp32)."""
    s32 = np.array(s, dtype=np.float32, copy=True)
    bad = ~np.isfinite(s32)
    if bad.any():
        good = s32[~bad]
        s32[bad] = good.min() if good.size else np.float32(0.0)
    return s32


def greedy(q: np.ndarray):
    """Test-time routing: each token to its highest-scoring expert, the lowest
    index on ties (Method, "Test time").  Returns (assign, counts)."""
    q = np.asarray(q)
    a = np.argmax(q, axis=1).astype(np.int32)  # first maximum = lowest index
    counts = np.bincount(a, minlength=q.shape[1]).astype(np.int32)
    return a, counts


# --------------------------------------------------------------------------
# balanced assignment
# --------------------------------------------------------------------------
def auction(q: np.ndarray, max_rounds: int = MAX_ROUNDS, trace: bool = False):
    """The integer Jacobi auction of ``base_oracle.c`` on quantised scores.

    Returns ``(assign int32[T], price int64[E], stats dict[, u_trace])`` where
    stats holds status, phases, rounds, final_eps, objective and bids."""
    q = np.ascontiguousarray(q, dtype=np.int32)
    T, E = q.shape
    assign = np.full(T, -1, dtype=np.int32)
    price = np.zeros(E, dtype=np.int64)
    st = np.zeros(6, dtype=np.int64)
    cap = min(int(max_rounds), 4_000_000) if trace else 0
    tr = np.zeros(max(cap, 1), dtype=np.int32)
    rc = lib().orc_auction(_p32(q), T, E, int(max_rounds), _p32(assign), _p64(price), _p64(st),
                           _p32(tr) if trace else None, cap)
    stats = dict(status=int(rc), phases=int(st[1]), rounds=int(st[2]), final_eps=int(st[3]),
                 objective=int(st[4]), bids=int(st[5]))
    if trace:
        return assign, price, stats, tr[: min(stats["rounds"], cap)].copy()
    return assign, price, stats


FIG9_MAX_ITERATIONS = 100  # the listing's default iteration cap


def fig9_auction(q: np.ndarray, max_iterations: int = FIG9_MAX_ITERATIONS,
                 max_rounds: int = MAX_ROUNDS):
    """The page's fig. 9 solver (experts bid for tokens, prices per token)
    with the released code's rules, as ``orc_fig9`` in ``base_oracle.c``
    states them.  Returns ``(assign int32[T], token price int64[T], stats)``
    with stats status, rounds, eps and objective."""
    q = np.ascontiguousarray(q, dtype=np.int32)
    T, E = q.shape
    assign = np.full(T, -1, dtype=np.int32)
    price = np.zeros(T, dtype=np.int64)
    st = np.zeros(4, dtype=np.int64)
    rc = lib().orc_fig9(_p32(q), T, E, int(max_iterations), int(max_rounds), _p32(assign),
                        _p64(price), _p64(st))
    return assign, price, dict(status=int(rc), rounds=int(st[1]), eps=int(st[2]),
                               objective=int(st[3]))


def hungarian(q: np.ndarray):
    """Exact optimum of eq. 2 by the Hungarian method on C replicated slots per
    expert.  Returns (objective, assign)."""
    q = np.ascontiguousarray(q, dtype=np.int32)
    T, E = q.shape
    a = np.full(T, -1, dtype=np.int32)
    obj = lib().orc_hungarian(_p32(q), T, E, _p32(a))
    return int(obj), a


def bruteforce(q: np.ndarray):
    """Exact optimum of eq. 2 by enumerating every balanced assignment.
    Returns (objective, one optimal assignment, #assignments, #optimal)."""
    q = np.ascontiguousarray(q, dtype=np.int32)
    T, E = q.shape
    a = np.full(T, -1, dtype=np.int32)
    na = ctypes.c_int64(0)
    no = ctypes.c_int64(0)
    obj = lib().orc_bruteforce(_p32(q), T, E, _p32(a), ctypes.byref(na), ctypes.byref(no))
    return int(obj), a, int(na.value), int(no.value)


def certificate(q: np.ndarray, assign: np.ndarray, price: np.ndarray) -> dict:
    """Optimality certificate of a balanced assignment with expert prices.

    * balance: every expert holds exactly C = T/E tokens;
    * 1-complementary slackness on the scaled values A = q (T+1):
      A[t,a_t] - p[a_t] >= max_e (A[t,e] - p[e]) - 1 for every token;
    * LP duality of eq. 2: OPT_scaled <= Dual = sum_t max_e (A[t,e] - p_e)
      + C sum_e p_e, so (T+1) P >= Dual - T proves P = OPT (both sides of
      OPT - P < 1 are integers once divided by T+1).
    Exact integer arithmetic (Python ints for the sums)."""
    q = np.asarray(q, dtype=np.int64)
    assign = np.asarray(assign, dtype=np.int64)
    price = np.asarray(price, dtype=np.int64)
    T, E = q.shape
    C = T // E
    scale = T + 1
    counts = np.bincount(assign, minlength=E) if assign.min() >= 0 else None
    balanced = bool(counts is not None and assign.max() < E and np.all(counts == C))
    A = q * scale                                   # fits int64 for |q| < 2^31, T < 2^31
    val = A - price[None, :]
    best = val.max(axis=1)
    own = val[np.arange(T), np.clip(assign, 0, E - 1)]
    cs = bool(np.all(own >= best - 1))
    P = int(sum(int(x) for x in q[np.arange(T), np.clip(assign, 0, E - 1)]))
    dual = sum(int(x) for x in best) + C * sum(int(x) for x in price)
    dual_ok = scale * P >= dual - T
    return dict(balanced=balanced, cs=cs, dual_ok=bool(dual_ok), objective=P, dual=dual,
                ok=bool(balanced and cs and dual_ok))


# --------------------------------------------------------------------------
# permutation (fig. 2 sort_by_expert / inverse_sort)
# --------------------------------------------------------------------------
def permutation(assign: np.ndarray, E: int):
    """Expert-major slot order, ascending token inside an expert.
    Returns (perm[slot] = t, inv[t] = slot, offsets[E+1])."""
    assign = np.asarray(assign, dtype=np.int64)
    T = assign.shape[0]
    perm = np.argsort(assign, kind="stable").astype(np.int32)
    inv = np.empty(T, dtype=np.int32)
    inv[perm] = np.arange(T, dtype=np.int32)
    counts = np.bincount(assign, minlength=E)
    offsets = np.zeros(E + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    return perm, inv, offsets


def gather_rows(x, perm: np.ndarray) -> np.ndarray:
    """``x_perm[slot] = x[perm[slot]]`` (fig. 2: features[sort_by_expert])."""
    return np.asarray(x)[np.asarray(perm, dtype=np.int64)]


def scatter_rows(y, perm: np.ndarray) -> np.ndarray:
    """``out[perm[slot]] = y[slot]`` (fig. 2: [inverse_sort(...)])."""
    y = np.asarray(y)
    out = np.empty_like(y)
    out[np.asarray(perm, dtype=np.int64)] = y
    return out


# --------------------------------------------------------------------------
# expert FFN and the eq. 1 combine
# --------------------------------------------------------------------------
def sigmoid(x):
    x = np.asarray(x, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(-x))


def act(x, kind: str):
    """ReLU, or GELU in its exact erf form 0.5 x (1 + erf(x / sqrt 2))."""
    x = np.asarray(x, dtype=np.float64)
    if kind == "relu":
        return np.maximum(x, 0.0)
    from scipy.special import erf
    return 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))


def act_grad(x, kind: str):
    """d act / dx; ReLU' (0) = 0; GELU' = Phi(x) + x phi(x)."""
    x = np.asarray(x, dtype=np.float64)
    if kind == "relu":
        return (x > 0).astype(np.float64)
    from scipy.special import erf
    return 0.5 * (1.0 + erf(x / np.sqrt(2.0))) + x * np.exp(-0.5 * x * x) / np.sqrt(2.0 * np.pi)


def expert_ffn(x_perm, offsets, W1, W2, kind: str, gate_s=None, experts=None):
    """Per expert segment: ``A1 = x W1_e^T``, ``H1 = act(A1)``, ``f = H1 W2_e^T``;
    with ``gate_s`` also ``y = sigmoid(gate_s) f + x`` (eq. 1).  float64.
    ``experts`` limits the work to some experts (rows of the others are NaN).
    Returns dict(a1, h1, f, y)."""
    x = _f64(x_perm)
    T, D = x.shape
    E, F, _ = W1.shape
    a1 = np.full((T, F), np.nan)
    f = np.full((T, D), np.nan)
    for e in (range(E) if experts is None else experts):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi == lo:
            continue
        a1[lo:hi] = x[lo:hi] @ _f64(W1[e]).T
        f[lo:hi] = act(a1[lo:hi], kind) @ _f64(W2[e]).T
    out = dict(a1=a1, h1=act(a1, kind), f=f)
    if gate_s is not None:
        out["y"] = sigmoid(gate_s)[:, None] * f + x
    return out


def layer_forward(h, w, W1, W2, kind: str, assign: np.ndarray, experts=None):
    """BASE layer forward with a given assignment (eq. 1, fig. 2).
    Returns dict(out, s, gate_s, perm, inv, offsets, x_perm, a1, f, y_perm)."""
    h64, w64 = _f64(h), _f64(w)
    E = w64.shape[0]
    s = h64 @ w64.T
    perm, inv, offsets = permutation(assign, E)
    x_perm = h64[perm]
    gate_s = s[perm, np.asarray(assign, dtype=np.int64)[perm]]
    r = expert_ffn(x_perm, offsets, W1, W2, kind, gate_s=gate_s, experts=experts)
    out = scatter_rows(r["y"], perm)
    return dict(out=out, s=s, gate_s=gate_s, perm=perm, inv=inv, offsets=offsets, x_perm=x_perm,
                a1=r["a1"], f=r["f"], y_perm=r["y"], assign=np.asarray(assign, dtype=np.int32))


def layer_backward(fw: dict, h, w, W1, W2, kind: str, dout, experts=None):
    """Gradients of ``L = <out, dout>`` with the assignment held fixed.
    With ``experts`` given, dW1 / dW2 are dicts {expert: array} of those
    experts only.

    dy = dout[perm]; dgate = <dy, f>; ds = dgate sigma (1 - sigma);
    dF = sigma dy; dH1 = dF W2_e; dW2_e = dF^T H1; dA1 = dH1 * act'(A1);
    dW1_e = dA1^T x; dx = dA1 W1_e + dy + ds w_{a_t}; dw_e = sum ds h_t;
    dh = dx[inv].  Returns dict(dh, dw, dW1, dW2)."""
    h64, w64 = _f64(h), _f64(w)
    E, F, D = W1.shape
    T = h64.shape[0]
    perm, offsets = fw["perm"], fw["offsets"]
    assign = np.asarray(fw["assign"], dtype=np.int64)
    dy = _f64(dout)[perm]
    x = fw["x_perm"]
    sg = sigmoid(fw["gate_s"])
    dgate = np.einsum("td,td->t", dy, fw["f"])
    ds = dgate * sg * (1.0 - sg)
    dF = sg[:, None] * dy
    dW1, dW2 = {}, {}
    dx = np.full((T, D), np.nan)
    for e in (range(E) if experts is None else experts):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        a1 = fw["a1"][lo:hi]
        h1 = act(a1, kind)
        dH1 = dF[lo:hi] @ _f64(W2[e])
        dW2[e] = dF[lo:hi].T @ h1
        dA1 = dH1 * act_grad(a1, kind)
        dW1[e] = dA1.T @ x[lo:hi]
        dx[lo:hi] = dA1 @ _f64(W1[e]) + dy[lo:hi] + ds[lo:hi, None] * w64[e][None, :]
    dw = np.zeros((E, D))
    ex = assign[perm]
    for e in (range(E) if experts is None else experts):
        m = ex == e
        dw[e] = (ds[m][:, None] * x[m]).sum(axis=0)
    dh = dx[fw["inv"]]
    if experts is None:  # every expert: full (E, F, D) / (E, D, F) arrays
        dW1 = np.stack([dW1[e] for e in range(E)])
        dW2 = np.stack([dW2[e] for e in range(E)])
    return dict(dh=dh, dw=dw, dW1=dW1, dW2=dW2, ds=ds, dgate=dgate)


# --------------------------------------------------------------------------
# the released code's layer variant
# --------------------------------------------------------------------------
LN_EPS = 1e-5  # the pages name no layer-norm epsilon; the common default


def layer_norm(x, gamma, beta, eps: float = LN_EPS) -> np.ndarray:
    """Layer norm of every row: ``(x - mean) / sqrt(var + eps) * gamma + beta``
    with the biased variance (the mean of squared deviations).  float64."""
    x = _f64(x)
    mu = x.mean(axis=-1, keepdims=True)
    d = x - mu
    var = (d * d).mean(axis=-1, keepdims=True)
    return d / np.sqrt(var + eps) * _f64(gamma) + _f64(beta)


def expert_stack(x, W1s, W2s, gammas, betas, kind: str = "relu"):
    """One expert as the released code builds it ("Placement and shape"): S
    sublayers, each ``x <- x + W2_i act(W1_i LN_i(x))``.  W1s (S, F, D), W2s
    (S, D, F), gammas / betas (S, D).  float64.  Returns the output."""
    x = _f64(x)
    for i in range(len(W1s)):
        u = layer_norm(x, gammas[i], betas[i])
        x = x + act(u @ _f64(W1s[i]).T, kind) @ _f64(W2s[i]).T
    return x


def layer_forward_blend(h, w, W1, W2, gamma, beta, kind: str, assign: np.ndarray, experts=None):
    """The released code's BASE layer with a given assignment ("Paper vs
    code", Mixing equation): ``out_t = alpha_t E_a(h_t) + (1 - alpha_t) h_t``
    with ``alpha_t = sigmoid(h_t . w_a)`` and ``E_a`` the expert stack of
    expert ``a = assign[t]``.  W1 (E, S, F, D), W2 (E, S, D, F), gamma / beta
    (E, S, D).  ``experts`` limits the work to some experts (the other tokens'
    outputs are NaN).  Returns dict(out, y_perm, perm, offsets, gate_s)."""
    h64, w64 = _f64(h), _f64(w)
    E = w64.shape[0]
    s = h64 @ w64.T
    assign = np.asarray(assign, dtype=np.int64)
    perm, inv, offsets = permutation(assign, E)
    x = h64[perm]
    gate_s = s[perm, assign[perm]]
    alpha = sigmoid(gate_s)[:, None]
    y = np.full_like(x, np.nan)
    g64, b64 = _f64(gamma), _f64(beta)
    for e in (range(E) if experts is None else experts):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi == lo:
            continue
        f = expert_stack(x[lo:hi], W1[e], W2[e], g64[e], b64[e], kind)
        y[lo:hi] = alpha[lo:hi] * f + (1.0 - alpha[lo:hi]) * x[lo:hi]
    return dict(out=scatter_rows(y, perm), y_perm=y, perm=perm, inv=inv, offsets=offsets,
                gate_s=gate_s)
