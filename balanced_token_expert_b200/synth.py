"""Seeded synthetic inputs for the BASE-layer hot path.

This module only draws random numbers; it holds none of the layer's
arithmetic, so the CUDA path and the CPU oracle can both be fed from it.
Every tensor comes from a CPU ``torch.Generator`` seeded with ``seed`` and is
drawn in a fixed order (h, w, W1, W2, dout), so a given (workload, seed) pair
always yields the same bits.

Workloads (the shapes follow the BASE layer of "BASE Layers: Simplifying
Training of Large, Sparse Models", Method and Placement sections: tokens h_t
of width D, E expert centroids w_e, expert FFNs D -> F -> D):

* ``routing_ref``: T=512, E=8, D=64, fp32, h ~ N(0,1), w ~ N(0,1/D).
* ``layer_fwd``: T=8192, E=16, D=1024, F=4096 ReLU, bf16; W1, W2 ~ N(0, 0.02^2).
* ``skewed``: T=32768, E=64, D=1024, bf16; tokens from a 64-component Gaussian
  mixture (means ~ N(0, I), noise 0.5 N(0, I), component k drawn with
  probability proportional to k^-1.2), and a seeded half of the tokens get
  +3.0 added to their affinity for expert 0 (``bump_tokens``/``bump_value``;
  the caller applies it to the quantised scores).
* ``large_routing``: T=131072, E=128, D=2048, bf16.
* ``layer_fwd_bwd``: T=32768, E=32, D=2048, F=8192 GELU, bf16, plus dout ~ N(0,1).
* ``layer_fwd_blend``: the layer_fwd shape through the released code's variant
  (one sublayer per expert; ``make_stack_params`` adds layer-norm gains and
  biases and the weights of further sublayers).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import torch

__all__ = ["Workload", "WORKLOADS", "make_inputs", "make_stack_params", "Inputs"]


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    E: int
    D: int
    F: int = 0                 # 0: no expert FFN in this workload
    act: str = "relu"          # "relu" | "gelu"
    dtype: str = "bf16"        # "f32" | "bf16"
    kind: str = "normal"       # "normal" | "mixture"
    backward: bool = False
    S: int = 0                 # > 0: the released code's variant with S sublayers per expert

    def scaled(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


WORKLOADS = {
    "routing_ref": Workload("routing_ref", T=512, E=8, D=64, dtype="f32"),
    "layer_fwd": Workload("layer_fwd", T=8192, E=16, D=1024, F=4096, act="relu"),
    "skewed": Workload("skewed", T=32768, E=64, D=1024, kind="mixture"),
    "large_routing": Workload("large_routing", T=131072, E=128, D=2048),
    "layer_fwd_bwd": Workload("layer_fwd_bwd", T=32768, E=32, D=2048, F=8192, act="gelu",
                              backward=True),
    # the layer_fwd shape through the released code's variant (one sublayer
    # per expert, the code's default, and the convex blend)
    "layer_fwd_blend": Workload("layer_fwd_blend", T=8192, E=16, D=1024, F=4096, act="relu", S=1),
}


@dataclass
class Inputs:
    wl: Workload
    seed: int
    h: torch.Tensor                      # (T, D) float32 or bfloat16
    w: torch.Tensor                      # (E, D)
    W1: Optional[torch.Tensor] = None    # (E, F, D) bfloat16
    W2: Optional[torch.Tensor] = None    # (E, D, F) bfloat16
    dout: Optional[torch.Tensor] = None  # (T, D) bfloat16
    bump_tokens: Optional[torch.Tensor] = None  # int64, sorted
    bump_value: float = 0.0              # added to the affinity of expert 0
    extra: dict = field(default_factory=dict)


def _cast(x: torch.Tensor, dtype: str) -> torch.Tensor:
    return x.contiguous() if dtype == "f32" else x.to(torch.bfloat16).contiguous()


def make_inputs(wl: Workload, seed: int = 0, with_weights: bool = True,
                with_dout: Optional[bool] = None) -> Inputs:
    """Draw the inputs of ``wl`` from a CPU generator seeded with ``seed``."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    T, E, D = wl.T, wl.E, wl.D
    if wl.kind == "mixture":
        K = 64
        mu = torch.randn(K, D, generator=g)
        probs = torch.tensor([(k + 1) ** -1.2 for k in range(K)], dtype=torch.float64)
        comp = torch.multinomial(probs / probs.sum(), T, replacement=True, generator=g)
        h = mu[comp] + 0.5 * torch.randn(T, D, generator=g)
    else:
        h = torch.randn(T, D, generator=g)
    w = torch.randn(E, D, generator=g) * (1.0 / math.sqrt(D))
    inp = Inputs(wl=wl, seed=seed, h=_cast(h, wl.dtype), w=_cast(w, wl.dtype))
    del h
    if wl.kind == "mixture":
        perm = torch.randperm(T, generator=g)
        inp.bump_tokens = perm[: T // 2].sort().values
        inp.bump_value = 3.0
    if wl.F and with_weights:
        F = wl.F
        inp.W1 = _cast(torch.randn(E, F, D, generator=g) * 0.02, "bf16")
        inp.W2 = _cast(torch.randn(E, D, F, generator=g) * 0.02, "bf16")
    if with_dout is None:
        with_dout = wl.backward
    if with_dout:
        inp.dout = _cast(torch.randn(T, D, generator=g), "bf16")
    return inp


def make_stack_params(wl: Workload, S: int, seed: int = 0) -> dict:
    """Parameters of the released code's expert stacks (S sublayers per
    expert): the weights of sublayers 1 .. S-1 (sublayer 0 uses the
    workload's W1 / W2), W ~ N(0, 0.02^2) bf16, and every sublayer's layer
    norm gain ~ 1 + 0.1 N(0,1) and bias ~ 0.1 N(0,1), fp32.  From a generator
    seeded with seed + 1000, so the workload's own draws are unchanged."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) + 1000)
    E, D, F = wl.E, wl.D, wl.F
    out = {}
    if S > 1:
        out["W1"] = _cast(torch.randn(E, S - 1, F, D, generator=g) * 0.02, "bf16")
        out["W2"] = _cast(torch.randn(E, S - 1, D, F, generator=g) * 0.02, "bf16")
    out["gamma"] = (1.0 + 0.1 * torch.randn(E, S, D, generator=g)).contiguous()
    out["beta"] = (0.1 * torch.randn(E, S, D, generator=g)).contiguous()
    return out
