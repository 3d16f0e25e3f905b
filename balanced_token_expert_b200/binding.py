"""ctypes binding of libbase (include/base.h), one Python function per C
entry point with the same name.  Argument marshalling only: every step runs
in the CUDA library; torch is used for device memory and the current stream.

The library must have been built (``balanced_token_expert_b200._build``); on a
machine without it every call raises ``LibraryMissing``.  There is no CPU
fallback."""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from . import _build

__all__ = [
    "LibraryMissing", "BaseError", "lib", "Stats", "LayerSaved",
    "BASE_OK", "BASE_F32", "BASE_BF16", "BASE_RELU", "BASE_GELU",
    "BASE_ROUTE_BALANCED", "BASE_ROUTE_GREEDY", "QSCALE",
    "base_status_string", "base_version", "base_workspace_size", "base_device_error",
    "base_scores", "base_assign_greedy", "base_assign_balanced", "base_assign_balanced_ex",
    "base_permute", "base_permute_noalloc", "base_expert_ffn", "base_combine", "base_layer_fwd",
    "base_layer_bwd", "base_test_inject", "BASE_TEST_WAIT_LIMIT_NS",
    "base_workspace_size_blend", "base_layer_fwd_blend", "base_expert_stack",
    "base_sanitize_scores", "BASE_ROUTE_SANITIZE", "base_workspace_size_fig9", "base_assign_fig9",
    "base_probe_workspace_size", "base_measure_latency", "base_scores_greedy",
    "BASE_TEST_AUCTION_ABSENT_CTA", "BASE_TEST_GEMM_DROP_FIRST_LOAD", "EXPORTED",
    "base_ep_dispatch", "base_ep_combine",
]

BASE_OK = 0
BASE_F32, BASE_BF16 = 0, 1
BASE_RELU, BASE_GELU = 0, 1
BASE_ROUTE_BALANCED, BASE_ROUTE_GREEDY = 0, 1
BASE_ROUTE_SANITIZE = 0x100
QSCALE = 65536.0
BASE_TEST_WAIT_LIMIT_NS, BASE_TEST_AUCTION_ABSENT_CTA, BASE_TEST_GEMM_DROP_FIRST_LOAD = 0, 1, 2

# every symbol include/base.h declares
EXPORTED = (
    "base_status_string", "base_device_error", "base_version", "base_workspace_size",
    "base_scores", "base_assign_greedy", "base_assign_balanced", "base_assign_balanced_ex",
    "base_permute", "base_permute_noalloc", "base_expert_ffn", "base_combine", "base_layer_fwd",
    "base_layer_bwd", "base_test_inject", "base_workspace_size_blend", "base_layer_fwd_blend",
    "base_expert_stack", "base_sanitize_scores", "base_workspace_size_fig9", "base_assign_fig9",
    "base_probe_workspace_size", "base_measure_latency", "base_scores_greedy",
    "base_ep_dispatch", "base_ep_combine",
)


class LibraryMissing(RuntimeError):
    pass


class BaseError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__("%s failed: %s (%d)" % (fn, base_status_string(status), status))
        self.status = status


class Stats(ctypes.Structure):
    _fields_ = [("status", ctypes.c_int64), ("phases", ctypes.c_int64),
                ("rounds", ctypes.c_int64), ("final_eps", ctypes.c_int64),
                ("objective", ctypes.c_int64), ("bids", ctypes.c_int64)]


class LayerSaved(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "s", "q", "assign", "price", "stats", "perm", "inv", "offsets", "gate", "x_perm", "a1",
        "h1", "f", "y_perm")]


_lib = None
_vp = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t

_SIGS = {
    "base_status_string": (ctypes.c_char_p, [_i]),
    "base_version": (ctypes.c_char_p, []),
    "base_device_error": (_i, [ctypes.POINTER(ctypes.c_int64), _i]),
    "base_workspace_size": (_sz, [_i, _i, _i, _i]),
    "base_test_inject": (_i, [_i, ctypes.c_longlong]),
    "base_workspace_size_blend": (_sz, [_i, _i, _i, _i]),
    "base_sanitize_scores": (_i, [_vp, _vp, _i, _i, _vp, _sz, _vp]),
    "base_scores_greedy": (_i, [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp]),
    "base_workspace_size_fig9": (_sz, [_i, _i]),
    "base_probe_workspace_size": (_sz, []),
    "base_measure_latency": (_i, [_vp, _vp, _sz, _vp]),
    "base_assign_fig9": (_i, [_vp, _i, _i, _vp, _vp, _vp, ctypes.c_longlong, _vp, _sz, _vp]),
    "base_expert_stack": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _i, _vp, _vp, _vp,
                               _vp, _sz, _vp]),
    "base_layer_fwd_blend": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp,
                                  ctypes.POINTER(LayerSaved), _vp, _sz, _vp]),
    "base_scores": (_i, [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp]),
    "base_assign_greedy": (_i, [_vp, _i, _i, _vp, _vp, _vp]),
    "base_assign_balanced": (_i, [_vp, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp]),
    "base_assign_balanced_ex": (_i, [_vp, _i, _i, _vp, _vp, _vp, ctypes.c_longlong, _vp, _vp,
                                     ctypes.c_longlong, _vp, _sz, _vp]),
    "base_permute": (_i, [_vp, _vp, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "base_permute_noalloc": (_i, [_vp, _vp, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "base_expert_ffn": (_i, [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _i, _vp, _vp, _vp, _vp, _vp, _vp,
                             _sz, _vp]),
    "base_combine": (_i, [_vp, _vp, _i, _i, _vp, _vp]),
    "base_ep_dispatch": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]),
    "base_ep_combine": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]),
    "base_layer_fwd": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp,
                            ctypes.POINTER(LayerSaved), _vp, _sz, _vp]),
    "base_layer_bwd": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, ctypes.POINTER(LayerSaved),
                            _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
}


def lib(build_if_missing: bool = False):
    """The loaded libbase (ctypes.CDLL)."""
    global _lib
    if _lib is not None:
        return _lib
    if build_if_missing:
        _build.build()
    if not os.path.exists(_build.SO):
        raise LibraryMissing("libbase.so is not built (run balanced_token_expert_b200._build)")
    L = ctypes.CDLL(_build.SO)
    for name, (res, args) in _SIGS.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(fn: str, st: int):
    if st != BASE_OK:
        raise BaseError(fn, st)


def base_status_string(status: int) -> str:
    return lib().base_status_string(int(status)).decode()


def base_version() -> str:
    return lib().base_version().decode()


def base_workspace_size(T: int, E: int, D: int = 0, F: int = 0) -> int:
    return int(lib().base_workspace_size(T, E, D, F))


def base_device_error(clear: bool = True) -> int:
    v = ctypes.c_int64(0)
    _check("base_device_error", lib().base_device_error(ctypes.byref(v), 1 if clear else 0))
    return int(v.value)


def base_test_inject(hook: int, value: int) -> None:
    """Test hooks of the bounded waits (include/base.h): a shorter wait limit,
    an auction CTA that never arrives, a GEMM load that is never issued."""
    _check("base_test_inject", lib().base_test_inject(int(hook), int(value)))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return BASE_F32
    if t.dtype == torch.bfloat16:
        return BASE_BF16
    raise TypeError("h / w must be float32 or bfloat16")


def base_scores(h, w, s=None, q=None, stream=None):
    T, D = h.shape
    E = w.shape[0]
    _check("base_scores", lib().base_scores(_ptr(h), _ptr(w), _dtype_code(h), T, D, E, _ptr(s),
                                            _ptr(q), _stream(stream)))


def base_scores_greedy(h, w, s, q, assign, counts=None, stream=None):
    T, D = h.shape
    E = w.shape[0]
    _check("base_scores_greedy", lib().base_scores_greedy(
        _ptr(h), _ptr(w), _dtype_code(h), T, D, E, _ptr(s), _ptr(q), _ptr(assign), _ptr(counts),
        _stream(stream)))


def base_sanitize_scores(s, q, ws, stream=None):
    T, E = s.shape
    _check("base_sanitize_scores", lib().base_sanitize_scores(
        _ptr(s), _ptr(q), T, E, _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def base_assign_greedy(q, assign, counts=None, stream=None):
    T, E = q.shape
    _check("base_assign_greedy", lib().base_assign_greedy(_ptr(q), T, E, _ptr(assign), _ptr(counts),
                                                          _stream(stream)))


def base_assign_balanced(q, assign, price, stats=None, ws=None, stream=None):
    T, E = q.shape
    _check("base_assign_balanced", lib().base_assign_balanced(
        _ptr(q), T, E, _ptr(assign), _ptr(price), _ptr(stats), _ptr(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)))


def base_assign_balanced_ex(q, assign, price, stats, ws, max_rounds: int = 1000000,
                            u_trace=None, t_trace=None, stream=None):
    T, E = q.shape
    cap = 0
    for t in (u_trace, t_trace):
        if t is not None:
            cap = t.numel() if cap == 0 else min(cap, t.numel())
    _check("base_assign_balanced_ex", lib().base_assign_balanced_ex(
        _ptr(q), T, E, _ptr(assign), _ptr(price), _ptr(stats), int(max_rounds), _ptr(u_trace),
        _ptr(t_trace), cap, _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def base_probe_workspace_size() -> int:
    return int(lib().base_probe_workspace_size())


def base_measure_latency(out, ws, stream=None):
    """out: 4 float64 on the device (ns: grid barrier, block barrier, L2 load, shared load)."""
    _check("base_measure_latency", lib().base_measure_latency(
        _ptr(out), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def base_workspace_size_fig9(T: int, E: int) -> int:
    return int(lib().base_workspace_size_fig9(T, E))


def base_assign_fig9(q, assign, price, stats, ws, max_iterations: int = 100, stream=None):
    """The fig. 9 solver; price: T int64 token prices; stats: 4 int64 (device)."""
    T, E = q.shape
    _check("base_assign_fig9", lib().base_assign_fig9(
        _ptr(q), T, E, _ptr(assign), _ptr(price), _ptr(stats), int(max_iterations), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def base_permute(h, assign, E, perm, inv, offsets, x_perm, s=None, gate=None, ws=None,
                 stream=None):
    T = assign.shape[0]
    D = 0 if h is None else h.shape[1]
    _check("base_permute", lib().base_permute(
        _ptr(h), _ptr(assign), T, D, E, _ptr(perm), _ptr(inv), _ptr(offsets), _ptr(x_perm),
        _ptr(s), _ptr(gate), _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
        _stream(stream)))


def base_permute_noalloc(h, assign, E, perm, inv, offsets, x_perm, s=None, gate=None,
                         stream=None):
    """base_permute without a workspace (the library's own fixed scratch)."""
    T = assign.shape[0]
    D = 0 if h is None else h.shape[1]
    _check("base_permute_noalloc", lib().base_permute_noalloc(
        _ptr(h), _ptr(assign), T, D, E, _ptr(perm), _ptr(inv), _ptr(offsets), _ptr(x_perm),
        _ptr(s), _ptr(gate), _stream(stream)))


def base_expert_ffn(x_perm, offsets, W1, W2, act: int, gate, y_perm, h1, a1=None, f=None, ws=None,
                    stream=None):
    T, D = x_perm.shape
    E, F, _ = W1.shape
    _check("base_expert_ffn", lib().base_expert_ffn(
        _ptr(x_perm), _ptr(offsets), T, D, F, E, _ptr(W1), _ptr(W2), int(act), _ptr(gate),
        _ptr(y_perm), _ptr(h1), _ptr(a1), _ptr(f), _ptr(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)))


def base_combine(y_perm, perm, out, stream=None):
    T, D = y_perm.shape
    _check("base_combine", lib().base_combine(_ptr(y_perm), _ptr(perm), T, D, _ptr(out),
                                              _stream(stream)))


def _ptr_array(ts):
    """A host array of the tensors' device pointers (None for a missing list)."""
    if ts is None:
        return None
    return (ctypes.c_void_p * len(ts))(*[t.data_ptr() for t in ts])


def base_ep_dispatch(h, perm, gate, recv, recv_gate, g0: int, E: int, stream=None):
    """Sources g0 .. g0 + len(h) - 1 push their rows to every worker's receive
    buffer, expert-major (include/base.h).  h, perm, gate: lists over the
    sources; recv, recv_gate: lists over all G workers; gate and recv_gate
    None or given together."""
    T, D = h[0].shape
    G = len(recv)
    _check("base_ep_dispatch", lib().base_ep_dispatch(
        _ptr_array(h), _ptr_array(perm), _ptr_array(gate), _ptr_array(recv),
        _ptr_array(recv_gate), g0, len(h), G, T, D, E, _stream(stream)))


def base_ep_combine(y, perm, out, r0: int, E: int, stream=None):
    """Receivers r0 .. r0 + len(y) - 1 send every expert output row to its
    token in its source worker's out (include/base.h).  y: list over the
    receivers; perm, out: lists over all G workers."""
    T, D = y[0].shape
    G = len(out)
    _check("base_ep_combine", lib().base_ep_combine(
        _ptr_array(y), _ptr_array(perm), _ptr_array(out), r0, len(y), G, T, D, E,
        _stream(stream)))


def _saved(sv: dict) -> LayerSaved:
    st = LayerSaved()
    for name, _ in LayerSaved._fields_:
        t = sv.get(name)
        setattr(st, name, None if t is None else t.data_ptr())
    return st


def base_layer_fwd(h, w, W1, W2, act: int, routing: int, out, saved: dict, ws, stream=None):
    T, D = h.shape
    E, F, _ = W1.shape
    sv = _saved(saved)
    _check("base_layer_fwd", lib().base_layer_fwd(
        _ptr(h), _ptr(w), _ptr(W1), _ptr(W2), int(act), int(routing), T, D, E, F, _ptr(out),
        ctypes.byref(sv), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def base_workspace_size_blend(T: int, E: int, D: int, F: int) -> int:
    return int(lib().base_workspace_size_blend(T, E, D, F))


def base_expert_stack(x_perm, offsets, W1, W2, gamma, beta, act: int, gate, y_perm, h1, ws,
                      stream=None):
    T, D = x_perm.shape
    E, S, F, _ = W1.shape
    _check("base_expert_stack", lib().base_expert_stack(
        _ptr(x_perm), _ptr(offsets), T, D, F, E, S, _ptr(W1), _ptr(W2), _ptr(gamma), _ptr(beta),
        int(act), _ptr(gate), _ptr(y_perm), _ptr(h1), _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


def base_layer_fwd_blend(h, w, W1, W2, gamma, beta, act: int, routing: int, out, saved: dict, ws,
                         stream=None):
    """The released code's variant: W1 (E, S, F, D), W2 (E, S, D, F), gamma / beta (E, S, D)."""
    T, D = h.shape
    E, S, F, _ = W1.shape
    sv = _saved(saved)
    _check("base_layer_fwd_blend", lib().base_layer_fwd_blend(
        _ptr(h), _ptr(w), _ptr(W1), _ptr(W2), _ptr(gamma), _ptr(beta), S, int(act), int(routing),
        T, D, E, F, _ptr(out), ctypes.byref(sv), _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


def base_layer_bwd(h, w, W1, W2, act: int, saved: dict, dout, dh, dw, dW1, dW2, ws, stream=None):
    T, D = h.shape
    E, F, _ = W1.shape
    sv = _saved(saved)
    _check("base_layer_bwd", lib().base_layer_bwd(
        _ptr(h), _ptr(w), _ptr(W1), _ptr(W2), int(act), T, D, E, F, ctypes.byref(sv), _ptr(dout),
        _ptr(dh), _ptr(dw), _ptr(dW1), _ptr(dW2), _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))
