"""Caller-owned device buffers for the libbase entry points, allocated with
torch (the library itself never allocates)."""
from __future__ import annotations

import torch

from . import binding


def workspace(T: int, E: int, D: int = 0, F: int = 0, device="cuda") -> torch.Tensor:
    """A 256-byte-aligned uint8 workspace of base_workspace_size(T, E, D, F) bytes."""
    n = binding.base_workspace_size(T, E, D, F)
    ws = torch.empty(n + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    return ws[off:off + n]


def workspace_blend(T: int, E: int, D: int, F: int, device="cuda") -> torch.Tensor:
    """A 256-byte-aligned workspace of base_workspace_size_blend(T, E, D, F) bytes."""
    n = binding.base_workspace_size_blend(T, E, D, F)
    ws = torch.empty(n + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    return ws[off:off + n]


def workspace_fig9(T: int, E: int, device="cuda") -> torch.Tensor:
    """A 256-byte-aligned workspace of base_workspace_size_fig9(T, E) bytes."""
    n = binding.base_workspace_size_fig9(T, E)
    ws = torch.empty(n + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    return ws[off:off + n]


def stats(device="cuda") -> torch.Tensor:
    """Device storage for one base_auction_stats (6 int64)."""
    return torch.zeros(6, dtype=torch.int64, device=device)


def stats_dict(t: torch.Tensor) -> dict:
    v = t.tolist()
    return dict(status=v[0], phases=v[1], rounds=v[2], final_eps=v[3], objective=v[4], bids=v[5])


def layer_saved(T: int, E: int, D: int, F: int, device="cuda", for_backward: bool = True) -> dict:
    """The base_layer_saved buffers of one forward."""
    bf = torch.bfloat16
    sv = dict(
        s=torch.empty(T, E, dtype=torch.float32, device=device),
        q=torch.empty(T, E, dtype=torch.int32, device=device),
        assign=torch.empty(T, dtype=torch.int32, device=device),
        price=torch.empty(E, dtype=torch.int64, device=device),
        stats=stats(device),
        perm=torch.empty(T, dtype=torch.int32, device=device),
        inv=torch.empty(T, dtype=torch.int32, device=device),
        offsets=torch.empty(E + 1, dtype=torch.int32, device=device),
        gate=torch.empty(T, dtype=torch.float32, device=device),
        x_perm=torch.empty(T, D, dtype=bf, device=device),
        h1=torch.empty(T, F, dtype=bf, device=device),
        y_perm=torch.empty(T, D, dtype=bf, device=device),
    )
    if for_backward:
        sv["a1"] = torch.empty(T, F, dtype=bf, device=device)
        sv["f"] = torch.empty(T, D, dtype=bf, device=device)
    return sv
