"""Expert parallelism for the BASE layer: E/G experts on each of G workers.

"BASE Layers: Simplifying Training of Large, Sparse Models", wikillm.com
summary, Method (Sharding, Shuffling) and the fig. 2 listing: every worker
holds T tokens and E/G experts; a training forward makes four all-to-alls --

1. shuffle: every worker sends a seeded random T/G of its tokens to each
   worker, which breaks the correlation of a sequence's tokens;
2. route: each worker scores its shuffled tokens against all E centroids and
   solves its own balanced assignment (every expert gets T/E of this worker's
   tokens: the problem splits per worker, no exchange), sorts them by expert
   and sends each worker the C (E/G) tokens of that worker's experts, with
   their gate scores;
3. the experts run on the tokens they received (eq. 1's gated FFN with the
   residual), and the results go back the way they came;
4. combine (the inverse sort) and undo the shuffle.

This module is the exchange: the index maps, the equal-split all-to-alls and
their inverses.  The arithmetic of every step is delegated to a backend;
:class:`CudaBackend` runs each step in the library's kernels (the routing,
the permutation, the grouped FFN and the row moves), with torch used for
device memory and ``torch.distributed`` (NCCL on GPUs) for the all-to-alls.
With one worker the exchanges are identities and the layer is the single-GPU
path applied to the shuffled tokens.

:func:`ep_layer_fwd_fused` runs the same layer with the library's fused
exchange kernels instead of all-to-alls (base_ep_dispatch / base_ep_combine:
each permutation and its exchange in one pass over peer-addressable
buffers), for workers whose buffers are all on this device.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch
import torch.distributed as dist

__all__ = ["EPPlan", "shuffle_permutation", "receive_order", "exchange", "ep_layer_fwd",
           "CudaBackend", "ep_layer_fwd_fused"]


@dataclass(frozen=True)
class EPPlan:
    """Sizes of one expert-parallel layer call.  T tokens per worker, E experts
    in all, G workers (E/G experts each), C = T/E tokens per expert from each
    worker."""
    T: int
    E: int
    G: int

    def __post_init__(self):
        if self.E % self.G or self.T % self.G or self.T % self.E:
            raise ValueError("expert parallelism needs G | E, G | T and E | T (T=%d E=%d G=%d)"
                             % (self.T, self.E, self.G))

    @property
    def C(self) -> int:
        return self.T // self.E

    @property
    def El(self) -> int:
        return self.E // self.G


def shuffle_permutation(T: int, seed: int) -> torch.Tensor:
    """The shuffle's random permutation of a worker's T tokens (fig. 2:
    random_permutation(T)), from a CPU generator: int64, on the CPU."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return torch.randperm(T, generator=g)


def receive_order(plan: EPPlan) -> torch.Tensor:
    """Rows received in step 2 arrive grouped by source worker, then local
    expert, then token ([g][j][c]); the grouped FFN wants each local expert's
    rows together ([j][g][c]).  Returns idx with expert-major row i taken from
    received row idx[i] (int64, CPU)."""
    G, El, C = plan.G, plan.El, plan.C
    j = torch.arange(El).view(El, 1, 1)
    g = torch.arange(G).view(1, G, 1)
    c = torch.arange(C).view(1, 1, C)
    return (g * (El * C) + j * C + c).reshape(-1)


def inverse(idx: torch.Tensor) -> torch.Tensor:
    """inv with inv[idx[i]] = i."""
    inv = torch.empty_like(idx)
    inv[idx] = torch.arange(idx.numel(), dtype=idx.dtype, device=idx.device)
    return inv


def exchange(t: torch.Tensor, group=None) -> torch.Tensor:
    """All-to-all with equal splits along dim 0: block g of this worker's rows
    goes to worker g, and block g of the result came from worker g.  With one
    worker (or no process group) it returns t itself."""
    if not (dist.is_available() and dist.is_initialized()):
        return t
    if dist.get_world_size(group) == 1:
        return t
    out = torch.empty_like(t)
    dist.all_to_all_single(out, t.contiguous(), group=group)
    return out


def ep_layer_fwd(h, w, W1_local, W2_local, act: int, plan: EPPlan, seed: int, backend,
                 group=None, return_route: bool = False):
    """One expert-parallel BASE layer forward with balanced routing on this
    worker.  h: (T, D) this worker's tokens; w: (E, D) all centroids;
    W1_local / W2_local: this worker's E/G experts.  Every worker calls it
    with its own seed (the shuffle).  Returns (T, D) outputs in h's order
    (and, with return_route, the shuffled tokens and their assignment)."""
    T, E, G = plan.T, plan.E, plan.G
    dev = h.device
    perm = shuffle_permutation(T, seed)
    perm_inv = inverse(perm)
    ridx = receive_order(plan)
    ridx_inv = inverse(ridx)
    # 1. shuffle: block g of this worker's shuffled tokens goes to worker g
    x_sh = backend.gather_rows(h, perm, perm_inv)
    shuffled = exchange(x_sh, group)
    # 2. route the shuffled tokens: scores, balanced assignment, expert-major slots
    assign, s = backend.route(shuffled, w)
    order, x_perm, gate = backend.permute(shuffled, assign, s, E)
    recv_x = exchange(x_perm, group)    # [g][j][c]: worker g's tokens for local expert j
    recv_gate = exchange(gate, group)
    # 3. the local experts, each expert's rows together
    x_loc = backend.gather_rows(recv_x, ridx, ridx_inv)
    gate_loc = recv_gate[ridx.to(dev)]
    offsets = torch.arange(0, plan.El + 1, dtype=torch.int32) * (G * plan.C)
    y_loc = backend.expert_ffn(x_loc, offsets.to(dev), W1_local, W2_local, act, gate_loc)
    y_recv = backend.scatter_rows(y_loc, ridx)     # back to the [g][j][c] order
    y_perm = exchange(y_recv, group)               # this worker's slots
    # 4. combine (inverse sort), then undo the shuffle
    y_sh = backend.scatter_rows(y_perm, order)
    back = exchange(y_sh, group)
    out = backend.scatter_rows(back, perm)
    if return_route:
        return out, shuffled, assign
    return out


class CudaBackend:
    """The steps of :func:`ep_layer_fwd` in the library's kernels (through the
    C ABI); tensors on the current CUDA device, h / weights bf16."""

    def __init__(self, T: int, E: int, D: int, F: int):
        from . import binding as B
        from . import buffers
        self.B, self.bufs = B, buffers
        self.T, self.E, self.D, self.F = T, E, D, F
        self.ws = buffers.workspace(T, E, D, F)

    def _dev_idx(self, idx):
        return idx.to(device="cuda", dtype=torch.int32)

    def scatter_rows(self, y, idx):
        """out[idx[i]] = y[i] (the library's row scatter)."""
        out = torch.empty_like(y)
        self.B.base_combine(y, self._dev_idx(idx), out)
        return out

    def gather_rows(self, x, idx, idx_inv):
        """out[i] = x[idx[i]], as a scatter through the inverse permutation."""
        return self.scatter_rows(x, idx_inv)

    def route(self, x, w):
        T, E = x.shape[0], w.shape[0]
        s = torch.empty(T, E, device="cuda")
        q = torch.empty(T, E, dtype=torch.int32, device="cuda")
        self.B.base_scores(x, w, s, q)
        assign = torch.empty(T, dtype=torch.int32, device="cuda")
        price = torch.empty(E, dtype=torch.int64, device="cuda")
        self.B.base_assign_balanced(q, assign, price, self.bufs.stats(), self.ws)
        return assign, s

    def permute(self, x, assign, s, E):
        T, D = x.shape
        perm = torch.empty(T, dtype=torch.int32, device="cuda")
        inv = torch.empty_like(perm)
        offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
        x_perm = torch.empty_like(x)
        gate = torch.empty(T, device="cuda")
        self.B.base_permute(x, assign, E, perm, inv, offsets, x_perm, s, gate, self.ws)
        return perm, x_perm, gate

    def expert_ffn(self, x, offsets, W1, W2, act, gate):
        T, D = x.shape
        F = W1.shape[1]
        y = torch.empty_like(x)
        h1 = torch.empty(T, F, dtype=x.dtype, device="cuda")
        self.B.base_expert_ffn(x, offsets, W1, W2, act, gate, y, h1, None, None, self.ws)
        return y


def ep_layer_fwd_fused(hs, w, W1s, W2s, act: int, plan: EPPlan, seeds=None, stream=None):
    """The expert-parallel forward with the library's fused exchange kernels,
    for G workers whose buffers are all on this device.

    With seeds (one per worker), the shuffle comes first and the unshuffle
    last, each the same kind of exchange with one destination block per
    worker: base_ep_dispatch with G "experts" of T/G rows through the
    worker's shuffle permutation sends block r of its shuffled tokens to
    worker r, and base_ep_combine undoes it.  Without seeds the inputs are
    taken as already shuffled.

    Each worker scores its tokens against all E centroids, solves its own
    balanced assignment and sorts its slots by expert (no rows moved); one
    base_ep_dispatch call then moves every worker's rows straight into the
    receiving workers' expert-major buffers (the permutation, the route
    all-to-all and the regrouping in one pass), each worker runs its E/G
    experts with eq. 1's gate and residual, and one base_ep_combine call sends
    every output row to its token in its source worker (the return all-to-all
    and the inverse sort in one pass).  On one GPU this runs the whole
    exchange; across GPUs each worker would pass its own rank and the peer
    mappings of the others' buffers.

    hs: G (T, D) bf16 batches; w: (E, D) bf16 centroids; W1s / W2s: per worker
    (E/G, F, D) and (E/G, D, F) bf16 expert weights.  Returns the G (T, D)
    outputs in each worker's token order."""
    from . import binding as B
    from . import buffers
    T, E, G = plan.T, plan.E, plan.G
    D = hs[0].shape[1]
    F = W1s[0].shape[1]
    C, El = plan.C, plan.El
    ws = buffers.workspace(T, E, D, F)
    sperms = None
    if seeds is not None:
        # 1. shuffle: worker g's shuffled block r goes to worker r, position g T/G
        sperms = [shuffle_permutation(T, sd).to(device="cuda", dtype=torch.int32) for sd in seeds]
        shuffled = [torch.empty_like(hs[0]) for _ in range(G)]
        B.base_ep_dispatch(hs, sperms, None, shuffled, None, 0, G, stream)
        hs = shuffled
    perms, gates = [], []
    for g in range(G):
        s = torch.empty(T, E, device="cuda")
        q = torch.empty(T, E, dtype=torch.int32, device="cuda")
        B.base_scores(hs[g], w, s, q, stream)
        assign = torch.empty(T, dtype=torch.int32, device="cuda")
        price = torch.empty(E, dtype=torch.int64, device="cuda")
        B.base_assign_balanced(q, assign, price, buffers.stats(), ws, stream)
        perm = torch.empty(T, dtype=torch.int32, device="cuda")
        inv = torch.empty_like(perm)
        offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
        gate = torch.empty(T, device="cuda")
        B.base_permute(None, assign, E, perm, inv, offsets, None, s, gate, ws, stream)
        perms.append(perm)
        gates.append(gate)
    recv = [torch.empty(T, D, dtype=hs[0].dtype, device="cuda") for _ in range(G)]
    recv_gate = [torch.empty(T, device="cuda") for _ in range(G)]
    B.base_ep_dispatch(hs, perms, gates, recv, recv_gate, 0, E, stream)
    offs = (torch.arange(El + 1, dtype=torch.int32) * (G * C)).cuda()
    ys = []
    for r in range(G):
        y = torch.empty(T, D, dtype=hs[0].dtype, device="cuda")
        h1 = torch.empty(T, F, dtype=hs[0].dtype, device="cuda")
        B.base_expert_ffn(recv[r], offs, W1s[r], W2s[r], act, recv_gate[r], y, h1, None, None, ws,
                          stream)
        ys.append(y)
    outs = [torch.empty(T, D, dtype=hs[0].dtype, device="cuda") for _ in range(G)]
    B.base_ep_combine(ys, perms, outs, 0, E, stream)
    if sperms is not None:
        # 4. unshuffle: every row back to its worker and position
        back = [torch.empty_like(outs[0]) for _ in range(G)]
        B.base_ep_combine(outs, sperms, back, 0, G, stream)
        outs = back
    return outs
