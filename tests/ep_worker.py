"""One rank of the two-rank CPU (gloo) run of the expert-parallel layer,
started by test_expert_parallel_gloo.py.  The exchange is the package's; the
arithmetic of every step comes from the CPU oracle through a small backend
defined here (the test supplies it: the package never imports the oracle).
Writes the rank's outputs, shuffled tokens and assignment to the .npz given."""
import os
import sys
from datetime import timedelta

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

import oracle  # noqa: E402
from balanced_token_expert_b200 import expert_parallel as ep  # noqa: E402
from balanced_token_expert_b200 import replicas  # noqa: E402

T, E, D, F = 64, 4, 16, 32


def inputs(rank, G):
    g = torch.Generator().manual_seed(100)
    w = torch.randn(E, D, generator=g, dtype=torch.float64) / D ** 0.5
    W1 = torch.randn(E, F, D, generator=g, dtype=torch.float64) * 0.2
    W2 = torch.randn(E, D, F, generator=g, dtype=torch.float64) * 0.2
    h = torch.randn(T, D, generator=torch.Generator().manual_seed(rank), dtype=torch.float64)
    return h, w, W1, W2


class OracleBackend:
    """The steps in float64 with the CPU oracle (test infrastructure)."""

    def gather_rows(self, x, idx, idx_inv):
        return x[idx]

    def scatter_rows(self, y, idx):
        out = torch.empty_like(y)
        out[idx.long()] = y
        return out

    def route(self, x, w):
        s = oracle.scores(x.numpy(), w.numpy())
        a = oracle.auction(oracle.quantize(s))[0]
        return torch.from_numpy(a), torch.from_numpy(s)

    def permute(self, x, assign, s, E_):
        a = assign.numpy()
        perm, inv, offsets = oracle.permutation(a, E_)
        gate = s.numpy()[perm, a[perm]]
        return (torch.from_numpy(perm.astype(np.int64)), x[torch.from_numpy(perm.astype(np.int64))],
                torch.from_numpy(np.ascontiguousarray(gate)))

    def expert_ffn(self, x, offsets, W1, W2, act, gate):
        r = oracle.expert_ffn(x.numpy(), offsets.numpy(), W1.numpy(), W2.numpy(), "relu",
                              gate_s=gate.numpy())
        return torch.from_numpy(r["y"])


def main(out):
    rank, world, _ = replicas.rank_env()
    dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    plan = ep.EPPlan(T=T, E=E, G=world)
    h, w, W1, W2 = inputs(rank, world)
    lo, hi = rank * plan.El, (rank + 1) * plan.El
    y, shuffled, assign = ep.ep_layer_fwd(h, w, W1[lo:hi].contiguous(), W2[lo:hi].contiguous(), 0,
                                          plan, seed=1000 + rank, backend=OracleBackend(),
                                          return_route=True)
    dist.barrier()
    dist.destroy_process_group()
    np.savez(out, y=y.numpy(), shuffled=shuffled.numpy(), assign=assign.numpy())


if __name__ == "__main__":
    main(sys.argv[1])
