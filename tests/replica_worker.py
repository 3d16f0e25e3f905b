"""One rank of the two-rank CPU (gloo) run of the replica path, started as a
subprocess by test_replicas_gloo.py: the rank routes its own seeded batch
with the oracle, takes part in the max-over-ranks step time and gathers every
rank's objective.  Writes its results as JSON to the path given."""
import json
import os
import sys
from datetime import timedelta

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch.distributed as dist  # noqa: E402

import oracle  # noqa: E402
from balanced_token_expert_b200 import replicas, synth  # noqa: E402


def main(out):
    rank, world, _ = replicas.rank_env()
    dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    step_ms = replicas.max_over_ranks(1.0 + rank)  # rank r "took" 1 + r ms
    wl = synth.WORKLOADS["routing_ref"]
    inp = synth.make_inputs(wl, replicas.rank_seed(rank), with_weights=False, with_dout=False)
    q = oracle.quantize(oracle.scores(inp.h, inp.w))
    assign, price, st = oracle.auction(q)
    objectives = [None] * world
    dist.all_gather_object(objectives, int(st["objective"]))
    dist.barrier()
    dist.destroy_process_group()
    with open(out, "w") as fh:
        json.dump(dict(rank=rank, world=world, step_ms=step_ms, objective=int(st["objective"]),
                       objectives=objectives, assign=assign.tolist(), status=st["status"]), fh)


if __name__ == "__main__":
    main(sys.argv[1])
