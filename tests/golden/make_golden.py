"""Writes the stored expected values under tests/golden/ from the oracle only.

The pages ("BASE Layers: Simplifying Training of Large, Sparse Models")
print no worked numeric example of the assignment, so the stored values are
the oracle's own results on the seeded routing reference workload (T=512,
E=8, D=64, fp32), each also checked against the Hungarian optimum before it
is written.  They freeze the oracle's trajectory (rounds, phases, bids) so
that a later change to its arithmetic shows up as a failing test.

Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from balanced_token_expert_b200 import synth  # noqa: E402


def main():
    for seed in (0, 1, 2):
        inp = synth.make_inputs(synth.WORKLOADS["routing_ref"], seed)
        q = oracle.quantize(oracle.scores(inp.h, inp.w))
        a, p, st = oracle.auction(q)
        hv, _ = oracle.hungarian(q)
        assert st["objective"] == hv and oracle.certificate(q, a, p)["ok"]
        ga, gc = oracle.greedy(q)
        rec = dict(workload="routing_ref", seed=seed, T=512, E=8, D=64,
                   q_sum=int(q.astype(np.int64).sum()), q_min=int(q.min()), q_max=int(q.max()),
                   hungarian_objective=hv, stats=st, assign=a.tolist(), price=p.tolist(),
                   greedy_assign=ga.tolist(), greedy_counts=gc.tolist())
        with open(os.path.join(HERE, "routing_ref_seed%d.json" % seed), "w") as fh:
            json.dump(rec, fh, separators=(",", ":"))
            fh.write("\n")


if __name__ == "__main__":
    main()
