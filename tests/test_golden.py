"""The oracle reproduces its stored results on the routing reference
workload (written by tests/golden/make_golden.py from the oracle alone)."""
import json
import os

import numpy as np
import pytest

from balanced_token_expert_b200 import synth

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_routing_reference_fixture(orc, seed):
    rec = json.load(open(os.path.join(HERE, "routing_ref_seed%d.json" % seed)))
    inp = synth.make_inputs(synth.WORKLOADS["routing_ref"], seed)
    q = orc.quantize(orc.scores(inp.h, inp.w))
    assert int(q.astype(np.int64).sum()) == rec["q_sum"]
    a, p, st = orc.auction(q)
    assert a.tolist() == rec["assign"] and p.tolist() == rec["price"]
    assert st == rec["stats"]
    assert st["objective"] == rec["hungarian_objective"]
    ga, gc = orc.greedy(q)
    assert ga.tolist() == rec["greedy_assign"] and gc.tolist() == rec["greedy_counts"]
