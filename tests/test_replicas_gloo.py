"""The replica (data-parallel) path with two gloo ranks on the CPU: every rank
routes its own tokens with no exchange ("BASE Layers", Method, Sharding), the
job's step time is the slowest rank's and the throughput counts every rank's
tokens."""
import json
import os
import socket
import subprocess
import sys

from balanced_token_expert_b200 import replicas, synth

HERE = os.path.dirname(os.path.abspath(__file__))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_route_their_own_batches(orc, tmp_path):
    world, port = 2, _free_port()
    procs = []
    for r in range(world):
        env = dict(os.environ, RANK=str(r), WORLD_SIZE=str(world), LOCAL_RANK=str(r),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, os.path.join(HERE, "replica_worker.py"),
                                       str(tmp_path / ("rank%d.json" % r))], env=env))
    for p in procs:
        assert p.wait(timeout=180) == 0
    res = [json.load(open(tmp_path / ("rank%d.json" % r))) for r in range(world)]
    # the step time every rank reports is the slowest rank's
    assert [x["step_ms"] for x in res] == [2.0, 2.0]
    # each rank solved its own problem: the single-process result for its seed
    wl = synth.WORKLOADS["routing_ref"]
    for r, x in enumerate(res):
        inp = synth.make_inputs(wl, replicas.rank_seed(r), with_weights=False, with_dout=False)
        a, _, st = orc.auction(orc.quantize(orc.scores(inp.h, inp.w)))
        assert x["status"] == 0 and x["assign"] == a.tolist()
        assert x["objective"] == st["objective"]
    assert res[0]["assign"] != res[1]["assign"]  # different tokens on each rank
    assert res[0]["objectives"] == res[1]["objectives"] == [res[0]["objective"], res[1]["objective"]]


def test_job_throughput_counts_every_rank():
    assert replicas.job_tokens_per_s(8192, 4, 2.0) == 8192 * 4 / 2e-3
    assert replicas.max_over_ranks(3.5) == 3.5  # no process group: the value itself
    assert replicas.rank_seed(0) != replicas.rank_seed(1)
