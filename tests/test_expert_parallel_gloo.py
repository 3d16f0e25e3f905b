"""The expert-parallel exchange ("BASE Layers", wikillm.com summary: Method,
Sharding and Shuffling; fig. 2's four all-to-alls) with two gloo ranks on the
CPU.  Each rank holds E/2 experts; the outputs must equal what the layer gives
when every rank routes its shuffled tokens with its own balanced assignment and
runs them through all E experts locally, undone back to each rank's order."""
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch

from balanced_token_expert_b200 import expert_parallel as ep

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_plan_and_index_maps():
    with pytest.raises(ValueError):
        ep.EPPlan(T=64, E=6, G=4)
    plan = ep.EPPlan(T=24, E=4, G=2)   # C = 6, 2 experts per worker
    idx = ep.receive_order(plan)
    # received [g][j][c] -> expert-major [j][g][c]
    assert idx.tolist()[:12] == [0, 1, 2, 3, 4, 5, 12, 13, 14, 15, 16, 17]
    assert sorted(idx.tolist()) == list(range(24))
    p = ep.shuffle_permutation(24, 7)
    assert sorted(p.tolist()) == list(range(24))
    assert torch.equal(ep.shuffle_permutation(24, 7), p)
    inv = ep.inverse(p)
    assert torch.equal(p[inv], torch.arange(24))


def test_two_gloo_ranks_match_the_unsharded_layer(orc, tmp_path):
    import ep_worker as W
    world, port = 2, _free_port()
    procs = []
    for r in range(world):
        env = dict(os.environ, RANK=str(r), WORLD_SIZE=str(world), LOCAL_RANK=str(r),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, os.path.join(HERE, "ep_worker.py"),
                                       str(tmp_path / ("rank%d.npz" % r))], env=env))
    for p in procs:
        assert p.wait(timeout=180) == 0
    res = [np.load(tmp_path / ("rank%d.npz" % r)) for r in range(world)]
    T, G = W.T, world
    B = T // G
    ins = [W.inputs(r, G) for r in range(G)]
    w, W1, W2 = ins[0][1], ins[0][2], ins[0][3]
    x_sh = [ins[g][0].numpy()[ep.shuffle_permutation(T, 1000 + g).numpy()] for g in range(G)]
    for r in range(G):
        # rank r's shuffled tokens: block g came from rank g
        shuffled = np.concatenate([x_sh[g][r * B:(r + 1) * B] for g in range(G)])
        assert np.array_equal(res[r]["shuffled"], shuffled)
        a = orc.auction(orc.quantize(orc.scores(shuffled, w.numpy())))[0]
        assert np.array_equal(res[r]["assign"], a)
    for g in range(G):
        expect = np.empty((T, W.D))
        perm = ep.shuffle_permutation(T, 1000 + g).numpy()
        for r in range(G):
            shuffled = np.asarray(res[r]["shuffled"])
            ysh = orc.layer_forward(shuffled, w.numpy(), W1.numpy(), W2.numpy(), "relu",
                                    res[r]["assign"])["out"]
            expect[perm[r * B:(r + 1) * B]] = ysh[g * B:(g + 1) * B]
        assert np.allclose(res[g]["y"], expect, rtol=0, atol=1e-10)
