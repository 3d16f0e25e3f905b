"""Bounded device-side waits that give up.

Every spin-wait of the library has a limit; when it runs out, the kernel
records a code in the sticky device error word, lets its copies in flight
land, frees what it holds and returns, so the CUDA context stays usable.
These tests make a wait run out without any fault, through the library's
test hooks (base_test_inject): a short wait limit plus an arrival that never
comes -- an auction CTA that leaves before the first grid barrier, or a score
GEMM CTA whose first TMA load is never issued.  The next call on the same
context must then succeed and be exact.  (The pages' only failure rule is the
solver's iteration cap, "Solver", fig. 9 caption; these waits are this
library's hang guard.)"""
import time

import numpy as np
import pytest
import torch

from _util import close_scores, dev, to_np
from balanced_token_expert_b200 import binding as B
from balanced_token_expert_b200 import buffers, synth

pytestmark = pytest.mark.gpu

LIMIT_NS = 2_000_000  # 2 ms instead of the defaults (20 s grid barrier, 4 s pipeline)


def _reset_hooks():
    B.base_test_inject(B.BASE_TEST_WAIT_LIMIT_NS, 0)
    B.base_test_inject(B.BASE_TEST_AUCTION_ABSENT_CTA, -1)
    B.base_test_inject(B.BASE_TEST_GEMM_DROP_FIRST_LOAD, 0)


@pytest.fixture(autouse=True)
def hooks_off():
    _reset_hooks()
    B.base_device_error(clear=True)
    yield
    _reset_hooks()
    torch.cuda.synchronize()
    B.base_device_error(clear=True)


def test_hooks_reject_bad_values():
    for hook, value in ((B.BASE_TEST_WAIT_LIMIT_NS, -1), (B.BASE_TEST_AUCTION_ABSENT_CTA, -2),
                        (B.BASE_TEST_GEMM_DROP_FIRST_LOAD, 2), (7, 0)):
        with pytest.raises(B.BaseError) as ei:
            B.base_test_inject(hook, value)
        assert ei.value.status == 1


def test_auction_grid_barrier_gives_up_and_context_survives(orc):
    rng = np.random.default_rng(5)
    T, E = 4096, 16
    q_np = rng.integers(-300000, 300000, size=(T, E)).astype(np.int32)
    q = dev(q_np)
    assign = torch.full((T,), -1, dtype=torch.int32, device="cuda")
    price = torch.zeros(E, dtype=torch.int64, device="cuda")
    st = buffers.stats()
    ws = buffers.workspace(T, E)
    B.base_test_inject(B.BASE_TEST_WAIT_LIMIT_NS, LIMIT_NS)
    B.base_test_inject(B.BASE_TEST_AUCTION_ABSENT_CTA, 1)  # any CTA but the first
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    B.base_assign_balanced(q, assign, price, st, ws)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    _reset_hooks()
    assert B.base_device_error(clear=True) == 5001
    assert buffers.stats_dict(st)["status"] == 4  # BASE_ERR_TIMEOUT
    assert dt < 5.0  # gave up at the short limit, not after the 20 s default
    # the same context, the next call: exact again
    B.base_assign_balanced(q, assign, price, st, ws)
    torch.cuda.synchronize()
    assert B.base_device_error(clear=True) == 0
    ao, po, so = orc.auction(q_np)
    assert buffers.stats_dict(st) == so
    assert np.array_equal(to_np(assign), ao) and np.array_equal(to_np(price), po)


def test_gemm_pipeline_wait_gives_up_and_context_survives(orc):
    wl = synth.WORKLOADS["layer_fwd"]
    inp = synth.make_inputs(wl, 2, with_weights=False, with_dout=False)
    T, E = wl.T, wl.E
    h, w = dev(inp.h), dev(inp.w)
    s = torch.empty(T, E, device="cuda")
    q = torch.empty(T, E, dtype=torch.int32, device="cuda")
    B.base_test_inject(B.BASE_TEST_WAIT_LIMIT_NS, LIMIT_NS)
    B.base_test_inject(B.BASE_TEST_GEMM_DROP_FIRST_LOAD, 1)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    B.base_scores(h, w, s, q)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    _reset_hooks()
    # the MMA warp's wait for the stage that never filled (3003); the other
    # warps of that CTA see the error word and leave without a code of their own
    assert B.base_device_error(clear=True) == 3003
    assert dt < 5.0
    B.base_scores(h, w, s, q)
    torch.cuda.synchronize()
    assert B.base_device_error(clear=True) == 0
    ok, worst = close_scores(to_np(s), orc.scores(inp.h, inp.w), 1e-5)
    assert ok, worst
    sg = to_np(s)
    assert np.array_equal(to_np(q), np.rint(sg * np.float32(65536)).astype(np.int32))
