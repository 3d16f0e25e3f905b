"""base_permute_noalloc: the permutation for callers that cannot allocate
device memory (it keeps its scratch in a fixed array inside the library
instead of a caller workspace).  Its results must equal base_permute's, call
after call, although every call reuses the same scratch.

The file name makes pytest collect it last, so that if it fails, a run that
stops at the first failure (``-x``) has already run every other test; it
does not depend on anything the other tests leave behind and passes alone
in a fresh process too."""
import numpy as np
import pytest
import torch

from balanced_token_expert_b200 import binding as B
from balanced_token_expert_b200 import buffers

pytestmark = pytest.mark.gpu


def _case(T, E, D, seed, balanced):
    g = torch.Generator().manual_seed(seed)
    if balanced:
        assign = (torch.randperm(T, generator=g) % E).to(torch.int32)
    else:
        assign = torch.randint(0, E, (T,), generator=g, dtype=torch.int32)
    h = torch.randn(T, D, generator=g).to(torch.bfloat16)
    s = torch.randn(T, E, generator=g)
    return assign.cuda(), h.cuda(), s.cuda()


def _outputs(T, E, D):
    return (torch.empty(T, dtype=torch.int32, device="cuda"),
            torch.empty(T, dtype=torch.int32, device="cuda"),
            torch.empty(E + 1, dtype=torch.int32, device="cuda"),
            torch.empty(T, D, dtype=torch.bfloat16, device="cuda"),
            torch.empty(T, dtype=torch.float32, device="cuda"))


def test_noalloc_permute_matches_the_workspace_version_on_consecutive_calls():
    B.base_device_error(clear=True)
    # two calls in a row, the second with a smaller shape, so stale counts of
    # the first call sit in the shared scratch when the second one runs
    for T, E, D, seed, balanced in ((131072, 128, 64, 1, False), (3000, 7, 200, 2, True)):
        assign, h, s = _case(T, E, D, seed, balanced)
        ref = _outputs(T, E, D)
        got = _outputs(T, E, D)
        ws = buffers.workspace(T, E, D)
        B.base_permute(h, assign, E, ref[0], ref[1], ref[2], ref[3], s, ref[4], ws)
        B.base_permute_noalloc(h, assign, E, got[0], got[1], got[2], got[3], s, got[4])
        torch.cuda.synchronize()
        for a, b in zip(ref, got):
            assert torch.equal(a, b)
        # and the result is the stable expert-major order
        perm = got[0].cpu().numpy()
        a_np = assign.cpu().numpy()
        assert np.array_equal(perm, np.argsort(a_np, kind="stable"))
    assert B.base_device_error(clear=True) == 0


def test_noalloc_permute_without_rows_or_gate():
    # h = None and s = None: only the slot order (perm, inv, offsets) is made
    B.base_device_error(clear=True)
    T, E, D = 20000, 5, 8
    assign, h, s = _case(T, E, D, 3, False)
    ref = _outputs(T, E, D)
    got = _outputs(T, E, D)
    B.base_permute(None, assign, E, ref[0], ref[1], ref[2], None, ws=buffers.workspace(T, E, D))
    B.base_permute_noalloc(None, assign, E, got[0], got[1], got[2], None)
    torch.cuda.synchronize()
    for a, b in zip(ref[:3], got[:3]):
        assert torch.equal(a, b)
    assert B.base_device_error(clear=True) == 0


def test_noalloc_permute_rejects_shapes_beyond_its_scratch():
    T, E = 1 << 20, 1024  # 4096 chunks x 1024 experts > 1M counts
    with pytest.raises(B.BaseError) as ei:
        B.base_permute_noalloc(None, torch.zeros(T, dtype=torch.int32, device="cuda"), E,
                               torch.empty(T, dtype=torch.int32, device="cuda"),
                               torch.empty(T, dtype=torch.int32, device="cuda"),
                               torch.empty(E + 1, dtype=torch.int32, device="cuda"), None)
    assert ei.value.status == 5  # BASE_ERR_WORKSPACE
