"""The C ABI library (no GPU needed): it loads, exports every entry point
include/base.h declares, reports workspace sizes and status strings, and
rejects bad arguments on the host before launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from balanced_token_expert_b200 import _build, binding
    _build.build()
    return binding.lib()


def header_functions():
    src = open(os.path.join(ROOT, "include", "base.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(base_\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported(L):
    from balanced_token_expert_b200 import binding
    names = header_functions()
    assert len(names) >= 12
    assert sorted(binding.EXPORTED) == names
    for n in names:
        assert hasattr(L, n), n


def test_status_strings_and_version(L):
    from balanced_token_expert_b200 import binding as b
    assert b.base_status_string(0) == "ok"
    assert "converge" in b.base_status_string(3)
    assert b.base_status_string(99) == "unknown status"
    assert "sm_100a" in b.base_version()


def test_workspace_size_grows_with_the_problem(L):
    from balanced_token_expert_b200 import binding as b
    small = b.base_workspace_size(512, 8, 64, 0)
    big = b.base_workspace_size(131072, 128, 2048, 0)
    bwd = b.base_workspace_size(32768, 32, 2048, 8192)
    assert 0 < small < big
    # the backward keeps dy, dF (T x D bf16) and dA1 (T x F bf16)
    assert bwd >= 32768 * (2048 * 2 * 2 + 8192 * 2)
    assert b.base_workspace_size(0, 8, 64, 0) == 0
    assert b.base_workspace_size(64, 1, 64, 0) == 0


def test_bad_arguments_are_rejected_on_the_host(L):
    p = ctypes.c_void_p(4096)      # never dereferenced: the checks fail first
    odd = ctypes.c_void_p(4100)    # not 16-byte aligned
    ws = ctypes.c_void_p(1 << 20)
    # T % E != 0
    assert L.base_assign_balanced(p, 100, 8, p, p, None, ws, 1 << 30, None) == 1
    # null scores
    assert L.base_assign_balanced(None, 64, 8, p, p, None, ws, 1 << 30, None) == 1
    # E out of range
    assert L.base_assign_greedy(p, 64, 1, p, None, None) == 1
    assert L.base_assign_greedy(p, 64, 1025, p, None, None) == 1
    # workspace too small
    assert L.base_assign_balanced(p, 64, 8, p, p, None, ws, 16, None) == 5
    # bf16 scores need D % 8 == 0 and 16-byte aligned rows
    assert L.base_scores(p, p, 1, 64, 12, 8, p, None, None) == 1
    assert L.base_scores(odd, p, 1, 64, 16, 8, p, None, None) == 1
    assert L.base_scores(p, p, 7, 64, 16, 8, p, None, None) == 1
    # FFN: bad activation and bad widths
    assert L.base_expert_ffn(p, p, 64, 16, 32, 4, p, p, 5, p, p, p, None, None, ws, 1 << 20, None) == 1
    assert L.base_expert_ffn(p, p, 64, 12, 32, 4, p, p, 0, p, p, p, None, None, ws, 1 << 20, None) == 1
    # combine: misaligned output
    assert L.base_combine(p, p, 64, 16, odd, None) == 1
    # extended auction: cap out of range, trace without a capacity
    assert L.base_assign_balanced_ex(p, 64, 8, p, p, None, 0, None, None, 0, ws, 1 << 30, None) == 1
    assert L.base_assign_balanced_ex(p, 64, 8, p, p, None, 10, p, None, 0, ws, 1 << 30, None) == 1


def test_spec_constants_agree_between_library_and_oracle():
    # the two sides restate the spec constants independently; they must agree
    import oracle
    hdr = open(os.path.join(ROOT, "include", "base.h")).read()
    cu = open(os.path.join(ROOT, "balanced_token_expert_b200", "csrc", "auction.cu")).read()
    orc_c = open(os.path.join(ROOT, "oracle", "base_oracle.c")).read()
    assert float(re.search(r"BASE_QSCALE\s+([0-9.]+)f", hdr).group(1)) == oracle.QSCALE
    assert int(re.search(r"BASE_AUCTION_MAX_ROUNDS\s+(\d+)", hdr).group(1)) == oracle.MAX_ROUNDS
    assert int(re.search(r"kEpsDivisor = (\d+)", cu).group(1)) == oracle.EPS_DIVISOR
    assert int(re.search(r"kEpsFactor = (\d+)", cu).group(1)) == oracle.EPS_FACTOR
    assert int(re.search(r"ORC_EPS_DIVISOR (\d+)", orc_c).group(1)) == oracle.EPS_DIVISOR
    assert int(re.search(r"ORC_EPS_FACTOR (\d+)", orc_c).group(1)) == oracle.EPS_FACTOR


def test_product_path_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "balanced_token_expert_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, f
                assert "base_oracle" not in txt, f
