"""bench.py's reference arm on the CPU: one JSON line with the keys the
benchmark contract names (the oracle timed on the host, a small token count)."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line(orc):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "routing_ref", "--steps", "1", "--warmup", "1"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["n_gpus"] == 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["config"]["T"] == 512


def test_rounds_by_kind_groups_traced_rounds():
    sys.path.insert(0, ROOT)
    import bench
    # T = 8: a phase start (8 bidders), two narrow rounds, two one-bidder
    # rounds, a second phase start, and a last round with no successor
    u = [8, 3, 2, 1, 1, 8, 1]
    t = [0, 10000, 13000, 15000, 16000, 17500, 30000]
    k = bench._rounds_by_kind(u, t, rounds=7, T=8)
    assert k["phase start"] == dict(rounds=2, us_total=10.0 + 12.5, us_median=11.25)
    assert k["2-8 bidders"]["rounds"] == 2 and k["2-8 bidders"]["us_total"] == 5.0
    assert k["1 bidder"] == dict(rounds=2, us_total=2.5, us_median=1.25)
    assert "9-128 bidders" not in k


def test_latency_roofline_model():
    sys.path.insert(0, ROOT)
    import bench
    fl = dict(grid_barrier_ns=1000.0, block_barrier_ns=50.0, l2_load_ns=400.0, smem_load_ns=30.0)
    # T = 8192, E = 16: a phase start, a 300-bidder grid round, a 20-bidder
    # one-CTA round and two one-bidder rounds
    u = [8192, 300, 20, 1, 1]
    r = bench.latency_roofline(u, 8192, 16, auction_ms=0.01, fl=fl, hbm_gbs=6500.0)
    q_ns = 4.0 * 8192 * 16 / 6500.0
    expect = max(2800.0, q_ns) + 2800.0 + 500.0 + 400.0 + 400.0
    assert abs(r["floor_ms"] - expect / 1e6) < 1e-12
    assert abs(r["frac"] - expect / 1e6 / 0.01) < 1e-9
    # with E = 64 the one-CTA limit is 32 bidders: 40 bidders run grid-wide
    r2 = bench.latency_roofline([40], 8192, 64, auction_ms=1.0, fl=fl, hbm_gbs=6500.0)
    assert abs(r2["floor_ms"] - 2800.0 / 1e6) < 1e-12
