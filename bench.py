#!/usr/bin/env python
"""Benchmark of the BASE-layer forward hot path on B200.

One step = one pass of the whole forward path over one batch of synthetic
tokens: bf16 affinity scores + quantisation (tcgen05) -> balanced Jacobi
auction -> expert-major permutation -> expert FFNs with the gated residual
(tcgen05) -> combine.  Default workload: T=8192 tokens, E=16 experts,
D=1024, FFN 1024 -> 4096 -> 1024 ReLU (bf16, random N(0, 0.02) weights,
h ~ N(0,1), w ~ N(0, 1/D)).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

The same run then times the other workloads a few steps each (--extra-steps)
and reports them under "workloads": the skewed-affinity auction stress
(T=32768, E=64), large routing (T=131072, E=128: scores, auction, greedy,
permute), the training step (T=32768, E=32, D=2048, FFN 8192 GELU, forward +
backward) and the released code's layer variant on the default shape (layer
norm + FFN + residual expert, convex blend).  --workload NAME --only times one workload alone.

With N > 1 (torchrun, one rank per GPU) every rank runs its own independent
problem (the balanced assignment decomposes per worker, so no collective is
on the data path); the time is the max over ranks.  Rank 0 prints one JSON
line.  ``--impl reference`` times the CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "tokens routed/s (auction) & BASE-layer fwd tokens/s; % of HBM/TC roofline"
UNIT = "tokens/s"


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of a
# step component, from one ncu capture of this bench's own command on the
# named workload at its full size (the component's kernels summed); a
# component whose kernels changed after their capture has no entry.
NCU_TRAFFIC = {
    ("scores", "layer_fwd"): 16854272,
    ("auction", "layer_fwd"): 772608 + 1024,
    # slice histogram + slice rank + row gather; the rows' writes stay in L2
    ("permute", "layer_fwd"): 37376 + 588544 + 16816640,
    # GEMM1 (h1 written, partly kept in L2) + GEMM2
    ("ffn", "layer_fwd"): 151065600 + 35437824 + 222275840 + 6731776,
    ("combine", "layer_fwd"): 16815872,
}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="layer_fwd")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--flush-mb", type=int, default=256)
    p.add_argument("--only", action="store_true",
                   help="time the chosen workload alone (no other workloads in the same run)")
    p.add_argument("--extra-steps", type=int, default=5,
                   help="timed steps of each of the other workloads")
    p.add_argument("--tokens", type=int, default=0,
                   help="run the workload with this many tokens instead (profiling a small case)")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons.  Sampling runs
    from before the warm-up to after the timed region; the summary keeps the
    samples taken inside [t0 - 0.1 s, t1 + 0.1 s] of the timed region."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.t0 = self.t1 = None
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(index), "--query-gpu=" + self.FIELDS,
                                       "--format=csv,noheader,nounits", "-lms", "20"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        if self.p is None:
            return None
        time.sleep(0.15)
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except Exception:
            self.p.kill()
        self.f.flush()
        import datetime
        rows = []
        for line in open(self.f.name):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                continue
            rows.append((ts, parts))
        os.unlink(self.f.name)
        if self.t0 is not None and self.t1 is not None:
            inside = [r for ts, r in rows if self.t0 - 0.1 <= ts <= self.t1 + 0.1]
            if inside:
                rows = [(0, r) for r in inside]
        rows = [r for _, r in rows]
        if not rows:
            return None
        num = lambda x: float(x) if x.replace(".", "", 1).isdigit() else None  # noqa: E731
        sm = [num(r[2]) for r in rows if num(r[2]) is not None]
        mx = [num(r[3]) for r in rows if num(r[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i] == "Active"})
        return dict(sm_mhz=statistics.median(sm) if sm else None,
                    sm_max_mhz=max(mx) if mx else None, reasons=reasons, samples=len(rows))


def _oracle_step(oracle, wl, inp):
    s = oracle.scores(inp.h, inp.w)
    q = oracle.quantize(s)
    if inp.bump_tokens is not None:
        q[inp.bump_tokens.numpy(), 0] += int(round(inp.bump_value * oracle.QSCALE))
    a = oracle.auction(q)[0]
    if wl.F:
        oracle.layer_forward(inp.h, inp.w, inp.W1, inp.W2, wl.act, a)
    else:
        oracle.greedy(q)
        perm = oracle.permutation(a, wl.E)[0]
        oracle.gather_rows(inp.h, perm)


def cpu_baseline(wl, seed=0):
    """The oracle as it stands, one full forward of the workload on the host."""
    import oracle
    from balanced_token_expert_b200 import synth
    inp = synth.make_inputs(wl, seed)
    t0 = time.perf_counter()
    _oracle_step(oracle, wl, inp)
    dt = time.perf_counter() - t0
    return dict(value=wl.T / dt, unit=UNIT, cores=len(os.sched_getaffinity(0)), kind="oracle",
                sample="one full forward of the workload (T=%d tokens: float64 scores, integer "
                       "auction, float64 expert FFNs) on the host, %.2f s" % (wl.T, dt))


def run_reference(args, wl, rank, world):
    if rank != 0:
        return
    import oracle
    from balanced_token_expert_b200 import synth
    oracle.build()
    inp = synth.make_inputs(wl, 0)

    def step():
        _oracle_step(oracle, wl, inp)

    for _ in range(args.warmup):
        step()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        step()
        times.append(time.perf_counter() - t0)
    ms = 1e3 * statistics.mean(times)
    value = wl.T / (ms / 1e3)
    cores = len(os.sched_getaffinity(0))
    print(json.dumps(dict(
        impl="reference", metric=METRIC, value=value, unit=UNIT, n_gpus=world, steps=args.steps,
        warmup=args.warmup, ms_per_step=ms, higher_is_better=True, scaling="weak",
        vs_baseline=None, dtype="f64", data="synthetic",
        config=_config(wl, args),
        cpu_baseline=dict(value=value, unit=UNIT, cores=cores, kind="oracle",
                          sample="every step: one full forward of the workload on the host"),
        e2e=dict(value=value, unit=UNIT, h2d_bytes_per_step=0, d2h_bytes_per_step=0))))


def _config(wl, args):
    if wl.S:
        desc = ("%s: the released code's BASE layer variant, T=%d tokens, E=%d experts, D=%d, "
                "experts of %d sublayer(s) layer norm + FFN %d->%d->%d %s + residual, convex "
                "blend, balanced auction routing, bf16" % (wl.name, wl.T, wl.E, wl.D, wl.S, wl.D,
                                                          wl.F, wl.D, wl.act))
    elif wl.F:
        desc = ("%s: BASE layer %s, T=%d tokens, E=%d experts, D=%d, FFN %d->%d->%d %s, "
                "balanced auction routing, bf16" % (wl.name, "forward+backward" if wl.backward
                                                     else "forward", wl.T, wl.E, wl.D, wl.D, wl.F,
                                                     wl.D, wl.act))
    else:
        desc = ("%s: scores + balanced auction + greedy + permute, T=%d tokens, E=%d experts, "
                "D=%d, bf16%s" % (wl.name, wl.T, wl.E, wl.D,
                                  ", skewed mixture with +3 affinity on expert 0 for half the "
                                  "tokens" if wl.kind == "mixture" else ""))
    return dict(workload=desc,
                T=wl.T, E=wl.E, D=wl.D, F=wl.F, act=wl.act, routing="balanced",
                l2="flushed between timed steps (%d MiB write)" % args.flush_mb,
                parallelism="independent replica per GPU")


EXTRA_WORKLOADS = ("skewed", "large_routing", "layer_fwd_bwd", "layer_fwd_blend")


def measure(args, wl, steps, warmup, rank, world, local_rank):
    """Times one workload: every component with CUDA events on the launching
    stream (L2 flushed between steps, max over ranks), then end to end through
    the public call with host buffers.  Returns the result dict (rank 0) or
    None (other ranks); every rank takes the same collective steps."""
    import torch
    from balanced_token_expert_b200 import binding as B
    from balanced_token_expert_b200 import buffers, replicas, synth

    T, E, D, F = wl.T, wl.E, wl.D, wl.F
    inp = synth.make_inputs(wl, seed=replicas.rank_seed(rank))
    h = inp.h.cuda()
    w = inp.w.cuda()
    W1 = inp.W1.cuda() if F else None
    W2 = inp.W2.cuda() if F else None
    act = B.BASE_RELU if wl.act == "relu" else B.BASE_GELU
    sv = buffers.layer_saved(T, E, D, max(F, 8), for_backward=wl.backward)
    out = torch.empty(T, D, dtype=torch.bfloat16, device="cuda")
    ws = buffers.workspace_blend(T, E, D, F) if wl.S else buffers.workspace(T, E, D, F)
    if wl.S:  # the released code's variant: S sublayers per expert
        extra = synth.make_stack_params(wl, wl.S, seed=replicas.rank_seed(rank))
        W1 = torch.cat([inp.W1[:, None]] + ([extra["W1"]] if wl.S > 1 else []), 1).cuda()
        W2 = torch.cat([inp.W2[:, None]] + ([extra["W2"]] if wl.S > 1 else []), 1).cuda()
        gam, bet = extra["gamma"].cuda(), extra["beta"].cuda()
    flush = torch.empty(args.flush_mb * (1 << 20), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    q_bump = None
    if inp.bump_tokens is not None:  # test data: +bump on expert 0's quantised affinity
        q_bump = (inp.bump_tokens.cuda(), int(round(inp.bump_value * B.QSCALE)))
    greedy_assign = torch.empty(T, dtype=torch.int32, device="cuda")
    greedy_counts = torch.empty(E, dtype=torch.int32, device="cuda")

    fused_greedy = not F and inp.bump_tokens is None and E <= 256
    if fused_greedy:
        # the routing step's test-time argmax comes out of the score GEMM's epilogue
        comps = [("scores_greedy", lambda: B.base_scores_greedy(h, w, sv["s"], sv["q"],
                                                                 greedy_assign, greedy_counts), 1)]
    else:
        comps = [("scores", lambda: B.base_scores(h, w, sv["s"], sv["q"]), 1)]
    if q_bump is not None:
        comps.append(("bump", lambda: sv["q"][:, 0].index_add_(
            0, q_bump[0], torch.full_like(q_bump[0], q_bump[1], dtype=torch.int32)), 0))
    # third field: our kernels the call launches (the auction: one cooperative
    # kernel; the permute: two sort launches and the row gather)
    comps.append(("auction", lambda: B.base_assign_balanced(sv["q"], sv["assign"], sv["price"],
                                                             sv["stats"], ws), 1))
    if not F and not fused_greedy:
        comps.append(("greedy", lambda: B.base_assign_greedy(sv["q"], greedy_assign,
                                                              greedy_counts), 1))
    comps.append(("permute", lambda: B.base_permute(h, sv["assign"], E, sv["perm"], sv["inv"],
                                                     sv["offsets"], sv["x_perm"], sv["s"],
                                                     sv["gate"], ws), 3))
    if F and wl.S:
        comps.append(("stack", lambda: B.base_expert_stack(sv["x_perm"], sv["offsets"], W1, W2,
                                                           gam, bet, act, sv["gate"], sv["y_perm"],
                                                           sv["h1"], ws), 3 * wl.S))
        comps.append(("combine", lambda: B.base_combine(sv["y_perm"], sv["perm"], out), 1))
    elif F:
        comps.append(("ffn", lambda: B.base_expert_ffn(sv["x_perm"], sv["offsets"], W1, W2, act,
                                                       sv["gate"], sv["y_perm"], sv["h1"],
                                                       sv.get("a1"), sv.get("f"), ws), 2))
        comps.append(("combine", lambda: B.base_combine(sv["y_perm"], sv["perm"], out), 1))
    if wl.backward:
        dout = inp.dout.cuda()
        dh = torch.empty(T, D, dtype=torch.bfloat16, device="cuda")
        dw = torch.empty(E, D, device="cuda")
        dW1 = torch.empty(E, F, D, device="cuda")
        dW2 = torch.empty(E, D, F, device="cuda")
        comps.append(("backward", lambda: B.base_layer_bwd(h, w, W1, W2, act, sv, dout, dh, dw,
                                                           dW1, dW2, ws), 8))
    names = [n for n, _, _ in comps if n != "bump"]

    def step(ev):
        j = 0
        for n, fn, _ in comps:
            if n == "bump":
                fn()
                continue
            ev[2 * j].record(stream)
            fn()
            ev[2 * j + 1].record(stream)
            j += 1

    phys = 0
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        try:
            phys = int(vis.split(",")[local_rank])
        except ValueError:
            phys = local_rank
    else:
        phys = local_rank
    clocks = Clocks(phys) if rank == 0 else None
    kernels_per_step = sum(k for _, _, k in comps)
    mk = lambda: [torch.cuda.Event(enable_timing=True) for _ in range(2 * len(names))]  # noqa: E731
    for _ in range(max(3, warmup)):
        flush.zero_()
        step(mk())
    torch.cuda.synchronize()
    B.base_device_error(clear=True)

    evs = [mk() for _ in range(steps)]
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    if clocks:
        clocks.mark_start()
    wall0 = time.perf_counter()
    for i in range(steps):
        flush.zero_()
        step(evs[i])
    torch.cuda.synchronize()
    if clocks:
        clocks.mark_end()
    if world > 1:
        dist.barrier()
    wall = time.perf_counter() - wall0
    per = {n: [] for n in names}
    for ev in evs:
        for j, n in enumerate(names):
            per[n].append(ev[2 * j].elapsed_time(ev[2 * j + 1]))
    step_ms = [sum(per[n][i] for n in names) for i in range(steps)]
    ms = statistics.mean(step_ms)
    st = buffers.stats_dict(sv["stats"])
    err = B.base_device_error(clear=True)
    ms = replicas.max_over_ranks(ms, device=torch.device("cuda"))
    clk = clocks.stop() if clocks else None

    # the auction's rounds by kind (an untimed traced run of the same call):
    # time per round grouped by the number of bidders, from the GPU timer
    trace_cap = st["rounds"] + 1
    u_tr = torch.zeros(trace_cap, dtype=torch.int32, device="cuda")
    t_tr = torch.zeros(trace_cap, dtype=torch.int64, device="cuda")
    B.base_assign_balanced_ex(sv["q"], sv["assign"], sv["price"], sv["stats"], ws, 1000000,
                              u_trace=u_tr, t_trace=t_tr)
    torch.cuda.synchronize()
    u_list = u_tr.cpu().tolist()
    rounds_by_kind = _rounds_by_kind(u_list, t_tr.cpu().tolist(), st["rounds"], wl.T)

    # the fig. 9 solver on the same scores: the alternative the pages print,
    # compared on rounds, time and objective (it is not the exact optimum)
    f9_a = torch.empty(T, dtype=torch.int32, device="cuda")
    f9_p = torch.empty(T, dtype=torch.int64, device="cuda")
    f9_s = torch.zeros(4, dtype=torch.int64, device="cuda")
    ws9 = buffers.workspace_fig9(T, E)
    f9_ms = []
    for i in range(4):
        flush.zero_()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        B.base_assign_fig9(sv["q"], f9_a, f9_p, f9_s, ws9)
        a1.record(stream)
        torch.cuda.synchronize()
        if i:
            f9_ms.append(a0.elapsed_time(a1))
    f9 = f9_s.tolist()
    fig9 = dict(ms=statistics.mean(f9_ms), rounds=f9[1], status=f9[0], eps=f9[2],
                objective=f9[3], objective_below_auction=st["objective"] - f9[3])
    del ws9

    # end to end through the public call: every step copies its inputs in from
    # pinned host memory (the tokens; for a training step also the upstream
    # gradient) and reads its result back.  Measured two ways: step by
    # step (copy in, compute, copy out, synchronise), and as a serving loop runs
    # it (one copy stream each way and two device buffers: step i+1's input
    # copy and step i-1's output copy overlap step i's compute).  Both keep the
    # L2 flush between steps, on the compute stream inside the timed region.
    nbuf = 2
    h_host = [inp.h.pin_memory() for _ in range(nbuf)]
    h_dev = [torch.empty_like(h) for _ in range(nbuf)]
    ins = [[(h_dev[b], h_host[b])] for b in range(nbuf)]  # (device, pinned host) per input
    if F:
        res_dev = [torch.empty(T, D, dtype=torch.bfloat16, device="cuda") for _ in range(nbuf)]
        res_host = [torch.empty(T, D, dtype=torch.bfloat16).pin_memory() for _ in range(nbuf)]
        if wl.backward:
            # a training step: forward (saving what the backward reads), then
            # the backward; its inputs are h and the upstream gradient dout,
            # the result read back is dh, the weight gradients stay on the
            # device for an optimizer there
            dout_dev = [torch.empty_like(dout) for _ in range(nbuf)]
            for b in range(nbuf):
                ins[b].append((dout_dev[b], inp.dout.pin_memory()))

            def compute(b):
                B.base_layer_fwd(h_dev[b], w, W1, W2, act, B.BASE_ROUTE_BALANCED, out, sv, ws,
                                 stream=stream)
                B.base_layer_bwd(h_dev[b], w, W1, W2, act, sv, dout_dev[b], res_dev[b], dw, dW1,
                                 dW2, ws, stream=stream)
        elif wl.S:
            sv2 = buffers.layer_saved(T, E, D, F, for_backward=False)

            def compute(b):
                B.base_layer_fwd_blend(h_dev[b], w, W1, W2, gam, bet, act, B.BASE_ROUTE_BALANCED,
                                       res_dev[b], sv2, ws, stream=stream)
        else:
            sv2 = buffers.layer_saved(T, E, D, F, for_backward=False)

            def compute(b):
                B.base_layer_fwd(h_dev[b], w, W1, W2, act, B.BASE_ROUTE_BALANCED, res_dev[b], sv2,
                                 ws, stream=stream)
        d2h = T * D * 2
    else:
        res_dev = [torch.empty(T, dtype=torch.int32, device="cuda") for _ in range(nbuf)]
        res_host = [torch.empty(T, dtype=torch.int32).pin_memory() for _ in range(nbuf)]

        def compute(b):
            B.base_scores(h_dev[b], w, sv["s"], sv["q"], stream=stream)
            if q_bump is not None:
                comps[1][1]()
            B.base_assign_balanced(sv["q"], res_dev[b], sv["price"], sv["stats"], ws, stream=stream)
            B.base_permute(h_dev[b], res_dev[b], E, sv["perm"], sv["inv"], sv["offsets"],
                           sv["x_perm"], sv["s"], sv["gate"], ws, stream=stream)
        d2h = T * 4

    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(nbuf)]
    ev_done = [torch.cuda.Event() for _ in range(nbuf)]
    ev_out = [torch.cuda.Event() for _ in range(nbuf)]

    def pipelined(K):
        for i in range(K):
            b = i % nbuf
            with torch.cuda.stream(s_in):
                if i >= nbuf:  # step i-2's compute has read h_dev[b]
                    s_in.wait_event(ev_done[b])
                for dst, src in ins[b]:
                    dst.copy_(src, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if i >= nbuf:  # step i-2's output copy has read res_dev[b]
                stream.wait_event(ev_out[b])
            flush.zero_()
            compute(b)
            ev_done[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[b])
                res_host[b].copy_(res_dev[b], non_blocking=True)
                ev_out[b].record(s_out)

    def serial_step():
        flush.zero_()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for dst, src in ins[0]:
            dst.copy_(src, non_blocking=True)
        compute(0)
        res_host[0].copy_(res_dev[0], non_blocking=True)
        b_.record(stream)
        b_.synchronize()
        return a.elapsed_time(b_)

    for _ in range(3):
        serial_step()
    e2e_serial = statistics.mean([serial_step() for _ in range(steps)])
    pipelined(3)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    pipelined(steps)
    s_out.wait_stream(stream)
    t1.record(s_out)
    t1.synchronize()
    e2e = t0.elapsed_time(t1) / steps
    e2e = replicas.max_over_ranks(e2e, device=torch.device("cuda"))
    e2e_serial = replicas.max_over_ranks(e2e_serial, device=torch.device("cuda"))
    if rank != 0:
        return None

    pk = peaks()
    comp = {n: statistics.mean(per[n]) for n in names}
    dom = max(comp, key=comp.get)
    bids = st["bids"]
    alg = dict(  # algorithmic work per launch (bytes or flops)
        scores=("hbm", 2 * T * D + 2 * E * D + 8 * T * E),
        scores_greedy=("hbm", 2 * T * D + 2 * E * D + 8 * T * E + 4 * T + 4 * E),
        auction=("hbm", 4 * E * bids + 4 * T + 8 * E),
        permute=("hbm", 4 * T * D + 12 * T + 8 * T),
        ffn=("tensor", 4 * T * D * F),
        stack=("tensor", 4 * T * D * F * max(1, wl.S)),
        combine=("hbm", 4 * T * D + 4 * T),
        greedy=("hbm", 4 * T * E + 4 * T),
        backward=("tensor", 8 * T * D * F))

    def roof(n):
        bound, work = alg[n]
        traffic = None if args.tokens else NCU_TRAFFIC.get((n, wl.name))
        sec = comp[n] / 1e3
        if bound == "tensor":
            a_ = work / sec / 1e12
            return dict(bound="tensor", achieved=a_, peak=pk["bf16"], unit="TFLOP/s",
                        frac=a_ / pk["bf16"], traffic=traffic, kernel=n, ms=comp[n],
                        peak_source=pk["source"] + " burst bf16")
        a_ = work / sec / 1e9
        return dict(bound="hbm", achieved=a_, peak=pk["hbm"], unit="GB/s",
                    frac=a_ / pk["hbm"], traffic=traffic, kernel=n, ms=comp[n],
                    peak_source=pk["source"] + " hbm copy")

    lat = latency_roofline(u_list[:st["rounds"]], T, E, comp["auction"], args._floors, pk["hbm"])
    return dict(
        value=replicas.job_tokens_per_s(T, world, ms), ms_per_step=ms, steps=steps,
        warmup=warmup, config=_config(wl, args),
        roofline=roof(dom),
        per_kernel={n: roof(n) for n in names},
        auction=dict(tokens_per_s=replicas.job_tokens_per_s(T, world, comp["auction"]),
                     rounds=st["rounds"],
                     phases=st["phases"], bids=bids, status=st["status"],
                     us_per_round=1e3 * comp["auction"] / max(1, st["rounds"]),
                     rounds_by_kind=rounds_by_kind, objective=st["objective"], fig9=fig9,
                     latency_roofline=lat),
        e2e=dict(value=replicas.job_tokens_per_s(T, world, e2e), unit=UNIT,
                 mode="pipelined: copy streams each way, two device buffers",
                 serial_value=replicas.job_tokens_per_s(T, world, e2e_serial),
                 serial_ms_per_step=e2e_serial,
                 h2d_bytes_per_step=sum(d.numel() * d.element_size() for d, _ in ins[0]),
                 d2h_bytes_per_step=d2h, ms_per_step=e2e),
        gpu_launches=kernels_per_step * steps,
        clocks=clk, device_error=err, wall_s=wall,
    )


def measure_floors():
    """Latency floors (ns) of the auction's steps on this GPU, from the
    library's probe: grid barrier, block barrier, L2 load, shared load."""
    import torch
    from balanced_token_expert_b200 import binding as B
    out = torch.zeros(4, dtype=torch.float64, device="cuda")
    ws = torch.empty(B.base_probe_workspace_size() + 256, dtype=torch.uint8, device="cuda")
    off = (-ws.data_ptr()) % 256
    B.base_measure_latency(out, ws[off:])
    torch.cuda.synchronize()
    g, c, l2, sm = out.tolist()
    return dict(grid_barrier_ns=g, block_barrier_ns=c, l2_load_ns=l2, smem_load_ns=sm)


def measure_ep_exchange(G, T, D, E, steps, hbm_gbs):
    """The expert-parallel exchange kernels with G workers' buffers on this
    GPU (the emulation of the peer exchange): CUDA-event time of one
    base_ep_dispatch (rows only) and one base_ep_combine over all workers,
    against the HBM roofline of the bytes they move here (every row read once
    and written once: 2 G T D 2 bytes; the buffers, 3 G T D 2 bytes, exceed
    L2).  Across GPUs the bound is NVLink instead: (G-1)/G of those rows
    cross it in each direction."""
    import torch
    from balanced_token_expert_b200 import binding as B
    g = torch.Generator(device="cuda")
    g.manual_seed(1234)
    hs = [torch.randn(T, D, device="cuda", generator=g).to(torch.bfloat16) for _ in range(G)]
    perms = [torch.randperm(T, device="cuda", generator=g).to(torch.int32) for _ in range(G)]
    recv = [torch.empty(T, D, dtype=torch.bfloat16, device="cuda") for _ in range(G)]
    outs = [torch.empty(T, D, dtype=torch.bfloat16, device="cuda") for _ in range(G)]
    ms = {"dispatch": [], "combine": []}
    for i in range(3 + steps):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record()
        B.base_ep_dispatch(hs, perms, None, recv, None, 0, E)
        ev[1].record()
        B.base_ep_combine(recv, perms, outs, 0, E)
        ev[2].record()
        torch.cuda.synchronize()
        if i >= 3:
            ms["dispatch"].append(ev[0].elapsed_time(ev[1]))
            ms["combine"].append(ev[1].elapsed_time(ev[2]))
    ok = all(torch.equal(a, b) for a, b in zip(outs, hs))  # the round trip is the identity
    nbytes = 2.0 * G * T * D * 2
    res = dict(workers=G, T=T, D=D, E=E, bytes_per_exchange=nbytes, round_trip_identity=ok,
               note="all workers' buffers on one GPU; across GPUs NVLink bounds it")
    for k, v in ms.items():
        m = statistics.mean(v)
        res[k] = dict(ms=m, achieved_gbs=nbytes / m / 1e6, frac=nbytes / m / 1e6 / hbm_gbs)
    del hs, perms, recv, outs
    torch.cuda.empty_cache()
    return res


def latency_roofline(u, T, E, auction_ms, fl, hbm_gbs):
    """The auction against its latency floor: every round costs at least its
    synchronisation chain -- a grid-wide round two grid barriers and two
    dependent L2 loads (bids in, resolves out), a one-CTA round two block
    barriers and one L2 load (the rejected token's score row), a one-bidder
    round one L2 load -- and a phase start no less than reading q from HBM.
    Which mode a round runs in follows the kernel's rule: one bidder -> one
    warp; up to 256 bidders (E <= 16) or 32 (else) -> one CTA; more -> grid."""
    narrow_max = 256 if E <= 16 else 32
    wide = 2 * fl["grid_barrier_ns"] + 2 * fl["l2_load_ns"]
    narrow = 2 * fl["block_barrier_ns"] + fl["l2_load_ns"]
    chain = fl["l2_load_ns"]
    q_ns = 4.0 * T * E / hbm_gbs  # bytes / (GB/s) = ns
    floor_ns = 0.0
    for x in u:
        if x == T:
            floor_ns += max(wide, q_ns)
        elif x == 1 and E <= 128:
            floor_ns += chain
        elif x <= narrow_max:
            floor_ns += narrow
        else:
            floor_ns += wide
    return dict(floor_ms=floor_ns / 1e6, frac=floor_ns / 1e6 / auction_ms, floors_ns=fl,
                model="rounds x floor of their kind: grid round 2 grid barriers + 2 L2 loads, "
                      "one-CTA round 2 block barriers + 1 L2 load, one-bidder round 1 L2 load, "
                      "phase start at least q read from HBM")


def _rounds_by_kind(u, t, rounds, T):
    """Per-round durations of a traced auction run, grouped by how many tokens
    bid: the whole-grid rounds (every token bids: the phase starts), and the
    rest by bidder count.  The last round has no successor and is left out."""
    kinds = [("phase start", lambda x: x == T), ("1 bidder", lambda x: x == 1),
             ("2-8 bidders", lambda x: 2 <= x <= 8), ("9-128 bidders", lambda x: 9 <= x <= 128),
             ("129+ bidders", lambda x: 128 < x < T)]
    groups = {name: [] for name, _ in kinds}
    n = min(rounds, len(u), len(t))
    for r in range(n - 1):
        for name, test in kinds:  # the first kind that matches
            if test(u[r]):
                groups[name].append((t[r + 1] - t[r]) / 1e3)
                break
    return {name: dict(rounds=len(ds), us_total=sum(ds), us_median=statistics.median(ds))
            for name, ds in groups.items() if ds}


def main():
    args = parse()
    from balanced_token_expert_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    if args.tokens:
        wl = wl.scaled(T=args.tokens)
    from balanced_token_expert_b200 import replicas
    rank, world, local_rank = replicas.rank_env()
    if args.impl == "reference":
        run_reference(args, wl, rank, world)
        return

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    from balanced_token_expert_b200 import _build
    from balanced_token_expert_b200 import binding as B
    if rank == 0 or world == 1:
        _build.build()
    if world > 1:
        dist.barrier()
    B.lib()

    args._floors = measure_floors()
    head = measure(args, wl, args.steps, args.warmup, rank, world, local_rank)
    torch.cuda.empty_cache()
    extra = {}
    if args.workload == "layer_fwd" and not args.tokens and not args.only:
        # the other workloads on the same run, a few steps each
        for name in EXTRA_WORKLOADS:
            r = measure(args, synth.WORKLOADS[name], args.extra_steps, 3, rank, world, local_rank)
            torch.cuda.empty_cache()
            if r is not None:
                extra[name] = r
    if rank == 0:
        res = dict(
            metric=METRIC, value=head["value"], unit=UNIT, n_gpus=world, steps=args.steps,
            warmup=args.warmup, ms_per_step=head["ms_per_step"], higher_is_better=True,
            scaling="weak", vs_baseline=None, dtype="bf16", data="synthetic",
            config=head["config"], roofline=dict(head["roofline"], **(
                {"latency": head["auction"]["latency_roofline"]}
                if head["roofline"]["kernel"] == "auction" else {})),
            per_kernel=head["per_kernel"],
            auction=head["auction"], e2e=head["e2e"],
            gpu_launches=head["gpu_launches"] + sum(r["gpu_launches"] for r in extra.values()),
            clocks=head["clocks"], device_error=head["device_error"], wall_s=head["wall_s"])
        if extra:
            res["workloads"] = extra
        if world == 1 and args.workload == "layer_fwd" and not args.tokens and not args.only:
            res["ep_exchange"] = measure_ep_exchange(8, wl.T, wl.D, wl.E, args.extra_steps,
                                                     peaks()["hbm"])
        if world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(wl)
        print(json.dumps(res))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
