"""Benchmark of the fused SwiGLU gate/up projection on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--no-extra]

Headline workload (one "step"): decode at the AstrAI-1B MLP shape
(K = 1536, N = 6912), one fused call at each M in {1, 2, 4, 8}, every call on
the next of 16 rotated weight copies (680 MB, > 5x the 126 MB L2), so every
call streams its weights cold from HBM -- the cold-weight protocol of
AstrAI swiglu_benchmark.md ("HBM re-measurement and kernel simplification").
Metric: algorithmic bytes (Wg + Wu + X + H) / device time, GB/s.

Also measured on single-GPU runs (key "also", not part of the step): the
prefill at the LLaMA-3 8B shape and its variants (training forward storing
G and U, GEGLU with a gate multiplier, fp8 output), the backward GEMMs (dX,
dW, all three in one launch) and a whole training step of the projection
(TFLOP/s), dSwiGLU on [8192, 14336] bf16 (GB/s), the fp32 3xTF32 forward and
backward at the LLaMA-2 13B and GPT-NeoX 20B shapes, the LLaMA-2 7B
decode shape, and batched decode at M in {16, 32, 64} on both decode shapes
(the tcgen05 weight stream; GB/s), each with its roofline fraction and the
SM clock seen.

Timing: W untimed warm-up steps, then exactly K steps bracketed by a barrier
and cuda synchronize, CUDA events on the launching stream, max over ranks.
The steps are replayed from CUDA graphs holding 8 full rotations of the
copies (32 steps, 128 calls) so host launch overhead does not starve the GPU
and consecutive calls overlap under programmatic dependent launch (a graph
boundary costs about one call's overlap, ~4 us, which a decoding step that
captures a whole model amortises over all of its layers; 16 calls per graph
cost ~0.25 us per call against 64).  Multi-GPU (torchrun): every
rank runs the same per-GPU workload on its own GPU (independent problems, no
data-path collective): weak scaling, value = all ranks' bytes / max time.

``--impl reference`` times the fp64 CPU oracle (the only reference
implementation of this op here) on a bounded sample of the same workload, on
the host cores, rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# Page figure for this exact metric and shape: the fused decode kernel's
# cold-weight bandwidth at (N, K) = (6912, 1536) on an L20 (sm_89) -- AstrAI
# swiglu_benchmark.md, "HBM re-measurement and kernel simplification".
# Another machine's number: context for vs_baseline, not the target.
PAGE_DECODE_GBS = 702.0

DECODE_SHAPE = (1536, 6912)
DECODE_MS = (1, 2, 4, 8)
DECODE_COPIES = 16
# Full rotations of the copies held by each CUDA graph the decode timings
# replay (the headline, per-M, read-floor, comparator and e2e graphs alike).
GRAPH_ROTATIONS = 8
# batched decode: the tcgen05 weight-streaming route
BATCHED_MS = (16, 32, 64)

# DRAM traffic of the decode kernel per launch from one ncu capture, keyed by
# the sha256 of the kernel source it was measured on; reported as null when
# the source has changed since.
DECODE_TRAFFIC = {"src_sha256": "8c42f1ecbaff02c004ce5aa789167c3c5f494abb341d46f9c023ec901850b626",
                  # one ncu capture of this kernel per M (AstrAI-1B shape,
                  # weights-stable launch, launch 3 of 3 on its own copy):
                  # dram__bytes_read.sum 42524416 at M = 8 and 42502912 at
                  # M = 1, dram__bytes_write.sum 0 (H stays in L2 within the
                  # launch); M = 2 and 4 lie between (X differs by < 0.1 %)
                  # and are taken as the mean of the two.
                  "bytes_per_launch_by_M": {"1": 42502912, "2": 42513664, "4": 42513664,
                                            "8": 42524416}}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def decode_bytes(M, K, N, elem=2):
    """Algorithmic bytes of one fused call: both weight matrices once, X in,
    H out."""
    return elem * (2 * N * K + M * K + M * N)


def up_route_for(M, K, N):
    from up_projection_b200 import _capi
    return _capi.swiglu_route_for(M, K, N, 0)


def src_sha(name):
    path = os.path.join(ROOT, "up_projection_b200", "csrc", name)
    return hashlib.sha256(open(path, "rb").read()).hexdigest()


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None
        self.path = os.path.join("/tmp", f"swiglu_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v == "Active"})
        loaded = [r[0] for r in rows if r[2] > 300.0] or [r[0] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------ distributed

def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    from up_projection_b200.parallel import max_over_ranks as mor
    return mor(x) if world > 1 else x


# -------------------------------------------------------------- our arm

def timed_events(fn, iters, stream):
    """Run fn() iters times between two CUDA events on `stream`; returns ms."""
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    s.record(stream)
    for _ in range(iters):
        fn()
    e.record(stream)
    torch.cuda.synchronize()
    return s.elapsed_time(e)


def decode_workload(K, N, Ms, copies, seed=0):
    """Rotated weight copies (distinct buffers, same values) and X per M."""
    from up_projection_b200 import synth
    X8, Wg, Wu = synth.swiglu_inputs(max(Ms), K, N, "bf16", seed=seed)
    dev = torch.device("cuda")
    Wg_all = torch.empty((copies, N, K), dtype=torch.bfloat16, device=dev)
    Wu_all = torch.empty_like(Wg_all)
    Wg_all[:] = Wg.to(dev)
    Wu_all[:] = Wu.to(dev)
    Xs = {M: X8[:M].contiguous() for M in Ms}
    return Xs, Wg_all, Wu_all


def run_decode(args, world, K, N, Ms, copies, stream, with_e2e):
    import up_projection_b200 as up
    Xs_host, Wg_all, Wu_all = decode_workload(K, N, Ms, copies)
    dev = torch.device("cuda")
    Xd = {M: Xs_host[M].to(dev) for M in Ms}
    Hd = {M: torch.empty((M, N), dtype=torch.bfloat16, device=dev) for M in Ms}
    per_step = len(Ms)
    groups = copies // per_step   # steps per full rotation of the copies
    g_steps = groups * GRAPH_ROTATIONS   # steps per graph
    g_calls = copies * GRAPH_ROTATIONS   # calls per graph of the single-kind timings

    def step_calls(g):
        # step g's calls, each on the next copy (no copy is used again within
        # the copies - 1 calls that follow it)
        for i, M in enumerate(Ms):
            c = (g * per_step + i) % copies
            up.swiglu_fwd(Xd[M], Wg_all[c], Wu_all[c], Hd[M], stream=stream, weights_stable=True)

    # eager warm-up (tensor maps, function attributes), then capture: graphs
    # of g_steps steps (consecutive calls overlap under programmatic
    # dependent launch across the whole graph), plus a graph of the first r
    # steps for a remainder, so that exactly K steps are timed.
    with torch.cuda.stream(stream):
        for g in range(groups):
            step_calls(g)
    torch.cuda.synchronize()
    assert up.swiglu_sync_status(stream) == 0

    def capture(nsteps):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            for g in range(nsteps):
                step_calls(g)
        return gr

    full = capture(g_steps)
    partial = {r: capture(r) for r in sorted({args.warmup % g_steps, args.steps % g_steps}) if r}
    torch.cuda.synchronize()

    def run_steps(k):
        for _ in range(k // g_steps):
            full.replay()
        if k % g_steps:
            partial[k % g_steps].replay()

    with torch.cuda.stream(stream):
        run_steps(args.warmup)
    torch.cuda.synchronize()
    barrier(world)
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    gpu_id = "GPU-" + str(props.uuid) if hasattr(props, "uuid") else str(torch.cuda.current_device())
    with ClockSampler(gpu_id) as clk:
        with torch.cuda.stream(stream):
            ms = timed_events(lambda: run_steps(args.steps), 1, stream)
    torch.cuda.synchronize()
    barrier(world)
    st = up.swiglu_sync_status(stream)
    if st != 0:
        raise RuntimeError(f"device status after decode: {up.status_string(st)}")
    ms_max = max_over_ranks(ms, world)
    step_bytes = sum(decode_bytes(M, K, N) for M in Ms)
    out = {"ms": ms_max, "step_bytes": step_bytes, "clocks": clk.summary(),
           "launches": args.steps * per_step}

    # per-M launch time (eager, each M alone on rotated copies) for the record
    per_m = {}
    with torch.cuda.stream(stream):
        for M in Ms:
            j = {"c": 0}

            def call():
                c = j["c"] % copies
                up.swiglu_fwd(Xd[M], Wg_all[c], Wu_all[c], Hd[M], stream=stream,
                              weights_stable=True)
                j["c"] += 1
            gr = torch.cuda.CUDAGraph()
            # a graph of GRAPH_ROTATIONS full rotations of this M alone
            with torch.cuda.graph(gr, stream=stream):
                for _ in range(g_calls):
                    call()
            reps = max(1, min(500 * copies, 4 * args.steps) // g_calls)
            for _ in range(2):
                gr.replay()
            t = timed_events(gr.replay, reps, stream) / (reps * g_calls)
            per_m[M] = {"us": t * 1e3, "GB/s": decode_bytes(M, K, N) / (t * 1e-3) / 1e9}
            del gr
    out["per_M"] = per_m

    # The pure-read floor on the same rotated copies (the AstrAI page's
    # "pure-read floor" probe): graphs of GRAPH_ROTATIONS rotations of reads.
    sink = torch.empty(int(up.lib().swiglu_read_floor_sink_words()), dtype=torch.int32,
                       device=dev)
    with torch.cuda.stream(stream):
        for c in range(copies):
            up.swiglu_read_floor(Wg_all[c], Wu_all[c], sink, stream=stream)
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            for j in range(g_calls):
                c = j % copies
                up.swiglu_read_floor(Wg_all[c], Wu_all[c], sink, stream=stream)
        reps = max(1, min(500 * copies, 4 * args.steps) // g_calls)
        for _ in range(2):
            gr.replay()
        t = timed_events(gr.replay, reps, stream) / (reps * g_calls)
        del gr
    out["floor"] = {"us": t * 1e3, "GB/s": 4.0 * N * K / (t * 1e-3) / 1e9}

    # Eager single-call latency: one call at a time, device time between two
    # events, the stream drained in between (no overlap with other calls).
    lat = {}
    with torch.cuda.stream(stream):
        for M in (min(Ms), max(Ms)):
            samples = []
            for i in range(220):
                c = i % copies
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                up.swiglu_fwd(Xd[M], Wg_all[c], Wu_all[c], Hd[M], stream=stream)
                b.record(stream)
                b.synchronize()
                if i >= 20:
                    samples.append(a.elapsed_time(b) * 1e3)
            q = np.percentile(samples, [50, 90, 99])
            lat[M] = {"p50_us": round(float(q[0]), 2), "p90_us": round(float(q[1]), 2),
                      "p99_us": round(float(q[2]), 2)}
    out["latency"] = lat

    # Comparators for context at the largest M, timed A-B-C-C-B-A, each a
    # graph of GRAPH_ROTATIONS rotations of the copies: A = this library's fused call,
    # B = torch F.linear twice + silu * mul (library GEMMs, G and U through
    # HBM), C = torch F.linear on the stacked [2N, K] weights + silu * mul of
    # the two halves.
    M = max(Ms)
    F = torch.nn.functional
    Wcat_all = torch.cat([Wg_all, Wu_all], dim=1)   # [copies, 2N, K]

    def arm_a(c):
        up.swiglu_fwd(Xd[M], Wg_all[c], Wu_all[c], Hd[M], stream=stream, weights_stable=True)

    def arm_b(c):
        return F.silu(F.linear(Xd[M], Wg_all[c])) * F.linear(Xd[M], Wu_all[c])

    def arm_c(c):
        gu = F.linear(Xd[M], Wcat_all[c])
        return F.silu(gu[:, :N]) * gu[:, N:]
    graphs = {}
    with torch.cuda.stream(stream):
        for name, fn in (("A", arm_a), ("B", arm_b), ("C", arm_c)):
            for c in range(copies):
                fn(c)
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                for j in range(g_calls):
                    fn(j % copies)
            graphs[name] = gr
        reps = max(1, min(200 * copies, 2 * args.steps) // g_calls)
        samples = {"A": [], "B": [], "C": []}
        for name in "ABCCBA":
            for _ in range(2):
                graphs[name].replay()
            samples[name].append(timed_events(graphs[name].replay, reps, stream) /
                                 (reps * g_calls))
    del graphs, Wcat_all
    cmp_us = {k: 1e3 * sum(v) / len(v) for k, v in samples.items()}
    out["comparators"] = {"M": M, "order": "A-B-C-C-B-A", "us": cmp_us,
                          "GB/s": {k: decode_bytes(M, K, N) / (v * 1e-6) / 1e9
                                   for k, v in cmp_us.items()}}

    out["H"] = {M: Hd[M].cpu() for M in Ms}

    if with_e2e:
        # Through the public API with host buffers, every step: one pinned
        # host->device copy of the step's four X (packed rows), the four
        # calls on row views of the packed device buffer, one device->host
        # copy of the four H (packed rows) -- all inside the timed region.
        rows = sum(Ms)
        offs, o = {}, 0
        for M in Ms:
            offs[M] = o
            o += M
        Xpack_h = torch.cat([Xs_host[M] for M in Ms], 0).pin_memory()
        Hpack_h = torch.empty((rows, N), dtype=torch.bfloat16).pin_memory()
        Xpack_d = torch.empty((rows, K), dtype=torch.bfloat16, device=dev)
        Hpack_d = torch.empty((rows, N), dtype=torch.bfloat16, device=dev)
        Xv = {M: Xpack_d[offs[M]:offs[M] + M] for M in Ms}
        Hv = {M: Hpack_d[offs[M]:offs[M] + M] for M in Ms}
        h2d = Xpack_h.numel() * 2
        d2h = Hpack_h.numel() * 2
        cnt = {"c": 0}

        def e2e_step():
            Xpack_d.copy_(Xpack_h, non_blocking=True)
            for M in Ms:
                c = cnt["c"] % copies
                up.swiglu_fwd(Xv[M], Wg_all[c], Wu_all[c], Hv[M], stream=stream,
                              weights_stable=True)
                cnt["c"] += 1
            Hpack_h.copy_(Hpack_d, non_blocking=True)
        e_steps = min(args.steps, 2000)
        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                e2e_step()
            torch.cuda.synchronize()
            barrier(world)
            e_ms = timed_events(e2e_step, e_steps, stream)
        barrier(world)
        if not torch.equal(Hpack_h[offs[max(Ms)]:], out["H"][max(Ms)]):
            raise RuntimeError("e2e: H read back differs from the device-timed run")
        e_ms = max_over_ranks(e_ms, world)
        # The same steps replayed from a CUDA graph of g_steps steps, with the
        # copies pipelined on a second stream (two device buffer sets): step
        # g's input copy and step g-1's read-back overlap step g-1's / g's
        # calls.  Still, every step: one host->device copy of its X, its four
        # calls, one device->host copy of its H.
        cs = torch.cuda.Stream()
        Xd2 = [Xpack_d, torch.empty_like(Xpack_d)]
        Hd2 = [Hpack_d, torch.empty_like(Hpack_d)]
        Hh2 = [Hpack_h, torch.empty_like(Hpack_h).pin_memory()]
        Xv2 = [{M: b[offs[M]:offs[M] + M] for M in Ms} for b in Xd2]
        Hv2 = [{M: b[offs[M]:offs[M] + M] for M in Ms} for b in Hd2]

        def e2e_rotation():
            # software pipeline: the copy stream runs step g+1's input copy
            # and step g-1's read-back while step g's calls run
            ev_in = [torch.cuda.Event() for _ in range(g_steps)]
            ev_c = [torch.cuda.Event() for _ in range(g_steps)]
            ev_out = [torch.cuda.Event() for _ in range(g_steps)]
            cs.wait_stream(stream)

            def copy_in(g):
                with torch.cuda.stream(cs):
                    if g >= 2:
                        cs.wait_event(ev_c[g - 2])   # buffer g%2's last calls read X
                    Xd2[g % 2].copy_(Xpack_h, non_blocking=True)
                    ev_in[g].record(cs)
            copy_in(0)
            for g in range(g_steps):
                b = g % 2
                if g + 1 < g_steps:
                    copy_in(g + 1)
                stream.wait_event(ev_in[g])
                if g >= 2:
                    stream.wait_event(ev_out[g - 2])  # buffer b's H has been read back
                for i, M in enumerate(Ms):
                    c = (g * per_step + i) % copies
                    up.swiglu_fwd(Xv2[b][M], Wg_all[c], Wu_all[c], Hv2[b][M], stream=stream,
                                  weights_stable=True)
                ev_c[g].record(stream)
                with torch.cuda.stream(cs):
                    cs.wait_event(ev_c[g])
                    Hh2[b].copy_(Hd2[b], non_blocking=True)
                    ev_out[g].record(cs)
            stream.wait_stream(cs)
        with torch.cuda.stream(stream):
            e2e_rotation()
            torch.cuda.synchronize()
            eg = torch.cuda.CUDAGraph()
            with torch.cuda.graph(eg, stream=stream):
                e2e_rotation()
            g_reps = max(1, e_steps // g_steps)
            for _ in range(2):
                eg.replay()
            torch.cuda.synchronize()
            barrier(world)
            eg_ms = timed_events(eg.replay, g_reps, stream)
        barrier(world)
        torch.cuda.synchronize()
        last = (g_steps - 1) % 2
        if not torch.equal(Hh2[last][offs[max(Ms)]:], out["H"][max(Ms)]):
            raise RuntimeError("e2e: pipelined read-back differs from the device-timed run")
        eg_ms = max_over_ranks(eg_ms, world)
        del eg
        out["e2e"] = {"ms": eg_ms, "steps": g_reps * g_steps, "h2d": h2d, "d2h": d2h,
                      "eager_ms": e_ms, "eager_steps": e_steps}
    del full, partial
    del Wg_all, Wu_all
    torch.cuda.empty_cache()
    return out


def run_extras(stream, pk):
    """Single-GPU extra measurements (rank 0 only)."""
    import ctypes

    import up_projection_b200 as up
    from up_projection_b200 import _capi as up_capi
    dev = torch.device("cuda")
    gen = torch.Generator(device=dev)
    gen.manual_seed(1)
    res = []
    state = {"clocks": None}
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    gpu_id = "GPU-" + str(props.uuid) if hasattr(props, "uuid") else str(torch.cuda.current_device())

    def time_op(fn, iters=10):
        # Every input below is larger than the 126 MB L2 (prefill 537 MB,
        # dSwiGLU 1.17 GB, fp32 >= 721 MB), so back-to-back calls read cold
        # operands; the calls are timed together to amortise launch latency.
        # One idle second first, so that one workload's power draw does not
        # lower the clocks of the next; the SM clock seen while timing is
        # kept with the result.
        torch.cuda.synchronize()
        time.sleep(1.0)
        with torch.cuda.stream(stream):
            for _ in range(3):
                fn()
            with ClockSampler(gpu_id) as clk:
                ms = timed_events(fn, iters, stream) / iters
        state["clocks"] = clk.summary()
        return ms

    def add(entry):
        entry["clocks"] = state["clocks"]
        res.append(entry)

    # prefill LLaMA-3 8B
    M, K, N = 8192, 4096, 14336
    X = torch.randn((M, K), generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)
    Wg = (torch.randn((N, K), generator=gen, device=dev) / K ** 0.5).to(torch.bfloat16)
    Wu = (torch.randn((N, K), generator=gen, device=dev) / K ** 0.5).to(torch.bfloat16)
    H = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ms = time_op(lambda: up.swiglu_fwd(X, Wg, Wu, H, stream=stream))
    fl = 4.0 * M * N * K
    tf = fl / (ms * 1e-3) / 1e12
    add({"workload": "prefill LLaMA-3 8B M=8192 K=4096 N=14336 bf16",
                "metric": "TFLOP/s", "value": round(tf, 1), "ms": round(ms, 4),
                "roofline": {"bound": "tensor", "achieved": round(tf, 1),
                             "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                             "frac": round(tf / pk["bf16_tflops"], 4)}})
    # context: the unfused library chain (two cuBLAS GEMMs, G and U through
    # HBM, then silu * mul)
    F = torch.nn.functional
    with torch.no_grad():
        ms_t = time_op(lambda: F.silu(F.linear(X, Wg)) * F.linear(X, Wu), iters=5)
    res[-1]["torch_unfused_ms"] = round(ms_t, 4)
    res[-1]["speedup_vs_torch_unfused"] = round(ms_t / ms, 3)
    # training forward: the same call also storing G and U for the backward
    Gs = torch.empty_like(H)
    Us = torch.empty_like(H)
    ms = time_op(lambda: up.lib().swiglu_fwd_epilogue(
        X.data_ptr(), Wg.data_ptr(), Wu.data_ptr(), H.data_ptr(), M, K, N, 0,
        ctypes.byref(up_capi.Epilogue(0, 1.0, Gs.data_ptr(), Us.data_ptr())), 0,
        stream.cuda_stream))
    tf = fl / (ms * 1e-3) / 1e12
    add({"workload": "prefill training forward (also stores G, U) LLaMA-3 8B bf16",
                "metric": "TFLOP/s", "value": round(tf, 1), "ms": round(ms, 4),
                "roofline": {"bound": "tensor", "achieved": round(tf, 1),
                             "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                             "frac": round(tf / pk["bf16_tflops"], 4)}})
    # GEGLU (GELU-tanh) epilogue with a gate multiplier
    ms = time_op(lambda: up.swiglu_fwd(X, Wg, Wu, H, stream=stream,
                                       activation=up.SWIGLU_ACT_GELU_TANH, gate_multiplier=1.5))
    tf = fl / (ms * 1e-3) / 1e12
    add({"workload": "prefill GEGLU (GELU-tanh, gate multiplier 1.5) LLaMA-3 8B bf16",
                "metric": "TFLOP/s", "value": round(tf, 1), "ms": round(ms, 4),
                "roofline": {"bound": "tensor", "achieved": round(tf, 1),
                             "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                             "frac": round(tf / pk["bf16_tflops"], 4)}})
    # fp8 output: e4m3 H with UE8M0 scales per (1,32) block
    Hq = torch.empty((M, N), dtype=torch.uint8, device=dev)
    Hs = torch.empty((M, N // 32), dtype=torch.uint8, device=dev)
    ms = time_op(lambda: up.lib().swiglu_fwd_fp8(
        X.data_ptr(), Wg.data_ptr(), Wu.data_ptr(), Hq.data_ptr(), Hs.data_ptr(), M, K, N,
        None, stream.cuda_stream))
    tf = fl / (ms * 1e-3) / 1e12
    add({"workload": "prefill, fp8 e4m3 H + UE8M0 (1,32) scales, LLaMA-3 8B bf16 in",
         "metric": "TFLOP/s", "value": round(tf, 1), "ms": round(ms, 4),
         "roofline": {"bound": "tensor", "achieved": round(tf, 1),
                      "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                      "frac": round(tf / pk["bf16_tflops"], 4)}})
    del Hq, Hs
    # backward GEMMs at the same size: dX = dG Wg + dU Wu and dWg, dWu
    dGb = torch.randn((M, N), generator=gen, device=dev).to(torch.bfloat16)
    dUb = torch.randn((M, N), generator=gen, device=dev).to(torch.bfloat16)
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    ms = time_op(lambda: up.swiglu_bwd_dx(dGb, dUb, Wg, Wu, dX, stream=stream))
    tf = fl / (ms * 1e-3) / 1e12
    add({"workload": "backward dX = dG Wg + dU Wu, LLaMA-3 8B M=8192 bf16",
                "metric": "TFLOP/s", "value": round(tf, 1), "ms": round(ms, 4),
                "roofline": {"bound": "tensor", "achieved": round(tf, 1),
                             "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                             "frac": round(tf / pk["bf16_tflops"], 4)}})
    dWg = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
    dWu = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
    ms = time_op(lambda: up.swiglu_bwd_dw(dGb, dUb, X, dWg, dWu, stream=stream))
    tf = fl / (ms * 1e-3) / 1e12
    add({"workload": "backward dWg = dG^T X, dWu = dU^T X, LLaMA-3 8B M=8192 bf16",
                "metric": "TFLOP/s", "value": round(tf, 1), "ms": round(ms, 4),
                "roofline": {"bound": "tensor", "achieved": round(tf, 1),
                             "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                             "frac": round(tf / pk["bf16_tflops"], 4)}})
    # all three backward GEMMs in one scheduled launch
    ms = time_op(lambda: up.lib().swiglu_bwd_gemms(
        dGb.data_ptr(), dUb.data_ptr(), Wg.data_ptr(), Wu.data_ptr(), X.data_ptr(), dX.data_ptr(),
        dWg.data_ptr(), dWu.data_ptr(), M, K, N, 0, stream.cuda_stream))
    tf = 2 * fl / (ms * 1e-3) / 1e12
    add({"workload": "backward dX, dWg, dWu in one launch (swiglu_bwd_gemms), LLaMA-3 8B M=8192 bf16",
         "metric": "TFLOP/s", "value": round(tf, 1), "ms": round(ms, 4),
         "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": pk["bf16_tflops"],
                      "unit": "TFLOP/s", "frac": round(tf / pk["bf16_tflops"], 4)}})
    # one whole training step of the projection: forward storing G and U,
    # dSwiGLU, dX, dWg/dWu (dH stands in for the gradient from above)
    dHb = torch.randn((M, N), generator=gen, device=dev).to(torch.bfloat16)
    epi_gu = up_capi.Epilogue(0, 1.0, Gs.data_ptr(), Us.data_ptr())

    def train_step():
        up.lib().swiglu_fwd_epilogue(X.data_ptr(), Wg.data_ptr(), Wu.data_ptr(), H.data_ptr(),
                                     M, K, N, 0, ctypes.byref(epi_gu), 0, stream.cuda_stream)
        up.dswiglu_bwd(dHb, Gs, Us, dGb, dUb, stream=stream)
        up.lib().swiglu_bwd_gemms(dGb.data_ptr(), dUb.data_ptr(), Wg.data_ptr(), Wu.data_ptr(),
                                  X.data_ptr(), dX.data_ptr(), dWg.data_ptr(), dWu.data_ptr(),
                                  M, K, N, 0, stream.cuda_stream)
    ms = time_op(train_step, iters=5)
    tf = 3 * fl / (ms * 1e-3) / 1e12
    add({"workload": "training step (forward storing G, U; dSwiGLU; dX; dWg, dWu), "
                     "LLaMA-3 8B M=8192 bf16",
         "metric": "TFLOP/s", "value": round(tf, 1), "ms": round(ms, 4),
         "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": pk["bf16_tflops"],
                      "unit": "TFLOP/s", "frac": round(tf / pk["bf16_tflops"], 4),
                      "note": "3 x 4MNK GEMM FLOPs; the dSwiGLU pass (1.17 GB) is counted as time only"}})
    del X, Wg, Wu, H, Gs, Us, dGb, dUb, dX, dWg, dWu, dHb
    # dSwiGLU on [8192, 14336] bf16
    n = 8192 * 14336
    dH = torch.randn(n, generator=gen, device=dev).to(torch.bfloat16)
    G = torch.randn(n, generator=gen, device=dev).to(torch.bfloat16)
    U = torch.randn(n, generator=gen, device=dev).to(torch.bfloat16)
    dG = torch.empty_like(G)
    dU = torch.empty_like(U)
    ms = time_op(lambda: up.dswiglu_bwd(dH, G, U, dG, dU, stream=stream))
    gbs = 10.0 * n / (ms * 1e-3) / 1e9
    add({"workload": "dSwiGLU n=8192*14336 bf16", "metric": "GB/s", "value": round(gbs, 1),
                "ms": round(ms, 4),
                "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"],
                             "unit": "GB/s", "frac": round(gbs / pk["hbm_gbs"], 4)}})
    del dH, G, U, dG, dU
    # fp32 3xTF32 at the 13B and NeoX-20B shapes
    for K, N, name in ((5120, 13824, "LLaMA-2 13B"), (6144, 24576, "GPT-NeoX 20B")):
        M = 2048
        X = torch.randn((M, K), generator=gen, device=dev)
        Wg = torch.randn((N, K), generator=gen, device=dev) / K ** 0.5
        Wu = torch.randn((N, K), generator=gen, device=dev) / K ** 0.5
        H = torch.empty((M, N), dtype=torch.float32, device=dev)
        try:
            ms = time_op(lambda: up.swiglu_fwd(X, Wg, Wu, H, stream=stream), iters=5)
        except Exception as exc:  # noqa: BLE001 - report, do not hide
            add({"workload": f"fp32 3xTF32 {name}", "error": str(exc)})
            continue
        fl = 4.0 * M * N * K
        tf = fl / (ms * 1e-3) / 1e12
        tf32_peak = pk["bf16_tflops"] * 0.5   # nominal dense TF32/BF16 ratio
        add({"workload": f"fp32 3xTF32 {name} M=2048 K={K} N={N}",
                    "metric": "TFLOP/s (fp32-equivalent)", "value": round(tf, 1),
                    "ms": round(ms, 4),
                    "roofline": {"bound": "tensor", "achieved": round(3 * tf, 1),
                                 "peak": round(tf32_peak, 1), "unit": "TFLOP/s (tf32 MMA)",
                                 "frac": round(3 * tf / tf32_peak, 4),
                                 "frac_vs_bf16_peak_literal": round(tf / pk["bf16_tflops"], 4)}})
        if K == 5120:
            # the fp32 backward GEMMs at the same shape (3xTF32)
            dGf = torch.randn((M, N), generator=gen, device=dev)
            dUf = torch.randn((M, N), generator=gen, device=dev)
            dXf = torch.empty((M, K), device=dev)
            dWgf = torch.empty((N, K), device=dev)
            dWuf = torch.empty((N, K), device=dev)
            for what, fn in (("dX = dG Wg + dU Wu",
                              lambda: up.swiglu_bwd_dx(dGf, dUf, Wg, Wu, dXf, stream=stream)),
                             ("dWg = dG^T X, dWu = dU^T X",
                              lambda: up.swiglu_bwd_dw(dGf, dUf, X, dWgf, dWuf, stream=stream))):
                ms = time_op(fn, iters=5)
                tf = fl / (ms * 1e-3) / 1e12
                add({"workload": f"fp32 3xTF32 backward {what}, {name} M=2048",
                     "metric": "TFLOP/s (fp32-equivalent)", "value": round(tf, 1),
                     "ms": round(ms, 4),
                     "roofline": {"bound": "tensor", "achieved": round(3 * tf, 1),
                                  "peak": round(tf32_peak, 1), "unit": "TFLOP/s (tf32 MMA)",
                                  "frac": round(3 * tf / tf32_peak, 4)}})
            ms = time_op(lambda: up.lib().swiglu_bwd_gemms(
                dGf.data_ptr(), dUf.data_ptr(), Wg.data_ptr(), Wu.data_ptr(), X.data_ptr(),
                dXf.data_ptr(), dWgf.data_ptr(), dWuf.data_ptr(), M, K, N, 1, stream.cuda_stream),
                iters=5)
            tf = 2 * fl / (ms * 1e-3) / 1e12
            add({"workload": f"fp32 3xTF32 backward dX, dWg, dWu in one launch, {name} M=2048",
                 "metric": "TFLOP/s (fp32-equivalent)", "value": round(tf, 1), "ms": round(ms, 4),
                 "roofline": {"bound": "tensor", "achieved": round(3 * tf, 1),
                              "peak": round(tf32_peak, 1), "unit": "TFLOP/s (tf32 MMA)",
                              "frac": round(3 * tf / tf32_peak, 4)}})
            del dGf, dUf, dXf, dWgf, dWuf
        del X, Wg, Wu, H
    torch.cuda.empty_cache()
    return res


def cpu_baseline_decode(K, N, Ms, budget_s=12.0, gpu_H=None):
    """Time the fp64 oracle (as it stands) on the decode step, bounded; and,
    given the GPU's H of the same step, report its agreement with the
    oracle's (max / mean absolute error, cosine, share within the bf16
    tolerance 1e-2 |ref| + 1e-3)."""
    import oracle
    from up_projection_b200 import synth
    X8, Wg, Wu = synth.swiglu_inputs(max(Ms), K, N, "bf16", seed=0)
    Xd = oracle.decode_bf16(X8)
    Wgd = oracle.decode_bf16(Wg)
    Wud = oracle.decode_bf16(Wu)
    o = oracle.default()
    t0 = time.perf_counter()
    steps = 0
    ref = {}
    while True:
        for M in Ms:
            ref[M] = o.swiglu_fwd_f64(Xd[:M], Wgd, Wud)["H"]
        steps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    step_bytes = sum(decode_bytes(M, K, N) for M in Ms)
    threads = int(os.environ.get("OMP_NUM_THREADS", len(os.sched_getaffinity(0))))
    # the same oracle on one thread, on a smaller bounded sample (M = 8 only)
    o.set_num_threads(1)
    t1 = time.perf_counter()
    n1 = 0
    while time.perf_counter() - t1 < budget_s / 3:
        o.swiglu_fwd_f64(Xd[:max(Ms)], Wgd, Wud)
        n1 += 1
    dt1 = time.perf_counter() - t1
    o.set_num_threads(0)
    single = {"value": round(decode_bytes(max(Ms), K, N) * n1 / dt1 / 1e9, 4), "unit": "GB/s",
              "cores": 1, "sample": f"{n1} decode calls at M={max(Ms)}, {dt1:.1f} s"}
    # informative, not a gate: the shift of the "eager" trajectory that rounds
    # G and U to bf16 before silu * mul, against the fused reference (which
    # keeps them unrounded), on the M = 8 call
    r8 = o.swiglu_fwd_f64(Xd[:max(Ms)], Wgd, Wud)
    g8 = torch.from_numpy(r8["G"]).to(torch.bfloat16).to(torch.float64).numpy()
    u8 = torch.from_numpy(r8["U"]).to(torch.bfloat16).to(torch.float64).numpy()
    eager = g8 / (1.0 + np.exp(-g8)) * u8
    shift = np.abs(eager - r8["H"])
    eager_shift = {"max_abs": float(shift.max()),
                   "rel_norm": float(np.linalg.norm(shift) / np.linalg.norm(r8["H"]))}
    parity = None
    if gpu_H is not None:
        g = np.concatenate([gpu_H[M].to(torch.float64).numpy().ravel() for M in Ms])
        r = np.concatenate([ref[M].ravel() for M in Ms])
        err = np.abs(g - r)
        parity = {"outputs": int(g.size), "max_abs_err": float(err.max()),
                  "mean_abs_err": float(err.mean()),
                  "cosine": float(g @ r / (np.linalg.norm(g) * np.linalg.norm(r))),
                  "within_bf16_tol": float(np.mean(err <= 1e-2 * np.abs(r) + 1e-3))}
    return {"value": round(step_bytes * steps / dt / 1e9, 4), "unit": "GB/s",
            "cores": min(threads, max(Ms)), "kind": "oracle", "parity_vs_gpu": parity,
            "single_thread": single, "eager_trajectory_shift": eager_shift,
            "sample": f"{steps} full decode steps (M=1,2,4,8 at K={K}, N={N}), fp64 C loops, "
                      f"OpenMP over output rows ({threads} threads available), {dt:.1f} s"}


def reference_arm(args, metric, config, K, N, budget_s=120.0):
    """The fp64 CPU oracle on the host cores, on a bounded sample of the decode
    step: the step's four calls restricted to the first N' output columns,
    N' chosen so that warm-up plus all timed steps take about budget_s."""
    import oracle
    from up_projection_b200 import synth
    X8, Wg, Wu = synth.swiglu_inputs(max(DECODE_MS), K, N, "bf16", seed=0)
    o = oracle.default()
    Xd, Wgd, Wud = o.decode_bf16(X8), o.decode_bf16(Wg), o.decode_bf16(Wu)
    t0 = time.perf_counter()
    for M in DECODE_MS:
        o.swiglu_fwd_f64(Xd[:M], Wgd, Wud)
    t_full = time.perf_counter() - t0
    frac = min(1.0, budget_s / (t_full * (args.steps + args.warmup)))
    n_s = max(8, int(N * frac) // 8 * 8)
    Wgs, Wus = Wgd[:n_s], Wud[:n_s]

    def step():
        for M in DECODE_MS:
            o.swiglu_fwd_f64(Xd[:M], Wgs, Wus)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    step_bytes = sum(decode_bytes(M, K, n_s) for M in DECODE_MS)
    value = step_bytes * args.steps / dt / 1e9
    threads = len(os.sched_getaffinity(0))
    sample = (f"each step: the four decode calls (M=1,2,4,8, K={K}) on the first {n_s} of "
              f"{N} output columns; fp64 C oracle, OpenMP over output rows")
    line = {"impl": "reference", "metric": metric, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt * 1e3 / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config,
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s",
                             "cores": min(threads, max(DECODE_MS)), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def summary_of(line):
    """Compact record of the line: value and roofline fraction per workload
    (decode GB/s, prefill and backward TFLOP/s, dSwiGLU GB/s, fp32 TFLOP/s),
    taken from the headline and the "also" entries."""
    out = {"decode_astrai_gbs": line["value"], "decode_astrai_frac": line["roofline"]["frac"],
           "decode_astrai_us_per_call": round(line["ms_per_step"] * 1e3 / len(DECODE_MS), 3),
           "e2e_gbs": line["e2e"]["value"]}
    keys = [("prefill LLaMA-3 8B", "prefill"),
            ("prefill training forward", "prefill_training_fwd"),
            ("prefill GEGLU", "prefill_geglu"),
            ("prefill, fp8", "prefill_fp8_out"),
            ("backward dX = ", "bwd_dx"),
            ("backward dWg", "bwd_dw"),
            ("backward dX, dWg, dWu in one launch", "bwd_gemms"),
            ("training step", "training_step"),
            ("dSwiGLU", "dswiglu"),
            ("fp32 3xTF32 LLaMA-2 13B", "fp32_13b"),
            ("fp32 3xTF32 GPT-NeoX 20B", "fp32_neox"),
            ("fp32 3xTF32 backward dX = ", "fp32_13b_bwd_dx"),
            ("fp32 3xTF32 backward dX, dWg, dWu in one launch", "fp32_13b_bwd_gemms"),
            ("decode LLaMA-2 7B", "decode_llama7b"),
            ("batched decode AstrAI", "batched_astrai"),
            ("batched decode LLaMA-2 7B", "batched_llama7b")]
    for entry in line.get("also", []):
        w = entry.get("workload", "")
        for prefix, key in keys:
            if w.startswith(prefix) and key + "_value" not in out:
                if "value" in entry:
                    out[key + "_value"] = entry["value"]
                    out[key + "_unit"] = entry.get("metric")
                    out[key + "_frac"] = entry.get("roofline", {}).get("frac")
                break
    if "cpu_baseline" in line:
        out["cpu_oracle_gbs"] = line["cpu_baseline"]["value"]
    return out


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extra", action="store_true", help="skip the 'also' measurements")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    K, N = DECODE_SHAPE
    metric = "SwiGLU gate/up: decode cold-weight GB/s, prefill TFLOP/s, % of roofline"
    config = {"workload": f"decode AstrAI-1B: M in {{1,2,4,8}}, K={K}, N={N}, bf16, "
                          f"{DECODE_COPIES} rotated weight copies",
              "global_batch": sum(DECODE_MS) * args.gpus, "seq_len": 1,
              "parallelism": f"independent replicas x{args.gpus} (no collective)",
              "l2": f"inputs larger than L2 ({DECODE_COPIES} rotated copies, "
                    f"{DECODE_COPIES * 4 * N * K / 1e6:.0f} MB)",
              "launch": "SWIGLU_FLAG_WEIGHTS_STABLE (programmatic dependent launch: weights "
                        "are model parameters no earlier work writes)",
              "graph": f"CUDA graphs of {GRAPH_ROTATIONS} rotations "
                       f"({GRAPH_ROTATIONS * DECODE_COPIES} calls), replayed"}

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return 0
        return reference_arm(args, metric, config, K, N)

    rank, world, local = dist_setup(args.gpus)
    import up_projection_b200 as up
    up.lib()  # fail loudly now if the CUDA library is missing
    pk = peaks()
    stream = torch.cuda.Stream()
    dec = run_decode(args, world, K, N, DECODE_MS, DECODE_COPIES, stream, with_e2e=True)
    total_bytes = dec["step_bytes"] * args.steps * world
    value = total_bytes / (dec["ms"] * 1e-3) / 1e9
    # dominant kernel: the decode kernel; average launch = timed region / launches
    per_launch_ms = dec["ms"] / dec["launches"]
    per_launch_bytes = dec["step_bytes"] / len(DECODE_MS)
    achieved = per_launch_bytes / (per_launch_ms * 1e-3) / 1e9
    sha = src_sha("decode_bf16.cu")
    traffic = None
    if DECODE_TRAFFIC["src_sha256"] == sha and DECODE_TRAFFIC["bytes_per_launch_by_M"]:
        vals = DECODE_TRAFFIC["bytes_per_launch_by_M"]
        traffic = sum(vals[str(M)] for M in DECODE_MS) / len(DECODE_MS)
    line = {
        "metric": metric, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dec["ms"] / args.steps, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": round(value / world / PAGE_DECODE_GBS, 3),
        "dtype": "bf16", "data": "synthetic", "config": config,
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"],
                     "unit": "GB/s", "frac": round(achieved / pk["hbm_gbs"], 4),
                     "traffic": traffic, "peak_source": pk["source"],
                     "kernel": "swiglu_decode_bf16_kernel",
                     "launch_time": "timed region / launches (graph replay)"},
        "per_M": {str(M): {k: round(v, 2) for k, v in d.items()} for M, d in dec["per_M"].items()},
        "e2e": {"value": round(dec["step_bytes"] * dec["e2e"]["steps"] * world
                               / (dec["e2e"]["ms"] * 1e-3) / 1e9, 1),
                "unit": "GB/s", "h2d_bytes_per_step": dec["e2e"]["h2d"],
                "d2h_bytes_per_step": dec["e2e"]["d2h"],
                "launch": "public API calls and the per-step pinned copies (on a second stream, "
                          "double-buffered, overlapping the calls) captured in CUDA graphs of "
                          f"{GRAPH_ROTATIONS} rotations, replayed",
                "eager_value": round(dec["step_bytes"] * dec["e2e"]["eager_steps"] * world
                                     / (dec["e2e"]["eager_ms"] * 1e-3) / 1e9, 1)},
        "gpu_launches": dec["launches"],
        "clocks": dec["clocks"],
        "read_floor": {"GB/s": round(dec["floor"]["GB/s"], 1), "us": round(dec["floor"]["us"], 2),
                       "what": "pure streaming read of the same Wg+Wu copies (swiglu_read_floor)",
                       "decode_frac_of_floor": round(achieved / dec["floor"]["GB/s"], 4)},
        "latency_single_call": {str(M): v for M, v in dec["latency"].items()},
        "comparators": {
            "what": {"A": "this library (fused decode call)",
                     "B": "torch F.silu(F.linear(X, Wg)) * F.linear(X, Wu)",
                     "C": "torch F.linear(X, [Wg; Wu]) then silu(g) * u"},
            "M": dec["comparators"]["M"], "order": dec["comparators"]["order"],
            "us": {k: round(v, 2) for k, v in dec["comparators"]["us"].items()},
            "GB/s": {k: round(v, 1) for k, v in dec["comparators"]["GB/s"].items()}},
    }
    # The extra single-GPU measurements take about a minute; under torchrun
    # the other ranks would idle in the closing barrier meanwhile, so they
    # run in single-GPU runs only.
    if rank == 0 and world == 1 and not args.no_extra:
        line["also"] = run_extras(stream, pk)
        # LLaMA-2 7B decode shape as a second cold-weight line
        s7 = max(40, min(2000, args.steps // 4))
        d7 = run_decode(argparse.Namespace(steps=s7, warmup=5), 1,
                        4096, 11008, DECODE_MS, 8, stream, with_e2e=False)
        v7 = d7["step_bytes"] * s7 / (d7["ms"] * 1e-3) / 1e9
        line["also"].append({"workload": "decode LLaMA-2 7B: M in {1,2,4,8}, K=4096, N=11008, "
                                         "8 rotated copies (1.44 GB)",
                             "metric": "GB/s", "value": round(v7, 1),
                             "per_M": {str(M): {k: round(v, 2) for k, v in d.items()}
                                       for M, d in d7["per_M"].items()},
                             "roofline": {"bound": "hbm", "achieved": round(v7, 1),
                                          "peak": pk["hbm_gbs"], "unit": "GB/s",
                                          "frac": round(v7 / pk["hbm_gbs"], 4)},
                             "read_floor_GB/s": round(d7["floor"]["GB/s"], 1),
                             "frac_of_floor": round(v7 / d7["floor"]["GB/s"], 4),
                             "latency_single_call": {str(M): v for M, v in d7["latency"].items()},
                             "comparators_us": {k: round(v, 2) for k, v in
                                                d7["comparators"]["us"].items()}})
        # Batched decode (M = 16, 32, 64): the tcgen05 weight stream, same
        # rotated cold copies, same comparators (at M = 64).
        for (Kb, Nb, cb, name) in ((1536, 6912, 16, "AstrAI 1B"), (4096, 11008, 8, "LLaMA-2 7B")):
            sb = max(48, min(1200, args.steps // 4)) // 3 * 3
            db = run_decode(argparse.Namespace(steps=sb, warmup=6), 1, Kb, Nb, BATCHED_MS, cb,
                            stream, with_e2e=False)
            vb = db["step_bytes"] * sb / (db["ms"] * 1e-3) / 1e9
            line["also"].append({
                "workload": f"batched decode {name}: M in {{16,32,64}}, K={Kb}, N={Nb}, "
                            f"{cb} rotated copies (tcgen05 weight stream)",
                "metric": "GB/s", "value": round(vb, 1),
                "route": up_route_for(BATCHED_MS[0], Kb, Nb),
                "per_M": {str(M): {k: round(v, 2) for k, v in d.items()}
                          for M, d in db["per_M"].items()},
                "roofline": {"bound": "hbm", "achieved": round(vb, 1), "peak": pk["hbm_gbs"],
                             "unit": "GB/s", "frac": round(vb / pk["hbm_gbs"], 4)},
                "read_floor_GB/s": round(db["floor"]["GB/s"], 1),
                "frac_of_floor": round(vb / db["floor"]["GB/s"], 4),
                "latency_single_call": {str(M): v for M, v in db["latency"].items()},
                "comparators_us": {k: round(v, 2) for k, v in db["comparators"]["us"].items()},
                "clocks": db["clocks"]})
    if rank == 0 and world == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline_decode(K, N, DECODE_MS, gpu_H=dec["H"])
    if rank == 0:
        # last key of the line: the headline figures of every workload in one
        # short object, so that a reader of the line's tail has all of them
        line["summary"] = summary_of(line)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
