#!/usr/bin/env python
"""Benchmark of the GLM-130B weight-only INT4 decode GEMM (and friends) on B200.

Default workload ("decode"): GLM-130B layer shapes QKV 12288->36864, attn-out
12288->12288, FFN-up 12288->65536 (GeGLU gate+value), FFN-down 32768->12288;
W ~ N(0, 0.02) fp16 quantized once to INT4 (one-shot, timed separately), X ~ N(0, 1)
fp16. One step = the decode GEMM for M in {1, 4, 16} on all four projections
(12 launches of glmq_gemm, weights resident in HBM). Metric: packed-weight GB/s
(decimal GB) over the step, plus the roofline of the decode kernel.

Other workloads: "sweep" (70 layers x 4 projections INT4-resident, one-shot
quantization layer by layer, then M=1 decode through all 280 projections in a
CUDA graph, tokens/s).

Timing: W >= 3 warm-up steps; K timed steps bracketed by a barrier and
torch.cuda.synchronize(); CUDA events on the launching stream; the max over
ranks. The step's working set (906 MB of packed weights) is larger than the
126 MB L2, so no separate flush is needed between steps.

`--impl reference` times the CPU oracle (the only reference this method has)
on a bounded sample of the same workload.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A16 GEMM weight GB/s (decode) and TFLOP/s (prefill) vs B200 roofline"
HIDDEN = 12288
DECODE_MS = (1, 4, 16)
EVENT_STEPS = 4          # steps of the separate event-carrying graph (per-launch shares)
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ----------------------------------------------------------------------------- helpers
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0, "source": "fallback"}


DECODE_SOURCES = ("decode.cuh", "glmq_ptx.cuh")


def source_digest(files=DECODE_SOURCES) -> str:
    """First 16 hex digits of the SHA-256 of the named kernel sources (the decode kernel's
    by default); a profile's DRAM counters are used only while this digest matches."""
    csrc = os.path.join(ROOT, "int8_quantized_glmq_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(files):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def profile_traffic_ratio(kernel_tag: str):
    """DRAM traffic / algorithmic bytes recorded by an ncu capture of this exact source, or None."""
    path = os.path.join(ROOT, "profiles", f"{kernel_tag}.md")
    if not os.path.exists(path):
        return None
    ratio, digest = None, None
    with open(path) as f:
        for line in f:
            if line.startswith("source_digest:"):
                digest = line.split(":", 1)[1].strip()
            if line.startswith("traffic_over_algorithmic:"):
                ratio = float(line.split(":", 1)[1].strip())
    if digest != source_digest():
        return None
    return ratio


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        import tempfile
        try:
            fd, self.path = tempfile.mkstemp(prefix="glmq_clocks_", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.15)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest x over all ranks (a device tensor under NCCL, a host tensor under gloo)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank_step: float, steps: int, elapsed_local_s: float, world: int):
    """(units/s over all ranks, slowest rank's seconds). Every rank runs its own replica of
    the workload (weak scaling: per-rank work is fixed), so the job processes
    world * units_per_rank_step * steps units in the slowest rank's time."""
    el = max_over_ranks(elapsed_local_s, world)
    return world * units_per_rank_step * steps / el, el


# ----------------------------------------------------------------------------- workloads
def make_weights(torch, seed_base: int):
    """fp16 GLM-130B projection weights ~ N(0, 0.02), generated on the device (seeded)."""
    from inputs import GLM_PROJECTIONS, PROJECTION_ORDER
    out = {}
    for i, name in enumerate(PROJECTION_ORDER):
        N, K = GLM_PROJECTIONS[name]
        g = torch.Generator(device="cuda").manual_seed(seed_base + i)
        w = torch.empty((N, K), dtype=torch.float16, device="cuda")
        w.normal_(0.0, 0.02, generator=g)
        out[name] = w
    return out


def time_launches(torch, fn, iters: int, warmup: int = 2):
    """Average device time of fn() per call, CUDA events on the current stream."""
    for _ in range(warmup):
        fn()
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(s)
    for _ in range(iters):
        fn()
    e1.record(s)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / 1e3 / iters


def settle(torch, seconds: float = 0.3):
    """Idle the GPU briefly between a tensor-heavy measurement and a memory-bound one:
    right after the M=2048 GEMMs the SM clock sits below its maximum under the power
    cap for a while, and the first memory-bound measurement after them read 10-25%
    slow."""
    torch.cuda.synchronize()
    time.sleep(seconds)


def time_launches_cold(torch, fn, iters: int, warmup: int = 8):
    """Average device time of fn() per call with L2 made cold before each call: a read
    of a 256 MB buffer between calls, outside the timed events. A read leaves clean
    lines behind, so the timed call does not pay the write-back of a flush buffer's
    dirty lines (a 256 MB write before each call added about 126 MB of DRAM writes to
    the timed call). Eight warm-up calls let the SM clock settle after the work that
    ran before."""
    flush = torch.ones((64 << 20,), dtype=torch.int32, device="cuda")
    for _ in range(warmup):
        flush.amax()
        fn()
    s = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
    torch.cuda.synchronize()
    for e0, e1 in ev:
        flush.amax()
        e0.record(s)
        fn()
        e1.record(s)
    torch.cuda.synchronize()
    del flush
    return sum(e0.elapsed_time(e1) for e0, e1 in ev) / 1e3 / iters


def run_decode(args, world, rank, local):
    import torch
    import int8_quantized_glmq_b200 as glmq
    from inputs import GLM_PROJECTIONS, PROJECTION_ORDER

    peaks = measured_peaks()
    torch.manual_seed(0)
    W16 = make_weights(torch, 1000)
    bits = 4
    # one-shot quantization (timed separately: not part of the decode step)
    quant = {}
    qstats = {}
    for name in PROJECTION_ORDER:
        N, K = GLM_PROJECTIONS[name]
        packed = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
        scale = torch.empty((N,), dtype=torch.float16, device="cuda")
        quant[name] = (packed, scale)
        t = time_launches(torch, lambda: glmq.quantize(W16[name], bits, out=(packed, scale)), 5)
        qbytes = N * K * 2 + N * K // 2 + N * 2
        qstats[name] = {"us": t * 1e6, "gbs": qbytes / t / 1e9}
    extras = {}
    if not args.no_extras:
        extras = run_extras(torch, glmq, W16, quant, peaks)
    del W16
    torch.cuda.empty_cache()

    # activations for the decode step
    xs = {}
    for M in DECODE_MS:
        for name in PROJECTION_ORDER:
            N, K = GLM_PROJECTIONS[name]
            g = torch.Generator(device="cuda").manual_seed(2000 + M)
            xs[(M, name)] = torch.randn((M, K), generator=g, device="cuda", dtype=torch.float32).half()
    ys = {(M, name): torch.empty((M, GLM_PROJECTIONS[name][0]), dtype=torch.float16, device="cuda")
          for M in DECODE_MS for name in PROJECTION_ORDER}
    launches = [(M, name) for M in DECODE_MS for name in PROJECTION_ORDER]
    weight_bytes = sum(quant[n][0].numel() for (_, n) in launches)
    alg_bytes = sum(quant[n][0].numel() + quant[n][1].numel() * 2 + xs[(M, n)].numel() * 2 + ys[(M, n)].numel() * 2
                    for (M, n) in launches)

    # Each call names the next call of the step (the last one the next step's first) in
    # glmq_gemm_decode_prefetch, which prefetches that call's first weight tiles into L2
    # while its own pipeline drains; the outputs are computed exactly as by the plain call.
    def call(j, hint=True, X=None, Y=None):
        M, n = launches[j]
        Mn, nn = launches[(j + 1) % len(launches)]
        X = xs[(M, n)] if X is None else X
        Y = ys[(M, n)] if Y is None else Y
        if not hint:
            return glmq.gemm(X, quant[n][0], quant[n][1], bits, out=Y)
        return glmq.gemm_decode_prefetch(X, quant[n][0], quant[n][1], bits, next_packed=quant[nn][0], next_M=Mn,
                                         out=Y)

    # The timed steps are captured into one CUDA graph: K steps of the 12 public calls,
    # nothing else between the kernels (so the programmatic-launch edges between them
    # stay intact). The per-launch split of the step comes from a separate graph of
    # EVENT_STEPS steps with timing-event record nodes (external events) around every
    # call; event nodes add gaps and cut the programmatic-launch edges, so those
    # durations are used only as shares of the step, scaled to the event-free step time.
    # The eager calls before capture size the library's scratch and set attributes.
    for j in range(len(launches)):
        call(j)
    torch.cuda.synchronize()
    cap_stream = torch.cuda.Stream()

    def capture(n_steps, with_events=False, hint=True, warmup=0):
        """One CUDA graph: `warmup` untimed steps, then n_steps steps between two timing
        events (so the graph's first-launch costs fall in the warm-up), optionally with
        event nodes around every call of the timed steps."""
        g = torch.cuda.CUDAGraph()
        evs = [[(torch.cuda.Event(enable_timing=True, external=True),
                 torch.cuda.Event(enable_timing=True, external=True)) for _ in launches]
               for _ in range(n_steps)] if with_events else None
        edge = (torch.cuda.Event(enable_timing=True, external=True),
                torch.cuda.Event(enable_timing=True, external=True))
        with torch.cuda.graph(g, stream=cap_stream):
            for _ in range(warmup):
                for j in range(len(launches)):
                    call(j, hint)
            edge[0].record()
            n0 = glmq.kernel_launches()
            for it in range(n_steps):
                for j in range(len(launches)):
                    if with_events:
                        evs[it][j][0].record()
                    call(j, hint)
                    if with_events:
                        evs[it][j][1].record()
            n_timed = glmq.kernel_launches() - n0
            edge[1].record()
        return g, evs, edge, n_timed

    def timed_replay(graph, edge):
        """Device seconds between the graph's two timing events (one replay, bracketed by a
        barrier and a device synchronize)."""
        barrier(world)
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        barrier(world)
        return edge[0].elapsed_time(edge[1]) / 1e3

    stream = torch.cuda.current_stream()
    timed_graph, _, edge, kernels_timed = capture(args.steps, warmup=args.warmup)

    clocks = ClockSampler(local)
    clocks.start()
    elapsed = timed_replay(timed_graph, edge)
    clk = clocks.stop()
    gpu_launches = kernels_timed
    value, elapsed_max = whole_job_rate(weight_bytes / 1e9, args.steps, elapsed, world)
    step_s = elapsed_max / args.steps
    del timed_graph

    # per-launch shares of the step (event-timed, separate graph)
    ev_graph, ev, ev_edge, _ = capture(EVENT_STEPS, with_events=True, warmup=args.warmup)
    ev_graph.replay()
    torch.cuda.synchronize()
    ev_s = [sum(ev[it][j][0].elapsed_time(ev[it][j][1]) for it in range(EVENT_STEPS)) / 1e3 / EVENT_STEPS
            for j in range(len(launches))]
    per_launch_s = [t / sum(ev_s) * step_s for t in ev_s]
    del ev_graph, ev, ev_edge

    # the same step with plain decode calls (no next-call hint), for comparison
    plain_graph, _, plain_edge, _ = capture(args.steps, hint=False, warmup=args.warmup)
    plain_value, _ = whole_job_rate(weight_bytes / 1e9, args.steps, timed_replay(plain_graph, plain_edge), world)
    del plain_graph, plain_edge
    extras["decode_step_without_prefetch_hint_gbs"] = round(plain_value, 2)

    # e2e through the public API: pinned host X in, pinned host Y out, every step
    hx = {k: v.cpu().pin_memory() for k, v in xs.items()}
    hy = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in ys.items()}
    h2d = sum(v.numel() * 2 for v in hx.values())
    d2h = sum(v.numel() * 2 for v in hy.values())

    # One e2e step -- for each of the 12 calls: copy X from pinned host memory to a
    # static device buffer (copy stream 1), the public glmq.gemm call, copy Y back into
    # pinned host memory (copy stream 2), ordered by events so one call's copies
    # overlap the others' compute -- is captured once into a CUDA graph, as a serving
    # loop would, and replayed every timed step. Every replay moves the bytes over PCIe.
    h2d_stream, d2h_stream = torch.cuda.Stream(), torch.cuda.Stream()
    xbuf = {k: torch.empty_like(v) for k, v in xs.items()}
    ybuf = {k: torch.empty_like(v) for k, v in ys.items()}
    ev_x = {k: torch.cuda.Event() for k in launches}
    ev_y = {k: torch.cuda.Event() for k in launches}
    e2e_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(e2e_graph, stream=cap_stream):
        h2d_stream.wait_stream(cap_stream)
        d2h_stream.wait_stream(cap_stream)
        for k in launches:
            M, n = k
            with torch.cuda.stream(h2d_stream):
                xbuf[k].copy_(hx[k], non_blocking=True)
            ev_x[k].record(h2d_stream)
            cap_stream.wait_event(ev_x[k])
            call(launches.index(k), X=xbuf[k], Y=ybuf[k])
            ev_y[k].record(cap_stream)
            d2h_stream.wait_event(ev_y[k])
            with torch.cuda.stream(d2h_stream):
                hy[k].copy_(ybuf[k], non_blocking=True)
        cap_stream.wait_stream(h2d_stream)
        cap_stream.wait_stream(d2h_stream)

    for _ in range(args.warmup):
        e2e_graph.replay()
    barrier(world)
    torch.cuda.synchronize()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(args.steps):
        e2e_graph.replay()
    a1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_value, _ = whole_job_rate(weight_bytes / 1e9, args.steps, a0.elapsed_time(a1) / 1e3, world)
    del e2e_graph

    # Dominant kernel: decode_kernel, with the finalize pass of the calls whose tiles are
    # split over K parts (one "launch" = one public call). Its time is the event-free
    # step time, so achieved is algorithmic bytes per step / step time: a lower bound on
    # the decode kernel's own rate (the step also holds the launches' gaps).
    achieved = alg_bytes / step_s / 1e9
    ratio = profile_traffic_ratio("decode_int4_glm_shapes")
    roofline = {"kernel": "decode_kernel (+ decode_finalize_kernel on split tiles), INT4, M in {1,4,16}",
                "bound": "hbm", "achieved": round(achieved, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "peak_source": peaks["source"],
                "traffic": (round(ratio * alg_bytes / len(launches)) if ratio else None),
                "algorithmic_bytes_per_launch": round(alg_bytes / len(launches)),
                "launch_time": "event-free step time / 12 calls"}
    per_launch = {f"{n}/M={M}": {"us": round(per_launch_s[j] * 1e6, 2),
                                 "gbs": round((quant[n][0].numel() + quant[n][1].numel() * 2 + xs[(M, n)].numel() * 2
                                               + ys[(M, n)].numel() * 2) / per_launch_s[j] / 1e9, 1)}
                  for j, (M, n) in enumerate(launches)}
    extras["decode_per_launch"] = per_launch
    extras["quantize_int4"] = {k: {"us": round(v["us"], 1), "gbs": round(v["gbs"], 1),
                                   "frac_hbm": round(v["gbs"] / peaks["hbm_gbs"], 4)} for k, v in qstats.items()}
    if not args.no_extras and world == 1:
        del xs, ys, hx, hy, xbuf, ybuf
        extras["sweep_70_layers_int4"] = sweep_summary(torch, glmq, peaks)
    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(elapsed_max / args.steps * 1e3, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp16", "weight_dtype": "int4", "data": "synthetic",
        "config": {"workload": "decode GEMV on GLM-130B layer shapes (QKV 12288->36864, attn-out 12288->12288, "
                               "FFN-up 12288->65536, FFN-down 32768->12288), M in {1,4,16}, INT4 weights",
                   "global_batch": list(DECODE_MS), "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
                   "weights": "N(0,0.02) fp16 on device, quantized once to INT4 (not in the step)",
                   "activations": "N(0,1) fp16",
                   "l2": "step working set 906 MB of packed weights > 126 MB L2 (no flush needed)"},
        "roofline": roofline,
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": gpu_launches,
        "clocks": clk,
        "extras": extras,
    }
    result["highlights"] = highlights(result, peaks)
    return result


def highlights(res, peaks):
    """The headline figures of the extras, repeated compactly at the end of the line."""
    ex = res.get("extras", {})
    h = {"decode_step_gbs": res["value"], "decode_frac_hbm": res["roofline"]["frac"]}
    pre = ex.get("prefill_int4_m2048")
    if pre:
        h["prefill_int4_m2048_tflops"] = {k: v["tflops"] for k, v in pre.items()}
        h["prefill_frac_burst_min"] = min(v["frac_burst"] for v in pre.values())
    m64 = ex.get("int4_m64")
    if m64:
        h["int4_m64_frac_binding_roof"] = {k: v["frac_binding_roof"] for k, v in m64.items()}
    i8 = ex.get("int8")
    if i8:
        h["int8_m64_frac_hbm"] = {k: v["M=64"].get("frac_hbm") for k, v in i8.items()}
    q = ex.get("quantize_int4")
    if q:
        h["quantize_int4_frac_hbm"] = {k: v["frac_hbm"] for k, v in q.items()}
    sw = ex.get("sweep_70_layers_int4")
    if sw and "tokens_per_s" in sw:
        h["sweep_70_layers"] = {"tokens_per_s": sw["tokens_per_s"], "frac_hbm": sw["frac_hbm"],
                                "quantize_all_ms": sw["quantize_all_ms"]}
    per = ex.get("decode_per_launch")
    if per:
        h["decode_min_call_frac_hbm"] = round(min(v["gbs"] for v in per.values()) / peaks["hbm_gbs"], 4)
    return h


def run_extras(torch, glmq, W16, quant, peaks):
    """Short, separately timed numbers: quantize roofline, prefill TFLOP/s, INT8."""
    from inputs import GLM_PROJECTIONS, PROJECTION_ORDER
    out = {"prefill_int4_m2048": {}, "int8": {}}
    for name in PROJECTION_ORDER:
        N, K = GLM_PROJECTIONS[name]
        packed, scale = quant[name]
        g = torch.Generator(device="cuda").manual_seed(3000)
        X = torch.randn((2048, K), generator=g, device="cuda", dtype=torch.float32).half()
        Y = torch.empty((2048, N), dtype=torch.float16, device="cuda")
        t = time_launches(torch, lambda: glmq.gemm(X, packed, scale, 4, out=Y), 5)
        tf = 2.0 * 2048 * N * K / t / 1e12
        out["prefill_int4_m2048"][name] = {"us": round(t * 1e6, 1), "tflops": round(tf, 1),
                                           "frac_burst": round(tf / peaks["bf16_tflops"], 4)}
        del X, Y
    # INT4 at M=64 (the skinny tensor-core kernel): arithmetic intensity ~249 flop/B, at the
    # ridge of the roofline, so both roofs are reported with the one that binds. L2 is
    # flushed before each timed call (attn-out's 75 MB of codes would otherwise stay in L2).
    out["int4_m64"] = {}
    settle(torch)
    for name in PROJECTION_ORDER:
        N, K = GLM_PROJECTIONS[name]
        packed, scale = quant[name]
        g = torch.Generator(device="cuda").manual_seed(3100)
        X = torch.randn((64, K), generator=g, device="cuda", dtype=torch.float32).half()
        Y = torch.empty((64, N), dtype=torch.float16, device="cuda")
        t = time_launches_cold(torch, lambda: glmq.gemm(X, packed, scale, 4, out=Y), 5)
        nbytes = packed.numel() + scale.numel() * 2 + X.numel() * 2 + Y.numel() * 2
        flops = 2.0 * 64 * N * K
        t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
        t_tc = flops / (peaks["bf16_tflops"] * 1e12)
        out["int4_m64"][name] = {"us": round(t * 1e6, 1), "weight_gbs": round(packed.numel() / t / 1e9, 1),
                                 "tflops": round(flops / t / 1e12, 1), "t_hbm_us": round(t_hbm * 1e6, 1),
                                 "t_tensor_us": round(t_tc * 1e6, 1),
                                 "binding": "hbm" if t_hbm >= t_tc else "tensor",
                                 "frac_binding_roof": round(max(t_hbm, t_tc) / t, 4)}
        del X, Y
    # FFN-up with the fused GeGLU epilogue (plus an fp16 bias) against the plain call
    N, K = GLM_PROJECTIONS["ffn_up"]
    pg, sg = glmq.quantize(W16["ffn_up"], 4, geglu=True)
    gb = torch.Generator(device="cuda").manual_seed(5000)
    bias = (torch.randn((N,), generator=gb, device="cuda", dtype=torch.float32) * 0.1).half()
    out["ffn_up_geglu_int4"] = {}
    for M in (1, 16, 2048):
        g = torch.Generator(device="cuda").manual_seed(6000 + M)
        X = torch.randn((M, K), generator=g, device="cuda", dtype=torch.float32).half()
        Yg = torch.empty((M, N // 2), dtype=torch.float16, device="cuda")
        Yp = torch.empty((M, N), dtype=torch.float16, device="cuda")
        tg = time_launches(torch, lambda: glmq.gemm_fused(X, pg, sg, 4, bias=bias, epilogue="geglu", out=Yg), 5)
        tp = time_launches(torch, lambda: glmq.gemm(X, pg, sg, 4, out=Yp), 5)
        out["ffn_up_geglu_int4"][f"M={M}"] = {"fused_us": round(tg * 1e6, 1), "plain_us": round(tp * 1e6, 1),
                                               "fused_weight_gbs": round(pg.numel() / tg / 1e9, 1)}
        del X, Yg, Yp
    del pg, sg
    # zero-point INT4 on QKV against the symmetric codes
    N, K = GLM_PROJECTIONS["qkv"]
    pz = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
    sz = torch.empty((N,), dtype=torch.float16, device="cuda")
    zz = torch.empty((N,), dtype=torch.uint8, device="cuda")
    tq = time_launches(torch, lambda: glmq.quantize_zp(W16["qkv"], out=(pz, sz, zz)), 3)
    out["zero_point_int4_qkv"] = {"quantize_us": round(tq * 1e6, 1),
                                  "quantize_gbs": round((N * K * 2 + N * K // 2 + N * 3) / tq / 1e9, 1)}
    for M in (1, 16, 2048):
        g = torch.Generator(device="cuda").manual_seed(7000 + M)
        X = torch.randn((M, K), generator=g, device="cuda", dtype=torch.float32).half()
        Y = torch.empty((M, N), dtype=torch.float16, device="cuda")
        t = time_launches(torch, lambda: glmq.gemm_zp(X, pz, sz, zz, out=Y), 5)
        out["zero_point_int4_qkv"][f"M={M}"] = {"us": round(t * 1e6, 1), "weight_gbs": round(pz.numel() / t / 1e9, 1),
                                                "tflops": round(2.0 * M * N * K / t / 1e12, 1)}
        del X, Y
    del pz, sz, zz
    # one rank's local GEMM under 4-way tensor parallelism (column: QKV, FFN-up; row:
    # attn-out, FFN-down); every rank's shard has the same shape, so rank 0's is timed.
    # The shards fit in L2, so L2 is flushed before each timed call.
    from int8_quantized_glmq_b200 import tensor_parallel as tpm
    out["tp4_local_int4"] = {}
    for name in PROJECTION_ORDER:
        N, K = GLM_PROJECTIONS[name]
        packed, scale = quant[name]
        if name in ("qkv", "ffn_up"):
            layer = tpm.ColumnParallelLinear(packed, scale, 4, 0, 4)
            Kl, Nl = K, N // 4
        else:
            layer = tpm.RowParallelLinear(packed, scale, 4, 0, 4)
            Kl, Nl = K // 4, N
        res = {"shard": f"{Nl}x{Kl}"}
        for M in (1, 16):
            g = torch.Generator(device="cuda").manual_seed(8000 + M)
            X = torch.randn((M, Kl), generator=g, device="cuda", dtype=torch.float32).half()
            Y = torch.empty((M, Nl), dtype=torch.float16, device="cuda")
            t = time_launches_cold(torch, lambda: glmq.gemm(X, layer.packed, layer.scale, 4, out=Y), 5)
            res[f"M={M}"] = {"us": round(t * 1e6, 1), "weight_gbs": round(layer.packed.numel() / t / 1e9, 1)}
            del X, Y
        out["tp4_local_int4"][name] = res
        del layer
    for name in PROJECTION_ORDER:
        N, K = GLM_PROJECTIONS[name]
        p8 = torch.empty((N, K), dtype=torch.uint8, device="cuda")
        s8 = torch.empty((N,), dtype=torch.float16, device="cuda")
        tq = time_launches(torch, lambda: glmq.quantize(W16[name], 8, out=(p8, s8)), 3)
        res = {"quantize_us": round(tq * 1e6, 1), "quantize_gbs": round((N * K * 3 + N * 2) / tq / 1e9, 1)}
        settle(torch)
        for M in (1, 64, 2048):
            g = torch.Generator(device="cuda").manual_seed(4000 + M)
            X = torch.randn((M, K), generator=g, device="cuda", dtype=torch.float32).half()
            Y = torch.empty((M, N), dtype=torch.float16, device="cuda")
            timer = time_launches if M == 2048 else time_launches_cold
            t = timer(torch, lambda: glmq.gemm(X, p8, s8, 8, out=Y), 5)
            res[f"M={M}"] = {"us": round(t * 1e6, 1), "weight_gbs": round(N * K / t / 1e9, 1),
                             "tflops": round(2.0 * M * N * K / t / 1e12, 1)}
            if M == 64:
                res["M=64"]["frac_hbm"] = round(N * K / t / 1e9 / peaks["hbm_gbs"], 4)
        out["int8"][name] = res
        del p8, s8
    return out


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, world, rank):
    """The CPU oracle, as it stands, on a bounded sample of the decode workload."""
    import numpy as np
    import oracle
    from inputs import GLM_PROJECTIONS, PROJECTION_ORDER, decode_activations, projection_weight

    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        cores = os.cpu_count() or 1
    rows = 256  # sampled output features per projection per step
    samples = {}
    for i, name in enumerate(PROJECTION_ORDER):
        N, K = GLM_PROJECTIONS[name]
        W = projection_weight(name, seed=1000 + i, rows=slice(0, rows))
        samples[name] = oracle.quantize_linear(W, 4)
    xs = {(M, n): decode_activations(M, GLM_PROJECTIONS[n][1], 2000 + M) for M in DECODE_MS for n in PROJECTION_ORDER}

    def step():
        for M in DECODE_MS:
            for n in PROJECTION_ORDER:
                p, s = samples[n]
                oracle.linear_forward(xs[(M, n)], p, s, 4)

    for _ in range(args.warmup):
        step()
    t = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t
    wbytes = sum(samples[n][0].nbytes for n in PROJECTION_ORDER) * len(DECODE_MS)
    value = wbytes * args.steps / el / 1e9
    sample = (f"{rows} output rows of each projection (of 12288..65536), M in {{1,4,16}}, INT4, "
              "oracle float64 dequantizing linear")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "decode GEMV on GLM-130B layer shapes, M in {1,4,16}, INT4 weights (sampled rows)"},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def cpu_baseline(budget_s: float = 12.0):
    """Oracle timing on the host cores for the cpu_baseline key (rank 0, N=1)."""
    import numpy as np
    import oracle
    from inputs import GLM_PROJECTIONS, decode_activations, projection_weight
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        cores = os.cpu_count() or 1
    N, K = GLM_PROJECTIONS["qkv"]
    rows = 2048
    W = projection_weight("qkv", seed=1000, rows=slice(0, rows))
    packed, s = oracle.quantize_linear(W, 4)
    X = decode_activations(1, K, 2001)
    t0 = time.perf_counter()
    n = 0
    while time.perf_counter() - t0 < budget_s:
        oracle.linear_forward(X, packed, s, 4)
        n += 1
    el = time.perf_counter() - t0
    return {"value": round(packed.nbytes * n / el / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"QKV decode M=1, {rows} of 36864 output rows x K=12288, INT4, repeated {n}x for {el:.1f} s"}


# ----------------------------------------------------------------------------- sweep
SWEEP_LAYERS = 70


def sweep_weight(torch, layer: int, proj_index: int, out):
    """Fills out with the fp16 weights of one projection of the layer sweep, N(0, 0.02),
    seeded by (layer, projection): seed 10000 + 4 * layer + proj_index."""
    g = torch.Generator(device="cuda").manual_seed(10000 + 4 * layer + proj_index)
    return out.normal_(0.0, 0.02, generator=g)


class Sweep:
    """The INT4 layer sweep: every projection of every layer quantized once (one-shot,
    layer by layer, each call timed) and resident in HBM, plus one CUDA graph that runs
    the M=1 decode GEMM through all of them in layer order. Each projection p reads the
    same seeded activation row xs[p]; the outputs of the layers in ``keep`` go to their
    own buffers (kept[(layer, name)]) so they can be checked after a replay."""

    def __init__(self, torch, glmq, layers: int, keep=()):
        from inputs import GLM_PROJECTIONS, PROJECTION_ORDER
        self.layers = layers
        self.quant = []
        self.qtime = 0.0
        self.qbytes = 0
        wbuf = {n: torch.empty(GLM_PROJECTIONS[n], dtype=torch.float16, device="cuda") for n in PROJECTION_ORDER}
        s = torch.cuda.current_stream()
        for layer in range(layers):
            row = []
            for p, n in enumerate(PROJECTION_ORDER):
                N, K = GLM_PROJECTIONS[n]
                sweep_weight(torch, layer, p, wbuf[n])
                packed = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
                scale = torch.empty((N,), dtype=torch.float16, device="cuda")
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(s)
                glmq.quantize(wbuf[n], 4, out=(packed, scale))
                e1.record(s)
                torch.cuda.synchronize()
                self.qtime += e0.elapsed_time(e1) / 1e3
                self.qbytes += N * K * 2 + N * K // 2 + N * 2
                row.append((packed, scale))
            self.quant.append(row)
        del wbuf
        torch.cuda.empty_cache()
        self.xs = {}
        for p, n in enumerate(PROJECTION_ORDER):
            g = torch.Generator(device="cuda").manual_seed(20000 + p)
            self.xs[n] = torch.randn((1, GLM_PROJECTIONS[n][1]), generator=g, device="cuda").half()
        self.ys = {n: torch.empty((1, GLM_PROJECTIONS[n][0]), dtype=torch.float16, device="cuda")
                   for n in PROJECTION_ORDER}
        self.kept = {(layer, n): torch.full((1, GLM_PROJECTIONS[n][0]), float("nan"), dtype=torch.float16,
                                            device="cuda")
                     for layer in keep for n in PROJECTION_ORDER}
        self.order = [(layer, p, n) for layer in range(layers) for p, n in enumerate(PROJECTION_ORDER)]
        self.wbytes = sum(q[0].numel() for row in self.quant for q in row)
        cs = torch.cuda.Stream()
        cs.wait_stream(s)
        with torch.cuda.stream(cs):
            for _ in range(2):
                self._step(glmq)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        n0 = glmq.kernel_launches()
        with torch.cuda.graph(self.graph, stream=cs):
            self._step(glmq)
        self.kernels_per_replay = glmq.kernel_launches() - n0

    def _step(self, glmq):
        # each call names the next one (the next projection, or layer 0's first after the
        # last layer) so that its weights' first tiles are prefetched into L2 while this
        # call's ring drains, as a serving loop through the layers would call it
        for i, (layer, p, n) in enumerate(self.order):
            out = self.kept.get((layer, n), self.ys[n])
            nl, np_, _ = self.order[(i + 1) % len(self.order)]
            glmq.gemm_decode_prefetch(self.xs[n], self.quant[layer][p][0], self.quant[layer][p][1], 4,
                                      next_packed=self.quant[nl][np_][0], next_M=1, out=out)

    def time_replays(self, torch, steps: int, warmup: int, world: int = 1):
        """Device seconds of `steps` replays (CUDA events on the current stream)."""
        for _ in range(warmup):
            self.graph.replay()
        torch.cuda.synchronize()
        barrier(world)
        s = torch.cuda.current_stream()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(steps):
            self.graph.replay()
        e1.record(s)
        torch.cuda.synchronize()
        barrier(world)
        return e0.elapsed_time(e1) / 1e3


def run_sweep(args, world, rank, local):
    """70 layers x 4 projections resident as INT4; M=1 decode through all 280 in one CUDA graph."""
    import torch
    import int8_quantized_glmq_b200 as glmq

    sw = Sweep(torch, glmq, args.layers)
    clocks = ClockSampler(local)
    clocks.start()
    el_local = sw.time_replays(torch, args.steps, args.warmup, world)
    clk = clocks.stop()
    tok_s, el = whole_job_rate(1.0, args.steps, el_local, world)
    peaks = measured_peaks()
    gbs = sw.wbytes * args.steps / el / 1e9
    res = {"metric": "GLM-130B 70-layer INT4 decode sweep (M=1, 280 projections), tokens/s",
           "value": round(tok_s, 2), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 4), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "fp16", "weight_dtype": "int4", "data": "synthetic",
           "config": {"workload": f"{args.layers}-layer GLM-130B projection sweep, M=1, "
                                  f"CUDA graph of {4 * args.layers} calls",
                      "packed_weight_bytes": sw.wbytes, "l2": "63 GB working set >> L2"},
           "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": round(gbs / peaks["hbm_gbs"], 4), "peak_source": peaks["source"], "traffic": None},
           "quantize_all_layers": {"ms": round(sw.qtime * 1e3, 2), "gbs": round(sw.qbytes / sw.qtime / 1e9, 1)},
           "gpu_launches": sw.kernels_per_replay * args.steps, "clocks": clk}
    del sw
    return res


def sweep_summary(torch, glmq, peaks, layers: int = SWEEP_LAYERS, steps: int = 10, warmup: int = 3):
    """Compact result of the layer sweep for the default bench line's extras."""
    free, _ = torch.cuda.mem_get_info()
    if free < 72e9 * layers / SWEEP_LAYERS:
        return {"skipped": f"needs about {72 * layers // SWEEP_LAYERS} GB free on the device"}
    sw = Sweep(torch, glmq, layers)
    el = sw.time_replays(torch, steps, warmup)
    gbs = sw.wbytes * steps / el / 1e9
    out = {"layers": layers, "tokens_per_s": round(steps / el, 2), "ms_per_token": round(el / steps * 1e3, 3),
           "weight_gbs": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
           "quantize_all_ms": round(sw.qtime * 1e3, 2), "quantize_gbs": round(sw.qbytes / sw.qtime / 1e9, 1)}
    del sw
    torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------------------- one launch (profiling)
def run_one(args, world, rank, local):
    """A handful of glmq_gemm (or glmq_quantize) launches on one GLM projection, for ncu captures."""
    import torch
    import int8_quantized_glmq_b200 as glmq
    from inputs import GLM_PROJECTIONS

    N, K = GLM_PROJECTIONS[args.proj]
    g = torch.Generator(device="cuda").manual_seed(1000)
    W = torch.empty((N, K), dtype=torch.float16, device="cuda").normal_(0.0, 0.02, generator=g)
    packed, scale = glmq.quantize(W, args.bits)
    if args.op == "gemm":
        del W
        X = torch.randn((args.m, K), generator=g, device="cuda", dtype=torch.float32).half()
        Y = torch.empty((args.m, N), dtype=torch.float16, device="cuda")
        fn = lambda: glmq.gemm(X, packed, scale, args.bits, out=Y, route=args.route)  # noqa: E731
        work = {"bytes": packed.numel() + scale.numel() * 2 + X.numel() * 2 + Y.numel() * 2,
                "flops": 2.0 * args.m * N * K}
    else:
        fn = lambda: glmq.quantize(W, args.bits, out=(packed, scale))  # noqa: E731
        work = {"bytes": W.numel() * 2 + packed.numel() + scale.numel() * 2, "flops": 0.0}
    t = time_launches(torch, fn, args.steps, warmup=args.warmup)
    return {"workload": "one", "op": args.op, "route": args.route, "proj": args.proj, "N": N, "K": K, "M": args.m,
            "bits": args.bits,
            "us": round(t * 1e6, 2), "gbs": round(work["bytes"] / t / 1e9, 1),
            "tflops": round(work["flops"] / t / 1e12, 1), "algorithmic_bytes": work["bytes"]}


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode", choices=["decode", "sweep", "one"])
    ap.add_argument("--proj", default="attn_out", choices=["qkv", "attn_out", "ffn_up", "ffn_down"])
    ap.add_argument("--op", default="gemm", choices=["gemm", "quantize"])
    ap.add_argument("--m", type=int, default=1)
    ap.add_argument("--bits", type=int, default=4, choices=[4, 8])
    ap.add_argument("--route", default="auto", choices=["auto", "decode", "prefill"],
                    help="glmq_gemm entry point for --workload one")
    ap.add_argument("--layers", type=int, default=70)
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        print(json.dumps(run_reference(args, world, rank)), flush=True)
        return

    world, rank, local = dist_setup()
    if args.workload == "sweep":
        res = run_sweep(args, world, rank, local)
    elif args.workload == "one":
        res = run_one(args, world, rank, local)
    else:
        res = run_decode(args, world, rank, local)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline()
        res["highlights"] = res.pop("highlights")       # keep the compact summary last on the line
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
