#!/usr/bin/env python
"""Benchmark of the SVDQuant W4A4 NVFP4 linear layer on B200.

Workload: the fused-QKV projection of a DiT block at 1024x1024 (M = 4608
tokens = 4096 image + 512 text, K = 3072, N = 9216, rank 32, NVFP4 group 16),
seeded synthetic inputs (synth/). One step = the whole hot path over one batch:
svdq_quantize_act (smoothing + NVFP4 quantisation + x_hat L1) followed by
svdq_w4a4_linear (block-scaled FP4 GEMM + P L2 + bias). The weight pack is
offline and not timed.

Metric: TFLOPS counted as 2 M N K per step (the low-rank flops are not
counted), and that value as a fraction of the dense FP4 peak.

Timing: W untimed warm-up steps, then K timed steps. Before every step a
512 MiB buffer is written (L2 is 126 MB) outside the step's events, so each
step starts with a cold L2. Steps are timed with CUDA events on the launching
stream; the timed loop is bracketed by a barrier and a device synchronise on
both sides; with several GPUs every rank runs its own replica (independent
batches: weak scaling, no collective on the data path) and the per-step time
is the maximum over ranks.

``--impl reference`` times the CPU oracle (the only reference implementation
of this path) on a bounded row sample of the same workload.

Roofline traffic: DRAM bytes per launch of the GEMM kernel as read by one
`ncu --set full` capture (dram__bytes_read.sum + dram__bytes_write.sum). The
figure is tied to the SHA-256 of the kernel source it was taken on and is
reported as null once that source has changed.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

WORKLOAD = "c3_qkv_nvfp4"
METRIC = "SVDQ W4A4-NVFP4 linear TFLOPS, % dense FP4 peak (M4608 K3072 N9216 r32)"
FP4_DENSE_SPEC_TFLOPS = 9000.0
NOMINAL_FP4_OVER_BF16 = 4.0     # 9 PF / 2.25 PF dense
NOMINAL_INT8_OVER_BF16 = 2.0    # 4.5 POPS / 2.25 PF dense
L2_FLUSH_BYTES = 512 << 20
GEMM_SOURCES = [os.path.join(ROOT, "bit_w4a4_quantized_nvfp4_b200", "csrc", f) for f in ("gemm_nvfp4.cu", "device.cuh")]
# {sha256 over the GEMM kernel's sources: DRAM bytes per launch from an ncu capture of the workload}
GEMM_TRAFFIC = {
    # profiles/gemm_nvfp4_c3.md: 25,554,944 B read + 31,602,432 B written
    "dc49122f1ef557b053c0051dea957ca15b67793316a8a7aa51c304a8aad672e1": 57157376,
}


def gemm_traffic():
    h = hashlib.sha256()
    try:
        for path in GEMM_SOURCES:
            with open(path, "rb") as f:
                h.update(f.read())
    except OSError:
        return None
    return GEMM_TRAFFIC.get(h.hexdigest())


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sustained=float(p["bf16_tflops_sustained"]), source="measured")
    except Exception:
        return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self._t.join(timeout=2)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(n_gpus: int, timeout_s: float = 120.0):
    """Join the torchrun job (one rank per GPU, NCCL); without a GPU the same
    host logic runs over gloo (used by the CPU tests)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    cuda = torch.cuda.is_available()
    if world > 1:
        import datetime

        import torch.distributed as dist

        if cuda:
            torch.cuda.set_device(local)
        dist.init_process_group("nccl" if cuda else "gloo", timeout=datetime.timedelta(seconds=timeout_s))
    elif cuda:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(world, v: float) -> float:
    if world == 1:
        return v
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world: int, flops_per_rank_step: float, ms_per_step: float) -> float:
    """Throughput of all ranks together: every rank runs one step of the same
    size, and the step time is the slowest rank's."""
    return world * flops_per_rank_step / (ms_per_step * 1e-3) / 1e12


def trimmed_mean(xs, frac: float = 0.1) -> float:
    """Mean after dropping the lowest and highest `frac` of the samples. CUDA
    event times come in ticks of about a microsecond, so a median sits on one
    tick; the trimmed mean averages the ticks out and still ignores outliers."""
    ys = sorted(xs)
    k = int(len(ys) * frac)
    ys = ys[k:len(ys) - k] if len(ys) > 2 * k else ys
    return statistics.mean(ys)


def bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


# --------------------------------------------------------------------------- CUDA arm
def run_cuda(args):
    import bit_w4a4_quantized_nvfp4_b200 as svdq

    world, rank, local = dist_setup(args.gpus)
    svdq.load()
    c = synth.CONFIGS[WORKLOAD]
    M, K, N, r = c["M"], c["K"], c["N"], c["r"]
    d = synth.config_layer(WORKLOAD)
    W = torch.from_numpy(d["W"]).cuda()
    lam = torch.from_numpy(d["lam"]).cuda()
    L1, L2, b = bf16_dev(d["L1"]), bf16_dev(d["L2"]), bf16_dev(d["b"])
    x = bf16_dev(d["x"])
    pw = svdq.pack_weight("nvfp4", W, lam, L1, L2)
    del W
    stream = torch.cuda.current_stream()
    qa = svdq.quantize_act(x, pw, L1)
    y = svdq.w4a4_linear(qa, pw, b)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    svdq.device_error()

    def step():
        svdq.quantize_act(x, pw, L1, out=qa)
        svdq.w4a4_linear(qa, pw, b, out=y)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()

    K_steps = args.steps

    def timed(split: bool):
        """K timed steps, each after an L2 flush, timed by events on the
        launching stream. split=False: events around the step only, so the
        GEMM's launch may overlap the activation pass's tail (dependent
        launch), as in use; split=True: one more event between the two
        kernels, which serialises them and times each alone."""
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
               torch.cuda.Event(enable_timing=True)) for _ in range(K_steps)]
        barrier(world)
        torch.cuda.synchronize()
        for i in range(K_steps):
            flush.zero_()
            e0, e1, e2 = ev[i]
            e0.record(stream)
            svdq.quantize_act(x, pw, L1, out=qa)
            if split:
                e1.record(stream)
            svdq.w4a4_linear(qa, pw, b, out=y)
            e2.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        return ev

    clocks = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    wall0 = time.perf_counter()
    ev = timed(split=False)
    wall = time.perf_counter() - wall0
    ev_split = timed(split=True)
    clk = clocks.stop() if clocks else None
    svdq.device_error()

    step_ms = [e0.elapsed_time(e2) for e0, _, e2 in ev]
    k1_ms = [e0.elapsed_time(e1) for e0, e1, _ in ev_split]
    k2_ms = [e1.elapsed_time(e2) for _, e1, e2 in ev_split]
    # the median of the timed steps (one slow step does not move it), max over ranks
    ms = max_over_ranks(world, statistics.median(step_ms))
    k1 = max_over_ranks(world, statistics.median(k1_ms))
    k2 = max_over_ranks(world, statistics.median(k2_ms))
    flops = 2.0 * M * N * K
    value = whole_job_tflops(world, flops, ms)

    # end to end through the public API with host buffers
    xh = torch.from_numpy(np.ascontiguousarray(d["x"]).view(np.int16)).pin_memory()
    e2e_steps = max(3, min(20, K_steps))
    e2e_ms = max_over_ranks(world, e2e_pipelined(svdq, pw, L1, b, xh, M, N, K, e2e_steps, world))

    P = peaks()
    fp4_peak = P["bf16"] * NOMINAL_FP4_OVER_BF16
    k2_tflops = flops / (k2 * 1e-3) / 1e12
    probe = mma_probe(svdq) if rank == 0 and not args.no_probe else None
    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "value_with_low_rank": round(whole_job_tflops(world, flops + 2.0 * M * r * (K + N), ms), 2),
        "unit": "TFLOPS",
        "n_gpus": world,
        "steps": K_steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4",
        "data": "synthetic",
        "config": {"workload": f"svdq_w4a4 nvfp4 fused-QKV projection M{M} K{K} N{N} r{r} (seeded DiT-shaped "
                               "inputs, 0.5% outlier channels x30)",
                   "M": M, "K": K, "N": N, "r": r, "group": 16,
                   "l2": "flushed before every timed step (512 MiB write, outside the step's events)",
                   "parallelism": f"{world} independent replicas (weak scaling, no collective)"},
        "pct_dense_fp4_peak_spec": round(100.0 * value / world / FP4_DENSE_SPEC_TFLOPS, 2),
        "kernels_ms": {"quantize_act": round(k1, 5), "w4a4_gemm": round(k2, 5),
                       "timing": "second timed loop of the same K steps with an event between the two kernels "
                                 "(serialised), medians"},
        "step_ms_stats": {"median": round(statistics.median(step_ms), 5), "mean": round(statistics.mean(step_ms), 5),
                          "trimmed_mean_10pct": round(trimmed_mean(step_ms), 5),
                          "kernels_trimmed_mean_10pct": {"quantize_act": round(trimmed_mean(k1_ms), 5),
                                                         "w4a4_gemm": round(trimmed_mean(k2_ms), 5)},
                          "min": round(min(step_ms), 5), "max": round(max(step_ms), 5), "n": len(step_ms),
                          "statistic": "median of the timed steps (rank 0's spread shown)"},
        "roofline": {"kernel": "w4a4_gemm (tcgen05 mxf4nvf4)", "bound": "tensor",
                     "achieved": round(k2_tflops, 1),
                     "peak": round(fp4_peak, 1), "unit": "TFLOP/s",
                     "frac": round(k2_tflops / fp4_peak, 4),
                     "peak_source": f"{P['source']} bf16 burst {P['bf16']} x nominal fp4/bf16 ratio 4",
                     "traffic": gemm_traffic(),
                     "probe_peak": probe,
                     "frac_of_probe": round(k2_tflops / probe["tflops"], 4) if probe else None},
        "e2e": {"value": round(whole_job_tflops(world, flops, e2e_ms), 3), "unit": "TFLOPS",
                "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2, "ms_per_step": round(e2e_ms, 4),
                "overlap": "copy in, compute and copy out of consecutive steps on three streams, two device buffers"},
        "gpu_launches": 2 * K_steps,
        "gpu_launches_note": "2 per step (activation pass, GEMM) in the headline timed loop; the split loop "
                             "for kernels_ms launches the same 2 per step",
        "wall_s_timed_region": round(wall, 4),
    }
    if clk:
        out["clocks"] = clk
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(d, rows=args.cpu_rows)
    if rank == 0 and not args.no_qkv:
        out["qkv_epilogue"] = bench_qkv(svdq, pw, L1, b, x, qa, flush, M, N, K)
    if rank == 0 and not args.no_mlp:
        del d
        out["mlp_gelu"] = bench_mlp(svdq, flush)
    if rank == 0 and not args.no_awq:
        out["awq_gemv"] = [bench_awq(svdq, P, m) for m in synth.CONFIGS["c2_awq_gemv"]["Ms"]]
    if rank == 0 and not args.no_int4:
        out["int4_linear"] = bench_int4(svdq, P)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def mma_probe(svdq, iters=4096, reps=5):
    """The device's own rate for the GEMM's MMA instruction (block-scaled
    NVFP4, 256 x 256 x 64 per CTA pair), from the library's probe kernel:
    operands resident in shared memory, no loads, no epilogue. mode 0 = MMAs
    only; mode 1 adds the GEMM's per-stage scale copies. Median of `reps`
    launches timed with CUDA events."""
    out = {}
    for mode in (0, 1):
        svdq.probe_mma_peak(iters, mode)
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fl = svdq.probe_mma_peak(iters, mode)
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        svdq.device_error()
        out[f"mode{mode}"] = round(fl / (statistics.median(ts) * 1e-3) / 1e12, 1)
    return {"tflops": out["mode0"], "tflops_with_scale_copies": out["mode1"], "unit": "TFLOP/s",
            "what": "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 256x256x64 back to back on "
                    "shared-memory operands, every SM pair (library probe kernel), median of 5 launches"}


def e2e_pipelined(svdq, pw, L1, b, xh, M, N, K, steps, world):
    """ms per step of the layer fed from, and read back to, pinned host memory:
    each step copies its x in (H2D), runs svdq_quantize_act + svdq_w4a4_linear
    and copies its y out (D2H). Consecutive steps overlap on three streams
    (copy in, compute, copy out) with two device buffers each, as a serving
    loop would; the timed region runs from before the first copy in to after
    the last copy out."""
    s_in, s_c, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    xd = [torch.empty((M, K), dtype=torch.int16, device="cuda") for _ in range(2)]
    yd = [torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    yh = torch.empty((M, N), dtype=torch.int16).pin_memory()
    for k in range(2):
        xd[k].copy_(xh)
    qa = [svdq.quantize_act(xd[k].view(torch.bfloat16), pw, L1) for k in range(2)]
    torch.cuda.synchronize()

    def run(n):
        ev_in = [torch.cuda.Event() for _ in range(n)]
        ev_c = [torch.cuda.Event() for _ in range(n)]
        ev_out = [torch.cuda.Event() for _ in range(n)]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(s_in)
        for i in range(n):
            k = i % 2
            if i >= 2:
                s_in.wait_event(ev_c[i - 2])  # step i-2 has finished reading xd[k]
            with torch.cuda.stream(s_in):
                xd[k].copy_(xh, non_blocking=True)
            ev_in[i].record(s_in)
            s_c.wait_event(ev_in[i])
            if i >= 2:
                s_c.wait_event(ev_out[i - 2])  # yd[k] of step i-2 has been copied out
            svdq.quantize_act(xd[k].view(torch.bfloat16), pw, L1, stream=s_c, out=qa[k])
            svdq.w4a4_linear(qa[k], pw, b, stream=s_c, out=yd[k])
            ev_c[i].record(s_c)
            s_out.wait_event(ev_c[i])
            with torch.cuda.stream(s_out):
                yh.copy_(yd[k].view(torch.int16), non_blocking=True)
            ev_out[i].record(s_out)
        end.record(s_out)
        torch.cuda.synchronize()
        return start.elapsed_time(end) / n

    run(2)
    barrier(world)
    ms = run(steps)
    barrier(world)
    return ms


def bench_qkv(svdq, pw, L1, b, x, qa, flush, M, N, K, steps=30):
    """The workload as the grouped Q/K/V projection of a DiT block (24 heads
    of 128 per section) followed by per-head RMSNorm of Q and K and the rotary
    embedding: fused into the GEMM's epilogue (svdq_w4a4_linear_qkv) against
    the plain layer followed by the separate pass (svdq_qkv_norm_rope). One
    step = activation pass + GEMM (+ pass), L2 flushed before each step,
    medians of CUDA-event times."""
    heads = N // 384
    e = synth.qkv_epilogue_inputs(synth.CONFIGS[WORKLOAD]["seed"], M, 128, heads)
    wq, wk = bf16_dev(e["wq"]), bf16_dev(e["wk"])
    cos, sin = torch.from_numpy(e["cos"]).cuda(), torch.from_numpy(e["sin"]).cuda()
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    rope = svdq.pack_rope(cos, sin)

    def fused():
        svdq.quantize_act(x, pw, L1, out=qa)
        svdq.w4a4_linear_qkv(qa, pw, heads, wq, wk, e["eps"], rope, b, out=y)

    def pack():
        svdq.pack_rope(cos, sin)

    def unfused():
        svdq.quantize_act(x, pw, L1, out=qa)
        svdq.w4a4_linear(qa, pw, b, out=y)
        svdq.qkv_norm_rope(y, heads, wq, wk, e["eps"], cos, sin)

    res = {}
    for name, fn in (("fused_ms", fused), ("unfused_ms", unfused), ("rope_pack_ms", pack)):
        ts = []
        for i in range(steps + 3):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            if i >= 3:
                ts.append(e0.elapsed_time(e1))
        res[name] = round(statistics.median(ts), 5)
    svdq.device_error()
    res["speedup"] = round(res["unfused_ms"] / res["fused_ms"], 4)
    res["workload"] = (f"fused-QKV projection M{M} K{K} N{N} ({heads} heads of 128 per section) + RMSNorm of Q, K "
                       "+ rotary embedding")
    res["note"] = ("the fused step reads the rotary tables packed by svdq_rope_pack, once per set of positions "
                   "(shared by every attention layer of a forward pass): rope_pack_ms is that pack, not in fused_ms")
    return res


def bench_mlp(svdq, flush, steps=30):
    """The MLP pair of a DiT block at full size: up-projection 4608x3072 ->
    12288, GELU, down-projection 4608x12288 -> 3072, both svdq_w4a4 NVFP4
    layers with rank-32 branches. Fused: the up-projection's epilogue computes
    GELU before its one rounding (bf16_gelu output) and its output is the
    down-projection's activation-pass input (4 launches). Unfused: the plain
    up-projection, then GELU as a separate elementwise pass (torch's
    gelu, the non-fused stand-in), then the down-projection (4 launches + 1).
    L2 flushed before each step; medians of CUDA-event times."""
    up = synth.config_layer("c4_mlp_up_nvfp4")
    down = synth.config_layer("c4_mlp_down_nvfp4")
    M, K, F = up["M"], up["K"], up["N"]

    def prep(d):
        L1, L2 = bf16_dev(d["L1"]), bf16_dev(d["L2"])
        pw = svdq.pack_weight("nvfp4", torch.from_numpy(d["W"]).cuda(), torch.from_numpy(d["lam"]).cuda(), L1, L2)
        return pw, L1, bf16_dev(d["b"])

    pw_u, L1u, bu = prep(up)
    pw_d, L1d, bd = prep(down)
    x = bf16_dev(up["x"])
    qa_u = svdq.quantize_act(x, pw_u, L1u)
    h = svdq.w4a4_linear(qa_u, pw_u, bu, out_dtype="bf16_gelu")
    qa_d = svdq.quantize_act(h, pw_d, L1d)
    y = svdq.w4a4_linear(qa_d, pw_d, bd)
    yu = torch.empty_like(h)
    torch.cuda.synchronize()

    def fused():
        svdq.quantize_act(x, pw_u, L1u, out=qa_u)
        svdq.w4a4_linear(qa_u, pw_u, bu, out_dtype="bf16_gelu", out=h)
        svdq.quantize_act(h, pw_d, L1d, out=qa_d)
        svdq.w4a4_linear(qa_d, pw_d, bd, out=y)

    def unfused():
        svdq.quantize_act(x, pw_u, L1u, out=qa_u)
        svdq.w4a4_linear(qa_u, pw_u, bu, out=yu)
        hu = torch.nn.functional.gelu(yu, approximate="none")
        svdq.quantize_act(hu, pw_d, L1d, out=qa_d)
        svdq.w4a4_linear(qa_d, pw_d, bd, out=y)

    res = {}
    for name, fn in (("fused_ms", fused), ("unfused_ms", unfused)):
        ts = []
        for i in range(steps + 3):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            if i >= 3:
                ts.append(e0.elapsed_time(e1))
        res[name] = round(statistics.median(ts), 5)
    svdq.device_error()
    flops = 2.0 * M * K * F * 2
    res["fused_tflops"] = round(flops / (res["fused_ms"] * 1e-3) / 1e12, 1)
    res["speedup"] = round(res["unfused_ms"] / res["fused_ms"], 4)
    res["workload"] = (f"MLP pair M{M}: up K{K} -> N{F} (GELU) and down K{F} -> N{K}, NVFP4, r32 "
                       "(seeded DiT-shaped inputs; the down-projection's input is the up-projection's output)")
    res["unfused_gelu"] = "torch.nn.functional.gelu (erf) as a separate pass, the non-fused comparison"
    return res


def bench_int4(svdq, P, steps=10):
    """The INT4 variant of the layer (M4608 K3072 N9216 r32, symmetric INT4
    g64 activations and weights): one step = svdq_quantize_act + svdq_w4a4_linear,
    L2 flushed before each step, against the dense INT8 tensor peak (the int4
    codes are widened to int8 for the MMA)."""
    name = "c5_qkv_int4"
    c = synth.CONFIGS[name]
    M, K, N, r = c["M"], c["K"], c["N"], c["r"]
    d = synth.config_layer(name)
    L1, L2, b = bf16_dev(d["L1"]), bf16_dev(d["L2"]), bf16_dev(d["b"])
    x = bf16_dev(d["x"])
    pw = svdq.pack_weight("int4", torch.from_numpy(d["W"]).cuda(), torch.from_numpy(d["lam"]).cuda(), L1, L2)
    qa = svdq.quantize_act(x, pw, L1)
    y = svdq.w4a4_linear(qa, pw, b)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    ms = []
    for i in range(steps + 3):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        svdq.quantize_act(x, pw, L1, out=qa)
        svdq.w4a4_linear(qa, pw, b, out=y)
        e1.record()
        torch.cuda.synchronize()
        if i >= 3:
            ms.append(e0.elapsed_time(e1))
    svdq.device_error()
    t = statistics.median(ms)
    tops = 2.0 * M * N * K / (t * 1e-3) / 1e12
    peak = P["bf16"] * NOMINAL_INT8_OVER_BF16
    return {"workload": f"svdq_w4a4 int4 g64 M{M} K{K} N{N} r{r}", "ms_per_step": round(t, 4),
            "value": round(tops, 1), "unit": "TOPS", "peak": round(peak, 1),
            "peak_source": f"{P['source']} bf16 burst {P['bf16']} x nominal int8/bf16 ratio 2",
            "frac": round(tops / peak, 4), "steps": steps}


def bench_awq(svdq, P, M=1):
    """AWQ W4A16 modulation projection (M rows, K 3072, N 18432): HBM-bound at
    small M. Weights rotate over copies totalling > 3x L2 so every launch
    streams from HBM; the launches are replayed from a CUDA graph, since one
    launch takes less device time than the host needs to issue it."""
    c = synth.CONFIGS["c2_awq_gemv"]
    K, N = c["K"], c["N"]
    d = synth.awq_inputs(c["seed"], M, K, N)
    w0 = svdq.awq_pack_weight(torch.from_numpy(d["W"]).cuda())
    copies = []
    for _ in range(12):  # 12 x 31.9 MB = 383 MB
        copies.append(svdq.AwqWeight(K, N, w0.q.clone(), w0.scales.clone(), w0.zeros.clone()))
    x = bf16_dev(d["x"])
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        for w in copies:
            svdq.awq_w4a16_linear(x, w, out=y)
    torch.cuda.synchronize()
    rounds = 5
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for _ in range(rounds):
            for w in copies:
                svdq.awq_w4a16_linear(x, w, out=y)
    g.replay()
    torch.cuda.synchronize()
    reps = 4
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(reps):
        g.replay()
    e.record()
    torch.cuda.synchronize()
    svdq.device_error()
    launches = reps * rounds * len(copies)
    us = s.elapsed_time(e) * 1e3 / launches
    byts = N * K // 2 + 2 * 2 * N * (K // 64) + M * K * 2 + M * N * 2
    gbs = byts / (us * 1e-6) / 1e9
    return {"M": M, "K": K, "N": N, "us_per_launch": round(us, 3), "algorithmic_bytes": byts,
            "achieved_gbs": round(gbs, 1), "peak_gbs": P["hbm_gbs"], "frac": round(gbs / P["hbm_gbs"], 4),
            "tflops": round(2.0 * M * N * K / (us * 1e-6) / 1e12, 3),
            "timing": f"CUDA graph of {rounds * len(copies)} launches over 12 rotating weight copies, replayed {reps}x"}


# --------------------------------------------------------------------------- oracle
def cpu_baseline(d, rows: int, tag="oracle"):
    import oracle

    c = synth.CONFIGS[WORKLOAD]
    K, N = c["K"], c["N"]
    w = oracle.pack_weight("nvfp4", d["W"], d["lam"], d["L1"], d["L2"])
    x = d["x"][:rows]
    t0 = time.perf_counter()
    a = oracle.quantize_act("nvfp4", x, w["inv_lam"], 1.0, d["L1"])
    oracle.linear("nvfp4", a, w, 1.0, d["L2"], d["b"])
    dt = time.perf_counter() - t0
    return {"value": round(2.0 * rows * N * K / dt / 1e12, 6), "unit": "TFLOPS", "cores": oracle.threads(),
            "kind": tag, "sample": f"first {min(rows, c['M'])} of {c['M']} rows of the workload (quantize_act + "
                                    "linear, float64 accumulation); weight pack untimed", "seconds": round(dt, 3)}


def oracle_configs():
    """Wall time of the CPU oracle on every workload, in full (the weight pack
    untimed): svdq workloads = quantize_act + linear over all M rows; the AWQ
    GEMV at each M of its sweep. The small workloads are also timed on one
    thread. One JSON line; a reported baseline, not a target."""
    import oracle

    nthreads = oracle.threads()
    out = {"kind": "oracle wall time per workload", "threads": nthreads, "nproc": os.cpu_count(), "workloads": {}}

    def svdq_time(name, threads=None):
        c = synth.CONFIGS[name]
        d = synth.config_layer(name)
        w = oracle.pack_weight(c["prec"], d["W"], d["lam"], d["L1"], d["L2"])
        if threads:
            oracle.set_threads(threads)
        t0 = time.perf_counter()
        a = oracle.quantize_act(c["prec"], d["x"], w["inv_lam"], 1.0, d["L1"])
        oracle.linear(c["prec"], a, w, 1.0, d["L2"], d["b"])
        dt = time.perf_counter() - t0
        oracle.set_threads(nthreads)
        return dt, 2.0 * c["M"] * c["N"] * c["K"]

    for name in ("c1_smoke_nvfp4", "c3_qkv_nvfp4", "c4_mlp_up_nvfp4", "c4_mlp_down_nvfp4", "c5_qkv_int4"):
        dt, fl = svdq_time(name)
        e = {"seconds": round(dt, 3), "tflops": round(fl / dt / 1e12, 6), "threads": nthreads}
        if name == "c1_smoke_nvfp4":
            dt1, _ = svdq_time(name, threads=1)
            e["seconds_1_thread"] = round(dt1, 3)
        out["workloads"][name] = e
    c = synth.CONFIGS["c2_awq_gemv"]
    for m in c["Ms"]:
        d = synth.awq_inputs(c["seed"], m, c["K"], c["N"])
        pk = oracle.awq_pack_weight(d["W"])
        t0 = time.perf_counter()
        oracle.awq_linear(d["x"], pk)
        dt = time.perf_counter() - t0
        oracle.set_threads(1)
        t0 = time.perf_counter()
        oracle.awq_linear(d["x"], pk)
        dt1 = time.perf_counter() - t0
        oracle.set_threads(nthreads)
        out["workloads"][f"c2_awq_gemv_m{m}"] = {"seconds": round(dt, 4), "seconds_1_thread": round(dt1, 4),
                                                 "threads": nthreads}
    print(json.dumps(out), flush=True)


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle

    c = synth.CONFIGS[WORKLOAD]
    M, K, N, r = c["M"], c["K"], c["N"], c["r"]
    d = synth.config_layer(WORKLOAD)
    w = oracle.pack_weight("nvfp4", d["W"], d["lam"], d["L1"], d["L2"])
    rows = args.ref_rows
    times = []
    for i in range(args.warmup + args.steps):
        lo = (i * rows) % M
        x = d["x"][lo:lo + rows]
        t0 = time.perf_counter()
        a = oracle.quantize_act("nvfp4", x, w["inv_lam"], 1.0, d["L1"])
        oracle.linear("nvfp4", a, w, 1.0, d["L2"], d["b"])
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    s = statistics.median(times)
    value = 2.0 * rows * N * K / s / 1e12
    sample = f"{rows} rows per step of the M{M} K{K} N{N} r{r} workload (CPU oracle, float64 accumulation)"
    out = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOPS",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(s * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"svdq_w4a4 nvfp4 fused-QKV projection M{M} K{K} N{N} r{r}", "M": M, "K": K,
                   "N": N, "r": r, "rows_per_step": rows},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOPS", "cores": oracle.threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--cpu-rows", type=int, default=4608)
    ap.add_argument("--ref-rows", type=int, default=128)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-awq", action="store_true")
    ap.add_argument("--no-int4", action="store_true")
    ap.add_argument("--no-probe", action="store_true")
    ap.add_argument("--no-qkv", action="store_true")
    ap.add_argument("--no-mlp", action="store_true")
    ap.add_argument("--oracle-configs", action="store_true",
                    help="only time the CPU oracle on every workload (no GPU needed) and exit")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.oracle_configs:
        oracle_configs()
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_cuda(args)


if __name__ == "__main__":
    main()
