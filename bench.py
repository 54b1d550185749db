"""Benchmark: exact tiled attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-extra] [--no-cpu]

A step is one pass of the hot path over the headline workload, the largest single-GPU configuration of the
method: prefill MHA with B=8, H=32, N=4096, d=128, causal (bf16 Q/K/V iid N(0,1), bf16 O + fp32 lse;
the ops-transformer page's measured shape, batch 8, seq 4096, head_dim 128).  `value` is TFLOP/s with the
4 n^2 d convention, halved for causal, over the whole job; the inputs (805 MiB) are larger than L2, and a
256 MiB write also flushes L2 before every timed step, outside the timed events.  The same JSON line
carries the roofline of the prefill kernel (per-launch CUDA events), an end-to-end number through the
public API with host buffers, the oracle timed on the host cores (sampled, extrapolated by the FLOP ratio,
plus the tiny configuration on one core and the other workloads' oracle rates), the SM clocks seen during
timing, and (unless --no-extra) the other workloads of the method, each with the clocks seen while it ran:
prefill d=64 (B=1, non-causal + causal), the d=128 N sweep, HSTU over jagged and dense sequences, head dims
96 and 256, e4m3 inputs, and the decode steps over a contiguous and a paged cache (GB/s).

--impl reference times the fp64 CPU oracle (the only reference implementation this method has) on the
same workload and metric, each step a bounded sample of it.
Multi-GPU: one process per GPU (torchrun); every rank runs the same workload on its own GPU (weak
scaling, no data-path collective); time = max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

HEADLINE = dict(B=8, H=32, N=4096, d=128, causal=True)
HBM_SPEC_GBS = 8000.0  # B200 HBM3e nominal (DGX figure), the denominator the decode target is stated against
METRIC = "attn fwd TFLOP/s (4n²d) & % of B200 BF16 peak; decode HBM GB/s"
L2_FLUSH_BYTES = 256 << 20


# ------------------------------------------------------------------------------------------------ utils
def attn_flops(B, H, N, d, causal):
    f = 4.0 * B * H * N * N * d
    return f / 2 if causal else f


def hstu_flops(lengths, H, d):
    return sum(2.0 * H * int(L) * int(L) * d for L in lengths)


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def kernel_source_hash():
    """Hash of the prefill kernel's code (ptx.cuh, prefill.cuh, decode.cuh) with comments and blank lines
    left out, so that an edit of comments alone keeps recorded profiler counters valid."""
    h = hashlib.sha256()
    for f in ("ptx.cuh", "prefill.cuh", "decode.cuh"):
        with open(os.path.join(ROOT, "exact_tiled_attention_43_b200", "csrc", f)) as fh:
            for line in fh:
                code = re.sub(r"/\*.*?\*/", "", line).split("//", 1)[0].rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def recorded_traffic(kernel_tag):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    want = kernel_source_hash()
    for line in open(path):
        parts = line.split()
        if len(parts) >= 3 and parts[0] == kernel_tag and parts[1] == want:
            return float(parts[2])
    return None


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    BAD = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40, "sw_power_cap": 0x4,
           "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                r = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.BAD.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def timed_steps(step_fn, steps, warmup, flush_buf, stream, dist_ctx):
    """W untimed warm-up steps; then K steps, each preceded by an L2 flush outside its CUDA events.
    Returns (total ms of the K steps on the device, per-step ms list)."""
    for _ in range(warmup):
        step_fn()
    torch.cuda.synchronize()
    dist_ctx.barrier()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    with torch.cuda.stream(stream):
        for a, b in evs:
            flush_buf.fill_(1)
            a.record(stream)
            step_fn()
            b.record(stream)
    torch.cuda.synchronize()
    dist_ctx.barrier()
    torch.cuda.synchronize()
    per = [a.elapsed_time(b) for a, b in evs]
    return sum(per), per


class DistCtx:
    """One process per GPU: rank/world from the torchrun environment; the process group is used only for
    barriers and the max-over-ranks of the device time (no data-path collective: every rank runs the whole
    workload on its own GPU).  `backend="gloo"` runs the same logic on CPU (tests)."""

    def __init__(self, backend="nccl"):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.on = self.world > 1
        self.device = "cuda" if backend == "nccl" else "cpu"
        if self.on:
            import datetime

            import torch.distributed as dist

            if backend == "nccl":
                torch.cuda.set_device(self.local)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.dist = dist

    def barrier(self):
        if self.on:
            self.dist.barrier()

    def max(self, x: float) -> float:
        if not self.on:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.on:
            self.dist.barrier()
            self.dist.destroy_process_group()


def job_throughput(units_per_step: float, steps: int, world: int, t_max_ms: float) -> float:
    """Whole-job throughput: the units all ranks processed divided by the slowest rank's device time."""
    return units_per_step * steps * world / (t_max_ms * 1e-3)


# ------------------------------------------------------------------------------------------------ CPU
def cpu_oracle_sample(budget_s=12.0):
    """Times the fp64 oracle (as it stands) on the host cores.  Headline: whole (batch, head) units of the
    headline workload, as many as fit in about `budget_s` seconds; the rate (TFLOP/s, 4 n^2 d halved for
    causal -- the oracle does exactly the causal half) is the line's value and the whole-workload time is
    extrapolated from it by the FLOP ratio.  Also: the tiny configuration (B1 H2 N256 d64, both modes) on
    all cores and on one core, the prefill d=64 workload on one unit, the HSTU jagged workload in full, and
    the decode step on two sequences of its length distribution (GB/s of K/V bytes)."""
    import oracle
    from exact_tiled_attention_43_b200 import inputs

    oracle.build()
    out = {"kind": "oracle", "cores": oracle.num_threads()}
    B, H, N, d = HEADLINE["B"], HEADLINE["H"], HEADLINE["N"], HEADLINE["d"]
    q, k, v = inputs.dense_qkv(inputs.PREFILL_D128, B, H, N, d)
    qf, kf, vf = (t.reshape(B * H, 1, N, d) for t in (q, k, v))
    scale = float(torch.tensor(1.0 / math.sqrt(d), dtype=torch.float32))
    t0 = time.perf_counter()
    oracle.attn(qf[:1], kf[:1], vf[:1], scale, True)
    t1 = time.perf_counter() - t0
    nu = int(max(1, min(B * H - 1, budget_s // max(t1, 1e-3))))
    t0 = time.perf_counter()
    oracle.attn(qf[1:1 + nu], kf[1:1 + nu], vf[1:1 + nu], scale, True)
    el = time.perf_counter() - t0
    rate = attn_flops(1, nu, N, d, True) / el
    full_s = attn_flops(B, H, N, d, True) / rate
    out.update({"value": rate / 1e12, "unit": "TFLOP/s", "seconds": el,
                "sample": f"{nu} of {B * H} (batch, head) units of B={B} H={H} N={N} d={d} causal, full rows, "
                          f"{el:.1f} s; the whole workload would take {full_s:.1f} s (extrapolated by the FLOP "
                          f"ratio)",
                "extrapolated_full_workload_s": full_s})
    del q, k, v, qf, kf, vf
    # tiny configuration, both modes, on all cores and on one core
    q, k, v = inputs.dense_qkv(inputs.TINY, 1, 2, 256, 64)
    sc = float(torch.tensor(0.125, dtype=torch.float32))
    tiny = {}
    for label, nthreads in (("all_cores", 0), ("one_core", 1)):
        oracle.set_num_threads(nthreads if nthreads else out["cores"])
        t0 = time.perf_counter()
        reps = 5
        for _ in range(reps):
            for causal in (False, True):
                oracle.attn(q, k, v, sc, causal)
        tiny[label + "_s"] = (time.perf_counter() - t0) / reps
    oracle.set_num_threads(out["cores"])
    tiny["tflops_one_core"] = (attn_flops(1, 2, 256, 64, False) + attn_flops(1, 2, 256, 64, True)) / \
        tiny["one_core_s"] / 1e12
    out["tiny_B1_H2_N256_d64"] = tiny
    # prefill d=64 (B1 H32 N4096): one unit, both modes
    q, k, v = inputs.dense_qkv(inputs.PREFILL_D64, 1, 32, 4096, 64)
    t0 = time.perf_counter()
    for causal in (False, True):
        oracle.attn(q[:, :1], k[:, :1], v[:, :1], sc, causal)
    el = time.perf_counter() - t0
    out["prefill_B1_H32_N4096_d64"] = {
        "value": (attn_flops(1, 1, 4096, 64, False) + attn_flops(1, 1, 4096, 64, True)) / el / 1e12,
        "unit": "TFLOP/s", "sample": "1 of 32 heads, non-causal + causal, full rows"}
    # HSTU jagged (16 sequences, H=4, d=64, lengths U[256, 4096]) in full
    lens = inputs.uniform_lengths(inputs.HSTU_JAGGED, 16, 256, 4096)
    cu = inputs.cu_seqlens(lens)
    q, k, v = inputs.jagged_qkv(inputs.HSTU_JAGGED, int(lens.sum()), 4, 64, std=0.5)
    t0 = time.perf_counter()
    oracle.hstu_jagged(q, k, v, cu, 0.125, 1.0 / 4096)
    el = time.perf_counter() - t0
    out["hstu_jagged_S16_H4_d64"] = {"value": hstu_flops(lens.tolist(), 4, 64) / el / 1e12, "unit": "TFLOP/s",
                                     "sample": "the whole workload"}
    # decode: two sequences (the workload's first two lengths), all 32 heads, d=128
    dl = inputs.uniform_lengths(inputs.DECODE, 64, 8192, 32768)[:2]
    qd, kc, vc, kl = inputs.decode_inputs(inputs.DECODE, 2, 32, int(dl.max()), 128, dl)
    t0 = time.perf_counter()
    oracle.decode(qd, kc, vc, kl, float(torch.tensor(1.0 / math.sqrt(128), dtype=torch.float32)))
    el = time.perf_counter() - t0
    out["decode_B64_H32_d128_L8k-32k"] = {"value": 2.0 * 32 * 128 * 2 * float(dl.sum()) / el / 1e9, "unit": "GB/s",
                                          "sample": f"2 of 64 sequences (lengths {dl.tolist()}), all heads"}
    return out


def run_reference(args):
    """The reference arm: the fp64 oracle on the host cores, same workload and metric."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from exact_tiled_attention_43_b200 import inputs

    oracle.build()
    B, H, N, d = HEADLINE["B"], HEADLINE["H"], HEADLINE["N"], HEADLINE["d"]
    q, k, v = inputs.dense_qkv(inputs.PREFILL_D128, B, H, N, d)
    scale = float(torch.tensor(1.0 / math.sqrt(d), dtype=torch.float32))
    # each step: four (batch, head) units of one batch index, causal, every 8th query row (a bounded CPU time
    # per step, ~0.1 s, large enough for the oracle's threads to share); the batch index rotates so that
    # successive steps read different data
    rows = list(range(0, N, 8))
    per_unit = sum(4.0 * (r + 1) * d for r in rows)
    step_units = 4
    step_flops = per_unit * step_units

    def step(i):
        b = i % B
        hs = slice((i * step_units) % H, (i * step_units) % H + step_units)
        oracle.attn(q[b:b + 1, hs], k[b:b + 1, hs], v[b:b + 1, hs], scale, True, rows=rows)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    el = time.perf_counter() - t0
    val = step_flops * args.steps / el / 1e12
    cores = oracle.num_threads()
    sample = (f"per step: {step_units} of {B * H} (batch, head) units, every 8th query row ({len(rows)} rows "
              f"each), causal, N={N}, d={d}")
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": _config(),
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _config():
    return {"workload": "prefill MHA B=8 H=32 N=4096 d=128 causal, bf16 Q/K/V iid N(0,1), one forward per step",
            "B": 8, "H": 32, "N": 4096, "d": 128, "causal": True, "o_dtype": "bf16", "lse": "fp32",
            "scale": "1/sqrt(d)",
            "l2": "inputs (805 MiB of Q/K/V) larger than L2; a 256 MiB write also flushes L2 before every timed "
                  "step, outside the events",
            "parallelism": "replicas: each rank runs the whole workload on its own GPU"}


# ------------------------------------------------------------------------------------------------ GPU
def run_ours(args):
    import exact_tiled_attention_43_b200 as eta
    from exact_tiled_attention_43_b200 import inputs

    ctx = DistCtx("nccl")
    dev = torch.device("cuda", ctx.local)
    torch.cuda.set_device(dev)
    eta.lib()
    peaks = load_peaks()
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    B, H, N, d, causal = HEADLINE["B"], HEADLINE["H"], HEADLINE["N"], HEADLINE["d"], HEADLINE["causal"]
    q, k, v = inputs.dense_qkv(inputs.PREFILL_D128, B, H, N, d, device=dev)
    scale = eta.default_scale(d)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    step_flops = attn_flops(B, H, N, d, causal)

    def step():
        eta.attn_fwd(q, k, v, causal=causal, scale=scale, out=o, lse=lse)

    with ClockSampler(ctx.local) as clk:
        total_ms, per = timed_steps(step, args.steps, args.warmup, flush, stream, ctx)
    clocks = clk.summary()
    assert eta.status() == 0

    t_max = ctx.max(total_ms)
    value = job_throughput(step_flops, args.steps, ctx.world, t_max) / 1e12
    # A step is one launch of the prefill kernel, timed by its own pair of CUDA events on the launching
    # stream: the per-launch duration of the roofline is the mean of those.
    launch_ms = statistics.mean(per)
    achieved = step_flops / (launch_ms * 1e-3) / 1e12
    traffic = recorded_traffic("prefill_d128_b8")

    # ---- end to end through the public API with pinned host buffers.  Every step copies its own Q, K, V in
    # and its O and lse out.  Steps are pipelined the way a caller streaming batches would run them: the
    # copy-in of step i+1 and the copy-out of step i-1 (each on its own stream) run while step i computes,
    # with two sets of device buffers.  The L2 flush stays in front of every compute.
    h_in = [tuple(t.cpu().pin_memory() for t in (q, k, v)) for _ in range(2)]
    h_out = [tuple(torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (o, lse)) for _ in range(2)]
    d_in = [tuple(torch.empty_like(t) for t in (q, k, v)) for _ in range(2)]
    d_out = [tuple(torch.empty_like(t) for t in (o, lse)) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = {name: [torch.cuda.Event() for _ in range(2)] for name in ("in", "comp", "out")}

    def e2e_run(nsteps):
        for i in range(nsteps):
            b = i % 2
            if i >= 2:
                s_in.wait_event(ev["comp"][b])  # step i-2 has finished reading this input set
            with torch.cuda.stream(s_in):
                for dst, src in zip(d_in[b], h_in[b]):
                    dst.copy_(src, non_blocking=True)
                ev["in"][b].record(s_in)
            stream.wait_event(ev["in"][b])
            if i >= 2:
                stream.wait_event(ev["out"][b])  # the copy-out of step i-2 has read this output set
            with torch.cuda.stream(stream):
                flush.fill_(1)
                qd, kd, vd = d_in[b]
                od, ld = d_out[b]
                eta.attn_fwd(qd, kd, vd, causal=causal, scale=scale, out=od, lse=ld)
                ev["comp"][b].record(stream)
            s_out.wait_event(ev["comp"][b])
            with torch.cuda.stream(s_out):
                for dst, src in zip(h_out[b], d_out[b]):
                    dst.copy_(src, non_blocking=True)
                ev["out"][b].record(s_out)

    e2e_steps = max(3, min(args.steps, 20))
    e2e_run(args.warmup)
    torch.cuda.synchronize()
    ctx.barrier()
    torch.cuda.synchronize()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    s_in.wait_event(e_start)
    s_out.wait_event(e_start)
    e2e_run(e2e_steps)
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)
    e_end.record(stream)
    torch.cuda.synchronize()
    ctx.barrier()
    torch.cuda.synchronize()
    e2e_ms = ctx.max(e_start.elapsed_time(e_end))
    h2d = 3 * q.numel() * 2
    d2h = o.numel() * 2 + lse.numel() * 4
    # the last step's results are the device's: check the copy-out carried them
    b_last = (e2e_steps - 1) % 2
    assert torch.equal(h_out[b_last][1], d_out[b_last][1].cpu()), "e2e copy-out mismatch"
    assert eta.status() == 0
    del h_in, h_out, d_in, d_out
    torch.cuda.empty_cache()

    extra = {} if args.no_extra else run_extras(args, eta, inputs, dev, flush, stream, ctx, peaks)

    line = None
    if ctx.rank == 0:
        cpu = None
        if ctx.world == 1 and not args.no_cpu:
            cpu = cpu_oracle_sample()
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ctx.world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t_max / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (iid N(0,1) bf16, fixed seeds)",
            "config": _config(),
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": achieved / peaks["bf16_tflops"], "traffic": traffic,
                         "kernel": "prefill_kernel<128, dense>",
                         "peak_source": f"{peaks['source']} bf16 burst (MEASURED_PEAKS.json)",
                         "launch_ms": launch_ms,
                         "algorithmic_bytes": 4.0 * B * H * N * d * 2 + 4.0 * B * H * N},
            "cpu_baseline": cpu,
            "e2e": {"value": step_flops * e2e_steps * ctx.world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "overlap": "copy-in of step i+1 and copy-out of step i-1 on their own streams during step i"},
            "gpu_launches": args.steps,
            "clocks": clocks,
            "extra": extra,
        }
        print(json.dumps(line), flush=True)
    ctx.close()
    return line


def run_extras(args, eta, inputs, dev, flush, stream, ctx, peaks):
    """The method's other workloads, each timed the same way (few steps)."""
    out = {}
    K, W = max(3, min(args.steps, 20)), max(3, args.warmup)
    pk = peaks["bf16_tflops"]

    def timed(fn):
        # An idle half second first, so that a case does not inherit the power-capped clocks of the
        # previous (possibly seconds-long) one.  Short cases run more steps (about 25 ms of timed work,
        # the same count on every rank) so that the clock sampler sees them, while the long ones stay in
        # the burst regime that the measured peak describes; the clocks are reported with each case.
        # Returns the device time scaled to K steps (the callers divide by K).
        torch.cuda.synchronize()
        time.sleep(0.5)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            fn()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        est = ctx.max(a.elapsed_time(b))
        k = int(min(2000, max(K, math.ceil(25.0 / max(est, 1e-3)))))
        with ClockSampler(ctx.local) as clk:
            ms, _ = timed_steps(fn, k, W, flush, stream, ctx)
        return ms / k * K, clk.summary()

    # the headline workload launched back to back (no flush between launches, ~50 ms of continuous tensor
    # work): the rate a caller sees in a long loop, against the sustained bf16 peak, with the clocks it ran at
    q, k, v = inputs.dense_qkv(inputs.PREFILL_D128, 8, 32, 4096, 128, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    f = attn_flops(8, 32, 4096, 128, True)
    nb = 50
    for _ in range(W):
        eta.attn_fwd(q, k, v, causal=True, out=o, lse=lse)
    torch.cuda.synchronize()
    time.sleep(0.5)
    ctx.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(ctx.local) as clk:
        a.record(stream)
        for _ in range(nb):
            eta.attn_fwd(q, k, v, causal=True, out=o, lse=lse)
        b.record(stream)
        torch.cuda.synchronize()
    bb_ms = ctx.max(a.elapsed_time(b)) / nb
    tf = f / (bb_ms * 1e-3) / 1e12
    out["prefill_B8_H32_N4096_d128_causal_back_to_back"] = {
        "clocks": clk.summary(), "value": tf, "unit": "TFLOP/s", "ms_per_launch": bb_ms, "launches": nb,
        "frac_of_sustained_peak": tf / peaks["bf16_tflops_sustained"], "frac_of_peak": tf / pk}
    del q, k, v, o, lse

    # prefill d=64, B=1, H=32, N=4096 (the ai6s.net page's call example): one non-causal and one causal
    # forward per step; inputs fit in L2, which the flush clears before every step
    q, k, v = inputs.dense_qkv(inputs.PREFILL_D64, 1, 32, 4096, 64, device=dev)
    o_nc, o_c = torch.empty_like(q), torch.empty_like(q)
    l_nc = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    l_c = torch.empty_like(l_nc)

    def c2_step():
        eta.attn_fwd(q, k, v, causal=False, out=o_nc, lse=l_nc)
        eta.attn_fwd(q, k, v, causal=True, out=o_c, lse=l_c)

    ms, ck = timed(c2_step)
    f = attn_flops(1, 32, 4096, 64, False) + attn_flops(1, 32, 4096, 64, True)
    tf = f * K / (ctx.max(ms) * 1e-3) / 1e12
    # per-launch durations of the two launches (events on the launching stream)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    lm = []
    for _ in range(20):
        flush.fill_(1)
        ev[0].record(stream)
        eta.attn_fwd(q, k, v, causal=False, out=o_nc, lse=l_nc)
        ev[1].record(stream)
        eta.attn_fwd(q, k, v, causal=True, out=o_c, lse=l_c)
        ev[2].record(stream)
        torch.cuda.synchronize()
        lm.append((ev[0].elapsed_time(ev[1]), ev[1].elapsed_time(ev[2])))
    nc_ms, c_ms = statistics.mean(a for a, _ in lm), statistics.mean(b for _, b in lm)
    out["prefill_B1_H32_N4096_d64_noncausal+causal"] = {
        "clocks": ck, "value": tf, "unit": "TFLOP/s", "ms_per_step": ms / K, "frac_of_peak": tf / pk,
        "launch_ms": {"noncausal": nc_ms, "causal": c_ms},
        "launch_frac_of_peak": f / ((nc_ms + c_ms) * 1e-3) / 1e12 / pk,
        "traffic": recorded_traffic("prefill_d64")}
    del q, k, v, o_nc, o_c, l_nc, l_c
    for N in (1024, 8192, 32768):
        q, k, v = inputs.dense_qkv(inputs.PREFILL_D128, 1, 32, N, 128, device=dev)
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
        ms, ck = timed(lambda: eta.attn_fwd(q, k, v, causal=True, out=o, lse=lse))
        tf = attn_flops(1, 32, N, 128, True) * K / (ctx.max(ms) * 1e-3) / 1e12
        out[f"prefill_B1_H32_N{N}_d128_causal"] = {"clocks": ck, "value": tf, "unit": "TFLOP/s", "ms_per_step": ms / K,
                                                   "frac_of_peak": tf / pk}
        del q, k, v, o, lse

    # HSTU jagged: 16 sequences, H=4, d=64, lengths U[256, 4096]
    lens = inputs.uniform_lengths(inputs.HSTU_JAGGED, 16, 256, 4096)
    cu = inputs.cu_seqlens(lens).to(dev)
    T = int(lens.sum())
    q, k, v = inputs.jagged_qkv(inputs.HSTU_JAGGED, T, 4, 64, std=0.5, device=dev)
    o = torch.empty_like(q)
    ms, ck = timed(lambda: eta.hstu_fwd_jagged(q, k, v, cu, 4096, 0.125, 1.0 / 4096, out=o))
    tf = hstu_flops(lens.tolist(), 4, 64) * K / (ctx.max(ms) * 1e-3) / 1e12
    out["hstu_jagged_S16_H4_d64"] = {"clocks": ck, "value": tf, "unit": "TFLOP/s", "ms_per_step": ms / K, "frac_of_peak": tf / pk,
                                     "T": T}
    del q, k, v, o

    # HSTU at the HSTU page's own shape (QKV = 16, 4, 4096, 64: every sequence 4096 long) and at N = 8192
    for S_, N_ in ((16, 4096), (16, 8192)):
        lens = torch.full((S_,), N_, dtype=torch.int32)
        cu = inputs.cu_seqlens(lens).to(dev)
        q, k, v = inputs.jagged_qkv(inputs.HSTU_JAGGED, S_ * N_, 4, 64, std=0.5, device=dev)
        o = torch.empty_like(q)
        ms, ck = timed(lambda: eta.hstu_fwd_jagged(q, k, v, cu, N_, 0.125, 1.0 / N_, out=o))
        tf = hstu_flops(lens.tolist(), 4, 64) * K / (ctx.max(ms) * 1e-3) / 1e12
        out[f"hstu_dense_S{S_}_H4_N{N_}_d64"] = {"clocks": ck, "value": tf, "unit": "TFLOP/s", "ms_per_step": ms / K,
                                                  "frac_of_peak": tf / pk}
        del q, k, v, o

    # head dim 96 (rows of 192 B: one and a half swizzle chunks), the d=128 line's shape B8 H32 N4096 causal
    B_, H_, N_ = 8, 32, 4096
    q, k, v = inputs.dense_qkv(inputs.PREFILL_D128, B_, H_, N_, 96, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((B_, H_, N_), dtype=torch.float32, device=dev)
    ms, ck = timed(lambda: eta.attn_fwd(q, k, v, causal=True, out=o, lse=lse))
    tf = 2.0 * B_ * H_ * N_ * N_ * 96 * K / (ctx.max(ms) * 1e-3) / 1e12
    out["prefill_B8_H32_N4096_d96_causal"] = {"clocks": ck, "value": tf, "unit": "TFLOP/s", "ms_per_step": ms / K,
                                              "frac_of_peak": tf / pk}
    del q, k, v, o, lse

    # head dim 256 (the FlashAttention-2 head size), B4 H16 N4096 causal: the same H*d as the d=128 line
    B_, H_, N_ = 4, 16, 4096
    q, k, v = inputs.dense_qkv(inputs.PREFILL_D128, B_, H_, N_, 256, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((B_, H_, N_), dtype=torch.float32, device=dev)
    ms, ck = timed(lambda: eta.attn_fwd(q, k, v, causal=True, out=o, lse=lse))
    tf = 2.0 * B_ * H_ * N_ * N_ * 256 * K / (ctx.max(ms) * 1e-3) / 1e12
    out["prefill_B4_H16_N4096_d256_causal"] = {"clocks": ck, "value": tf, "unit": "TFLOP/s", "ms_per_step": ms / K,
                                               "frac_of_peak": tf / pk}
    del q, k, v, o, lse

    # e4m3 inputs with per-tensor descales, B8 H32 N4096 d128 causal (the d=128 line's shape); the fraction is
    # of the e4m3 tensor peak, taken as twice the measured bf16 figure (the nominal dense ratio)
    q8, k8, v8, (dq, dk, dv) = inputs.fp8_dense_qkv(inputs.PREFILL_FP8, 8, 32, 4096, 128, device=dev)
    o = torch.empty((8, 32, 4096, 128), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((8, 32, 4096), dtype=torch.float32, device=dev)
    ms, ck = timed(lambda: eta.attn_fwd_fp8(q8, k8, v8, dq, dk, dv, causal=True, out=o, lse=lse))
    tf = 2.0 * 8 * 32 * 4096 * 4096 * 128 * K / (ctx.max(ms) * 1e-3) / 1e12
    out["prefill_fp8_B8_H32_N4096_d128_causal"] = {"clocks": ck, "value": tf, "unit": "TFLOP/s", "ms_per_step": ms / K,
                                                   "frac_of_peak": tf / (2.0 * pk),
                                                   "peak_note": "e4m3 peak = 2 x measured bf16"}
    del q8, k8, v8, o, lse

    # decode: batch 64, H=32, d=128, lengths U[8192, 32768] (inputs far larger than L2: no flush needed)
    B, H, d, Lmax = 64, 32, 128, 32768
    lens = inputs.uniform_lengths(inputs.DECODE, B, 8192, 32768)
    q, kc, vc, kl = inputs.decode_inputs(inputs.DECODE, B, H, Lmax, d, lens, device=dev)
    kl = kl.to(dev)
    ws = torch.empty(eta.attn_decode_workspace_size(B, H, Lmax, d), dtype=torch.uint8, device=dev)
    od = torch.empty((B, H, d), dtype=torch.bfloat16, device=dev)
    ld = torch.empty((B, H), dtype=torch.float32, device=dev)
    ms, ck = timed(lambda: eta.attn_decode(q, kc, vc, kl, workspace=ws, out=od, lse=ld))
    nbytes = 2.0 * H * d * 2 * float(lens.sum()) + q.numel() * 2 + od.numel() * 2 + ld.numel() * 4
    gbs = nbytes * K / (ctx.max(ms) * 1e-3) / 1e9
    out["decode_B64_H32_d128_L8k-32k"] = {"clocks": ck, "value": gbs, "unit": "GB/s", "ms_per_step": ms / K,
                                          "frac_of_peak": gbs / peaks["hbm_gbs"],
                                          "frac_of_spec": gbs / HBM_SPEC_GBS, "bytes_per_step": nbytes}
    del q, kc, vc, ws
    torch.cuda.empty_cache()

    # decode over a paged cache with grouped query heads: batch 64, Hq=32 query heads sharing Hkv=8 kv heads,
    # d=128, 64-row pages in a shuffled pool, lengths U[8192, 32768]
    B, Hq, Hkv, d, ps = 64, 32, 8, 128, 64
    lens = inputs.uniform_lengths(inputs.DECODE_PAGED, B, 8192, 32768)
    q, kp, vp, table, kl = inputs.paged_decode_inputs(inputs.DECODE_PAGED, B, Hq, Hkv, d, ps, lens, spare_pages=0,
                                                      device=dev)
    table, kl = table.to(dev), kl.to(dev)
    ws = torch.empty(eta.attn_decode_paged_workspace_size(B, Hq, table.shape[1], ps, d), dtype=torch.uint8,
                     device=dev)
    od = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=dev)
    ld = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    ms, ck = timed(lambda: eta.attn_decode_paged(q, kp, vp, table, kl, workspace=ws, out=od, lse=ld))
    nbytes = (2.0 * Hkv * d * 2 * float(lens.sum()) + q.numel() * 2 + od.numel() * 2 + ld.numel() * 4 +
              table.numel() * 4)
    gbs = nbytes * K / (ctx.max(ms) * 1e-3) / 1e9
    out["decode_paged_gqa_B64_Hq32_Hkv8_d128_page64_L8k-32k"] = {"clocks": ck,
        "value": gbs, "unit": "GB/s", "ms_per_step": ms / K, "frac_of_peak": gbs / peaks["hbm_gbs"],
        "frac_of_spec": gbs / HBM_SPEC_GBS, "bytes_per_step": nbytes}
    del q, kp, vp, ws
    torch.cuda.empty_cache()
    assert eta.status() == 0
    return out


CASES = {
    # name: (kind, shape) -- small named cases for profiler captures (no JSON line, just launches)
    "prefill_d128_b8": ("dense_causal", dict(B=8, H=32, N=4096, d=128)),
    "prefill_d64_b1": ("dense", dict(B=1, H=32, N=4096, d=64)),
    "prefill_d64_b4": ("dense", dict(B=4, H=32, N=4096, d=64)),
    "prefill_d128_b2": ("dense", dict(B=2, H=32, N=4096, d=128)),
    "prefill_d96_b2": ("dense", dict(B=2, H=32, N=4096, d=96)),
    "prefill_d256_b2": ("dense", dict(B=2, H=16, N=4096, d=256)),
    "prefill_fp8_b2": ("fp8", dict(B=2, H=32, N=4096, d=128)),
    "hstu_jagged": ("hstu", dict(S=16, H=4, d=64)),
    "decode_b2": ("decode", dict(B=2, H=32, d=128, Lmax=32768)),
    "decode_paged_b4": ("decode_paged", dict(B=4, Hq=32, Hkv=8, d=128, ps=64)),
}


def run_case(args):
    """Runs one named case `--warmup` + `--steps` times (both causal modes for dense prefill); used as the
    target of ncu captures."""
    import exact_tiled_attention_43_b200 as eta
    from exact_tiled_attention_43_b200 import inputs

    kind, s = CASES[args.case]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if kind in ("dense", "dense_causal"):
        q, k, v = inputs.dense_qkv(inputs.PREFILL_D64 if s["d"] == 64 else inputs.PREFILL_D128, s["B"], s["H"],
                                   s["N"], s["d"], device=dev)
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
        fns = [lambda: eta.attn_fwd(q, k, v, causal=True, out=o, lse=lse)]
        if kind == "dense":
            fns.insert(0, lambda: eta.attn_fwd(q, k, v, causal=False, out=o, lse=lse))
    elif kind == "fp8":
        q8, k8, v8, (dq, dk, dv) = inputs.fp8_dense_qkv(inputs.PREFILL_FP8, s["B"], s["H"], s["N"], s["d"], device=dev)
        fns = [lambda: eta.attn_fwd_fp8(q8, k8, v8, dq, dk, dv, causal=False),
               lambda: eta.attn_fwd_fp8(q8, k8, v8, dq, dk, dv, causal=True)]
    elif kind == "hstu":
        lens = inputs.uniform_lengths(inputs.HSTU_JAGGED, s["S"], 256, 4096)
        cu = inputs.cu_seqlens(lens).to(dev)
        q, k, v = inputs.jagged_qkv(inputs.HSTU_JAGGED, int(lens.sum()), s["H"], s["d"], std=0.5, device=dev)
        fns = [lambda: eta.hstu_fwd_jagged(q, k, v, cu, 4096, 0.125, 1.0 / 4096)]
    elif kind == "decode_paged":
        lens = inputs.uniform_lengths(inputs.DECODE_PAGED, 64, 8192, 32768)[: s["B"]]
        q, kp, vp, table, kl = inputs.paged_decode_inputs(inputs.DECODE_PAGED, s["B"], s["Hq"], s["Hkv"], s["d"],
                                                          s["ps"], lens, spare_pages=0, device=dev)
        table, kl = table.to(dev), kl.to(dev)
        fns = [lambda: eta.attn_decode_paged(q, kp, vp, table, kl)]
    else:
        lens = inputs.uniform_lengths(inputs.DECODE, 64, 8192, 32768)[: s["B"]]
        q, kc, vc, kl = inputs.decode_inputs(inputs.DECODE, s["B"], s["H"], s["Lmax"], s["d"], lens, device=dev)
        kl = kl.to(dev)
        fns = [lambda: eta.attn_decode(q, kc, vc, kl)]
    for _ in range(args.warmup + args.steps):
        for f in fns:
            f()
    torch.cuda.synchronize()
    assert eta.status() == 0
    print(f"case {args.case}: ok", flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extra", action="store_true", help="only the headline workload")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--case", choices=sorted(CASES), help="run one small named case (profiling target)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.case:
        run_case(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
