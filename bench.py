"""Benchmark of the CCA / CCGQA layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl cca|reference]

A step is one prefill forward (down-projection, latent stencil, latent attention,
up-projection) of the whole batch of the workload (default: CCGQA bf16 long prefill,
B=2 x 16384 tokens, E=2048, 16 query / 4 kv heads, C=2), inputs resident in HBM.  The L2
is flushed (256 MiB write) between timed steps, outside each step's CUDA events.  The
single-token decode step over the compressed cache (B=64, 8192 cached tokens) is timed in
the same run and reported under "decode".  One JSON line is printed by rank 0.

With --gpus N > 1 (under torchrun) every rank runs its own replica of the workload (the
path has no exchange step); times are the max over ranks.

--impl reference times the CPU oracle (the plain float64 restatement of the method) on a
bounded sample of the same workload, on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "CCA/CCGQA prefill tokens/s & TFLOP/s (% bf16 peak); decode GB/s (% HBM) on 1 B200"
DEFAULT_WORKLOAD = "ccgqa_prefill_16k"
DECODE_WORKLOAD = "ccgqa_decode_8k"


def prefill_flops(w) -> float:
    """Algorithmic flops of one prefill forward: 2 E (n_q + 2 n_kv) + 2 n_q E per token for
    the projections, 4 d~ per visible (query, key, head) for the causal attention."""
    tokens = w.batch * w.seq
    proj = 2.0 * tokens * w.d_model * (w.n_q + 2 * w.n_kv) + 2.0 * tokens * w.n_q * w.d_model
    return proj + attention_flops(w)


def attention_flops(w) -> float:
    return 2.0 * w.batch * w.n_heads * w.dl * w.seq * (w.seq + 1)


def decode_bytes(w, es=2) -> float:
    """Algorithmic HBM bytes of one decode step: the K/V cache read (L+1 rows, 16-bit), both
    weight matrices, the float32 conv / value-shift state read and written, x read and y
    written."""
    B, ctx = w.batch, w.seq
    cache = 2.0 * B * w.n_kv_heads * (ctx + 1) * w.dl * es
    weights = ((w.n_q + 2 * w.n_kv) * w.d_model + w.d_model * w.n_q) * es
    state = 2.0 * B * ((w.conv_kernel - 1) * (w.n_q + w.n_kv) + (w.n_kv - w.n_kv // 2)) * 4
    io = 2.0 * B * w.d_model * es
    return cache + weights + state + io


# Rated dense bf16 tensor throughput of one B200 (the sparsity-free half of NVIDIA's figure),
# reported beside the measured cuBLAS peak.
RATED_BF16_TFLOPS = 2250.0


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def measured_peak_clock():
    """Median SM clock under load while MEASURED_PEAKS.json's GEMM peak was taken (or None)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        return json.load(open(p)).get("clocks_under_load", {}).get("sm_mhz_median")
    return None


class ClockSampler:
    """nvidia-smi clock / throttle samples while the GPU is busy."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out = ""
        else:
            self.out = ""

    def summary(self):
        rows = []
        for line in self.out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[3:7]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
        loaded = [r for r in rows if r[0] > 0.5 * r[1]] or rows
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": rows[0][1],
                "reasons": reasons, "samples": len(rows)}


def dist_setup(n):
    if n <= 1:
        return 0, 1, 0
    import torch.distributed as dist
    rank = int(os.environ["RANK"])
    world = int(os.environ["WORLD_SIZE"])
    local = int(os.environ.get("LOCAL_RANK", rank))
    torch.cuda.set_device(local)
    from datetime import timedelta
    dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                            device_id=torch.device("cuda", local))
    return rank, world, local


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """The slowest rank's time: every rank contributes, every rank gets the max."""
    if world <= 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, ms: float) -> float:
    """Whole-job rate of weak-scaled replicas: every rank's units over the slowest rank's time."""
    return units_per_rank * world / (ms * 1e-3)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ the CUDA arm
def bench_prefill(cls, w, steps, warmup, world, seed, e2e=True):
    inp = W.make_inputs(w, seed=seed)
    layer = cls.CCALayer.from_workload(w, inp)
    x = inp.x.cuda()
    y = torch.empty_like(x)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    for _ in range(warmup):
        layer.prefill(x, out=y)
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    cls.cca_stage_timing(True)
    for i in range(steps):
        flush.fill_(i & 0xFF)
        starts[i].record()
        layer.prefill(x, out=y)
        ends[i].record()
    torch.cuda.synchronize()
    barrier(world)
    cls.cca_stage_timing(False)
    stage_ms, calls = cls.cca_stage_times(8)
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms = statistics.median(step_ms)
    names = (["weights_to_16bit", "qkv_projection", "latent_stencil", "latent_attention",
              "out_projection"] if len(stage_ms) == 5 else
             ["weights_to_16bit", "qkv_projection_stencil", "latent_attention", "out_projection"])
    stages = {n: t / max(calls, 1) for n, t in zip(names, stage_ms)}
    # kernels per forward: one per timed slot, plus the channel-filter split that shares the
    # first slot with the W_o conversion (layers with convolutions)
    per_step = len(stage_ms) + (0 if w.flags & 16 else 1)

    if not e2e:
        return dict(ms=ms, stages=stages, calls=calls, launches=per_step * steps)

    # end to end through the public API, the way a serving loop overlaps the copies: step i's
    # x goes host -> device on one copy stream, its forward (the whole batch, the launch
    # configuration of the device-timed steps above) runs on the compute stream, and its y goes
    # device -> host on a second copy stream.  With two device buffers each for x and y, step
    # i+1's input copy and step i-1's output copy run under step i's forward (the two copy
    # directions use separate copy engines).  Every step copies all of its x in and all of its
    # y out from / to pinned host memory inside the timed region, which runs from before the
    # first step's input copy to after the last step's output copy: the rate is the steps'
    # tokens over that time (so it includes the pipeline's fill and drain).
    xh = inp.x.pin_memory()
    yh = torch.empty(xh.shape, dtype=xh.dtype).pin_memory()
    xd = [torch.empty_like(x) for _ in range(2)]
    yd = [torch.empty_like(y) for _ in range(2)]
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_run(n):
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record()
        for st in (s_in, s_cmp, s_out):
            st.wait_event(start)
        cmp_done, out_done = [], []
        for i in range(n):
            k = i % 2
            if i >= 2:
                s_in.wait_event(cmp_done[i - 2])     # step i-2's forward has read xd[k]
                s_cmp.wait_event(out_done[i - 2])    # step i-2's y has left yd[k]
            with torch.cuda.stream(s_in):
                xd[k].copy_(xh, non_blocking=True)
            landed = torch.cuda.Event()
            landed.record(s_in)
            s_cmp.wait_event(landed)
            layer.prefill(xd[k], out=yd[k], stream=s_cmp)
            cmp_done.append(torch.cuda.Event())
            cmp_done[-1].record(s_cmp)
            s_out.wait_event(cmp_done[-1])
            with torch.cuda.stream(s_out):
                yh.copy_(yd[k], non_blocking=True)
            out_done.append(torch.cuda.Event())
            out_done[-1].record(s_out)
        for st in (s_in, s_cmp, s_out):
            torch.cuda.current_stream().wait_stream(st)
        end.record()
        torch.cuda.synchronize()
        return start.elapsed_time(end) / n

    e2e_run(3)
    e2e_ms = e2e_run(steps)
    # the last step's y as it reached the host against the device-timed forward of the same x
    # (the forward has no atomics, so equal; a copy racing a buffer's reuse would show here)
    yc = y.float().cpu()
    e2e_err = float((yh.float() - yc).abs().max() / yc.pow(2).mean().sqrt())
    if not e2e_err <= 1e-3:
        raise RuntimeError(f"end-to-end output differs from the device-timed forward ({e2e_err:.3g})")
    nbytes = x.numel() * x.element_size()
    return dict(ms=ms, stages=stages, calls=calls, e2e_ms=e2e_ms, h2d=nbytes, d2h=nbytes,
                launches=per_step * steps)


# Decode steps rotate over this many independent layers (weights and caches), in the order a
# model of that depth issues them: between two uses of a layer, 31 other layers' caches
# (8 GB) and weights (160 MB) pass through L2, so no step finds its own in L2 from its
# previous use, as in a real decode.
DECODE_LAYERS = 32
# The decode step is timed over at least this many steps back to back: the window's first step
# has no earlier kernel to start under (about 24 us of the chain's start are paid once per
# window), so a short window overstates the per-step time a serving loop sees.  200 steps
# are 12 ms of device time.
DECODE_MIN_STEPS = 200


def decode_launches(cls, layer, batch, max_seq):
    """Kernels one decode step launches, as the library reports them for this shape."""
    n = cls.cca_decode_kernel_count(layer.cfg, batch, max_seq)
    if n <= 0:
        raise RuntimeError(cls.cca_last_error_string())
    return n


def bench_decode(cls, w, steps, warmup, seed, layers=DECODE_LAYERS):
    inp = W.make_inputs(w, seed=seed)
    max_seq = w.seq + 2 * steps + warmup + 8
    k0, v0 = inp.k_cache.cuda(), inp.v_cache.cuda()
    stack = []
    for _ in range(layers):
        layer = cls.CCALayer.from_workload(w, inp)
        cache = layer.new_cache(w.batch, max_seq)
        cache.k[:, :, :w.seq] = k0
        cache.v[:, :, :w.seq] = v0
        cache.conv_state.copy_(inp.conv_state.cuda())
        cache.vshift_state.copy_(inp.vshift_state.cuda())
        cache.lengths.copy_(inp.lengths.cuda())
        layer.workspace(cls.cca_decode_workspace_size(layer.cfg, w.batch, max_seq))  # not in a step
        stack.append((layer, cache))
    del k0, v0
    x = inp.x.cuda()
    y = torch.empty_like(x)
    for i in range(warmup):
        layer, cache = stack[i % layers]
        layer.decode(x, cache, out=y)
    torch.cuda.synchronize()
    # The steps run back to back between one pair of events, as a serving loop issues them
    # (each step's first kernel then starts under the previous step's last one).
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record()
    for i in range(steps):
        layer, cache = stack[(warmup + i) % layers]
        layer.decode(x, cache, out=y)
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    # per-kernel breakdown from a separate loop: the stage events between the kernels keep
    # each from starting under the previous one, so these add up to a little more than ms
    cls.cca_stage_timing(True)
    for i in range(min(steps, 10)):
        layer, cache = stack[(warmup + steps + i) % layers]
        layer.decode(x, cache, out=y)
    torch.cuda.synchronize()
    cls.cca_stage_timing(False)
    stage_ms, calls = cls.cca_stage_times(8)
    for layer, cache in stack:
        cls.cca_cache_check(cache.struct)
    nk = decode_launches(cls, stack[0][0], w.batch, max_seq)
    names = {5: ["qkv_projection", "stencil_append", "split_kv_attention", "merge", "out_projection"],
             4: ["qkv_projection", "stencil_append", "attention", "out_projection"],
             3: ["qkv_projection", "stencil_append_attention", "out_projection"]}[nk]
    return dict(ms=ms, stages={n: t / max(calls, 1) for n, t in zip(names, stage_ms)},
                launches=nk * steps, layers=layers, steps=steps)


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_cores() -> int:
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()


# The oracle's sample of a prefill workload: the causal prefix of sequence 0, this many tokens
# (the whole workload when it is smaller).  Both the CUDA arm's cpu_baseline and the reference
# arm time exactly this sample.
CPU_SAMPLE_TOKENS = 4096


def cpu_oracle_sample(w, seed=0, full=False):
    """Times the float64 oracle once on a fixed sample of the workload and returns the rate.

    Prefill: a full forward of the first CPU_SAMPLE_TOKENS tokens of sequence 0 (all B*S
    tokens with full=True); per-token attention cost grows with the prefix, so a prefix sample
    overstates the oracle's full-length rate.  Decode: one decode step of the whole batch."""
    import numpy as np
    import oracle.cca_oracle as O
    from oracle.cca_oracle import OracleConfig, OracleWeights
    inp = W.make_inputs(w, seed=seed)
    cfg = OracleConfig(d_model=w.d_model, n_heads=w.n_heads, n_kv_heads=w.n_kv_heads,
                       compression=w.compression, conv_kernel=w.conv_kernel)
    f64 = lambda t: t.to(torch.float64).numpy()
    ow = OracleWeights.from_arrays(cfg, f64(inp.w_qkv), f64(inp.w_o), f64(inp.conv_seq),
                                   f64(inp.conv_chan))
    base = dict(unit="tokens/s", cores=host_cores(), kind="oracle", cpu=cpu_model())
    if w.decode:
        t0 = time.perf_counter()
        O.decode_batch(cfg, ow, f64(inp.x), f64(inp.k_cache), f64(inp.v_cache),
                       inp.lengths.numpy(), f64(inp.conv_state), f64(inp.vshift_state))
        dt = time.perf_counter() - t0
        return dict(base, value=w.batch / dt, seconds=dt,
                    sample=f"float64 oracle decode step of all {w.batch} sequences of {w.name} "
                           f"({w.seq} cached tokens each; {dt:.2f} s)")
    if full or w.batch * w.seq <= CPU_SAMPLE_TOKENS:
        t0 = time.perf_counter()
        O.prefill(cfg, ow, f64(inp.x))
        dt = time.perf_counter() - t0
        return dict(base, value=w.batch * w.seq / dt, seconds=dt,
                    sample=f"float64 oracle full forward of {w.name} ({w.batch} x {w.seq} "
                           f"tokens; {dt:.2f} s)")
    T = min(CPU_SAMPLE_TOKENS, w.seq)
    x0 = f64(inp.x[0, :T])
    t0 = time.perf_counter()
    O.prefill_sequence(cfg, ow, x0)
    dt = time.perf_counter() - t0
    return dict(base, value=T / dt, seconds=dt,
                sample=f"float64 oracle forward of the first {T} tokens of sequence 0 of "
                       f"{w.name} ({dt:.2f} s; per-token attention cost grows with the prefix, "
                       f"so this overstates the oracle's full-length rate)")


# DRAM bytes (read + write) of one latent-attention launch on a workload, from an ncu
# capture of the current kernel (scaled by tokens from a smaller case of the same shape); a
# workload without one reports null.
ATTN_TRAFFIC = {
    # 25.66 MB read, 0 written on one 8192-token sequence (B=1) of the same shape (the kernel
    # with part of its exponentials on the FMA pipes), x 4 for 2 x 16384 tokens
    "ccgqa_prefill_16k": 4 * 25.658112e6,
}


def workload_from_args(args):
    w = W.WORKLOADS[args.workload]
    over = {k: v for k, v in (("batch", args.batch), ("seq", args.seq)) if v is not None}
    if over:
        w = w.with_(name=w.name + "[" + ",".join(f"{k}={v}" for k, v in over.items()) + "]", **over)
    return w


def run_decode_only(args):
    """Only the decode step (a profiling case for the decode kernels): one JSON line."""
    import compressed_latent_space_b200 as cls
    cls.load()
    hbm, _, _, peak_src = measured_peaks()
    dw = W.WORKLOADS[DECODE_WORKLOAD]
    with ClockSampler(0) as clk:
        dec = bench_decode(cls, dw, args.steps, args.warmup, seed=0, layers=args.decode_layers)
    gbs = decode_bytes(dw) / (dec["ms"] * 1e-3) / 1e9
    line = {"metric": "decode GB/s", "value": gbs, "unit": "GB/s",
            "ms_per_step": dec["ms"], "frac_of_hbm": gbs / hbm, "peak_source": peak_src,
            "tokens_per_s": dw.batch / (dec["ms"] * 1e-3), "bytes_per_step": decode_bytes(dw),
            "workload": dw.name, "stages_ms": dec["stages"], "layers": dec["layers"],
            "gpu_launches": dec["launches"], "clocks": clk.summary()}
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_sample(dw)
    print(json.dumps(line), flush=True)


def result_line(w, world, steps, warmup, pre, ms, e2e_ms, dec, dms, peaks):
    """The JSON line of the CUDA arm from the per-rank results (`pre` / `dec` as the bench
    functions return them) and the step times already maximised over ranks."""
    hbm, bf16_peak, _, peak_src = peaks
    tokens = w.batch * w.seq
    flops = prefill_flops(w)
    attn_ms = pre["stages"].get("latent_attention", float("nan"))
    attn_tflops = attention_flops(w) / (attn_ms * 1e-3) / 1e12
    line = {
        "metric": METRIC,
        "value": job_throughput(tokens, world, ms),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": steps,
        "warmup": warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic (seeded N(0,1) x, N(0,0.02^2) weights)",
        "config": {"workload": w.name, "description": w.description, "batch": w.batch,
                   "seq_len": w.seq, "d_model": w.d_model, "n_heads": w.n_heads,
                   "n_kv_heads": w.n_kv_heads, "compression": w.compression,
                   "latent_head_dim": w.dl, "conv_kernel": w.conv_kernel,
                   "parallelism": f"replicas x{world}",
                   "l2": "flushed between timed steps (256 MiB write outside the step events)"},
        "tflops": flops / (ms * 1e-3) / 1e12,
        "tflops_frac_of_measured_bf16_peak": flops / (ms * 1e-3) / 1e12 / bf16_peak,
        "tflops_frac_of_rated_bf16_peak": flops / (ms * 1e-3) / 1e12 / RATED_BF16_TFLOPS,
        "stages_ms": pre["stages"],
        "roofline": {"kernel": "latent_attention", "bound": "tensor", "achieved": attn_tflops,
                     "peak": bf16_peak, "unit": "TFLOP/s", "frac": attn_tflops / bf16_peak,
                     "traffic": ATTN_TRAFFIC.get(w.name),
                     "peak_source": f"{peak_src} cuBLAS bf16 burst",
                     "frac_of_rated": attn_tflops / RATED_BF16_TFLOPS,
                     "rated_peak": RATED_BF16_TFLOPS},
        "e2e": {"value": job_throughput(tokens, world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": pre["h2d"], "d2h_bytes_per_step": pre["d2h"],
                "ms_per_step": e2e_ms,
                "pipeline": "steps back to back, each the whole batch's forward on a compute "
                            "stream with its x in and y out on two copy streams; step i+1's "
                            "input copy and step i-1's output copy overlap step i's forward"},
        "gpu_launches": pre["launches"] + (dec["launches"] if dec else 0),
    }
    if dec:
        dw = W.WORKLOADS[DECODE_WORKLOAD]
        gbs = decode_bytes(dw) / (dms * 1e-3) / 1e9
        line["decode"] = {"workload": dw.name, "description": dw.description, "ms_per_step": dms,
                          "tokens_per_s": job_throughput(dw.batch, world, dms), "GB/s": gbs,
                          "frac_of_hbm": gbs / hbm, "hbm_peak_GB/s": hbm,
                          "bytes_per_step": decode_bytes(dw), "stages_ms": dec["stages"],
                          "peak_source": peak_src, "steps": dec["steps"],
                          "layers": f"steps rotate over {dec['layers']} independent layers "
                                    "(weights + caches), so none is in L2 from its last use"}
    return line


def backward_flops(w) -> float:
    """Algorithmic flops of one backward pass: twice the forward projections' (the input and
    the weight gradient of each GEMM) and 2.5x the forward attention's (dS and dP, dQ, dK, dV:
    five S x S x d~ products against the forward's two), counted once each."""
    tokens = w.batch * w.seq
    proj = 2.0 * tokens * w.d_model * (w.n_q + 2 * w.n_kv) + 2.0 * tokens * w.n_q * w.d_model
    return 2.0 * proj + 2.5 * attention_flops(w)


def bench_backward(cls, w, steps, warmup, seed):
    """cca_backward on the workload (forward intermediates recomputed inside), median step."""
    inp = W.make_inputs(w, seed=seed)
    layer = cls.CCALayer.from_workload(w, inp)
    x = inp.x.cuda()
    dy = torch.randn(x.shape, generator=torch.Generator("cpu").manual_seed(seed + 1)).to(x.dtype).cuda()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    for _ in range(warmup):
        layer.backward(x, dy)
    torch.cuda.synchronize()
    cls.cca_stage_timing(True)
    times = []
    for i in range(steps):
        flush.fill_(i & 0xFF)
        s0 = torch.cuda.Event(enable_timing=True)
        e0 = torch.cuda.Event(enable_timing=True)
        s0.record()
        layer.backward(x, dy)
        e0.record()
        times.append((s0, e0))
    torch.cuda.synchronize()
    cls.cca_stage_timing(False)
    stage_ms, calls = cls.cca_stage_times(8)
    cls.cca_workspace_status(layer._ws)
    ms = statistics.median(s.elapsed_time(e) for s, e in times)
    names = ["forward_recompute", "dO_and_rowsum", "attention_backward", "stencil_backward",
             "gradient_gemms"]
    return {"workload": w.name, "ms_per_step": ms, "tokens_per_s": w.batch * w.seq / (ms * 1e-3),
            "tflops": backward_flops(w) / (ms * 1e-3) / 1e12,
            "flops_counted": "2x forward projections + 2.5x forward attention (algorithmic)",
            "stages_ms": {n: t / max(calls, 1) for n, t in zip(names, stage_ms)},
            "launches": 19 * steps}


def bench_baselines(cls, steps, warmup, world, seed, ccgqa_ms):
    """The systems the pages compare CCA / CCGQA prefill with at 16k tokens (MHA and GQA-8,
    head width 128, RoPE, same d_model / heads / batch as the CCGQA workload), run on this
    library's own GEMM, pointwise latent kernel and attention kernel, timed like the CCGQA
    step.  The ratios set this B200's numbers beside the pages' H100 ones (1.7x, 1.3x)."""
    out = {}
    for name, w in W.BASELINES.items():
        r = bench_prefill(cls, w, steps, warmup, world, seed, e2e=False)
        out[name] = {"description": w.description, "ms_per_step": r["ms"], "launches": r["launches"],
                     "tokens_per_s": job_throughput(w.batch * w.seq, world, r["ms"]),
                     "tflops": prefill_flops(w) / (r["ms"] * 1e-3) / 1e12,
                     "attention_tflops": attention_flops(w) / (r["stages"]["latent_attention"] * 1e-3) / 1e12,
                     "stages_ms": r["stages"],
                     "ccgqa_speedup": r["ms"] / ccgqa_ms}
    out["pages_h100"] = "CCA/CCGQA prefill 1.7x faster than MHA and 1.3x faster than GQA-8 at 16k (context only)"
    return out


def run_cuda(args):
    rank, world, local = dist_setup(args.gpus)
    import compressed_latent_space_b200 as cls
    cls.load()
    w = workload_from_args(args)
    if w.decode:                      # a decode workload named directly: its own line
        if world > 1:
            raise SystemExit("the decode workload line is a 1-GPU profiling case")
        return run_decode_only(args)
    with ClockSampler(local) as clk:
        pre = bench_prefill(cls, w, args.steps, args.warmup, world, seed=rank)
        dec = None
        if not args.no_decode:
            dw = W.WORKLOADS[DECODE_WORKLOAD]
            dec = bench_decode(cls, dw, max(args.steps, DECODE_MIN_STEPS), args.warmup,
                               seed=rank, layers=args.decode_layers)
        base = None
        if not args.no_baselines and w.name == DEFAULT_WORKLOAD:
            base = bench_baselines(cls, args.steps, args.warmup, world, rank, pre["ms"])
        bwd = None
        if not args.no_backward and w.dtype == "bf16" and not (w.flags & 16):
            bwd = bench_backward(cls, w, max(3, args.steps // 2), args.warmup, rank)
    ms = max_over_ranks(pre["ms"], world)
    e2e_ms = max_over_ranks(pre["e2e_ms"], world)
    dms = max_over_ranks(dec["ms"], world) if dec else None
    line = result_line(w, world, args.steps, args.warmup, pre, ms, e2e_ms, dec, dms,
                       measured_peaks())
    if bwd:
        bwd["ms_per_step"] = max_over_ranks(bwd["ms_per_step"], world)
        line["backward"] = bwd
        line["gpu_launches"] += bwd["launches"]
    if base:
        for name in W.BASELINES:
            base[name]["ms_per_step"] = max_over_ranks(base[name]["ms_per_step"], world)
        line["baselines"] = base
        line["gpu_launches"] += sum(base[name]["launches"] for name in W.BASELINES)
    line["clocks"] = clk.summary()
    peak_clk = measured_peak_clock()
    if peak_clk and line["clocks"].get("sm_mhz"):
        # the measured GEMM peak ran power-capped at a lower SM clock than this run: the
        # fraction at equal clocks scales the achieved rate by peak clock / this run's clock
        r = line["roofline"]
        r["sm_mhz"] = line["clocks"]["sm_mhz"]
        r["peak_sm_mhz"] = peak_clk
        r["frac_at_peak_clock"] = r["frac"] * peak_clk / line["clocks"]["sm_mhz"]
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_sample(w)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------------ the reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = workload_from_args(args)
    for _ in range(args.warmup if not args.cpu_full else 0):
        cpu_oracle_sample(w)
    runs = [cpu_oracle_sample(w, full=args.cpu_full) for _ in range(args.steps if not args.cpu_full else 1)]
    v = statistics.median(r["value"] for r in runs)
    line = {"metric": METRIC, "value": v, "unit": "tokens/s", "impl": "reference",
            "n_gpus": args.gpus, "steps": len(runs), "warmup": args.warmup,
            "ms_per_step": statistics.median(r["seconds"] for r in runs) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": w.name, "description": w.description},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": runs[-1]["cores"],
                             "kind": "oracle", "sample": runs[-1]["sample"],
                             "cpu": runs[-1]["cpu"]},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="cca", choices=["cca", "reference"])
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--decode-layers", type=int, default=DECODE_LAYERS,
                    help="independent layers the decode steps rotate over (fewer for profiling "
                         "captures that must stay small; the timing needs the default)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward-pass timing")
    ap.add_argument("--no-baselines", action="store_true",
                    help="skip the same-box MHA / GQA-8 prefill baselines")
    ap.add_argument("--cpu-full", action="store_true",
                    help="reference arm: one full forward of the whole workload instead of the "
                         "fixed prefix sample (minutes for the large workloads)")
    ap.add_argument("--decode-only", action="store_true",
                    help="time only the decode step (a profiling case for its kernels)")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (smaller cases for profiling)")
    ap.add_argument("--seq", type=int, default=None,
                    help="override the workload's sequence length (smaller cases for profiling)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)      # at least 3 untimed warm-up steps
    if args.impl == "reference":
        run_reference(args)
    elif args.decode_only:
        run_decode_only(args)
    else:
        run_cuda(args)


if __name__ == "__main__":
    main()
