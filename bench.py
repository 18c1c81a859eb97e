#!/usr/bin/env python
"""Throughput of block-causal ReLU linear attention at 720p on B200 (one JSON line on rank 0).

Workload (one "step"): the 720p block-causal prefill, B=1, H=20, D=128, 920 tokens per latent
frame (23 x 40), blocks of 3 frames = 2760 tokens, 20 blocks = 55,200 tokens; bf16 q, k, v drawn
N(0, 1) with numpy's seeded generator (seed = rank), fp32 accumulation, eps = 1e-6, final fp32
cache written. One step is one call of sv_block_causal_attn: state reduction -> prefix scan ->
output GEMM, i.e. every step of the hot path. Each step reads q, k and v (848 MB) and writes o
(283 MB); each kernel streams more than the 126 MB L2 (state: k and v, 565 MB; output: q and o),
so L2 is not flushed between steps.

  python bench.py [--gpus N --steps K --warmup W]        our CUDA path (torchrun for N > 1)
  python bench.py --impl reference [...]                 the fp64 CPU oracle on the host cores

With N > 1 every rank runs its own independent prefill (weak scaling, no data-path collective);
the timed region is bracketed by barriers and the reported time is the max over ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

B, H, N, D, L = 1, 20, 55200, 128, 2760
EPS = 1e-6
METRIC = "block-causal linear-attn tokens·heads/s at 720p; HBM GB/s & roofline fraction"
UNIT = "tokens*heads/s"
WORKLOAD = {
    "workload": "720p block-causal prefill: B=1 H=20 N=55200 (20 blocks x 2760 tokens = 3 latent frames "
                "x 23x40) D=128, bf16 q/k/v ~ N(0,1), fp32 accumulation, eps=1e-6, final fp32 cache out",
    "B": B, "H": H, "N": N, "D": D, "block_len": L,
    "seed": "rank",
    "l2": "per step q, k, v 848 MB read, o 283 MB written, each kernel streaming > 126 MB L2; not flushed",
}
ALG_BYTES_PER_TOKHEAD = 4 * D * 2              # read q, k, v once, write o once (bf16)
ALG_FLOPS_PER_TOKHEAD = 4 * D * D + 4 * D       # state 2D^2 + z D, numerator 2D^2 + den 2D + div D


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), float(j.get("bf16_tflops_sustained", j["bf16_tflops"])), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# ----------------------------------------------------------------------------------------------
# clocks during the timed region (NVML, the source nvidia-smi reads)
# ----------------------------------------------------------------------------------------------
_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
            0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
            0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, index: int, period_s: float = 0.02):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - NVML missing
            self._nv = None
            self.error = str(e)
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                bits = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for b, name in _REASONS.items():
                    if bits & b and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._nv is not None:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._nv is not None:
            self._t.join()

    def summary(self):
        if self._nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "error", "")}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------------------------------------
# the oracle on the host cores (reference arm and cpu_baseline)
# ----------------------------------------------------------------------------------------------
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def oracle_rate(q, k, v, budget_s: float, max_heads: int | None = None):
    """Time the fp64 oracle (as it stands) head by head on the stored inputs, cycling over the heads,
    until budget_s elapse (or max_heads heads are done). Returns (tokens*heads per second, heads
    done, tokens per head, seconds)."""
    import oracle
    from block_causal_linear_relu_b200.inputs import to_f64

    done, t0 = 0, time.perf_counter()
    while max_heads is None or done < max_heads:
        h = done % H
        qh, kh, vh = (to_f64(x[:, h:h + 1], "bf16") for x in (q, k, v))
        oracle.block_causal_attn(qh, kh, vh, L, EPS)
        done += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return done * N / dt, done, N, dt


def oracle_rates_other(budget_s: float):
    """The fp64 oracle (as it stands) on bounded samples of the other configurations, on the host
    cores, each sample repeated until budget_s elapse (at least once). Rates in the units of those
    configurations' GPU figures; a reported baseline, not a target."""
    import oracle
    from oracle import rope as R
    from block_causal_linear_relu_b200.inputs import draw_conv, draw_proj, draw_qkv, to_f64

    def run(fn):
        n, t0 = 0, time.perf_counter()
        while True:
            fn()
            n += 1
            dt = time.perf_counter() - t0
            if dt >= budget_s:
                return n, dt

    def attn_line(name, shape, fn, what):
        q, k, v = (to_f64(x, "bf16") for x in draw_qkv(shape, 0, "bf16"))
        n, dt = run(lambda: fn(q, k, v))
        out[name] = {"value": n * shape[1] * shape[2] / dt, "unit": UNIT,
                     "sample": f"fp64 numpy oracle, {what}, {n} run(s), {dt:.1f} s"}

    out = {}
    attn_line("480p_bidir", (1, 1, 8190, 112), lambda q, k, v: oracle.linattn_fwd(q, k, v, EPS),
              "one head of the 480p bidirectional layer [1, 1, 8190, 112]")
    S0, z0 = np.zeros((1, 1, D, D)), np.zeros((1, 1, D))
    attn_line("720p_stream", (1, 1, L, D), lambda q, k, v: oracle.cache_step(q, k, v, S0, z0, EPS),
              "one head of one streaming block [1, 1, 2760, 128] through the cache")
    ang = R.rope3d_angles(R.token_positions(N, 23, 40), R.default_pairs(D))
    attn_line("720p_prefill_rope", (1, 1, N, D), lambda q, k, v: R.block_causal_attn_rope(q, k, v, L, EPS, ang),
              "one head of the 720p prefill with 3D RoPE [1, 1, 55200, 128], blocks of 2760")
    xs, w, bias = draw_conv((1, 60, 920, 64), 0, "bf16")
    xf = to_f64(xs, "bf16")
    n, dt = run(lambda: oracle.temporal_conv_block_causal(xf, w, bias, 3))
    out["720p_temporal_conv"] = {"value": n * 2 * xf.size * 2 / dt / 1e9, "unit": "GB/s (bf16 bytes read + written)",
                                 "sample": f"fp64 numpy oracle, 64 of the 2560 channels of x [1, 60, 920, C], "
                                           f"blocks of 3 frames, {n} run(s), {dt:.1f} s"}
    xp, wp = draw_proj((1, 512, 2560), 3 * 2560, 0)
    xpf, wpf = to_f64(xp, "bf16"), to_f64(wp, "bf16")
    n, dt = run(lambda: oracle.qkv_projection(xpf, wpf, 20, 128))
    out["sv2_projections"] = {"value": n * 2 * 512 * 2560 * 7680 / dt / 1e12, "unit": "TFLOP/s",
                              "sample": f"fp64 numpy oracle, the Q/K/V projection of 512 of the 20240 rows "
                                        f"[512 x 2560] x [2560 x 7680], {n} run(s), {dt:.1f} s"}
    return out


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return 0
    from block_causal_linear_relu_b200.inputs import draw_qkv

    q, k, v = draw_qkv((B, H, N, D), 0, "bf16")
    # one warm-up head sizes the per-step sample so that the whole run stays within a few minutes
    r0, _, _, t_head = oracle_rate(q, k, v, 0.0, max_heads=1)
    per_step_budget = max(0.0, min(t_head * H, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(max(0, args.warmup - 1)):
        oracle_rate(q, k, v, 0.0, max_heads=1)
    tot_heads, tot_s = 0, 0.0
    for _ in range(args.steps):
        _, nh, _, dt = oracle_rate(q, k, v, per_step_budget)
        tot_heads, tot_s = tot_heads + nh, tot_s + dt
    value = tot_heads * N / tot_s
    cores = _blas_threads()
    sample = (f"fp64 numpy oracle (state form), {tot_heads} heads x {N} tokens of the seed-0 720p prefill "
              f"over {args.steps} steps (each step >= 1 head, bounded)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_s / max(1, args.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": WORKLOAD,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "cpu_model": _cpu_model(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------------------------
# our CUDA path
# ----------------------------------------------------------------------------------------------
def _source_sha():
    h = hashlib.sha256()
    for f in ("sv_kernels.cu", "sv_ptx.cuh", "sv_geometry.h"):
        with open(os.path.join(ROOT, "block_causal_linear_relu_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if taken on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(p) as f:
            j = json.load(f)
        ent = j.get(kernel)
        if ent and ent.get("source_sha") == _source_sha():
            return float(ent["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


def max_over_ranks(values, world: int, device=None):
    """Element-wise max of per-rank timings over all ranks (no-op for one rank). Works on any
    torch.distributed backend: CUDA tensors for NCCL, CPU tensors for gloo."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def aggregate_value(world: int, tokheads_per_rank: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput: the units every rank processed divided by the slowest rank's time."""
    return world * tokheads_per_rank * steps / (max_ms / 1e3)


def run_ours(args, rank: int, world: int):
    import torch
    import torch.distributed as dist

    import block_causal_linear_relu_b200 as sv
    from block_causal_linear_relu_b200.inputs import draw_qkv

    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)) if world > 1 else 0)
    dev = torch.device("cuda", torch.cuda.current_device())
    sv.load()
    hbm_gbs, tf_burst, tf_sust, peak_src = peaks()

    qs, ks, vs = draw_qkv((B, H, N, D), rank, "bf16")
    to_dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
    q, k, v = to_dev(qs), to_dev(ks), to_dev(vs)
    o = torch.empty_like(q)
    S_out = torch.zeros(B, H, D, D, device=dev)
    z_out = torch.zeros(B, H, D, device=dev)
    stream = torch.cuda.current_stream()
    ws = sv.make_workspace(sv.SV_OP_BLOCK_CAUSAL_ATTN, q, L)

    def step():
        sv.sv_block_causal_attn(q, k, v, L, o=o, eps=EPS, S_out=S_out, z_out=z_out, ws=ws, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()

    # (A) the timed region: K whole steps, nothing else on the stream
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        t_start.record(stream)
        for _ in range(args.steps):
            step()
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ms = t_start.elapsed_time(t_end)

    # (B) per-kernel durations: the same steps again with the library's timing hook recording an
    # event before/between/after its three kernels (events between kernels stop the programmatic
    # overlap of neighbouring kernels, so this pass is kept out of the timed region above)
    n_prof = max(1, min(args.steps, 100))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_prof)]
    for row in evs:
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()
    for i in range(n_prof):
        sv.sv_profile_events(evs[i])
        step()
    sv.sv_profile_events(None)
    torch.cuda.synchronize()
    st_ms = sum(r[0].elapsed_time(r[1]) for r in evs) / n_prof
    sc_ms = sum(r[1].elapsed_time(r[2]) for r in evs) / n_prof
    ou_ms = sum(r[2].elapsed_time(r[3]) for r in evs) / n_prof
    ms, st_ms, sc_ms, ou_ms = max_over_ranks([ms, st_ms, sc_ms, ou_ms], world, dev)
    if ws.status() != 0:
        raise RuntimeError("a kernel reported a device-side timeout")

    tokheads = B * H * N
    value = aggregate_value(world, tokheads, args.steps, ms)
    ms_step = ms / args.steps

    # end to end through the public API: every step copies its inputs from pinned host memory,
    # makes the call and reads its output back. The steps are pipelined over two sets of device
    # buffers: step i + 1's upload (own stream) overlaps step i's call and its download (own stream;
    # PCIe carries both directions at once). Each step's copies are inside the timed region.
    e2e = None
    if not args.no_e2e:
        pin = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
        qh, kh, vh = pin(qs), pin(ks), pin(vs)
        ohs = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]
        bufs = [(q, k, v, o)] + [tuple(torch.empty_like(q) for _ in range(4))]
        n_e2e = max(2, min(args.steps, args.e2e_steps))
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        up = [torch.cuda.Event() for _ in range(2)]      # inputs of buffer set j landed
        done = [torch.cuda.Event() for _ in range(2)]    # the call on buffer set j finished
        down = [torch.cuda.Event() for _ in range(2)]    # o of buffer set j read back

        def e2e_run(n):
            for i in range(n):
                j = i % 2
                qd, kd, vd, od = bufs[j]
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(done[j])            # the call two steps back has read this set
                    qd.copy_(qh, non_blocking=True)
                    kd.copy_(kh, non_blocking=True)
                    vd.copy_(vh, non_blocking=True)
                    up[j].record(s_in)
                stream.wait_event(up[j])
                if i >= 2:
                    stream.wait_event(down[j])              # o of this set was read back
                sv.sv_block_causal_attn(qd, kd, vd, L, o=od, eps=EPS, S_out=S_out, z_out=z_out, ws=ws, stream=stream)
                done[j].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(done[j])
                    ohs[j].copy_(od, non_blocking=True)
                    down[j].record(s_out)
            stream.wait_stream(s_in)
            stream.wait_stream(s_out)

        e2e_run(2)
        torch.cuda.synchronize()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        s_in.wait_stream(stream)
        e2e_run(n_e2e)
        b.record(stream)
        torch.cuda.synchronize()
        ems = max_over_ranks([a.elapsed_time(b)], world, dev)[0]
        e2e = {"value": world * tokheads * n_e2e / (ems / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": 3 * q.numel() * 2, "d2h_bytes_per_step": o.numel() * 2,
               "steps": n_e2e, "ms_per_step": ems / n_e2e,
               "pipelining": "two buffer sets; step i+1's upload overlaps step i's call and download"}

    if rank != 0:
        return 0
    io_bytes_half = 2 * tokheads * D * 2  # state kernel reads k, v; output kernel reads q, writes o
    kernels = {"state_reduce": st_ms, "prefix_scan": sc_ms, "out_gemm": ou_ms}
    dom = "state_reduce" if st_ms >= ou_ms else "out_gemm"
    dom_ms = kernels[dom]
    achieved = io_bytes_half / (dom_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                "frac": achieved / hbm_gbs, "traffic": _traffic(dom),
                "peak_source": f"{peak_src} HBM copy bandwidth (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured" else "fallback 6650 GB/s",
                "alg_bytes_per_launch": io_bytes_half, "avg_launch_ms": dom_ms,
                "timing": f"CUDA events around each kernel over {n_prof} instrumented steps"}
    step_bytes = tokheads * ALG_BYTES_PER_TOKHEAD
    step_flops = tokheads * ALG_FLOPS_PER_TOKHEAD
    t_roof = max(step_bytes / (hbm_gbs * 1e9), step_flops / (tf_burst * 1e12))
    step_roof = {"alg_bytes": step_bytes, "alg_flops": step_flops, "t_roof_us": t_roof * 1e6,
                 "t_meas_us": ms_step * 1e3, "frac": t_roof / (ms_step / 1e3),
                 "achieved_gbs": step_bytes / (ms_step / 1e3) / 1e9,
                 "achieved_tflops": step_flops / (ms_step / 1e3) / 1e12}
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        rate, nh, ntok, secs = oracle_rate(qs, ks, vs, args.cpu_budget)
        cpu = {"value": rate, "unit": UNIT, "cores": _blas_threads(), "cpu_model": _cpu_model(), "kind": "oracle",
               "sample": f"fp64 numpy oracle (state form), {nh} heads x {ntok} tokens cycling over this "
                         f"workload's {H} heads ({nh / H:.1f} passes), {secs:.1f} s"}
        if not args.no_extras:  # the oracle beside the other configurations' GPU figures
            cpu["other_configs"] = oracle_rates_other(1.5)
    extras = None
    if world == 1 and not args.no_extras:
        extras = {}
        for name, passes in EXTRA_PASSES.items():
            extras[name] = time_workload(name, passes, dev.index)
        extras["720p_temporal_conv"] = time_conv(5, dev.index)
        extras["sv2_projections"] = time_proj(20, dev.index)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": WORKLOAD,
        "roofline": roofline, "step_roofline": step_roof,
        "kernels_ms": kernels, "cpu_baseline": cpu, "e2e": e2e, "clocks": clk.summary(),
        "gpu_launches": 3 * args.steps, "impl": "ours",
        "other_configs": extras,
    }
    print(json.dumps(line), flush=True)
    return 0


EXTRA_WORKLOADS = {
    # name: (description, B, H, N, D, block_len, kind, repeats)
    "480p_bidir": ("480p bidirectional Linear DiT attention: B=2 H=20 N=8190 (21x15x26) D=112", 2, 20, 8190, 112,
                   8190, "fwd", 1),
    "720p_stream": ("autoregressive cache streaming: 60 blocks of B=1 H=20 N=2760 D=128 through the fp32 cache "
                    "(S [1,20,128,128], z [1,20,128]), one sv_cache_step per block", 1, 20, 2760, 128, 2760,
                    "stream", 60),
    "720p_denoise": ("autoregressive generation with several denoising steps per block: 12 blocks x 4 steps of "
                     "B=1 H=20 N=2760 D=128 through the fp32 cache; steps 1-3 of a block attend to it with "
                     "commit=0, step 4 commits the block's state; fresh q, k, v per step", 1, 20, 2760, 128, 2760,
                     "denoise", 48),
    "sv2_stack": ("SANA-Video 2.0-shaped stack: 24 bidirectional layers of B=2 H=20 N=10120 D=128, fresh inputs "
                  "per layer, back to back on one stream", 2, 20, 10120, 128, 10120, "fwd", 24),
    "720p_prefill_rope": ("720p block-causal prefill with the 3D rotary embedding on the numerator: B=1 H=20 "
                          "N=55200 (20 blocks of 3 frames of 23x40 tokens) D=128, pairs (22, 21, 21), "
                          "sv_block_causal_attn_rope", 1, 20, 55200, 128, 2760, "rope", 4),
    "720p_stream_rope": ("cache streaming with the 3D rotary embedding: 60 blocks of B=1 H=20 N=2760 (3 frames of "
                         "23x40) D=128 through the fp32 cache, frame0 = 3 x block, one sv_block_causal_attn_rope "
                         "per block", 1, 20, 2760, 128, 2760, "rope_stream", 60),
}
ROPE_GRID = (23, 40)  # tokens per 720p latent frame: rows x columns


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def time_workload(name, passes: int, dev_index: int = 0, heads: int | None = None):
    """Device time of one of the other configurations, as a dict for the bench line. Every call of a
    pass gets distinct inputs (torch's seeded CUDA generator, seed 0), so L2 never holds a call's
    inputs from an earlier call. Eager: CUDA events around each call issued from Python through the
    binding. Graph: one pass of the same calls captured in a CUDA graph and replayed (how a
    generation loop issues them), device time per call."""
    import torch

    import block_causal_linear_relu_b200 as sv

    desc, b, h, n, d, blen, kind, reps = EXTRA_WORKLOADS[name]
    if heads is not None:  # a smaller case of the same workload, for profiling captures only
        h = heads
        desc += f" (heads overridden to {heads}: not the configuration)"
    dev = torch.device("cuda", dev_index)
    hbm_gbs, _, _, _ = peaks()
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    sets = [tuple(torch.randn(b, h, n, d, device=dev, generator=gen).to(torch.bfloat16) for _ in range(3))
            for _ in range(reps)]
    outs = [torch.empty_like(x[0]) for x in sets]
    S = torch.zeros(b, h, d, d, device=dev)
    z = torch.zeros(b, h, d, device=dev)
    if kind.startswith("rope"):
        ws = sv.make_workspace(sv.SV_OP_BLOCK_CAUSAL_ATTN, sets[0][0], blen)
        fpb = n // (ROPE_GRID[0] * ROPE_GRID[1])  # frames per call
        tab = sv.sv_rope3d_table(fpb * (reps if kind == "rope_stream" else 1), ROPE_GRID[0], ROPE_GRID[1], d,
                                 sv.rope_pairs(d), device=dev)
    else:
        ws = sv.make_workspace(sv.SV_OP_LINATTN_FWD if kind == "fwd" else sv.SV_OP_CACHE_STEP, sets[0][0])
    stream = torch.cuda.current_stream()
    steps_per_block = 4 if kind == "denoise" else 1

    def call(i, st):
        q, k, v = sets[i]
        if kind == "fwd":
            sv.sv_linattn_fwd(q, k, v, o=outs[i], ws=ws, stream=st)
        elif kind == "rope":
            sv.sv_block_causal_attn_rope(q, k, v, blen, tab, o=outs[i], ws=ws, stream=st)
        elif kind == "rope_stream":  # block i sits at frames 3i .. 3i + 2 of the video
            sv.sv_block_causal_attn_rope(q, k, v, n, tab, frame0=i * fpb, o=outs[i], S_in=S, z_in=z, S_out=S,
                                         z_out=z, ws=ws, stream=st)
        else:  # a block's last step commits its state to the cache
            sv.sv_cache_step(q, k, v, S, z, commit=(i % steps_per_block == steps_per_block - 1), o=outs[i], ws=ws,
                             stream=st)

    for i in range(min(reps, 3)):
        call(i, stream)
    torch.cuda.synchronize()
    per = []
    with ClockSampler(dev.index) as clk_e:
        for _ in range(passes):
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
            evs[0].record(stream)
            for i in range(reps):
                call(i, stream)
                evs[i + 1].record(stream)
            torch.cuda.synchronize()
            per += [evs[i].elapsed_time(evs[i + 1]) for i in range(reps)]
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            for i in range(reps):
                call(i, side)
        graph.replay()
        side.synchronize()
        ga, gb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(dev.index) as clk_g:
            ga.record(side)
            for _ in range(passes):
                graph.replay()
            gb.record(side)
            side.synchronize()
        graph_ms = ga.elapsed_time(gb) / (passes * reps)
    del graph
    torch.cuda.synchronize()
    if ws.status() != 0:
        raise RuntimeError("a kernel reported a device-side timeout")
    per_ms = np.array(per)
    tokheads = b * h * n
    call_bytes = tokheads * 4 * d * 2
    t_roof_ms = call_bytes / (hbm_gbs * 1e9) * 1e3
    gl = 3 if blen < n or kind.startswith("rope") else 1
    return {
        "workload": desc, "B": b, "H": h, "N": n, "D": d, "block_len": blen, "calls_per_pass": reps,
        "passes": passes, "kernels_per_call": gl, "gpu_launches": gl * reps * passes * 2,
        "alg_bytes_per_call": call_bytes, "t_roof_ms": t_roof_ms,
        "graph": {"ms_per_call": graph_ms, "value": tokheads / (graph_ms / 1e3), "hbm_frac": t_roof_ms / graph_ms,
                  "clocks": clk_g.summary()},
        "eager": {"ms_per_call_mean": float(per_ms.mean()), "ms_per_call_median": float(np.median(per_ms)),
                  "ms_per_call_p90": float(np.percentile(per_ms, 90)), "value": tokheads / (per_ms.mean() / 1e3),
                  "hbm_frac": t_roof_ms / float(per_ms.mean()), "clocks": clk_e.summary()},
        "unit": UNIT, "data": "synthetic (torch CUDA generator, seed 0), distinct inputs per call",
        "timing": "CUDA events; eager = per call from Python, graph = one pass captured and replayed",
    }


# passes of each other configuration timed inside the default bench run (each pass: every call of
# the workload once, with distinct inputs)
EXTRA_PASSES = {"480p_bidir": 200, "720p_stream": 5, "sv2_stack": 8, "720p_denoise": 4, "720p_prefill_rope": 5,
                "720p_stream_rope": 3}


def time_conv(passes: int, dev_index: int = 0):
    """The block-causal temporal convolution (kernel width 3) on the 720p latent video the prefill
    covers: x [1, 60, 920, 2560] bf16 (60 latent frames of 23 x 40 tokens, hidden 2560), blocks of 3
    frames; one call over the whole sequence, and the same 20 blocks streamed with the carried frame.
    Algorithmic bytes: read x and write y once (plus the carried frame read and written per block)."""
    import torch

    import block_causal_linear_relu_b200 as sv

    dev = torch.device("cuda", dev_index)
    hbm_gbs, _, _, _ = peaks()
    B, T, S, C, Lb = 1, 60, 920, 2560, 3
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    xs = [torch.randn(B, T, S, C, device=dev, generator=gen).to(torch.bfloat16) for _ in range(2)]
    w = torch.randn(C, 3, device=dev, generator=gen) * 0.5
    b = torch.randn(C, device=dev, generator=gen) * 0.5
    y = torch.empty_like(xs[0])
    blocks = [[x[:, a:a + Lb].contiguous() for a in range(0, T, Lb)] for x in xs]
    yb = torch.empty_like(blocks[0][0])
    carry = torch.zeros(B, S, C, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    one_bytes = 2 * xs[0].numel() * 2
    blk_bytes = 2 * blocks[0][0].numel() * 2 + 2 * carry.numel() * 2

    def timed(fn, n):
        fn(0)
        torch.cuda.synchronize()
        a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(dev.index) as clk:
            a.record(stream)
            for i in range(n):
                fn(i)
            e.record(stream)
            torch.cuda.synchronize()
        return a.elapsed_time(e) / n, clk.summary()

    one_ms, clk1 = timed(lambda i: sv.sv_temporal_conv(xs[i % 2], w, Lb, bias=b, y=y, stream=stream), 10 * passes)
    # the 20 blocks of both sequences captured once in a CUDA graph and replayed (a generation loop's
    # way of issuing short calls): device time per block without the host's per-call work
    nb = len(blocks[0])
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            for seq in blocks:
                for blk in seq:
                    sv.sv_temporal_conv_step(blk, w, carry, bias=b, y=yb, stream=side)
        graph.replay()
        side.synchronize()
        ga, ge = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(dev.index) as clk2:
            ga.record(side)
            for _ in range(passes):
                graph.replay()
            ge.record(side)
            side.synchronize()
        blk_ms = ga.elapsed_time(ge) / (passes * 2 * nb)
        clk2 = clk2.summary()
    del graph
    torch.cuda.synchronize()
    return {
        "workload": "block-causal temporal conv (width 3, depthwise) over x [1, 60, 920, 2560] bf16, blocks of 3 "
                    "frames; one call, and 20 blocks streamed with the carried frame",
        "one_shot": {"ms": one_ms, "alg_bytes": one_bytes, "hbm_gbs_alg": one_bytes / (one_ms / 1e3) / 1e9,
                     "hbm_frac": one_bytes / (one_ms / 1e3) / 1e9 / hbm_gbs, "clocks": clk1},
        "per_block": {"ms": blk_ms, "alg_bytes": blk_bytes, "hbm_gbs_alg": blk_bytes / (blk_ms / 1e3) / 1e9,
                      "hbm_frac": blk_bytes / (blk_ms / 1e3) / 1e9 / hbm_gbs, "clocks": clk2},
        "inputs": "two x tensors alternated (each 283 MB, more than L2); torch CUDA generator seed 0",
        "timing": "CUDA events; one-shot: back-to-back calls on one stream, mean per call; per block: the 40 "
                  "block calls captured in a CUDA graph and replayed, mean per call",
    }


def time_proj(reps: int, dev_index: int = 0):
    """The projections of one SANA-Video 2.0-shaped layer: x [2, 10120, 2560] bf16 -> ReLU(q), ReLU(k), v
    [2, 20, 10120, 128] (W_qkv [7680, 2560]) and o [2, 20, 10120, 128] -> y [2, 10120, 2560] (W_o [2560,
    2560]). Tensor-bound: flops 2 * M * N * K; the roofline is the measured cuBLAS bf16 rate. cuBLAS
    on the same shapes (torch.matmul into a plain [M, N] output, no ReLU, no layout change) is timed
    beside it for context."""
    import torch

    import block_causal_linear_relu_b200 as sv

    dev = torch.device("cuda", dev_index)
    _, tf_burst, tf_sust, _ = peaks()
    B, N, C, H, D = 2, 10120, 2560, 20, 128
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    x = torch.randn(B, N, C, device=dev, generator=gen).to(torch.bfloat16)
    w = (torch.randn(3 * H * D, C, device=dev, generator=gen) / C ** 0.5).to(torch.bfloat16)
    wo = (torch.randn(C, H * D, device=dev, generator=gen) / (H * D) ** 0.5).to(torch.bfloat16)
    q, k, v = (torch.empty(B, H, N, D, dtype=torch.bfloat16, device=dev) for _ in range(3))
    y = torch.empty(B, N, C, dtype=torch.bfloat16, device=dev)
    ws = sv.Workspace(256, dev)
    stream = torch.cuda.current_stream()

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(dev.index) as clk:
            a.record(stream)
            for _ in range(reps):
                fn()
            e.record(stream)
            torch.cuda.synchronize()
        return a.elapsed_time(e) / reps, clk.summary()

    qkv_ms, clk_q = timed(lambda: sv.sv_qkv_projection(x, w, H, D, q=q, k=k, v=v, ws=ws, stream=stream))
    out_ms, clk_o = timed(lambda: sv.sv_out_projection(v, wo, y=y, ws=ws, stream=stream))
    x2 = x.view(B * N, C)
    ref_qkv_ms, _ = timed(lambda: torch.matmul(x2, w.t()))
    o2 = torch.empty(B * N, H * D, dtype=torch.bfloat16, device=dev)
    ref_out_ms, _ = timed(lambda: torch.matmul(o2, wo.t()))
    if ws.status() != 0:
        raise RuntimeError("a kernel reported a device-side timeout")
    f_qkv = 2.0 * B * N * C * 3 * H * D
    f_out = 2.0 * B * N * H * D * C
    res = {"workload": "SANA-Video 2.0 layer projections: x [2, 10120, 2560] -> q, k, v [2, 20, 10120, 128] (ReLU on "
                       "q, k); o [2, 20, 10120, 128] -> y [2, 10120, 2560]; bf16, fp32 accumulation",
           "peak_tflops": tf_burst, "peak_source": "MEASURED_PEAKS.json bf16_tflops (cuBLAS burst)"}
    for name, ms, f, ref_ms, clk in (("qkv", qkv_ms, f_qkv, ref_qkv_ms, clk_q), ("out", out_ms, f_out, ref_out_ms, clk_o)):
        tf = f / (ms / 1e3) / 1e12
        res[name] = {"ms": ms, "tflops": tf, "frac": tf / tf_burst, "cublas_ms": ref_ms,
                     "cublas_tflops": f / (ref_ms / 1e3) / 1e12, "clocks": clk}
    return res


def run_extra(args, name):
    """One configuration alone, as an informational JSON line (not the bench line)."""
    import torch

    import block_causal_linear_relu_b200 as sv

    torch.cuda.set_device(0)
    sv.load()
    r = time_workload(name, max(1, args.steps // EXTRA_WORKLOADS[name][-1]), heads=args.heads)
    line = {"metric": METRIC, "value": r["graph"]["value"], "unit": UNIT, "n_gpus": 1, "workload": name,
            "impl": "ours", "dtype": "bf16", **r}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="leave the other configurations (480p, streaming, 2.0 stack, denoising) out of the line")
    ap.add_argument("--workload", choices=["720p_prefill", "720p_temporal_conv", "sv2_projections"] + sorted(EXTRA_WORKLOADS),
                    default="720p_prefill",
                    help="the bench line is 720p_prefill; the others print an informational timing line")
    ap.add_argument("--heads", type=int, default=None,
                    help="override H (profiling captures of a smaller case only; not a bench line)")
    args = ap.parse_args()
    if args.heads is not None:
        global H
        H = args.heads
        WORKLOAD.update({"H": H, "workload": WORKLOAD["workload"].replace("H=20", f"H={H}")})

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.workload == "sv2_projections":
        import torch
        torch.cuda.set_device(0)
        print(json.dumps({"workload": "sv2_projections", "impl": "ours", **time_proj(max(3, args.steps // 10))}),
              flush=True)
        return 0
    if args.workload == "720p_temporal_conv":
        import torch
        torch.cuda.set_device(0)
        print(json.dumps({"workload": "720p_temporal_conv", "impl": "ours", **time_conv(max(1, args.steps // 20))}),
              flush=True)
        return 0
    if args.workload != "720p_prefill":
        return run_extra(args, args.workload)
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0))))
        try:
            return run_ours(args, rank, world)
        finally:
            dist.destroy_process_group()
    return run_ours(args, rank, world)


if __name__ == "__main__":
    sys.exit(main())
