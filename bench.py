#!/usr/bin/env python
"""Benchmark of the GDN token-mixer hot path on B200 (one JSON line on rank 0).

A step is one gdn_prefill over the model-shaped workload (one sequence of T = 4096 tokens,
16 QK / 32 value heads, d = 128, bf16 q/k/v/z, fp32 gates and state): conv + SiLU + L2 norm
+ gates, the chunked gated delta rule, the gated RMSNorm, the final state.  `value` is the
whole-job prefill throughput in Mtok/s (max device time over ranks).  The decode step
(256 sequences x 1 token on 512 MiB of resident fp32 state) is timed in the same run and
reported under "decode" as state GB/s against the measured HBM copy bandwidth.

Timing: W untimed warm-up steps, then K steps between a barrier + cuda synchronize on both
sides, timed with CUDA events on the launching stream.  Inputs rotate over three device
copies (3 x 97 MiB > 126 MB L2) so no step starts with its inputs in L2.  A second pass of
the same K steps brackets every kernel with CUDA events for the per-kernel durations of the
roofline.  "e2e" runs the public call on inputs copied in from pinned host memory and results
copied back every step, pipelined over three streams.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]
  python bench.py --configs      # one JSON line per workload: GPU time and the oracle beside it
Multi-GPU: launched with torch.distributed.run, one rank per GPU; every rank runs its own
full workload (weak scaling, no data-path collective: the mixer shards by sequence/head).
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDN prefill Mtok/s (T=4096, 32 V heads); decode state GB/s vs HBM peak"
WORKLOAD = "prefill_T4096_bf16"
DECODE_WORKLOAD = "decode_N256_bf16"
HBM_FALLBACK_GBS = 6650.0
SM_COUNT = 148
FP32_LANES_PER_SM = 128

# Algorithmic work per (token, value head) of each kernel at d = 128, chunk 64 (16 QK heads
# shared by 32 value heads; Q K^T and K K^T are counted once per QK head).
D, C = 128, 64
FLOP_PHASEA_PER_TOKEN = 16 * (2 * 2 * C * D) + 32 * (2 * 2 * C * D)      # K K^T, Q K^T; W, U'
FLOP_PHASEB_PER_TOKEN = 32 * (3 * 2 * D * D + 2 * C * D)                  # W S^T, Q S^T, U^T K, (MoQK^T) U
BYTES_PER_TOKEN_IO = 2 * (16 * D * 2) + 2 * (32 * D * 2) + 2 * 32 * 4 + 32 * D * 2  # q,k,v,z,a,b in; y out


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["gdn", "reference"], default="gdn")
    p.add_argument("--no-cpu-baseline", action="store_true", help="skip the timed oracle sample")
    p.add_argument("--decode-steps", type=int, default=None)
    p.add_argument("--profile", choices=["prefill", "decode", "decode_multi", "proj", "bwd"], default=None,
                   help="only run W + K calls of one workload (for ncu captures; prints no bench line)")
    p.add_argument("--configs", action="store_true",
                   help="time every workload (GPU and the oracle on a bounded sample) instead of the bench step")
    return p.parse_args(argv)


# ---- host-side helpers (also exercised by the CPU multi-process tests) -------------------

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def shard_units(n_units: int, rank: int, world: int) -> range:
    """Contiguous, balanced share of n_units independent work units (sequences or QK-head
    groups) for `rank`; shares differ by at most one unit and cover every unit once."""
    base, extra = divmod(n_units, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def max_over_ranks(x: float, device=None) -> float:
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device=None) -> float:
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier():
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": HBM_FALLBACK_GBS, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "sm_max_mhz": 1965.0}, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines: list[str] = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=5)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(names, parts[3:7]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# The source files each measured kernel is compiled from (its own header and what it includes).
# Launch configurations live in gdn_api.cu; a change there is re-captured with the kernel's.
KERNEL_SOURCES = {
    "chunk_prep_tc": ("k_chunk_tc.cuh", "tc_ptx.cuh", "gdn_common.cuh"),
    "chunk_scan_tc_norm": ("k_chunk_tc.cuh", "tc_ptx.cuh", "gdn_common.cuh"),
    "decode_multi": ("k_decode_multi.cuh", "gdn_common.cuh"),
    "proj_gemm": ("k_proj.cuh", "tc_ptx.cuh", "gdn_common.cuh"),
    "proj_gemm_out": ("k_proj.cuh", "tc_ptx.cuh", "gdn_common.cuh"),
    "recurrence_bwd": ("k_bwd.cuh", "gdn_common.cuh"),
    "decode": ("k_decode.cuh", "gdn_common.cuh"),
    "chunk_phaseB_simt": ("k_chunk_simt.cuh", "gdn_common.cuh"),
}


def source_sha(files=None) -> str:
    """Hash of the named kernel source files (default: every file of csrc/)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_deltanet_token_b200", "csrc")
    for name in sorted(files if files is not None else os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or None when the
    kernel's source files changed since those counters were taken."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel)
    except (OSError, ValueError):
        return None
    if not rec or kernel not in KERNEL_SOURCES or rec.get("src_sha") != source_sha(KERNEL_SOURCES[kernel]):
        return None
    return rec.get("dram_bytes_per_launch")


# ---- the timed oracle (CPU baseline and the reference arm) ---------------------------------

def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_model() -> str:
    """The host CPU's model name (first "model name" line of /proc/cpuinfo)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_sample(target_s: float, threads: int = 0):
    """Time the fp64 oracle on a prefix of the bench workload (all 32 value heads), sized
    to take about target_s seconds, on `threads` host threads (0: every core).  Returns
    (tokens/s, tokens, seconds, threads)."""
    import oracle
    from gated_deltanet_token_b200.inputs import make_inputs

    cores = threads if threads > 0 else cpu_cores()
    full = make_inputs(WORKLOAD)

    def run(T):
        inp = dict(full)
        for n in ("q", "k", "v", "z", "a", "b"):
            inp[n] = full[n][:T]
        t0 = time.perf_counter()
        oracle.prefill(inp, n_threads=cores, want_state=True)
        return time.perf_counter() - t0

    t_probe = run(64)
    per_tok = t_probe / 64
    T = int(min(4096, max(64, target_s / max(per_tok, 1e-9))))
    dt = run(T)
    reps = 1
    while dt < target_s and T == 4096:  # the whole workload is short: repeat it up to the budget
        dt += run(T)
        reps += 1
    return reps * T / dt, reps * T, dt, cores


def sample_text(Ts: int, secs: float) -> str:
    return (f"the T=4096 workload, all 32 value heads, run {Ts // 4096} times, {secs:.1f} s" if Ts >= 4096
            else f"first {Ts} tokens of the T=4096 workload, all 32 value heads, {secs:.1f} s")


def bench_config(world: int, n_sets: int = 3) -> dict:
    """The `config` of the bench line; the reference arm reports the same one."""
    return {"workload": WORKLOAD, "B": 1, "T": 4096, "h_qk": 16, "h_v": 32, "d": 128, "chunk": 64,
            "in_dtype": "bf16", "out_dtype": "bf16", "state_dtype": "f32",
            "l2": f"{n_sets} rotating input sets of 97 MiB (> 126 MB L2)",
            "parallelism": f"replicas x{world}"}


def reference_arm(args):
    """`--impl reference`: the oracle, as it stands, on the host cores; each step a bounded
    sample (a token prefix of the same workload)."""
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    budget = 120.0 / max(1, args.steps + args.warmup)
    import oracle
    from gated_deltanet_token_b200.inputs import make_inputs

    oracle.build()
    cores = cpu_cores()
    full = make_inputs(WORKLOAD)

    def step(T):
        inp = dict(full)
        for n in ("q", "k", "v", "z", "a", "b"):
            inp[n] = full[n][:T]
        t0 = time.perf_counter()
        oracle.prefill(inp, n_threads=cores)
        return time.perf_counter() - t0

    per_tok = step(32) / 32
    T = int(min(4096, max(8, budget / max(per_tok, 1e-9))))
    for _ in range(args.warmup):
        step(T)
    times = [step(T) for _ in range(args.steps)]
    total = sum(times)
    value = T * args.steps / total / 1e6
    sample = (f"the whole T=4096 workload, all 32 value heads, per step" if T >= 4096
              else f"first {T} of the 4096 tokens, all 32 value heads, per step")
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "Mtok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": bench_config(world),
        "cpu_baseline": {"value": value, "unit": "Mtok/s", "cores": cores, "kind": "oracle",
                         "sample": sample, "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": "Mtok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)
    return 0


# ---- the GPU arm ------------------------------------------------------------------------------

def to_dev(x, device):
    import numpy as np
    import torch

    if x is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(x))
    if x.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    return t.to(device)


def gpu_arm(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    from gated_deltanet_token_b200 import gdn
    from gated_deltanet_token_b200.inputs import make_inputs

    rank, local, world = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    peaks, peak_src = measured_peaks()
    hbm = float(peaks["hbm_gbs"])
    sm_max = float(peaks.get("sm_max_mhz", 1965.0))

    # --- prefill workload: every rank runs its own copy (weak scaling) -----------------------
    inp = make_inputs(WORKLOAD, seed=rank)
    names = ("q", "k", "v", "z", "a", "b")
    params = {n: to_dev(inp[n], dev) for n in ("A_log", "dt_bias", "conv_w", "norm_w")}
    n_sets = 3
    sets = [{n: to_dev(inp[n], dev) for n in names} for _ in range(n_sets)]
    T = inp["spec"]["T"]
    y = torch.empty((T, 32, 128), dtype=torch.bfloat16, device=dev)
    fs = torch.empty((1, 32, 128, 128), dtype=torch.float32, device=dev)
    dims = gdn.make_dims(1, T, 16, 32, gdn.GDN_DTYPE_BF16, gdn.GDN_DTYPE_BF16)
    ws = torch.empty(gdn.gdn_prefill_workspace_size(dims), dtype=torch.uint8, device=dev)

    def step(i):
        s = sets[i % n_sets]
        gdn.gdn_prefill(s["q"], s["k"], s["v"], s["z"], s["a"], s["b"], params["A_log"],
                        params["dt_bias"], params["conv_w"], params["norm_w"], None, None,
                        out_dtype=torch.bfloat16, y=y, final_state=fs, workspace=ws)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.2)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(args.steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_local = e0.elapsed_time(e1)
    ms = max_over_ranks(ms_local, dev)
    ms_per_step = ms / args.steps
    tokens_all = sum_over_ranks(float(T * args.steps), dev)
    value = tokens_all / (ms / 1e3) / 1e6
    # The same K steps again with every kernel bracketed by CUDA events on the call's stream:
    # the per-kernel durations of the roofline.  (The events order the kernels strictly, so the
    # launch overlap between them is absent from this pass and its step time is not reported.)
    gdn.gdn_profile_enable(True)
    gdn.gdn_profile_read()
    torch.cuda.synchronize()
    for i in range(args.steps):
        step(i)
    torch.cuda.synchronize()
    prof = gdn.gdn_profile_read()
    gdn.gdn_profile_enable(False)
    launches = sum(v[0] for v in prof.values())  # the same launches as the timed steps

    # --- roofline of the dominant kernel ------------------------------------------------------
    dom = max(prof.items(), key=lambda kv: kv[1][1])
    dom_name, (dom_n, dom_ms) = dom
    dom_avg_s = dom_ms / dom_n / 1e3
    if dom_name.startswith("chunk_phaseB") or dom_name.startswith("chunk_scan"):
        work, unit_kind = FLOP_PHASEB_PER_TOKEN * T, "flop"
    elif dom_name.startswith("chunk_phaseA") or dom_name.startswith("chunk_prep"):
        work, unit_kind = FLOP_PHASEA_PER_TOKEN * T, "flop"
    else:
        work, unit_kind = None, None
    if unit_kind == "flop" and "simt" in dom_name:
        peak_tflops = SM_COUNT * FP32_LANES_PER_SM * 2 * sm_max * 1e6 / 1e12
        roof = {"kernel": dom_name, "bound": "alu", "achieved": work / dom_avg_s / 1e12,
                "peak": peak_tflops, "unit": "TFLOP/s",
                "peak_source": f"derived: {SM_COUNT} SMs x {FP32_LANES_PER_SM} fp32 lanes x 2 x {sm_max:.0f} MHz"}
    elif unit_kind == "flop":
        pk = float(peaks["bf16_tflops"])
        roof = {"kernel": dom_name, "bound": "tensor", "achieved": work / dom_avg_s / 1e12, "peak": pk,
                "unit": "TFLOP/s", "peak_source": f"{peak_src} bf16_tflops"}
    else:
        roof = {"kernel": dom_name, "bound": "hbm", "achieved": BYTES_PER_TOKEN_IO * T / dom_avg_s / 1e9,
                "peak": hbm, "unit": "GB/s", "peak_source": f"{peak_src} hbm_gbs"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = ncu_traffic(dom_name)
    roof["avg_launch_us"] = dom_avg_s * 1e6
    roof["kernels"] = {k: {"launches": v[0], "avg_us": v[1] / v[0] * 1e3,
                           "share": v[1] / sum(x[1] for x in prof.values())} for k, v in prof.items()}

    # --- decode: 256 sequences x 1 token, resident fp32 state read and written in place --------
    dinp = make_inputs(DECODE_WORKLOAD, seed=rank)
    dd = {n: to_dev(dinp[n], dev) for n in ("q", "k", "v", "z", "a", "b", "A_log", "dt_bias", "conv_w",
                                            "norm_w", "conv_state", "state")}
    yd = torch.empty((256, 32, 128), dtype=torch.bfloat16, device=dev)
    del dinp

    def dstep():
        gdn.gdn_decode(dd["q"], dd["k"], dd["v"], dd["z"], dd["a"], dd["b"], dd["A_log"], dd["dt_bias"],
                       dd["conv_w"], dd["norm_w"], dd["conv_state"], dd["state"],
                       out_dtype=torch.bfloat16, y=yd)

    dsteps = args.decode_steps or max(args.steps, 20)
    for _ in range(max(3, args.warmup)):
        dstep()
    torch.cuda.synchronize()
    barrier()
    e0.record(stream)
    for _ in range(dsteps):
        dstep()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    dms = max_over_ranks(e0.elapsed_time(e1), dev) / dsteps
    # the same step through the pool-slot call: the 256 states as a pool, slots in reverse order
    slot_ids = torch.arange(255, -1, -1, dtype=torch.int32, device=dev)

    def dstep_slots():
        gdn.gdn_decode_slots(dd["q"], dd["k"], dd["v"], dd["z"], dd["a"], dd["b"], dd["A_log"], dd["dt_bias"],
                             dd["conv_w"], dd["norm_w"], dd["conv_state"], dd["state"], slot_ids,
                             out_dtype=torch.bfloat16, y=yd)

    try:
        for _ in range(3):
            dstep_slots()
        torch.cuda.synchronize()
        barrier()
        e0.record(stream)
        for _ in range(dsteps):
            dstep_slots()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        slots_ms = max_over_ranks(e0.elapsed_time(e1), dev) / dsteps
    except RuntimeError as exc:  # an auxiliary figure: report, do not lose the bench line
        slots_ms = f"failed: {exc}"
    # four decode tokens per sequence in one call (each state row read and written once)
    multi = None
    try:
        K4 = 4
        per_tok = [make_inputs(DECODE_WORKLOAD, seed=rank + 100 + i) for i in range(K4)]
        dm = {nm: to_dev(np.ascontiguousarray(np.stack([p_[nm] for p_ in per_tok], axis=1)), dev)
              for nm in ("q", "k", "v", "z", "a", "b")}
        del per_tok
        ym = torch.empty((256, K4, 32, 128), dtype=torch.bfloat16, device=dev)

        def dstep_multi():
            gdn.gdn_decode_multi(dm["q"], dm["k"], dm["v"], dm["z"], dm["a"], dm["b"], dd["A_log"], dd["dt_bias"],
                                 dd["conv_w"], dd["norm_w"], dd["conv_state"], dd["state"],
                                 out_dtype=torch.bfloat16, y=ym)

        for _ in range(3):
            dstep_multi()
        torch.cuda.synchronize()
        barrier()
        e0.record(stream)
        for _ in range(dsteps):
            dstep_multi()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        mms = max_over_ranks(e0.elapsed_time(e1), dev) / dsteps
        m_state = 256 * 32 * 128 * 128 * 4 * 2  # each state row read and written once per call
        m_other = 256 * (K4 * (2 * 16 * 128 * 2 + 2 * 32 * 128 * 2 + 2 * 32 * 4 + 32 * 128 * 2) + 2 * 3 * 8192 * 2)
        multi = {"tokens_per_sequence": K4, "ms_per_call": mms, "tokens_per_s": 256 * K4 / (mms / 1e3),
                 "state_GBps": m_state / (mms / 1e3) / 1e9,
                 "total_GBps": (m_state + m_other) / (mms / 1e3) / 1e9,
                 "frac_state": m_state / (mms / 1e3) / 1e9 / hbm,
                 "frac_total": (m_state + m_other) / (mms / 1e3) / 1e9 / hbm,
                 "traffic": ncu_traffic("decode_multi")}
    except RuntimeError as exc:  # an auxiliary figure: report, do not lose the bench line
        multi = f"failed: {exc}"
    clk = clocks.stop()
    state_bytes = 256 * 32 * 128 * 128 * 4 * 2
    other = 256 * (2 * 16 * 128 * 2 + 2 * 32 * 128 * 2 + 2 * 32 * 4 + 32 * 128 * 2 + 2 * 3 * 8192 * 2)
    decode = {"workload": DECODE_WORKLOAD, "ms_per_step": dms,
              "state_GBps": state_bytes / (dms / 1e3) / 1e9,
              "total_GBps": (state_bytes + other) / (dms / 1e3) / 1e9,
              "peak_GBps": hbm, "frac_state": state_bytes / (dms / 1e3) / 1e9 / hbm,
              "tokens_per_s": 256 / (dms / 1e3), "traffic": ncu_traffic("decode"),
              "slots_ms_per_step": slots_ms, "multi_token": multi}
    del dd

    # --- the projections around the mixer at T = 4096 (tcgen05 GEMMs), synthetic weights --------
    proj = None
    try:
        from gated_deltanet_token_b200.inputs import make_proj_inputs

        pp = make_proj_inputs(T, 2048, 16, 32, seed=rank)
        xp, wi, wo = to_dev(pp["x"], dev), to_dev(pp["w_in"], dev), to_dev(pp["w_out"], dev)
        del pp
        pouts = gdn.gdn_in_proj(xp, wi, 16, 32)
        yo = torch.empty((T, 2048), dtype=torch.bfloat16, device=dev)

        def time_call(fn, reps=20):
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            barrier()
            e0.record(stream)
            for _ in range(reps):
                fn()
            e1.record(stream)
            torch.cuda.synchronize()
            barrier()
            return max_over_ranks(e0.elapsed_time(e1), dev) / reps

        ms_in = time_call(lambda: gdn.gdn_in_proj(xp, wi, 16, 32, out=pouts))
        ms_out = time_call(lambda: gdn.gdn_out_proj(y, wo, 16, 32, out=yo))
        fl_in = 2.0 * T * 2048 * wi.shape[0]
        fl_out = 2.0 * T * 4096 * 2048
        pk = float(peaks["bf16_tflops"])
        proj = {"in_proj_us": ms_in * 1e3, "in_proj_tflops": fl_in / (ms_in / 1e3) / 1e12,
                "out_proj_us": ms_out * 1e3, "out_proj_tflops": fl_out / (ms_out / 1e3) / 1e12,
                "peak_tflops": pk, "peak_source": f"{peak_src} bf16_tflops",
                "in_proj_frac": fl_in / (ms_in / 1e3) / 1e12 / pk, "out_proj_frac": fl_out / (ms_out / 1e3) / 1e12 / pk,
                "shape": "x [4096, 2048] -> 12352 features; y [4096, 4096] -> 2048",
                "traffic_in": ncu_traffic("proj_gemm"), "traffic_out": ncu_traffic("proj_gemm_out")}
        del xp, wi, wo, pouts, yo
    except RuntimeError as exc:  # an auxiliary figure: report, do not lose the bench line
        proj = f"failed: {exc}"

    # --- the backward of the recurrence core at T = 4096 (fp32), synthetic inputs ---------------
    bwd = None
    try:
        from gated_deltanet_token_b200.inputs import make_bwd_inputs

        bi = make_bwd_inputs([T], 16, 32, seed=rank)
        bt = {k: to_dev(bi[k], dev) for k in ("qh", "kh", "v", "g", "beta", "init_state", "dy", "dS_T")}
        del bi
        bdims = gdn.make_dims(1, T, 16, 32, gdn.GDN_DTYPE_F32, gdn.GDN_DTYPE_F32)
        bws = torch.empty(gdn.lib().gdn_recurrence_backward_workspace_size(bdims), dtype=torch.uint8, device=dev)

        def bcall():
            gdn.gdn_recurrence_backward(bt["qh"], bt["kh"], bt["v"], bt["g"], bt["beta"], bt["init_state"], None,
                                        bt["dy"], bt["dS_T"], workspace=bws)

        for _ in range(2):
            bcall()
        torch.cuda.synchronize()
        barrier()
        e0.record(stream)
        for _ in range(5):
            bcall()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        bms = max_over_ranks(e0.elapsed_time(e1), dev) / 5
        bwd = {"ms_per_call": bms, "tokens_per_s": T / (bms / 1e3), "workspace_MB": bws.numel() / 1e6,
               "shape": "T=4096, 16 QK / 32 value heads, fp32, one sequence",
               "traffic": ncu_traffic("recurrence_bwd")}
        del bt, bws
    except RuntimeError as exc:  # an auxiliary figure: report, do not lose the bench line
        bwd = f"failed: {exc}"

    # --- end to end through the public call with host buffers ----------------------------------
    # Every step copies its own inputs in from pinned host memory and its y and final state back
    # out.  Three streams (host->device copies, the prefill, device->host copies) and two buffer
    # slots let step i+1's inputs cross the host link while step i computes and step i-1's
    # results return, as a serving loop would run them.
    host = {n: to_dev(inp[n], "cpu").pin_memory() for n in names}
    n_slots = 2
    dbuf = [{n: torch.empty_like(host[n], device=dev) for n in names} for _ in range(n_slots)]
    ys = [torch.empty_like(y) for _ in range(n_slots)]
    fss = [torch.empty_like(fs) for _ in range(n_slots)]
    y_host = [torch.empty(y.shape, dtype=y.dtype, pin_memory=True) for _ in range(n_slots)]
    fs_host = [torch.empty(fs.shape, dtype=fs.dtype, pin_memory=True) for _ in range(n_slots)]
    s_in, s_run, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(n_slots)]   # the slot's inputs are on the device
    ev_run = [torch.cuda.Event() for _ in range(n_slots)]  # the slot's prefill has finished
    ev_out = [torch.cuda.Event() for _ in range(n_slots)]  # the slot's results are on the host
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = y.numel() * y.element_size() + fs.numel() * fs.element_size()
    torch.cuda.synchronize()

    def e2e_step(i):
        k = i % n_slots
        b = dbuf[k]
        s_in.wait_event(ev_run[k])  # the prefill two steps back is done with this slot's inputs
        with torch.cuda.stream(s_in):
            for n in names:
                b[n].copy_(host[n], non_blocking=True)
        ev_in[k].record(s_in)
        s_run.wait_event(ev_in[k])
        s_run.wait_event(ev_out[k])  # this slot's results of two steps back are on the host
        gdn.gdn_prefill(b["q"], b["k"], b["v"], b["z"], b["a"], b["b"], params["A_log"],
                        params["dt_bias"], params["conv_w"], params["norm_w"], None, None,
                        out_dtype=torch.bfloat16, y=ys[k], final_state=fss[k], workspace=ws, stream=s_run)
        ev_run[k].record(s_run)
        s_out.wait_event(ev_run[k])
        with torch.cuda.stream(s_out):
            y_host[k].copy_(ys[k], non_blocking=True)
            fs_host[k].copy_(fss[k], non_blocking=True)
        ev_out[k].record(s_out)

    e2e_steps = max(3, min(args.steps, 50))
    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    e0.record(s_in)  # every step's work follows its input copies on s_in
    for i in range(e2e_steps):
        e2e_step(i)
    e1.record(s_out)  # ... and ends with its result copies on s_out
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    e2e_val = sum_over_ranks(float(T * e2e_steps), dev) / (e2e_ms / 1e3) / 1e6
    # the results that came back equal those of the device-resident timed steps (same inputs)
    last = (e2e_steps - 1) % n_slots
    e2e_match = bool(torch.equal(y_host[last], y.cpu()) and torch.equal(fs_host[last], fs.cpu()))

    # --- CPU baseline: the oracle on a bounded sample, rank 0 at N = 1 only ---------------------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tps, Ts, secs, cores = oracle_sample(12.0)
        tps1, Ts1, secs1, _ = oracle_sample(8.0, threads=1)
        cpu = {"value": tps / 1e6, "unit": "Mtok/s", "cores": cores, "kind": "oracle",
               "sample": sample_text(Ts, secs), "cpu_model": cpu_model(),
               "threads_1": {"value": tps1 / 1e6, "unit": "Mtok/s", "threads": 1, "sample": sample_text(Ts1, secs1)}}

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    out = {
        "metric": METRIC, "value": value, "unit": "Mtok/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16x3/f32", "data": "synthetic",
        "config": bench_config(world, n_sets),
        "roofline": roof, "cpu_baseline": cpu,
        "e2e": {"value": e2e_val, "unit": "Mtok/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "pipeline": "3 streams, 2 slots", "matches_device": e2e_match},
        "gpu_launches": launches, "clocks": clk, "decode": decode, "projections": proj,
        "backward": bwd,
    }
    print(json.dumps(out), flush=True)
    return 0


def configs_table(args):
    """`--configs`: for each workload, the GPU time of one call (median over repeats, inputs
    resident) and the oracle's tokens/s on the host cores for a bounded token sample."""
    import numpy as np
    import torch

    import oracle
    from gated_deltanet_token_b200 import gdn
    from gated_deltanet_token_b200.inputs import WORKLOADS, make_inputs

    oracle.build()
    cores = cpu_cores()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)

    def dev_t(a):
        if a is None:
            return None
        t = torch.from_numpy(np.ascontiguousarray(a))
        if a.dtype == np.uint16:
            t = t.view(torch.bfloat16)
        return t.to(dev)

    def gpu_time(fn, reps):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    def oracle_rate(inp, kind, sample_tokens):
        sub = dict(inp)
        if kind == "prefill":
            cu = inp.get("cu_seqlens")
            if cu is not None:  # the first sequences, up to the sample size
                keep = int(np.searchsorted(cu, sample_tokens, side="right"))
                keep = max(1, min(keep, len(cu) - 1))
                sub["cu_seqlens"] = cu[:keep + 1]
                T = int(cu[keep])
            else:
                T = min(sample_tokens, inp["q"].shape[0])
            for n in ("q", "k", "v", "z", "a", "b"):
                sub[n] = inp[n][:T]
            if sub.get("init_state") is not None and cu is not None:
                sub["init_state"] = inp["init_state"][:len(sub["cu_seqlens"]) - 1]
            t0 = time.perf_counter()
            oracle.prefill(sub, n_threads=cores, want_state=True)
            return T / (time.perf_counter() - t0), f"first {T} tokens"
        t0 = time.perf_counter()
        oracle.decode(sub, n_threads=cores)
        N = inp["q"].shape[0]
        return N / (time.perf_counter() - t0), f"all {N} sequences, one step"

    for name in WORKLOADS:
        inp = make_inputs(name)
        spec = inp["spec"]
        hq, hv = spec["h_qk"], spec["h_v"]
        d = {n: dev_t(inp.get(n)) for n in ("q", "k", "v", "z", "a", "b", "A_log", "dt_bias", "conv_w",
                                            "norm_w", "init_state", "state", "conv_state")}
        if spec["kind"] == "prefill":
            T = spec["T"]
            cu = inp.get("cu_seqlens")
            cu_t = None if cu is None else torch.from_numpy(cu.astype(np.int32)).to(dev)
            odt = torch.float32 if spec["dtype"] == "f32" else torch.bfloat16
            dims = gdn.make_dims(spec["n_seqs"], T, hq, hv, gdn.GDN_DTYPE_F32 if spec["dtype"] == "f32"
                                 else gdn.GDN_DTYPE_BF16, gdn.GDN_DTYPE_F32 if odt == torch.float32
                                 else gdn.GDN_DTYPE_BF16)
            ws = torch.empty(gdn.gdn_prefill_workspace_size(dims), dtype=torch.uint8, device=dev)
            y = torch.empty((T, hv, 128), dtype=odt, device=dev)
            fs = torch.empty((spec["n_seqs"], hv, 128, 128), dtype=torch.float32, device=dev)

            def call():
                gdn.gdn_prefill(d["q"], d["k"], d["v"], d["z"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                                d["conv_w"], d["norm_w"], d["init_state"], cu_t, out_dtype=odt, y=y,
                                final_state=fs, workspace=ws)
            ms = gpu_time(call, 5 if T > 100000 else 20)
            units = T
            rate, sample = oracle_rate(inp, "prefill", 1024 if hv >= 32 else T)
            del ws, y, fs
        else:
            N = spec["n_seqs"]
            yd = torch.empty((N, hv, 128), dtype=torch.bfloat16, device=dev)

            def call():
                gdn.gdn_decode(d["q"], d["k"], d["v"], d["z"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                               d["conv_w"], d["norm_w"], d["conv_state"], d["state"], out_dtype=torch.bfloat16,
                               y=yd)
            ms = gpu_time(call, 20)
            units = N
            rate, sample = oracle_rate(inp, "decode", N)
        print(json.dumps({"workload": name, "kind": spec["kind"], "tokens": units, "gpu_ms": ms,
                          "gpu_tok_s": units / (ms / 1e3), "oracle_tok_s": rate, "oracle_threads": cores,
                          "oracle_sample": sample, "speedup": units / (ms / 1e3) / rate}), flush=True)
        del d
        torch.cuda.empty_cache()
    return 0


def profile_case(args):
    """`--profile`: W + K calls of one workload and nothing else, with a small device footprint
    (one input set: the prefill holds ~0.5 GB, the decode the 512 MiB of resident state), for
    ncu captures of a single kernel."""
    import numpy as np
    import torch

    from gated_deltanet_token_b200 import gdn
    from gated_deltanet_token_b200.inputs import make_inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    n = args.warmup + args.steps
    if args.profile == "proj":
        from gated_deltanet_token_b200.inputs import make_proj_inputs

        pp = make_proj_inputs(4096, 2048, 16, 32)
        x, wi, wo, y = (to_dev(pp[k], dev) for k in ("x", "w_in", "w_out", "y"))
        for _ in range(n):
            gdn.gdn_in_proj(x, wi, 16, 32)
            gdn.gdn_out_proj(y, wo, 16, 32)
    elif args.profile == "bwd":
        from gated_deltanet_token_b200.inputs import make_bwd_inputs

        bi = make_bwd_inputs([4096], 16, 32)
        bt = {k: to_dev(bi[k], dev) for k in ("qh", "kh", "v", "g", "beta", "init_state", "dy", "dS_T")}
        bdims = gdn.make_dims(1, 4096, 16, 32, gdn.GDN_DTYPE_F32, gdn.GDN_DTYPE_F32)
        bws = torch.empty(gdn.lib().gdn_recurrence_backward_workspace_size(bdims), dtype=torch.uint8, device=dev)
        for _ in range(n):
            gdn.gdn_recurrence_backward(bt["qh"], bt["kh"], bt["v"], bt["g"], bt["beta"], bt["init_state"], None,
                                        bt["dy"], bt["dS_T"], workspace=bws)
    elif args.profile == "prefill":
        inp = make_inputs(WORKLOAD)
        d = {k: to_dev(inp[k], dev) for k in ("q", "k", "v", "z", "a", "b", "A_log", "dt_bias", "conv_w", "norm_w")}
        y = torch.empty((inp["spec"]["T"], 32, 128), dtype=torch.bfloat16, device=dev)
        for _ in range(n):
            gdn.gdn_prefill(d["q"], d["k"], d["v"], d["z"], d["a"], d["b"], d["A_log"], d["dt_bias"], d["conv_w"],
                            d["norm_w"], None, None, out_dtype=torch.bfloat16, y=y)
    else:
        K = 4 if args.profile == "decode_multi" else 1
        per_tok = [make_inputs(DECODE_WORKLOAD, seed=100 + i) for i in range(K)]
        d = {k: to_dev(per_tok[0][k], dev) for k in ("A_log", "dt_bias", "conv_w", "norm_w", "conv_state", "state")}
        for k in ("q", "k", "v", "z", "a", "b"):
            d[k] = to_dev(np.ascontiguousarray(np.stack([p_[k] for p_ in per_tok], axis=1)) if K > 1
                          else per_tok[0][k], dev)
        del per_tok
        for _ in range(n):
            if K > 1:
                gdn.gdn_decode_multi(d["q"], d["k"], d["v"], d["z"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                                     d["conv_w"], d["norm_w"], d["conv_state"], d["state"], out_dtype=torch.bfloat16)
            else:
                gdn.gdn_decode(d["q"], d["k"], d["v"], d["z"], d["a"], d["b"], d["A_log"], d["dt_bias"], d["conv_w"],
                               d["norm_w"], d["conv_state"], d["state"], out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    print(f"profile {args.profile}: {n} calls", flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.profile:
        return profile_case(args)
    if args.impl == "reference":
        return reference_arm(args)
    if args.configs:
        return configs_table(args)
    return gpu_arm(args)


if __name__ == "__main__":
    sys.exit(main())
