"""Benchmark of the forward delta-rule scan on B200: head-tokens/s and roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                    [--no-per-config]

One step = one dr_scan_fwd call over the whole workload (all B*H sequences, all T tokens),
inputs resident in HBM. Under torchrun each rank runs the same workload on its own GPU
(independent sequences, no collective on the data path: weak scaling); the time is the
max over ranks and `value` counts the head-tokens all ranks processed.
Rank 0 prints ONE JSON line. The headline workload is the largest single-GPU configuration
(KDA, B8 H16 T4096); on one GPU the line also carries every other configuration (the small
fp32 DeltaNet case, Gated DeltaNet, the long-context sweep, VLA, Gated DeltaNet-2 and the
decode step) under "per_config", each with its own roofline, e2e and cpu_baseline.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("scan fwd tokens/s per B200 (B·H·T/time) and % of roofline "
          "(TC FLOP/s or HBM GB/s)")
UNIT = "tokens/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# the largest single-GPU configuration (524,288 head-tokens, 816 MB of algorithmic traffic)
DEFAULT_WORKLOAD = "kda_bf16"
# every configuration, in the order the per_config object lists them
PER_CONFIG = ["deltanet_fp32", "gdn_bf16", "kda_bf16", "gdn_long_t4096", "gdn_long_t8192",
              "gdn_long_t16384", "gdn_long_t32768", "vla_fp32_d32", "vla_fp32_d96",
              "vla_ratio_fp32_d32", "vla_ratio_fp32_d96", "gdn2_bf16", "loglinear_bf16",
              "gdn_decode_bf16"]


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--e2e-steps", type=int, default=20)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-per-config", action="store_true")
    p.add_argument("--chained", action="store_true",
                   help="time the chained chunked kernel where the segmented scan would run")
    p.add_argument("--no-e2e", action="store_true",
                   help="skip the end-to-end leg (profiling runs: only the timed launches)")
    p.add_argument("--per-config-steps", type=int, default=0,
                   help="timed steps per extra configuration (0: --steps)")
    return p.parse_args(argv)


# ---------------------------------------------------------------------------------------
# workload accounting
# ---------------------------------------------------------------------------------------
def algorithmic_bytes(w, with_state_in=None, with_state_out=True) -> int:
    """Bytes the scan must move once: q, k, v in, out out, beta and gates in, S0 in (when
    given) and S_final out. Per head-token this is the figure the roofline uses. VLA: q, k,
    v, u in and out out (fp32), S_final and A_final out."""
    from delta_rule_recurrent_chunked_b200 import workloads as wl

    if isinstance(w, wl.VLAWorkload):
        return w.B * w.H * (w.T * 5 * w.d * 4 + (2 * w.d * w.d * 4 if with_state_out else 0))
    if isinstance(w, wl.LogLinearWorkload):  # q, k, v in and out (bf16), lambda in (fp32)
        return w.B * w.H * w.T * ((2 * w.dk + 2 * w.dv) * 2 + w.levels * 4)
    isz = 2 if w.dtype == "bf16" else 4
    BH, T = w.B * w.H, w.T
    per_head = T * (2 * w.dk + 2 * w.dv) * isz
    if w.mode != wl.LINEAR:
        per_head += T * 4
    if w.mode in (wl.GDN, wl.GDN2):
        per_head += T * 4
    elif w.mode == wl.KDA:
        per_head += T * w.dk * 4
    if w.mode == wl.GDN2:
        per_head += T * (w.dk + w.dv) * 4  # erase and write gates
    state = w.dv * w.dk * 4
    if with_state_in if with_state_in is not None else w.s0_std > 0:
        per_head += state
    if with_state_out:
        per_head += state
    return BH * per_head


def algorithmic_flops(w) -> int:
    """Dense-chunk FLOPs of the chunked form (C = 64), triangular halves counted once.
    VLA: about 12 d^2 per head-token (A u, the rank-1 update of A, A k, the write and the
    readout of S, each a d x d matrix-vector product or outer-product update)."""
    from delta_rule_recurrent_chunked_b200 import workloads as wl

    if isinstance(w, wl.VLAWorkload):
        return w.B * w.H * w.T * 12 * w.d * w.d
    if isinstance(w, wl.LogLinearWorkload):
        # per chunk of 64: Q K^T and P V halves, the chunk state V^T K, and one readout
        # Q M_b^T per set bit of the chunk index (on average half the chunk-index bits)
        C = 64
        nch = -(-w.T // C)
        bits = sum(bin(c).count("1") for c in range(nch)) / nch
        per_token = C * w.dk + C * w.dv + 2 * w.dk * w.dv + bits * 2 * w.dk * w.dv
        return int(w.B * w.H * w.T * per_token)
    C = 64
    per_token = 6 * w.dk * w.dv + C * (3 * w.dk + 2 * w.dv) + C * C // 3
    return w.B * w.H * w.T * per_token


def workload_config(w, world: int, nsets: int = 0, nbytes: int = 0) -> dict:
    """The `config` object of the JSON line (shared by both arms)."""
    from delta_rule_recurrent_chunked_b200 import workloads as wl

    cfg = {"workload": w.name, "B": w.B, "H": w.H, "T": w.T}
    if isinstance(w, wl.DRWorkload):
        cfg.update({"dk": w.dk, "dv": w.dv, "mode": wl.MODE_NAMES[w.mode]})
        if not w.decode:
            cfg["chunk"] = 64
    elif isinstance(w, wl.LogLinearWorkload):
        cfg.update({"dk": w.dk, "dv": w.dv, "mode": "loglinear", "levels": w.levels, "chunk": 64})
    else:
        cfg.update({"d": w.d, "mode": "vla_ratio" if w.ratio else "vla"})
    cfg["parallelism"] = f"replicas{world}" if world > 1 else "1gpu"
    if nsets:
        cfg["l2"] = (f"rotating {nsets} resident input sets ({nsets * nbytes / 2**20:.0f} MiB)"
                     " > 126 MiB L2")
    return cfg


def aggregate_value(world: int, head_tokens: int, steps: int, total_ms_max: float) -> float:
    """Whole-job head-tokens/s: every rank processes the full workload per step (weak
    scaling); the time is the slowest rank's."""
    return world * head_tokens * steps / (total_ms_max / 1e3)


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per launch from one ncu capture,
# keyed by workload and the sha256 prefix of the timed kernel's source (dr_chunked.cuh;
# dr_chunked.cuh and drscan.cu for Gated DeltaNet-2's two kernels and for the segmented
# scan's three launches, summed per call; dr_decode.cuh for the decode workload;
# loglinear.cuh for log-linear attention) at capture time; a changed source reports null.
# Summaries with the commands are under profiles/.
NCU_TRAFFIC = {
    ("kda_bf16", "b213a8f2dcd89007"): 673309440 + 119424512,
    ("gdn_bf16", "b213a8f2dcd89007"): 101836288 + 14326784,
    # Gated DeltaNet-2: the pre-scaling kernel and the chunked kernel of one call
    ("gdn2_bf16", "522518ff6411b1c8"): 201334272 + 45484544 + 101819136 + 9624832,
    # the segmented scan: the segment launch, the hand-off check, the conditional launch
    ("gdn_long_t4096", "522518ff6411b1c8"): 52038400 + 633600 + 3169024 + 67840,
    ("gdn_long_t8192", "522518ff6411b1c8"): 109064192 + 14753024 + 3172608 + 67840,
    ("gdn_long_t16384", "522518ff6411b1c8"): 210941440 + 47334400 + 3168512 + 67840,
    ("gdn_long_t32768", "522518ff6411b1c8"): 414370048 + 116414464 + 3169024 + 68096,
    ("kda_long_t32768", "522518ff6411b1c8"): 747991040 + 128194560 + 15752192 + 68352,
    ("gdn_decode_bf16", "6c9773f81f64a408"): 271627008 + 211260672,
    ("loglinear_bf16", "79c1bdb9297c23dc"): 107535616 + 22006784,
}


def kernel_source_sha(*names: str) -> str:
    """sha256 prefix of the timed kernels' sources (dr_chunked.cuh by default; several files
    are hashed in the order given)."""
    import hashlib

    h = hashlib.sha256()
    for name in names or ("dr_chunked.cuh",):
        with open(os.path.join(ROOT, "delta_rule_recurrent_chunked_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------------------
# clocks during the timed region (NVML reads only; nothing is changed)
# ---------------------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, device_index, period_s=0.002):
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()
        reasons = [k for k, bit in self.REASONS.items() if self.reasons & bit and k != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples)}


# ---------------------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------------------
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, group=None, device=None) -> float:
    """Max of a per-rank float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized():
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on the host cores, on a bounded sample of the workload
# ---------------------------------------------------------------------------------------
def oracle_sample(inputs, heads, T):
    from delta_rule_recurrent_chunked_b200 import workloads as wl

    sub = wl.head_slice(inputs, heads)
    for key in ("q", "k", "v", "beta", "gate", "u", "erase", "write", "lam"):
        if sub.get(key) is not None:
            sub[key] = np.ascontiguousarray(sub[key][:, :, :T])
    return sub


def run_oracle(sub):
    import oracle
    from delta_rule_recurrent_chunked_b200 import workloads as wl

    w = sub["workload"]
    if isinstance(w, wl.VLAWorkload) and w.ratio:
        oracle.vla_scan_ratio(sub["q"], sub["k"], sub["v"], sub["u"], lambda0=w.lambda0)
    elif isinstance(w, wl.VLAWorkload):
        oracle.vla_scan(sub["q"], sub["k"], sub["v"], sub["u"], lambda0=w.lambda0)
    elif isinstance(w, wl.LogLinearWorkload):
        oracle.loglinear_scan(sub["q"], sub["k"], sub["v"], sub["lam"])
    elif w.mode == wl.GDN2:
        oracle.dr_scan_ex(sub["q"], sub["k"], sub["v"], sub["beta"], sub["gate"], sub["S0"],
                          w.mode, erase=sub["erase"], write=sub["write"])
    else:
        oracle.dr_scan(sub["q"], sub["k"], sub["v"], sub["beta"], sub["gate"], sub["S0"], w.mode)


def cpu_baseline(inputs, target_s=10.0):
    """Time the oracle on whole heads (all T tokens), as many as fit ~target_s."""
    import oracle

    w = inputs["workload"]
    cores = oracle.num_threads()
    BH = w.B * w.H
    probe = oracle_sample(inputs, list(range(min(BH, cores))), min(w.T, 512))
    run_oracle(probe)  # first call: library load and thread start-up, not timed
    t0 = time.perf_counter()
    run_oracle(probe)
    dt = max(time.perf_counter() - t0, 1e-6)
    rate = min(BH, cores) * min(w.T, 512) / dt  # head-tokens/s with all cores busy
    heads = int(max(1, min(BH, round(rate * target_s / w.T))))
    heads = max(1, (heads // cores) * cores) if heads >= cores else heads
    # when every head fits well inside the target, repeat whole passes to reach it
    reps = int(max(1, min(100, round(rate * target_s / (heads * w.T)))))
    sub = oracle_sample(inputs, list(range(heads)), w.T)
    t0 = time.perf_counter()
    n = 0
    # the estimate sets the minimum; whole passes continue until the target time (<= 100)
    while n < reps or (time.perf_counter() - t0 < target_s and n < 100):
        run_oracle(sub)
        n += 1
    reps = n
    dt = time.perf_counter() - t0
    passes = f"{reps} passes over " if reps > 1 else ""
    return {"value": reps * heads * w.T / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{passes}{heads} of {BH} heads x all {w.T} tokens (fp64 oracle, {dt:.1f} s)"}


# ---------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------
def make_device_inputs(inputs, device):
    import torch

    w = inputs["workload"]
    dev = {}
    for name in ("q", "k", "v"):
        raw = inputs[name + "_raw"]
        t = torch.from_numpy(np.ascontiguousarray(raw).view(np.int16)).view(torch.bfloat16) \
            if w.dtype == "bf16" else torch.from_numpy(np.ascontiguousarray(raw))
        dev[name] = t.to(device)
    for name in ("beta", "gate", "S0", "erase", "write"):
        arr = inputs.get(name)
        dev[name] = None if arr is None else torch.from_numpy(np.ascontiguousarray(arr)).to(device)
    return dev


def rotation(nbytes: int):
    """(input sets to rotate over, whether an L2 flush is needed between timed steps): enough
    resident copies that a set is evicted before it comes round again (>= 3x the 126 MiB L2
    across the rotation, at most 4 copies); workloads too small for that flush L2 instead."""
    nsets = max(1, min(4, -(-3 * L2_BYTES // max(nbytes, 1))))
    return nsets, nsets * nbytes < 2 * L2_BYTES


def l2_note(nsets: int, nbytes: int, flush: bool) -> str:
    if flush:
        return ("L2 flushed between timed steps (256 MiB write outside the timed launches); "
                "value from the summed launch times")
    if nsets == 1:
        return f"one resident input set of {nbytes / 2**20:.0f} MiB > 126 MiB L2"
    return (f"rotating {nsets} resident input sets ({nsets * nbytes / 2**20:.0f} MiB)"
            " > 126 MiB L2")


def timed_loop(step, K, device, stream, local, flush=None):
    """Time K steps with CUDA events on `stream` (warm-up done by the caller), NVML clocks
    sampled meanwhile. With `flush` (a callable that writes more than L2), the flush runs
    between timed steps, outside the events, and the total is the sum of the launch times.
    Returns (total_ms, per-launch ms list, clocks, wall seconds)."""
    import torch

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    clocks = ClockSampler(local)
    barrier(device)
    torch.cuda.synchronize(device)
    clocks.start()
    t_wall = time.perf_counter()
    for i in range(K):
        if flush is not None:
            flush()
        starts[i].record(stream)
        step(i)
        ends[i].record(stream)
    torch.cuda.synchronize(device)
    t_wall = time.perf_counter() - t_wall
    barrier(device)
    clk = clocks.stop()
    per_launch = [starts[i].elapsed_time(ends[i]) for i in range(K)]
    total = sum(per_launch) if flush is not None else starts[0].elapsed_time(ends[-1])
    return total, per_launch, clk, t_wall


def make_flush(device):
    import torch

    buf = torch.empty(256 * 2**20 // 4, dtype=torch.float32, device=device)

    def flush():
        buf.fill_(1.0)

    return flush


def fp32_alu_peak_tflops(device) -> float:
    """FP32 FMA peak of the device from its unit counts and clock: SMs x 128 FP32 lanes x
    2 FLOP x the maximum SM clock (148 x 128 x 2 x 1.965 GHz = 74.4 TFLOP/s on B200)."""
    import torch

    props = torch.cuda.get_device_properties(device)
    mhz = None
    try:
        import pynvml

        pynvml.nvmlInit()
        h = pynvml.nvmlDeviceGetHandleByIndex(device.index or 0)
        mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
    except Exception:
        pass
    mhz = mhz or 1965
    return props.multi_processor_count * 128 * 2 * mhz * 1e6 / 1e12


def base_line(args, w, world, K, total_ms_max, clk, e2e_ms, e2e_h2d, e2e_d2h, config, dtype,
              t_wall, launches_per_step=1):
    return {
        "metric": METRIC, "value": aggregate_value(world, w.head_tokens, K, total_ms_max),
        "unit": UNIT, "n_gpus": world, "steps": K, "warmup": max(3, args.warmup),
        "ms_per_step": total_ms_max / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": dtype, "data": "synthetic", "config": config,
        "clocks": {k: clk[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
        "e2e": {"value": world * w.head_tokens / (e2e_ms / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": e2e_h2d, "d2h_bytes_per_step": e2e_d2h},
        "gpu_launches": K * launches_per_step,
        "wall_s": t_wall,
    }


def measure_dr(args, w, world, rank, local, device, K, cpu_target):
    """The delta-rule scan (dr_scan_fwd; Gated DeltaNet-2 through dr_scan_fwd_ex) on one
    workload: device-timed steps on resident inputs, e2e through the C ABI with host
    buffers, the roofline of the launch and the oracle on the host cores."""
    import torch

    import delta_rule_recurrent_chunked_b200 as drs
    from delta_rule_recurrent_chunked_b200 import workloads as wl

    inputs = wl.generate_dr(w, seed=rank)
    mode = wl.MODE_NAMES[w.mode]
    nbytes = algorithmic_bytes(w)
    nsets, needs_flush = rotation(nbytes)
    flush = make_flush(device) if needs_flush else None
    sets = [make_device_inputs(inputs, device) for _ in range(nsets)]
    outs = [torch.empty_like(st["v"]) for st in sets]
    Sfs = [torch.empty((w.B, w.H, w.dv, w.dk), dtype=torch.float32, device=device) for _ in sets]

    def step(i):
        st = sets[i % nsets]
        if w.mode == wl.GDN2:
            drs.scan_ex(st["q"], st["k"], st["v"], st["beta"], st["gate"], st["S0"], mode=mode,
                        erase=st["erase"], write=st["write"], want_u=False,
                        out=outs[i % nsets], S_final=Sfs[i % nsets])
        else:
            drs.scan(st["q"], st["k"], st["v"], st["beta"], st["gate"], st["S0"], mode=mode,
                     out=outs[i % nsets], S_final=Sfs[i % nsets], chained=args.chained)

    stream = torch.cuda.current_stream(device)
    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize(device)
    if drs.poll_error(device) != 0:
        raise RuntimeError("device status set during warm-up")
    seg0 = drs.segment_counters(device)
    total_ms, per_launch, clk, t_wall = timed_loop(step, K, device, stream, local, flush)
    seg1 = drs.segment_counters(device)
    status = drs.poll_error(device)
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")
    total_ms_max = max_over_ranks(total_ms, device=device)
    launch_ms = statistics.mean(per_launch)
    del sets, outs, Sfs

    e2e = skipped_e2e() if args.no_e2e else run_e2e(args, w, inputs, mode, device, stream)
    e2e_ms = max_over_ranks(e2e["ms"], device=device)

    peaks, peak_src = load_peaks()
    achieved = nbytes / (launch_ms / 1e3) / 1e9
    tflops = algorithmic_flops(w) / (launch_ms / 1e3) / 1e12
    chunked = drs.chunked_applies(mode, w.dtype == "bf16", w.dk, w.dv)
    # Gated DeltaNet-2 on the chunked path is two launches per call: the pre-scaling of k and
    # v by the erase and write gates, then the chunked kernel; the roofline is the call's
    prescaled = chunked and w.mode == wl.GDN2
    # the segmented scan (few heads, long sequences) is three launches of this library per
    # call: all segments at once, the hand-off check and the chained kernel's conditional
    # launch (which returns at once when the checks pass)
    nseg = (drs.chunked_plan_ex(mode, w.B * w.H, w.T, w.dk, w.dv, chained=args.chained)[2]
            if chunked else 1)
    kname = "chunked" if nseg == 1 else f"segmented chunked ({nseg} segments per head)"
    config = dict(workload_config(w, world), l2=l2_note(nsets, nbytes, needs_flush),
                  kernel=("prescale+" + kname if prescaled else kname) if chunked
                  else "sequential")
    if nseg > 1:
        # timed calls that took the segmented scan, and how many of them a failed hand-off
        # check sent back to the chained kernel
        config["segmented"] = {"calls": seg1[0] - seg0[0], "chained_reruns": seg1[1] - seg0[1]}
    line = base_line(args, w, world, K, total_ms_max, clk, e2e_ms, e2e["h2d"], e2e["d2h"], config,
                     w.dtype, t_wall,
                     launches_per_step=(1 if prescaled else 0) + (3 if nseg > 1 else 1))
    line["roofline"] = {
        "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
        "frac": achieved / peaks["hbm_gbs"],
        # a call of several launches (pre-scaling, segments) is keyed by both sources
        "traffic": (NCU_TRAFFIC.get((w.name, kernel_source_sha("dr_chunked.cuh", "drscan.cu")))
                    if prescaled or nseg > 1 else NCU_TRAFFIC.get((w.name, kernel_source_sha()))
                    if chunked else None),
        "peak_source": f"{peak_src} hbm_gbs", "bytes_per_launch": nbytes,
        "launch_ms": launch_ms, "tensor_tflops": tflops,
        "tensor_frac": tflops / peaks["bf16_tflops"]}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(inputs, cpu_target)
    return line


def measure_vla(args, w, world, rank, local, device, K, cpu_target):
    """The VLA Sherman-Morrison scan (fp32) through vla_scan_fwd_ex: the chunked scan as one
    fused cluster kernel per step (the Woodbury A-phase and the WY S-phase at once, on CUDA
    cores), reported against the FP32 ALU peak over the whole step."""
    import torch

    import delta_rule_recurrent_chunked_b200 as drs
    from delta_rule_recurrent_chunked_b200 import workloads as wl

    inputs = wl.generate_vla(w, seed=rank)
    nbytes = algorithmic_bytes(w)
    nsets, needs_flush = rotation(nbytes)
    flush = make_flush(device) if needs_flush else None
    sets = [{k: torch.from_numpy(np.ascontiguousarray(inputs[k])).to(device)
             for k in ("q", "k", "v", "u")} for _ in range(nsets)]
    outs = [torch.empty_like(st["v"]) for st in sets]

    def step(i):
        st = sets[i % nsets]
        if w.ratio:
            drs.vla_scan_ratio(st["q"], st["k"], st["v"], st["u"], lambda0=w.lambda0,
                               out=outs[i % nsets])
        else:
            drs.vla_scan(st["q"], st["k"], st["v"], st["u"], lambda0=w.lambda0,
                         out=outs[i % nsets])

    stream = torch.cuda.current_stream(device)
    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize(device)
    if drs.poll_error(device) != 0:
        raise RuntimeError("device status set during warm-up")
    total_ms, per_launch, clk, t_wall = timed_loop(step, K, device, stream, local, flush)
    if drs.poll_error(device) != 0:
        raise RuntimeError("device status set in the timed region")
    total_ms_max = max_over_ranks(total_ms, device=device)
    launch_ms = statistics.mean(per_launch)
    del sets, outs

    # end to end: pinned host q/k/v/u in, out/S_final/A_final back, every step (pipelined)
    host = {k: torch.from_numpy(np.ascontiguousarray(inputs[k])).pin_memory()
            for k in ("q", "k", "v", "u")}

    def make_outputs():
        return [torch.empty(host["v"].shape, dtype=torch.float32, device=device),
                torch.empty((w.B, w.H, w.d, w.d), dtype=torch.float32, device=device),
                torch.empty((w.B, w.H, w.d, w.d), dtype=torch.float32, device=device)]

    def launch(d, o):
        if w.ratio:
            _, Sf, Af, _ = drs.vla_scan_ratio(d["q"], d["k"], d["v"], d["u"], lambda0=w.lambda0,
                                              out=o[0])
        else:
            _, Sf, Af = drs.vla_scan(d["q"], d["k"], d["v"], d["u"], lambda0=w.lambda0, out=o[0])
        o[1].copy_(Sf)
        o[2].copy_(Af)

    pipe = CopyPipeline(device, host, make_outputs, launch)
    e2e_ms = max_over_ranks(float("nan") if args.no_e2e else pipe.run(max(1, args.e2e_steps)),
                            device=device)

    flops = algorithmic_flops(w)
    peak = fp32_alu_peak_tflops(device)
    achieved = flops / (launch_ms / 1e3) / 1e12
    config = dict(workload_config(w, world), l2=l2_note(nsets, nbytes, needs_flush),
                  kernel="vla_fused")
    line = base_line(args, w, world, K, total_ms_max, clk, e2e_ms, pipe.h2d, pipe.d2h, config,
                     "f32", t_wall)
    line["roofline"] = {
        "bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
        "frac": achieved / peak, "traffic": None,
        "peak_source": "derived: SMs x 128 FP32 lanes x 2 x max SM clock",
        "flops_per_launch": flops, "launch_ms": launch_ms,
        "hbm_gbs": nbytes / (launch_ms / 1e3) / 1e9}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(inputs, cpu_target)
    return line


def measure_decode(args, w, world, rank, local, device, K, cpu_target):
    """Streaming decode through dr_decode_step: one token per head per step on an fp32 state
    that stays resident in HBM and is updated in place (HBM-bound: the state is read and
    written once per step)."""
    import torch

    import delta_rule_recurrent_chunked_b200 as drs
    from delta_rule_recurrent_chunked_b200 import workloads as wl

    inputs = wl.generate_dr(w, seed=rank)
    mode = wl.MODE_NAMES[w.mode]
    nbytes = algorithmic_bytes(w)  # per step: the state in and out plus one token's tensors
    dev = make_device_inputs(inputs, device)  # [B, H, T=1, ...]: drop the token axis
    tok = {"q": dev["q"].reshape(w.B, w.H, w.dk), "k": dev["k"].reshape(w.B, w.H, w.dk),
           "v": dev["v"].reshape(w.B, w.H, w.dv), "beta": dev["beta"].reshape(w.B, w.H),
           "gate": None if dev["gate"] is None else
           dev["gate"].reshape((w.B, w.H) + ((w.dk,) if w.mode == wl.KDA else ()))}
    S = dev["S0"].clone()
    out = torch.empty_like(tok["v"])

    def step(i):
        drs.decode_step(tok["q"], tok["k"], tok["v"], tok["beta"], tok["gate"], S, mode=mode,
                        out=out)

    stream = torch.cuda.current_stream(device)
    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize(device)
    if drs.poll_error(device) != 0:
        raise RuntimeError("device status set during warm-up")
    total_ms, per_launch, clk, t_wall = timed_loop(step, K, device, stream, local)
    if drs.poll_error(device) != 0:
        raise RuntimeError("device status set in the timed region")
    total_ms_max = max_over_ranks(total_ms, device=device)
    launch_ms = statistics.mean(per_launch)

    # end to end: each step's token (q, k, v, beta, gate) from pinned host memory and its
    # output back; the state is the model's and stays resident on the device
    host = {k: t.cpu().pin_memory() for k, t in tok.items() if t is not None}

    def make_outputs():
        return [torch.empty_like(out)]

    def launch(d, o):
        drs.decode_step(d["q"], d["k"], d["v"], d["beta"], d.get("gate"), S, mode=mode, out=o[0])

    pipe = CopyPipeline(device, host, make_outputs, launch)
    e2e_ms = max_over_ranks(float("nan") if args.no_e2e else pipe.run(max(1, args.e2e_steps)),
                            device=device)

    peaks, peak_src = load_peaks()
    achieved = nbytes / (launch_ms / 1e3) / 1e9
    config = dict(workload_config(w, world), kernel="decode",
                  l2=f"resident state {w.B * w.H * w.dv * w.dk * 4 / 2**20:.0f} MiB > 126 MiB L2")
    line = base_line(args, w, world, K, total_ms_max, clk, e2e_ms, pipe.h2d, pipe.d2h, config,
                     w.dtype, t_wall)
    line["roofline"] = {
        "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
        "frac": achieved / peaks["hbm_gbs"],
        "traffic": NCU_TRAFFIC.get((w.name, kernel_source_sha("dr_decode.cuh"))),
        "peak_source": f"{peak_src} hbm_gbs", "bytes_per_launch": nbytes,
        "launch_ms": launch_ms}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(inputs, cpu_target)
    return line


def measure_loglinear(args, w, world, rank, local, device, K, cpu_target):
    """Log-linear attention (loglinear_scan_fwd) on one workload: resident inputs timed on the
    device, e2e through the C ABI with host buffers, HBM roofline, oracle on the host."""
    import torch

    import delta_rule_recurrent_chunked_b200 as drs
    from delta_rule_recurrent_chunked_b200 import workloads as wl

    inputs = wl.generate_loglinear(w, seed=rank)
    nbytes = algorithmic_bytes(w)
    nsets, needs_flush = rotation(nbytes)
    flush = make_flush(device) if needs_flush else None

    def upload():
        d = {}
        for name in ("q", "k", "v"):
            raw = np.ascontiguousarray(inputs[name + "_raw"])
            d[name] = torch.from_numpy(raw.view(np.int16)).view(torch.bfloat16).to(device)
        d["lam"] = torch.from_numpy(np.ascontiguousarray(inputs["lam"])).to(device)
        return d

    sets = [upload() for _ in range(nsets)]
    outs = [torch.empty_like(st["v"]) for st in sets]

    def step(i):
        st = sets[i % nsets]
        drs.loglinear_scan(st["q"], st["k"], st["v"], st["lam"], out=outs[i % nsets])

    stream = torch.cuda.current_stream(device)
    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize(device)
    if drs.poll_error(device) != 0:
        raise RuntimeError("device status set during warm-up")
    total_ms, per_launch, clk, t_wall = timed_loop(step, K, device, stream, local, flush)
    if drs.poll_error(device) != 0:
        raise RuntimeError("device status set in the timed region")
    total_ms_max = max_over_ranks(total_ms, device=device)
    launch_ms = statistics.mean(per_launch)
    del sets, outs

    host = {}
    for name in ("q", "k", "v"):
        raw = np.ascontiguousarray(inputs[name + "_raw"])
        host[name] = torch.from_numpy(raw.view(np.int16)).view(torch.bfloat16).pin_memory()
    host["lam"] = torch.from_numpy(np.ascontiguousarray(inputs["lam"])).pin_memory()

    def make_outputs():
        return [torch.empty(host["v"].shape, dtype=torch.bfloat16, device=device)]

    def launch(d, o):
        drs.loglinear_scan(d["q"], d["k"], d["v"], d["lam"], out=o[0])

    pipe = CopyPipeline(device, host, make_outputs, launch)
    e2e_ms = max_over_ranks(float("nan") if args.no_e2e else pipe.run(max(1, args.e2e_steps)),
                            device=device)

    peaks, peak_src = load_peaks()
    achieved = nbytes / (launch_ms / 1e3) / 1e9
    tflops = algorithmic_flops(w) / (launch_ms / 1e3) / 1e12
    config = dict(workload_config(w, world), l2=l2_note(nsets, nbytes, needs_flush),
                  kernel="loglinear")
    line = base_line(args, w, world, K, total_ms_max, clk, e2e_ms, pipe.h2d, pipe.d2h, config,
                     "bf16", t_wall)
    line["roofline"] = {
        "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
        "frac": achieved / peaks["hbm_gbs"],
        "traffic": NCU_TRAFFIC.get((w.name, kernel_source_sha("loglinear.cuh"))),
        "peak_source": f"{peak_src} hbm_gbs", "bytes_per_launch": nbytes,
        "launch_ms": launch_ms, "tensor_tflops": tflops,
        "tensor_frac": tflops / peaks["bf16_tflops"]}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(inputs, cpu_target)
    return line


def measure(args, name, world, rank, local, device, K, cpu_target):
    from delta_rule_recurrent_chunked_b200 import workloads as wl

    w = wl.workload(name)
    if isinstance(w, wl.LogLinearWorkload):
        return measure_loglinear(args, w, world, rank, local, device, K, cpu_target)
    if isinstance(w, wl.VLAWorkload):
        return measure_vla(args, w, world, rank, local, device, K, cpu_target)
    if w.decode:
        return measure_decode(args, w, world, rank, local, device, K, cpu_target)
    return measure_dr(args, w, world, rank, local, device, K, cpu_target)


# keys of a per_config entry (the rest of a line is shared by all configurations)
PER_CONFIG_KEYS = ("value", "unit", "ms_per_step", "steps", "dtype", "config", "clocks", "e2e",
                   "gpu_launches", "roofline", "cpu_baseline")


def run_ours(args, world, rank, local):
    import torch
    import torch.distributed as dist

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", device_id=device, timeout=timedelta(seconds=120))

    line = measure(args, args.workload, world, rank, local, device, args.steps, 10.0)
    if world == 1 and not args.no_per_config:
        K = args.per_config_steps or min(args.steps, 200)
        per = {}
        for name in PER_CONFIG:
            if name == args.workload:
                continue
            sub = measure(args, name, world, rank, local, device, K, 3.0)
            per[name] = {k: sub[k] for k in PER_CONFIG_KEYS if k in sub}
            torch.cuda.empty_cache()
        line["per_config"] = per
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def skipped_e2e():
    return {"ms": float("nan"), "h2d": 0, "d2h": 0}


class CopyPipeline:
    """End-to-end steps through the public API, pipelined over three streams: the host->device
    copy of step i+1 and the device->host copy of step i-1 overlap the scan of step i (PCIe
    carries both directions at once). Every step still copies its inputs in and its results
    out inside the timed region; two buffer sets and events keep the steps apart."""

    def __init__(self, device, host_in, make_outputs, launch):
        import torch

        self.torch = torch
        self.host_in = host_in                                  # name -> pinned host tensor
        self.dev_in = [{k: (None if t is None else torch.empty_like(t, device=device))
                        for k, t in host_in.items()} for _ in range(2)]
        self.dev_out = [make_outputs() for _ in range(2)]       # list of device tensors
        self.host_out = [[torch.empty_like(t, device="cpu").pin_memory() for t in outs]
                         for outs in self.dev_out]
        self.launch = launch                                    # (dev_in, dev_out) -> None
        self.s_in, self.s_run, self.s_out = (torch.cuda.Stream(device) for _ in range(3))
        self.ev_in = [torch.cuda.Event() for _ in range(2)]
        self.ev_run = [torch.cuda.Event() for _ in range(2)]
        self.ev_out = [torch.cuda.Event() for _ in range(2)]
        self.started = [False, False]
        self.h2d = sum(t.numel() * t.element_size() for t in host_in.values() if t is not None)
        self.d2h = sum(t.numel() * t.element_size() for t in self.dev_out[0])

    def step(self):
        torch = self.torch
        j = self.i % 2
        with torch.cuda.stream(self.s_in):
            if self.started[j]:
                self.s_in.wait_event(self.ev_run[j])       # the scan of step i-2 read dev_in[j]
            for k, t in self.host_in.items():
                if t is not None:
                    self.dev_in[j][k].copy_(t, non_blocking=True)
            self.ev_in[j].record(self.s_in)
        with torch.cuda.stream(self.s_run):
            self.s_run.wait_event(self.ev_in[j])
            if self.started[j]:
                self.s_run.wait_event(self.ev_out[j])      # step i-2's results are copied out
            self.launch(self.dev_in[j], self.dev_out[j])
            self.ev_run[j].record(self.s_run)
        with torch.cuda.stream(self.s_out):
            self.s_out.wait_event(self.ev_run[j])
            for h, d in zip(self.host_out[j], self.dev_out[j]):
                h.copy_(d, non_blocking=True)
            self.ev_out[j].record(self.s_out)
        self.started[j] = True
        self.i += 1

    def run(self, n, warmup=3):
        torch = self.torch
        self.i = 0
        for _ in range(warmup):
            self.step()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(self.s_in)
        for _ in range(n):
            self.step()
        b.record(self.s_out)  # after the last step's device->host copy, which follows all work
        b.synchronize()
        return a.elapsed_time(b) / n


def run_e2e(args, w, inputs, mode, device, stream):
    """Same workload through the public API with pinned host buffers: per step copy the
    inputs host->device, run the scan, copy out and S_final device->host (pipelined)."""
    import torch

    import delta_rule_recurrent_chunked_b200 as drs

    host = {}
    for name in ("q", "k", "v"):
        raw = np.ascontiguousarray(inputs[name + "_raw"])
        t = torch.from_numpy(raw.view(np.int16)).view(torch.bfloat16) if w.dtype == "bf16" \
            else torch.from_numpy(raw)
        host[name] = t.pin_memory()
    for name in ("beta", "gate", "S0", "erase", "write"):
        a = inputs.get(name)
        host[name] = None if a is None else torch.from_numpy(np.ascontiguousarray(a)).pin_memory()

    def make_outputs():
        return [torch.empty(host["v"].shape, dtype=host["v"].dtype, device=device),
                torch.empty((w.B, w.H, w.dv, w.dk), dtype=torch.float32, device=device)]

    def launch(d, o):
        if d.get("erase") is not None:
            drs.scan_ex(d["q"], d["k"], d["v"], d["beta"], d["gate"], d["S0"], mode=mode,
                        erase=d["erase"], write=d["write"], want_u=False, out=o[0], S_final=o[1])
        else:
            drs.scan(d["q"], d["k"], d["v"], d["beta"], d["gate"], d["S0"], mode=mode,
                     out=o[0], S_final=o[1], chained=args.chained)

    pipe = CopyPipeline(device, host, make_outputs, launch)
    ms = pipe.run(max(1, args.e2e_steps))
    return {"ms": ms, "h2d": pipe.h2d, "d2h": pipe.d2h}


# ---------------------------------------------------------------------------------------
# reference arm: the fp64 oracle as it stands, on the host cores
# ---------------------------------------------------------------------------------------
def run_reference(args, world, rank):
    if rank != 0:
        return
    import oracle
    from delta_rule_recurrent_chunked_b200 import workloads as wl

    w = wl.workload(args.workload)
    inputs = wl.generate(w, seed=0)
    cores = oracle.num_threads()
    BH = w.B * w.H
    heads = list(range(min(BH, cores)))
    probe = oracle_sample(inputs, heads, min(w.T, 256))
    t0 = time.perf_counter()
    run_oracle(probe)
    rate = len(heads) * min(w.T, 256) / max(time.perf_counter() - t0, 1e-6)
    steps_total = args.steps + max(3, args.warmup)
    budget_s = 120.0
    T_s = int(max(1, min(w.T, rate * budget_s / steps_total / len(heads))))
    sub = oracle_sample(inputs, heads, T_s)
    for _ in range(max(3, args.warmup)):
        run_oracle(sub)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run_oracle(sub)
    dt = time.perf_counter() - t0
    value = len(heads) * T_s * args.steps / dt
    sample = f"{len(heads)} of {BH} heads x first {T_s} of {w.T} tokens per step (fp64 oracle)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": dt * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    args = parse_args(argv)
    world, rank, local = dist_env()
    if args.impl == "reference":
        run_reference(args, world, rank)
    else:
        run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
