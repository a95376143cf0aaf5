"""Benchmark of split-KV tail-padded attention on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload long_gqa]

A step is one call of attn_fwd_split_kv over one batch of the workload (the
whole hot path: one kernel).  The default workload is the largest one
(long GQA self-attention: B 1, Hq 32 / Hkv 8, D 128, 512 prefix + 24576
suffix keys of which the last 40 are tail pad).  Inputs are synthetic (seeded, see workloads/)
and rotate over 4 device copies (> 126 MB L2) so no step reads another step's
data from L2.  Device time is measured with CUDA events on the launching
stream, W warm-up steps first, barrier + synchronize on both sides, max over
ranks.  N > 1 (torchrun) runs one independent copy of the workload per rank
(weak scaling, no collective on the data path).

--impl reference times the CPU oracle (the slow, obviously-correct fp64
definition) on the host cores, each step a bounded sample of query rows of
the same workload, reported in the same unit.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "split-KV attention TFLOP/s and % of B200 dense-bf16 peak; max-abs err vs CPU oracle"
DEFAULT_WORKLOAD = "long_gqa"
FALLBACK_BF16_TFLOPS = 1590.0
KERNEL_SOURCES = ["varlen_flash_attention_b200/csrc/attn_common.cuh",
                  "varlen_flash_attention_b200/csrc/attn_fwd_persistent.cuh",
                  "varlen_flash_attention_b200/csrc/ptx.cuh",
                  "varlen_flash_attention_b200/csrc/splitkv_attn.cu"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
PROLOGUE_SOURCES = ["varlen_flash_attention_b200/csrc/qk_norm_rope.cuh"]


def q_valid_of(w):
    rl = w.real_lens()
    return list(rl) if w.Sq == w.Skv else [w.Sq] * w.B


def flops_of(w, rows=None):
    """Algorithmic FLOPs: 4 * D * Hq * sum_b (valid query rows) * real_len[b]."""
    rl = w.real_lens()
    qv = q_valid_of(w)
    if rows is not None:
        qv = [sum(1 for r in rows if r < qv[b]) for b in range(w.B)]
    return 4.0 * w.D * w.Hq * sum(q * n for q, n in zip(qv, rl))


def hbm_bytes_of(w):
    """Algorithmic DRAM bytes of one call: the valid query rows read once,
    the valid K/V rows read once per (batch row, KV head), every output row
    written once (pad rows as zeros)."""
    rl = w.real_lens()
    qv = q_valid_of(w)
    row = w.D * 2
    q = sum(qv) * w.Hq * row
    kv = 2 * sum(rl) * w.Hkv * row
    o = w.B * w.Sq * w.Hq * row
    return q + kv + o


def forced_rows(w):
    """Rows every oracle check includes: the first row, the rows on either
    side of the prefix/suffix boundary, the last valid query row and every
    pad query row."""
    qv = min(q_valid_of(w))
    rows = {0, w.Sp - 1, w.Sp, qv - 1} | set(range(qv, w.Sq))
    return sorted(r for r in rows if 0 <= r < w.Sq)


def measured_hbm():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured copy"
    return 6650.0, "fallback copy"


def kernel_source_sha(sources=None):
    h = hashlib.sha256()
    for f in (KERNEL_SOURCES if sources is None else sources):
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def captured_traffic(key, sources=None):
    """DRAM bytes of one launch from profiles/traffic.json, or None when the
    entry is missing or the kernel sources changed since the capture."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        e = json.load(f).get(key)
    if not e or e.get("kernel_source_sha") != kernel_source_sha(sources):
        return None
    return int(e["dram_bytes_per_launch"])


SUSTAINED_AFTER_S = 1.0  # a timed region longer than this runs under the power cap


def measured_peaks(timed_s: float = 0.0):
    """(peak TFLOP/s, description): the measured cuBLAS bf16 burst figure for a
    kernel timed briefly, the sustained (power-capped) one for a timed region
    longer than SUSTAINED_AFTER_S; the recipe's fallback if no measurement."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if timed_s > SUSTAINED_AFTER_S and "bf16_tflops_sustained" in d:
            return float(d["bf16_tflops_sustained"]), "measured bf16 sustained"
        return float(d["bf16_tflops"]), "measured bf16 burst"
    return FALLBACK_BF16_TFLOPS, "fallback bf16 burst"


def traffic_per_launch(workload):
    return captured_traffic(workload)


class ClockSampler:
    """Polls NVML (SM clock, clock-event reasons) from a thread while running."""

    REASONS = {
        "hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
        "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
        "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
        "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
        "hw_power_brake": "nvmlClocksEventReasonHwPowerBrakeSlowdown",
    }

    def __init__(self, device_index):
        self.samples = []
        self.power_w = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:  # no NVML: clocks reported as unavailable
            self._ok = False

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.power_w.append(nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0)
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, attr in self.REASONS.items():
                    if r & getattr(nv, attr, 0):
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.0005)

    def __enter__(self):
        if self._ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def mark(self):
        """Drop what was sampled so far (the summary covers what follows)."""
        self.samples.clear()
        self.power_w.clear()
        self.reasons.clear()

    def __exit__(self, *a):
        self._stop.set()
        if self._ok:
            self.t.join()

    def summary(self):
        if not self._ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples)}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples),
                "power_w_max": max(self.power_w) if self.power_w else None}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        return rank, world, local, dist
    return 0, 1, 0, None


def barrier(dist):
    if dist is not None:
        dist.barrier()


def max_over_ranks(x, dist, device="cuda"):
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, dist, device="cuda"):
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def combine_ranks(flop_per_step, steps, dt_ms, dist, device="cuda"):
    """Whole-job throughput: all ranks' FLOPs over the slowest rank's time.

    Returns (slowest time in ms, TFLOP/s)."""
    dt_max = max_over_ranks(dt_ms, dist, device)
    total = sum_over_ranks(flop_per_step * steps, dist, device)
    return dt_max, total / (dt_max / 1e3) / 1e12


def cpu_model():
    """The host CPU's model name (for the CPU baseline's record)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_oracle_sample(w, gpu_out=None, target_s=10.0, seed=0):
    """Time the fp64 oracle on a bounded row sample of the workload (host cores).

    With ``gpu_out`` (the kernel's output on the same inputs), also compare the
    sampled rows with it: (cpu_baseline dict, oracle_check dict)."""
    import numpy as np

    import oracle

    t = workloads.make_inputs(w)
    rl = w.real_lens()
    rng = np.random.default_rng(seed)
    n = max(1, min(w.Sq, 16))
    rows = sorted(int(r) for r in rng.choice(w.Sq, size=n, replace=False))
    t0 = time.perf_counter()
    oracle.attn_split_kv(**t, real_len=rl, rows=rows)
    dt = time.perf_counter() - t0
    n2 = int(min(w.Sq, max(n, n * target_s / max(dt, 1e-3))))
    rows = sorted(set(int(r) for r in rng.choice(w.Sq, size=n2, replace=False)) | set(forced_rows(w)))
    t0 = time.perf_counter()
    ref = oracle.attn_split_kv(**t, real_len=rl, rows=rows)
    dt = time.perf_counter() - t0
    fl = flops_of(w, rows)
    cpu = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
           "sample": f"{len(rows)} of {w.Sq} query rows x {w.Hq} heads x {w.B} batch rows of {w.name} "
                     f"({fl / 1e9:.1f} GFLOP, {dt:.1f} s)",
           "cpu": cpu_model(),
           "all_rows_s": flops_of(w) / (fl / dt)}  # linear extrapolation to every valid row
    if gpu_out is None:
        return cpu, None
    got = gpu_out[:, rows].float().cpu().numpy().astype(np.float64)
    diff = got - ref
    max_abs = float(np.abs(diff).max())
    rel_l2 = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
    qv = q_valid_of(w)
    pad_zero = all(bool((gpu_out[b, qv[b]:] == 0).all()) for b in range(w.B))
    check = {"max_abs": max_abs, "rel_l2": rel_l2,
             "rows": f"{len(rows)} of {w.Sq} x {w.Hq} heads x {w.B} (seeded sample + forced rows "
                     f"0, prefix/suffix boundary, last valid, all pad)",
             "bound": {"max_abs": 2e-2, "rel_l2": 1e-2}, "pad_rows_exactly_zero": pad_zero,
             "pass": max_abs <= 2e-2 and rel_l2 <= 1e-2 and pad_zero}
    return cpu, check


def run_reference(args, w):
    """The CPU oracle as the reference arm: each step a bounded row sample."""
    import numpy as np

    import oracle

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    t = workloads.make_inputs(w)
    rl = w.real_lens()
    rng = np.random.default_rng(1)
    # about 3 s of CPU work per step at this machine's oracle speed
    probe = sorted(int(r) for r in rng.choice(w.Sq, size=min(w.Sq, 8), replace=False))
    t0 = time.perf_counter()
    oracle.attn_split_kv(**t, real_len=rl, rows=probe)
    dt = max(time.perf_counter() - t0, 1e-3)
    per_step = int(min(w.Sq, max(1, len(probe) * 3.0 / dt)))
    samples = [sorted(int(r) for r in rng.choice(w.Sq, size=per_step, replace=False))
               for _ in range(args.warmup + args.steps)]
    for rows in samples[: args.warmup]:
        oracle.attn_split_kv(**t, real_len=rl, rows=rows)
    fl = 0.0
    t0 = time.perf_counter()
    for rows in samples[args.warmup:]:
        oracle.attn_split_kv(**t, real_len=rl, rows=rows)
        fl += flops_of(w, rows)
    dt = time.perf_counter() - t0
    value = fl / dt / 1e12
    sample = f"{per_step} of {w.Sq} query rows x {w.Hq} heads x {w.B} batch rows of {w.name} per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "batch": w.B, "seq_q": w.Sq, "prefix": w.Sp, "suffix": w.Ss,
                   "real_len": rl, "heads_q": w.Hq, "heads_kv": w.Hkv, "head_dim": w.D},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args, w):
    import varlen_flash_attention_b200 as sk

    rank, world, local, dist = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    rl = w.real_lens()
    n_copies = 4
    host = workloads.make_inputs(w, seed=w.seed + 1000 * rank)
    keys = ("q", "k_prefix", "v_prefix", "k_suffix", "v_suffix")
    copies = [{k: host[k].to(dev) for k in keys} for _ in range(n_copies)]
    outs = [torch.empty(w.B, w.Sq, w.Hq, w.D, dtype=torch.bfloat16, device=dev) for _ in range(n_copies)]
    stream = torch.cuda.current_stream(dev)

    def step(i):
        c = copies[i % n_copies]
        sk.attn_fwd_split_kv(c["q"], c["k_prefix"], c["v_prefix"], c["k_suffix"], c["v_suffix"],
                             real_len=rl, out=outs[i % n_copies], stream=stream)

    sk.sk_device_status(local, clear=True)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    # The sampler starts first and the warm-up runs right up to the timed
    # region: an idle GPU drops its clocks, and the first launch after even a
    # short idle runs at half speed while they ramp back up.
    with ClockSampler(local) as clk:
        for i in range(args.warmup):
            step(i)
        barrier(dist)
        torch.cuda.synchronize(dev)
        clk.mark()
        ev0.record(stream)
        for i in range(args.steps):
            step(i)
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        barrier(dist)
    dt_ms = ev0.elapsed_time(ev1)
    status = sk.sk_device_status(local, clear=True)
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")
    fl = flops_of(w)
    dt_ms_max, value = combine_ranks(fl, args.steps, dt_ms, dist)
    per_launch_ms = dt_ms / args.steps
    achieved = fl / (per_launch_ms / 1e3) / 1e12

    # ---- end to end through the public API with host buffers (pinned): every
    # step copies its inputs host -> device, runs the kernel and reads its
    # output back.  Three streams pipeline consecutive steps (step i+1's
    # inputs upload while step i computes and step i-1's output downloads),
    # with two device buffer sets and two pinned output buffers.
    pinned = {k: host[k].pin_memory() for k in keys}
    outs_host = [torch.empty(w.B, w.Sq, w.Hq, w.D, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    h2d = sum(pinned[k].numel() * 2 for k in keys)
    d2h = outs_host[0].numel() * 2
    dbufs = [{k: torch.empty_like(copies[0][k]) for k in keys} for _ in range(2)]
    douts = [torch.empty_like(outs[0]) for _ in range(2)]
    s_up, s_run, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_run = [torch.cuda.Event() for _ in range(2)]
    ev_down = [torch.cuda.Event() for _ in range(2)]
    primed = [False, False]

    def e2e_step(i):
        b = i % 2
        with torch.cuda.stream(s_up):
            if primed[b]:
                s_up.wait_event(ev_run[b])  # the kernel of step i-2 has read this buffer set
            for k in keys:
                dbufs[b][k].copy_(pinned[k], non_blocking=True)
            ev_up[b].record(s_up)
        s_run.wait_event(ev_up[b])
        if primed[b]:
            s_run.wait_event(ev_down[b])    # step i-2's output has been read back
        sk.attn_fwd_split_kv(dbufs[b]["q"], dbufs[b]["k_prefix"], dbufs[b]["v_prefix"], dbufs[b]["k_suffix"],
                             dbufs[b]["v_suffix"], real_len=rl, out=douts[b], stream=s_run)
        ev_run[b].record(s_run)
        with torch.cuda.stream(s_down):
            s_down.wait_event(ev_run[b])
            outs_host[b].copy_(douts[b], non_blocking=True)
            ev_down[b].record(s_down)
        primed[b] = True

    for i in range(max(2, args.warmup)):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    barrier(dist)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    for i in range(args.steps):
        e2e_step(i)
    e1.record(s_down)  # the d2h stream ends after every step's read-back
    torch.cuda.synchronize(dev)
    barrier(dist)
    _, e2e_value = combine_ranks(fl, args.steps, e0.elapsed_time(e1), dist)
    if sk.sk_device_status(local, clear=True) != 0:
        raise RuntimeError("device status set during the end-to-end run")
    # same inputs, deterministic kernel: the last read-back equals the device-timed output
    if not torch.equal(outs_host[(args.steps - 1) % 2].view(torch.int16), outs[0].cpu().view(torch.int16)):
        raise RuntimeError("end-to-end output differs from the device-timed output")

    peak, peak_kind = measured_peaks(dt_ms_max / 1e3)
    hbm_peak, hbm_kind = measured_hbm()
    hbm_b = hbm_bytes_of(w)
    hbm_gbs = hbm_b / (per_launch_ms / 1e3) / 1e9
    clocks = clk.summary()
    line = None
    if rank == 0:
        cpu, check = (cpu_oracle_sample(w, outs[0]) if world == 1 and not args.no_cpu_baseline
                      else (None, None))
        line = {
            "metric": METRIC,
            "value": value,
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": dt_ms_max / args.steps,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "batch": w.B, "seq_q": w.Sq, "prefix": w.Sp, "suffix": w.Ss,
                       "real_len": rl, "heads_q": w.Hq, "heads_kv": w.Hkv, "head_dim": w.D,
                       "flop_per_step": fl, "l2": "inputs rotate over 4 device copies (> 126 MB L2)",
                       "parallelism": f"replica x{world}" if world > 1 else "single"},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "peak_kind": peak_kind,
                         "traffic": traffic_per_launch(w.name)},
            "hbm": {"bytes_per_step": hbm_b, "achieved": hbm_gbs, "peak": hbm_peak, "unit": "GB/s",
                    "frac": hbm_gbs / hbm_peak, "peak_kind": hbm_kind,
                    "bytes": "valid Q rows + valid K/V once per KV head + every output row"},
            "cpu_baseline": cpu,
            "oracle_check": check,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": args.steps,
            "clocks": clocks,
        }
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


def run_prologue(args, w):
    """The optional A0 prologue (fused Q/K RMSNorm + RoPE, in place) on the
    workload's q and k: HBM GB/s against the measured copy bandwidth.  Bytes
    = one read and one write of every q and k element."""
    import numpy as np

    import varlen_flash_attention_b200 as sk

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    g = torch.Generator().manual_seed(w.seed)
    S = w.Sq
    per_copy = 2 * w.B * S * (w.Hq + w.Hkv) * w.D  # q + k bytes
    n_copies = max(2, -(-2 * 126 * 2 ** 20 // per_copy))  # rotating copies > 2x L2
    qs = [torch.randn(w.B, S, w.Hq, w.D, generator=g).to(torch.bfloat16).to(dev) for _ in range(n_copies)]
    ks = [torch.randn(w.B, S, w.Hkv, w.D, generator=g).to(torch.bfloat16).to(dev) for _ in range(n_copies)]
    wq = torch.ones(w.D, dtype=torch.bfloat16, device=dev)
    wk = torch.ones(w.D, dtype=torch.bfloat16, device=dev)
    rot = w.D
    ang = np.arange(S)[:, None] * 10000.0 ** (-np.arange(0, rot, 2) / rot)
    table = torch.from_numpy(np.concatenate([np.cos(ang), np.sin(ang)], 1).astype(np.float32)).to(dev)
    step = lambda i: sk.qk_rmsnorm_rope(qs[i % n_copies], ks[i % n_copies], wq, wk, table, rot_dim=rot,
                                        exact=args.exact)
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(0) as clk:
        e0.record()
        for i in range(args.steps):
            step(i)
        e1.record()
        torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / args.steps
    nbytes = 2 * 2 * w.B * S * (w.Hq + w.Hkv) * w.D
    gbs = nbytes / (ms / 1e3) / 1e9
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    peak, kind = (json.load(open(p))["hbm_gbs"], "measured copy") if os.path.exists(p) else (6650.0, "fallback")
    print(json.dumps({
        "metric": "qk_rmsnorm_rope (A0 prologue) HBM GB/s", "value": gbs, "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "dtype": ("f32 (sum of squares, r and undecided bf16 roundings in f64)" if args.exact else "f32"),
        "data": "synthetic", "instance": "exact" if args.exact else "fp32 (default)",
        "config": {"workload": w.name, "batch": w.B, "seq": S, "heads_q": w.Hq, "heads_kv": w.Hkv,
                   "head_dim": w.D, "rot_dim": rot, "bytes_per_step": nbytes,
                   "l2": f"{n_copies} rotating q/k copies, {n_copies * per_copy / 1e6:.0f} MB > 2x L2"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                     "peak_kind": kind, "traffic": captured_traffic("prologue:" + w.name, PROLOGUE_SOURCES)},
        "gpu_launches": args.steps, "clocks": clk.summary()}), flush=True)
    return 0


def run_scatter(args, w):
    """The attention with its output scattered over ``args.scatter`` destination
    buffers on this GPU (the stores of the fused output all-to-all; on several
    GPUs the buffers would be the ranks' receive buffers): TFLOP/s against
    the same roofline as the plain line."""
    import varlen_flash_attention_b200 as sk

    n = args.scatter
    if w.Sq % n:
        raise SystemExit(f"{w.name}: Sq={w.Sq} does not split into {n} chunks")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    rl = w.real_lens()
    n_copies = 4
    host = workloads.make_inputs(w)
    keys = ("q", "k_prefix", "v_prefix", "k_suffix", "v_suffix")
    copies = [{k: host[k].to(dev) for k in keys} for _ in range(n_copies)]
    dsts = [[torch.empty(w.B, w.Sq // n, w.Hq, w.D, dtype=torch.bfloat16, device=dev) for _ in range(n)]
            for _ in range(n_copies)]

    def step(i):
        c = copies[i % n_copies]
        sk.attn_fwd_split_kv_scatter(c["q"], c["k_prefix"], c["v_prefix"], c["k_suffix"], c["v_suffix"],
                                     dsts[i % n_copies], real_len=rl)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(0) as clk:
        e0.record()
        for i in range(args.steps):
            step(i)
        e1.record()
        torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / args.steps
    fl = flops_of(w)
    value = fl / (ms / 1e3) / 1e12
    peak, peak_kind = measured_peaks(ms * args.steps / 1e3)
    ref = sk.attn_fwd_split_kv(copies[0]["q"], copies[0]["k_prefix"], copies[0]["v_prefix"],
                               copies[0]["k_suffix"], copies[0]["v_suffix"], real_len=rl)
    torch.cuda.synchronize(dev)
    same = all(torch.equal(d.view(torch.int16), ref[:, r * (w.Sq // n):(r + 1) * (w.Sq // n)].view(torch.int16))
               for r, d in enumerate(dsts[0]))
    print(json.dumps({
        "metric": METRIC + " (output scattered over destination buffers)", "value": value, "unit": "TFLOP/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "out_scatter": n, "rows_per_destination": w.Sq // n,
                   "l2": "inputs rotate over 4 device copies (> 126 MB L2)"},
        "roofline": {"bound": "tensor", "achieved": value, "peak": peak, "unit": "TFLOP/s", "frac": value / peak,
                     "peak_kind": peak_kind, "traffic": None},
        "scattered_equals_plain_output": same, "gpu_launches": args.steps, "clocks": clk.summary()}), flush=True)
    return 0


def run_packed(args, pw):
    """Packed variable-length attention (attn_fwd_varlen): ``pw.n_seg``
    samples of unequal length in one call, each attending to itself only.
    TFLOP/s = 4 * D * Hq * sum(len_i^2) / t, with an oracle check on sampled
    rows (the first and last row of every segment plus a seeded sample)."""
    import numpy as np

    import oracle
    import varlen_flash_attention_b200 as sk

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    t = workloads.make_packed(pw)
    cu, lens = t["cu_seqlens"], t["lens"]
    n_copies = 4
    copies = [{k: t[k].to(dev) for k in ("q", "k", "v")} for _ in range(n_copies)]
    outs = [torch.empty_like(copies[0]["q"]) for _ in range(n_copies)]
    fl = 4.0 * pw.D * pw.Hq * sum(float(n) * n for n in lens)

    def step(i):
        c = copies[i % n_copies]
        sk.attn_fwd_varlen(c["q"], c["k"], c["v"], cu, cu, out=outs[i % n_copies])

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    sk.sk_device_status(0, clear=True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(0) as clk:
        e0.record()
        for i in range(args.steps):
            step(i)
        e1.record()
        torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / args.steps
    if sk.sk_device_status(0, clear=True) != 0:
        raise RuntimeError("device status set during the packed run")
    value = fl / (ms / 1e3) / 1e12
    peak, peak_kind = measured_peaks(ms * args.steps / 1e3)
    rng = np.random.default_rng(11)
    rows = set(rng.choice(cu[-1], size=min(cu[-1], 96), replace=False).tolist())
    rows |= set(cu[:-1]) | set(c - 1 for c in cu[1:])
    rows = sorted(int(r) for r in rows)
    t0 = time.perf_counter()
    ref = oracle.attn_varlen(t["q"], t["k"], t["v"], cu, cu, rows=rows)
    cpu_s = time.perf_counter() - t0
    got = outs[(args.steps - 1) % n_copies][rows].float().cpu().numpy().astype(np.float64)
    diff = got - ref
    max_abs = float(np.abs(diff).max())
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
    seg_of = np.searchsorted(np.asarray(cu), np.asarray(rows), side="right") - 1
    fl_rows = 4.0 * pw.D * pw.Hq * sum(float(lens[s]) for s in seg_of)
    print(json.dumps({
        "metric": METRIC + " (packed varlen segments)", "value": value, "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": pw.name, "segments": pw.n_seg, "tokens": cu[-1], "min_len": min(lens),
                   "max_len": max(lens), "heads_q": pw.Hq, "heads_kv": pw.Hkv, "head_dim": pw.D,
                   "flop_per_step": fl, "l2": "inputs rotate over 4 device copies (> 126 MB L2)"},
        "roofline": {"bound": "tensor", "achieved": value, "peak": peak, "unit": "TFLOP/s", "frac": value / peak,
                     "peak_kind": peak_kind, "traffic": None},
        "oracle_check": {"max_abs": max_abs, "rel_l2": rel, "rows": f"{len(rows)} of {cu[-1]} x {pw.Hq} heads "
                         "(first and last row of every segment + 96 seeded)", "bound": {"max_abs": 2e-2, "rel_l2": 1e-2},
                         "pass": max_abs <= 2e-2 and rel <= 1e-2},
        "cpu_baseline": {"value": fl_rows / cpu_s / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": f"{len(rows)} query rows x {pw.Hq} heads ({cpu_s:.1f} s)"},
        "gpu_launches": args.steps, "clocks": clk.summary()}), flush=True)
    return 0


def run_host(args, w):
    """Host cost of one call (validation, per-row metadata, five tensor-map
    encodings, launch) on the tiny workload, whose kernel is far shorter than
    that: wall time of back-to-back calls, which the host then bounds
    (``--workload`` is ignored: a longer kernel would bound the loop instead)."""
    import varlen_flash_attention_b200 as sk

    w = workloads.get("tiny")

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    t = {k: v.to(dev) for k, v in workloads.make_inputs(w).items()}
    out = torch.empty(w.B, w.Sq, w.Hq, w.D, dtype=torch.bfloat16, device=dev)
    rl = w.real_lens()
    call = lambda: sk.attn_fwd_split_kv(t["q"], t["k_prefix"], t["v_prefix"], t["k_suffix"], t["v_suffix"],
                                        real_len=rl, out=out)
    for _ in range(max(args.warmup, 50)):
        call()
    torch.cuda.synchronize(dev)
    n = max(args.steps, 2000)
    t0 = time.perf_counter()
    for _ in range(n):
        call()
    t1 = time.perf_counter()
    torch.cuda.synchronize(dev)
    t2 = time.perf_counter()
    print(json.dumps({"metric": "host cost per attn_fwd_split_kv call (Python binding + C ABI + launch)",
                      "value": (t1 - t0) / n * 1e6, "unit": "us", "calls": n, "higher_is_better": False,
                      "drain_after_last_call_us": (t2 - t1) * 1e6,
                      "config": {"workload": w.name}}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=list(workloads.WORKLOADS) + list(workloads.PACKED))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--op", choices=["attention", "prologue", "host"], default="attention",
                    help="prologue: time the optional fused Q/K RMSNorm+RoPE kernel instead; "
                         "host: host cost of one attention call (always the tiny workload)")
    ap.add_argument("--exact", action="store_true",
                    help="with --op prologue: time the bit-exact instance instead of the default fp32 one")
    ap.add_argument("--scatter", type=int, default=0,
                    help="N > 1: scatter the attention output over N destination buffers (fused all-to-all stores)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.workload in workloads.PACKED:
        return run_packed(args, workloads.PACKED[args.workload])
    w = workloads.get(args.workload)
    if args.op == "prologue":
        return run_prologue(args, w)
    if args.op == "host":
        return run_host(args, w)
    if args.scatter > 1:
        return run_scatter(args, w)
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
