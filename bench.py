"""Benchmark of the DCP exchange hot path on B200: fused pack -> all-to-all ->
stable log-sum-exp combine, through the C-ABI of libcplse.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config stress]
                    [--per-config decode,mla,ulysses] [--impl ours|reference]

One step = one call of cp_pack_permute_combine_fused over one batch: the whole
DCP path (LSE formation, head-chunk pack, the W x W block exchange, combine)
in one pass. `value` is the effective HBM throughput of that step, algorithmic
bytes W*T*H*(2D+8) + T*H*(2D+4) per call over the device time of K
back-to-back steps, summed over ranks (each rank runs its own independent
batch: weak scaling, no collective on the data path).

The headline workload is the largest single-GPU one (stress, 18.8 GB per
call). The other large workloads (decode, mla, ulysses) are measured in the
same run and reported under `per_config`, each with its own roofline, CPU
baseline and kernel breakdown. The roofline of each comes from a dedicated
pass of separately event-bracketed launches (median, p10, p90), independent
of --steps.

--impl reference times the float64 CPU oracle (rank 0 only) on a bounded
sample of the same workload, on the host cores.

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import datetime
import gc
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "pack+permute+combine µs/call and effective HBM GB/s (% of B200 peak)"
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 128 << 20          # at least the B200's L2 (126 MB); fixes the rotation policy
ROOFLINE_LAUNCHES = 50
KERNEL_SOURCES = ["lse_pack_stable_b200/csrc/rowcombine_async.cuh",
                  "lse_pack_stable_b200/csrc/rowcombine_async.cu",
                  "lse_pack_stable_b200/csrc/rowcombine.cuh", "lse_pack_stable_b200/csrc/common.cuh"]
PER_CONFIG_DEFAULT = "decode,mla,ulysses"


def parse(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="stress", choices=sorted(synth.CONFIGS))
    ap.add_argument("--per-config", default=PER_CONFIG_DEFAULT,
                    help="comma-separated workloads measured after the headline one "
                         "(one GPU only); 'none' for the headline alone")
    ap.add_argument("--launches", type=int, default=ROOFLINE_LAUNCHES,
                    help="event-bracketed launches of the roofline pass (at least 50)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="cut the headline workload to this many tokens (small cases for "
                         "profiler captures; 0: the workload's own T)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-breakdown", action="store_true")
    return ap.parse_args(argv)


def env_rank():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def rotation_sets(wl: synth.Workload) -> int:
    """Device copies of one call's inputs and outputs that consecutive calls
    rotate over, so that every call reads cold HBM: one when a call's bytes
    exceed 3x the L2 already, else enough copies to cover 3x the L2."""
    set_bytes = wl.fused_bytes()
    if set_bytes >= 3 * L2_BYTES:
        return 1
    return max(2, math.ceil(3 * L2_BYTES / set_bytes) + 1)


def l2_note(wl: synth.Workload) -> str:
    n = rotation_sets(wl)
    b = wl.fused_bytes()
    if n == 1:
        return ("one set of inputs and outputs, %.1f GB per call (> 3x the L2): every call "
                "streams cold HBM" % (b / 1e9))
    return ("inputs and outputs rotate over %d device sets of %.0f MB (%.0f MB in all, > 3x the L2)"
            % (n, b / 1e6, n * b / 1e6))


def workload_for(name: str, world: int) -> synth.Workload:
    """The workload a run on `world` GPUs measures: on one GPU the configured
    one, W ranks emulated; on N > 1 GPUs the same T, H, D and distributions
    with W = N real ranks, rank r holding plane r (one per GPU)."""
    wl = synth.CONFIGS[name]
    if world == 1:
        return wl
    if wl.H % world:
        raise SystemExit("%s: H = %d is not a multiple of %d GPUs" % (name, wl.H, world))
    return synth.Workload(**{**wl.__dict__, "W": world})


def config_block(wl: synth.Workload, world: int):
    """The workload's description; identical in both arms of the benchmark."""
    if world == 1:
        return {"workload": "%s: W=%d simulated ranks, T=%d, H=%d, D=%d, %s payload, fp32 max/sum"
                            % (wl.name, wl.W, wl.T, wl.H, wl.D, wl.dtype),
                "W": wl.W, "T": wl.T, "H": wl.H, "D": wl.D, "payload_dtype": wl.dtype,
                "global_batch": 1, "parallelism": "replicas1",
                "bytes_per_call": wl.fused_bytes(), "l2": l2_note(wl)}
    return {"workload": "%s shape across %d GPUs: W=%d real ranks (KV shard r on GPU r), T=%d, "
                        "H=%d, D=%d, %s payload, fp32 max/sum; destination j combines head chunk j"
                        % (wl.name, world, wl.W, wl.T, wl.H, wl.D, wl.dtype),
            "W": wl.W, "T": wl.T, "H": wl.H, "D": wl.D, "payload_dtype": wl.dtype,
            "global_batch": 1, "parallelism": "dcp%d" % world,
            "bytes_per_call": wl.fused_bytes(),
            "l2": "one set per rank, %.2f GB of planes per GPU (> 3x the L2)"
                  % (wl.T * wl.H * (2 * wl.D + 8) / 1e9)}


def reduce_max(values, world, device):
    """Element-wise max of `values` over all ranks (the device time of a
    multi-GPU step is the slowest rank's); identity on one rank."""
    if world == 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(world, bytes_per_step, steps, total_ms):
    """Whole-job GB/s: every rank's bytes over the (max-over-ranks) time."""
    return world * bytes_per_step * steps / (total_ms * 1e-3) / 1e9


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def peak_source(kind: str) -> str:
    return ("measured (MEASURED_PEAKS.json hbm_gbs)" if kind == "measured"
            else "fallback 6.65 TB/s (MEASURED_PEAKS.json absent)")


def host_cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def kernel_source_hash():
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(config: str):
    """DRAM bytes per full-size launch of the fused kernel from the committed
    ncu summary, if it was taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "fused_%s.md" % config)
    try:
        text = open(path).read()
    except OSError:
        return None
    src = re.search(r"kernel source sha256/16:\s*([0-9a-f]{16})", text)
    tr = re.search(r"dram bytes per launch:\s*([0-9]+)", text)
    if not src or not tr or src.group(1) != kernel_source_hash():
        return None
    return int(tr.group(1))


def merge_kernel_name(W: int, D: int) -> str:
    """The merge kernel the library launches for W ranks and head dim D."""
    return ("rowcombine_kernel (register-staged, fused mode)" if W > 8 or D > 256
            else "rowcombine_async_kernel (shared-memory-staged, fused mode)")


def pct(ms, q):
    return float(np.percentile(np.asarray(ms, dtype=np.float64), q))


# --------------------------------------------------------------------------------------------
# clocks during the timed regions (NVML)

class ClockSampler:
    """Samples the SM clock and the clock-event reasons in a background thread
    while it is running; start()/stop() may be called several times and the
    samples accumulate (the timed region and the roofline pass)."""
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, index: int, period_s: float = 0.01):
        self.samples, self.reasons, self.ok = [], set(), False
        self.period = period_s
        self._stop = threading.Event()
        self.t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = None
            try:   # NVML numbers devices in PCI order, CUDA may not: match by UUID
                import torch
                uuid = str(torch.cuda.get_device_properties(index).uuid)
                self.h = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + uuid)
            except Exception:  # noqa: BLE001
                self.h = None
            if self.h is None:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = str(e)
            self.max_mhz = None

    def _sample(self):
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            mask = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            for name, bit in self.REASONS.items():
                if mask & bit and name != "gpu_idle":
                    self.reasons.add(name)
        except Exception:  # noqa: BLE001
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._stop.clear()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok and self.t is not None:
            self._stop.set()
            self.t.join()
            self._sample()          # at least one sample taken under load per window
            self.t = None

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.err}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# --------------------------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and --impl reference)

def _oracle_fmt(wl):
    import oracle
    return oracle.get(), (oracle.BF16 if wl.dtype == "bf16" else oracle.FP16)


def oracle_seconds_per_token(wl, o, m, s):
    """Per-token cost of the oracle, from a sample large enough (~0.2 s of work)
    that thread start-up does not dominate."""
    orc, fmt = _oracle_fmt(wl)
    t_cal = min(wl.T, 16, o.shape[1])
    while True:
        t0 = time.perf_counter()
        orc.fused(o[:, :t_cal], m[:, :t_cal], s[:, :t_cal], fmt)
        el = time.perf_counter() - t0
        if el > 0.2 or t_cal >= min(wl.T, o.shape[1]):
            return max(el, 1e-6) / t_cal
        t_cal = min(wl.T, o.shape[1], t_cal * 4)


def time_oracle(wl: synth.Workload, budget_s: float, o=None, m=None, s=None):
    """Time the float64 oracle's direct pack->a2a->combine on a token sample of the
    workload. Returns (GB/s over the sample's algorithmic bytes, seconds per pass,
    sample text, cores)."""
    orc, fmt = _oracle_fmt(wl)
    per_tok = wl.fused_bytes() / wl.T
    if o is None:
        o, m, s = sample_inputs(wl, min(wl.T, 256))
    dt = oracle_seconds_per_token(wl, o, m, s)
    toks = int(max(1, min(wl.T, budget_s / dt)))
    if o.shape[1] < toks:
        o, m, s = sample_inputs(wl, toks)
    reps = max(1, int(budget_s / (dt * toks)))
    t0 = time.perf_counter()
    for _ in range(reps):
        orc.fused(o[:, :toks], m[:, :toks], s[:, :toks], fmt)
    el = time.perf_counter() - t0
    gbs = per_tok * toks * reps / el / 1e9
    sample = ("first %d of %d tokens (all W=%d ranks, all %d heads), %d pass(es), %.1f s"
              % (toks, wl.T, wl.W, wl.H, reps, el))
    return gbs, el / reps, sample, orc.threads()


def time_oracle_threads(wl, budget_s, threads, o, m, s):
    """time_oracle with the oracle's parallel loops on `threads` threads (the
    previous count is restored afterwards)."""
    orc, _ = _oracle_fmt(wl)
    prev = orc.threads()
    orc.set_threads(threads)
    try:
        return time_oracle(wl, budget_s, o, m, s)
    finally:
        orc.set_threads(prev)


def sample_inputs(wl, toks):
    o = np.stack([synth.o_block(wl, r, 0, toks) for r in range(wl.W)])
    ms = [synth.stats_block(wl, r, 0, toks) for r in range(wl.W)]
    return o, np.stack([a for a, _ in ms]), np.stack([b for _, b in ms])


def cpu_baseline(wl, o, m, s, budget_s, single_thread_s):
    """The oracle on a bounded token sample: all host threads, and (if
    single_thread_s > 0) one thread."""
    gbs, _, sample, cores = time_oracle(wl, budget_s, o, m, s)
    rec = {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
           "sample": sample, "cpu_model": host_cpu_model()}
    if single_thread_s > 0:
        gbs1, _, sample1, _ = time_oracle_threads(wl, single_thread_s, 1, o, m, s)
        rec["single_thread"] = {"value": round(gbs1, 4), "unit": "GB/s", "cores": 1,
                                "sample": sample1}
    return rec


def run_reference(args):
    rank, _, world = env_rank()
    if rank != 0:
        return 0
    wl = workload_for(args.config, world)
    steps, warm = max(1, args.steps), max(0, args.warmup)
    orc, fmt = _oracle_fmt(wl)
    o, m, s = sample_inputs(wl, min(wl.T, 16))
    dt = oracle_seconds_per_token(wl, o, m, s)
    budget = 90.0 / (steps + warm)            # the whole run: about 1.5 minutes of CPU
    toks = int(max(1, min(wl.T, budget / dt)))
    o, m, s = sample_inputs(wl, toks)
    per_tok = wl.fused_bytes() / wl.T
    per_step = []
    for i in range(warm + steps):
        t0 = time.perf_counter()
        orc.fused(o, m, s, fmt)
        sec = time.perf_counter() - t0
        if i >= warm:
            per_step.append((per_tok * toks / sec / 1e9, sec))
    sample = "first %d of %d tokens (all W=%d ranks, all %d heads) per step" % (toks, wl.T, wl.W, wl.H)
    cores = orc.threads()
    value = statistics.median(g for g, _ in per_step)
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus,
        "steps": steps, "warmup": warm,
        "ms_per_step": round(1e3 * statistics.median(sec for _, sec in per_step), 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "payload_dtype": wl.dtype,
        "data": "synthetic (seeded counter-based generator, the workload's shapes and distributions)",
        "config": config_block(wl, world), "impl": "reference",
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores,
                         "kind": "oracle", "sample": sample, "cpu_model": host_cpu_model()},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------------------------
# GPU arm

class Inputs:
    """One workload's inputs: generated on the host (into pinned memory when
    the end-to-end leg copies from there), uploaded once, plus the device sets
    that consecutive calls rotate over."""

    def __init__(self, wl, dev, pinned):
        import torch
        W, T, H, D, Hc = wl.W, wl.T, wl.H, wl.D, wl.Hc
        self.tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float16
        self.o_h = torch.empty((W, T, H, D), dtype=torch.int16, pin_memory=pinned)
        self.m_h = torch.empty((W, T, H), dtype=torch.float32, pin_memory=pinned)
        self.s_h = torch.empty((W, T, H), dtype=torch.float32, pin_memory=pinned)
        tb = max(1, (256 << 20) // (H * D * 2))
        on = self.o_h.numpy().view(np.uint16)
        for r in range(W):
            for t0 in range(0, T, tb):
                t1 = min(T, t0 + tb)
                synth.o_block(wl, r, t0, t1, out=on[r, t0:t1])
            mr, sr = synth.stats_block(wl, r)
            self.m_h[r].numpy()[...] = mr
            self.s_h[r].numpy()[...] = sr
        self.in_bytes = self.o_h.numel() * 2 + self.m_h.numel() * 4 + self.s_h.numel() * 4
        self.nsets = rotation_sets(wl)
        o_d = self.o_h.to(dev).view(self.tdt)
        m_d = self.m_h.to(dev)
        s_d = self.s_h.to(dev)
        self.sets = []
        for i in range(self.nsets):
            oi = o_d if i == 0 else o_d.clone()
            mi = m_d if i == 0 else m_d.clone()
            si = s_d if i == 0 else s_d.clone()
            out = torch.empty((W, T, Hc, D), dtype=self.tdt, device=dev)
            ol = torch.empty((W, T, Hc), dtype=torch.float32, device=dev)
            self.sets.append((oi, mi, si, out, ol))

    def host(self):
        return self.o_h.numpy().view(np.uint16), self.m_h.numpy(), self.s_h.numpy()


def fused_stepper(cp, wl, sets, stream):
    """step(i): one fused call on set i mod len(sets), with pre-marshalled
    C-ABI arguments (one ctypes call per step)."""
    sh = stream.cuda_stream

    def cargs(oi, mi, si, out, ol):
        return (oi.data_ptr(), cp._strides3(oi), mi.data_ptr(), cp._strides3(mi), si.data_ptr(),
                cp._strides3(si), wl.W, wl.T, wl.H, wl.D, cp._dtype(oi), 1, out.data_ptr(),
                ol.data_ptr(), sh)
    call_args = [cargs(*st) for st in sets]
    fused = cp._lib.cp_pack_permute_combine_fused
    n = len(sets)

    def step(i):
        st = fused(*call_args[i % n])
        if st != 0:
            raise cp.CplseError(st, cp.last_error())
    return step


def hold_device(stream, ms):
    """Keep the stream busy for about `ms` milliseconds (a bounded clock spin),
    so that the host enqueues the launches that follow before the device
    reaches them: a timed launch then never includes host-side issue time,
    whatever the cost of marshalling and validating one call."""
    import torch
    with torch.cuda.stream(stream):
        torch.cuda._sleep(int(ms * 1e-3 * 2.0e9))


def time_back_to_back(step, stream, K, Wm, barrier):
    """Device time (ms) of K back-to-back steps after Wm untimed ones, one event
    pair around the whole region, barriers and synchronisations on both sides."""
    import torch
    for i in range(Wm):
        step(i)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    hold_device(stream, 2.0)
    a.record(stream)
    for i in range(K):
        step(i)
    b.record(stream)
    torch.cuda.synchronize()
    barrier()
    return a.elapsed_time(b)


def time_launches(fn, stream, reps, warm=3, hold_ms=None):
    """Device time (ms) of each of `reps` calls, each bracketed by its own event
    pair on the launching stream; calls follow each other with no host wait,
    one synchronisation at the end."""
    import torch
    for i in range(warm):
        fn(i)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    hold_device(stream, hold_ms if hold_ms is not None else max(2.0, 0.2 * reps))
    for i in range(reps):
        ev[i][0].record(stream)
        fn(i)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def launch_stats(ms, nbytes, peak):
    """Median / p10 / p90 of per-launch times and the median's throughput."""
    med = statistics.median(ms)
    gbs = nbytes / (med * 1e-3) / 1e9
    return {"us": round(med * 1e3, 3),
            "us_p10_p50_p90": [round(1e3 * pct(ms, q), 3) for q in (10, 50, 90)],
            "bytes": nbytes, "GB/s": round(gbs, 1), "frac": round(gbs / peak, 4),
            "launches": len(ms)}


def measure_workload(cp, wl, dev, stream, args, world, barrier, peak, peak_kind, headline):
    """Everything the line reports for one workload: K back-to-back steps (the
    throughput), a roofline pass of separately bracketed launches, and, as
    asked for, the end-to-end leg, the kernel breakdown and the CPU baseline."""
    import torch
    rank, local_rank, _ = env_rank()
    inp = Inputs(wl, dev, pinned=headline and not args.no_e2e)
    step = fused_stepper(cp, wl, inp.sets, stream)
    bytes_per_call = wl.fused_bytes()
    K, Wm = max(1, args.steps), max(3, args.warmup)

    clocks = ClockSampler(dev.index)
    clocks.start()
    total_ms = time_back_to_back(step, stream, K, Wm, barrier)
    launch_ms = time_launches(step, stream, max(ROOFLINE_LAUNCHES, args.launches))
    clocks.stop()
    med_launch = statistics.median(launch_ms)
    total_ms, med_launch = reduce_max([total_ms, med_launch], world, dev)
    ms_per_step = total_ms / K
    value = job_throughput(world, bytes_per_call, K, total_ms)

    achieved = bytes_per_call / (med_launch * 1e-3) / 1e9
    overlapped = bytes_per_call / (ms_per_step * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": recorded_traffic(wl.name),
                "peak_source": peak_source(peak_kind), "kernel": merge_kernel_name(wl.W, wl.D),
                "algorithmic_bytes_per_launch": bytes_per_call,
                "us_per_launch": round(med_launch * 1e3, 3),
                "us_per_launch_p10_p50_p90": [round(1e3 * pct(launch_ms, q), 3)
                                              for q in (10, 50, 90)],
                "launches_timed": len(launch_ms),
                "overlapped": {"us_per_call": round(ms_per_step * 1e3, 3),
                               "GB/s": round(overlapped, 2),
                               "frac": round(overlapped / peak, 4),
                               "note": "K back-to-back calls, each scheduled while the previous "
                                       "drains (programmatic dependent launch)"}}
    res = {"value": value, "ms_per_step": ms_per_step, "K": K, "Wm": Wm, "roofline": roofline,
           "clocks": clocks.summary(), "bytes_per_call": bytes_per_call}

    if headline and not args.no_e2e:
        res["e2e"] = measure_e2e(cp, wl, inp, stream, dev, K, Wm, barrier, world)
    if not args.no_breakdown and world == 1:
        res["breakdown"] = measure_breakdown(cp, wl, inp.sets, stream, dev, peak)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        o, m, s = inp.host()
        res["cpu_baseline"] = cpu_baseline(wl, o, m, s, 15.0 if headline else 8.0,
                                           5.0 if headline else 0.0)
    del inp, step
    gc.collect()
    torch.cuda.empty_cache()
    return res


def run_ours(args):
    import torch
    import torch.distributed as dist

    import lse_pack_stable_b200 as cp

    rank, local_rank, world = env_rank()
    # one process per GPU; with fewer GPUs than ranks (the host-collective test
    # of this path) ranks share devices
    device_index = local_rank % torch.cuda.device_count()
    torch.cuda.set_device(device_index)
    dev = torch.device("cuda", device_index)
    peak, peak_kind = measured_peak()
    if world > 1:
        # the communicator's own log stays on; no NVLink multicast (NVLS) objects
        os.environ.setdefault("NCCL_DEBUG", "INFO")
        os.environ.setdefault("NCCL_NVLS_ENABLE", "0")
        backend = os.environ.get("CPLSE_BENCH_BACKEND", "nccl")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120),
                                device_id=dev if backend == "nccl" else None)
        try:
            return run_exchange(args, cp, dev, rank, local_rank, world, peak, peak_kind)
        finally:
            dist.destroy_process_group()

    def barrier():
        pass

    wl = synth.CONFIGS[args.config]
    if args.tokens > 0:
        wl = synth.Workload(**{**wl.__dict__, "T": args.tokens})
    stream = torch.cuda.current_stream(dev)

    head = measure_workload(cp, wl, dev, stream, args, 1, barrier, peak, peak_kind, True)

    per_config = None
    names = [] if args.per_config in ("", "none") else args.per_config.split(",")
    if names:
        per_config = {}
        for name in names:
            if name == args.config:
                continue
            r = measure_workload(cp, synth.CONFIGS[name], dev, stream, args, 1, barrier, peak,
                                 peak_kind, False)
            per_config[name] = {
                "config": config_block(synth.CONFIGS[name], 1),
                "us_per_call": round(r["ms_per_step"] * 1e3, 3),
                "GB/s": round(r["value"], 2), "steps": r["K"], "roofline": r["roofline"],
                "clocks": r["clocks"], "cpu_baseline": r.get("cpu_baseline"),
                "breakdown": r.get("breakdown")}

    line = {
        "metric": METRIC, "value": round(head["value"], 2), "unit": "GB/s", "n_gpus": world,
        "steps": head["K"], "warmup": head["Wm"], "ms_per_step": round(head["ms_per_step"], 5),
        "us_per_call": round(head["ms_per_step"] * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "payload_dtype": wl.dtype,
        "data": "synthetic (seeded counter-based generator, the workload's shapes and distributions)",
        "config": config_block(wl, 1),
        "roofline": head["roofline"], "clocks": head["clocks"], "gpu_launches": head["K"],
        "e2e": head.get("e2e"), "cpu_baseline": head.get("cpu_baseline"),
        "breakdown": head.get("breakdown"), "per_config": per_config,
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------------------------
# N > 1 GPUs: the exchange across real ranks

NVLINK_PEER_GBS = 770.0        # measured B200 peer copy over NVLink 5, per direction per GPU


def run_exchange(args, cp, dev, rank, local_rank, world, peak, peak_kind):
    """One rank per GPU, W = N. Each step is the whole exchange for every
    destination at once: rank j pulls head chunk j of every rank's planes
    (PullExchange: barrier, cp_pull_combine, barrier). The NCCL path (pack,
    two all-to-alls, combine) is timed the same way as the baseline, and the
    two must agree bit for bit on every rank."""
    import torch
    import torch.distributed as dist
    from lse_pack_stable_b200.exchange import A2aExchange, PeerMapError, PullExchange

    wl = workload_for(args.config, world)
    if args.tokens > 0:
        wl = synth.Workload(**{**wl.__dict__, "T": args.tokens})
    T, H, D, Hc = wl.T, wl.H, wl.D, wl.H // world
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float16
    stream = torch.cuda.current_stream(dev)

    # this rank's plane of the N-rank workload, generated on the host (pinned:
    # the end-to-end leg uploads from there)
    o_h = torch.empty((T, H, D), dtype=torch.int16, pin_memory=True)
    on = o_h.numpy().view(np.uint16)
    tb = max(1, (256 << 20) // (H * D * 2))
    for t0 in range(0, T, tb):
        synth.o_block(wl, rank, t0, min(T, t0 + tb), out=on[t0:min(T, t0 + tb)])
    mr, sr = synth.stats_block(wl, rank)
    m_h = torch.from_numpy(mr).pin_memory()
    s_h = torch.from_numpy(sr).pin_memory()

    # The pull path needs every rank's planes mapped into every process. If that
    # fails on any rank, every rank learns it at the same point (PeerMapError)
    # and the line times the NCCL path instead, saying why.
    try:
        pull, pull_error = PullExchange(T, H, D, tdt, dev), None
        planes = (pull.o, pull.smax, pull.ssum)
    except PeerMapError as e:
        pull, pull_error = None, str(e)
        planes = (torch.empty((T, H, D), dtype=tdt, device=dev),
                  torch.empty((T, H), dtype=torch.float32, device=dev),
                  torch.empty((T, H), dtype=torch.float32, device=dev))
    planes[0].view(torch.int16).copy_(o_h)
    planes[1].copy_(m_h)
    planes[2].copy_(s_h)
    a2a = A2aExchange(T, H, D, tdt, dev)
    out_p = torch.empty((T, Hc, D), dtype=tdt, device=dev)
    lse_p = torch.empty((T, Hc), dtype=torch.float32, device=dev)
    out_a = torch.empty_like(out_p)
    lse_a = torch.empty_like(lse_p)

    def barrier():
        dist.barrier()

    def a2a_step(i):
        a2a(*planes, out_a, lse_a)

    if pull is not None:
        def step(i):
            pull(out_p, lse_p)
    else:
        step = a2a_step

    K, Wm = max(1, args.steps), max(3, args.warmup)
    # the two paths agree bit for bit (checked on every rank, then reduced)
    step(0)
    a2a_step(0)
    torch.cuda.synchronize()
    same = torch.tensor([float(pull is not None
                               and torch.equal(out_p.view(torch.int16), out_a.view(torch.int16))
                               and torch.equal(lse_p.view(torch.int32), lse_a.view(torch.int32)))],
                        device=dev)
    dist.all_reduce(same, op=dist.ReduceOp.MIN)

    clocks = ClockSampler(dev.index)
    clocks.start()
    pull_ms = time_back_to_back(step, stream, K, Wm, barrier)
    a2a_ms = time_back_to_back(a2a_step, stream, K, Wm, barrier)
    # per call, the slowest rank (the FastVideo page's rank-max p50/p95)
    pull_calls = rank_max_calls(step, stream, K, world, dev) if pull is not None else None
    a2a_calls = rank_max_calls(a2a_step, stream, K, world, dev)
    clocks.stop()
    pull_ms, a2a_ms = reduce_max([pull_ms, a2a_ms], world, dev)
    bytes_per_call = wl.fused_bytes()                 # every rank's reads and writes together
    value = bytes_per_call * K / (pull_ms * 1e-3) / 1e9
    # NVLink roofline: each destination reads (W-1) of its W contributions from
    # peers (pull); the all-to-all sends (W-1) of its W packet blocks
    if pull is not None:
        remote = (world - 1) * T * Hc * (2 * D + 8)
    else:
        remote = (world - 1) * T * Hc * (2 * D + 4)
    achieved = remote / (pull_ms / K * 1e-3) / 1e9

    # end to end through the public API: upload this rank's plane into its
    # shared buffers, exchange, download this destination's rows
    ho = torch.empty((T, Hc, D), dtype=torch.int16, pin_memory=True)
    hl = torch.empty((T, Hc), dtype=torch.float32, pin_memory=True)

    def e2e_step(i):
        planes[0].view(torch.int16).copy_(o_h, non_blocking=True)
        planes[1].copy_(m_h, non_blocking=True)
        planes[2].copy_(s_h, non_blocking=True)
        step(i)
        res_o, res_l = (out_p, lse_p) if pull is not None else (out_a, lse_a)
        ho.copy_(res_o.view(torch.int16), non_blocking=True)
        hl.copy_(res_l, non_blocking=True)
    ke = max(3, min(K, 20))
    e2e_ms = reduce_max([time_back_to_back(e2e_step, stream, ke, 3, barrier)], world, dev)[0]
    h2d = o_h.numel() * 2 + m_h.numel() * 4 + s_h.numel() * 4
    d2h = ho.numel() * 2 + hl.numel() * 4

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": Wm, "ms_per_step": round(pull_ms / K, 5),
        "us_per_call": round(pull_ms / K * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "payload_dtype": wl.dtype,
        "data": "synthetic (seeded counter-based generator, the workload's shapes and distributions)",
        "config": config_block(wl, world),
        "roofline": {"bound": "nvlink", "achieved": round(achieved, 2), "peak": NVLINK_PEER_GBS,
                     "unit": "GB/s", "frac": round(achieved / NVLINK_PEER_GBS, 4),
                     "traffic": None,
                     "kernel": ("pull_combine_kernel (plain loads over NVLink)" if pull is not None
                                else "NCCL all-to-all between cp_pack_lse_rank and "
                                     "cp_lse_combine_rank (pull path unavailable)"),
                     "peak_source": "measured B200 peer copy per direction (770 GB/s)",
                     "nvlink_bytes_per_rank_per_call": remote},
        "clocks": clocks.summary(),
        # this package's kernels per step: the pull kernel, or the per-rank pack and combine
        "gpu_launches": K if pull is not None else 2 * K,
        "e2e": {"value": round(bytes_per_call * ke / (e2e_ms * 1e-3) / 1e9, 3), "unit": "GB/s",
                "h2d_bytes_per_step": h2d * world, "d2h_bytes_per_step": d2h * world,
                "ms_per_step": round(e2e_ms / ke, 4), "steps": ke},
        "exchange": {"timed_path": "pull" if pull is not None else "a2a",
                     "pull_unavailable": pull_error,
                     "pull_equals_a2a": bool(same.item() == 1.0) if pull is not None else None,
                     "pull_rank_max_us_p50_p95": ([round(1e3 * pct(pull_calls, q), 3) for q in (50, 95)]
                                                  if pull_calls is not None else None),
                     "a2a_rank_max_us_p50_p95": [round(1e3 * pct(a2a_calls, q), 3) for q in (50, 95)],
                     "a2a_us_per_call": round(a2a_ms / K * 1e3, 3),
                     "a2a_GB/s": round(bytes_per_call * K / (a2a_ms * 1e-3) / 1e9, 2),
                     "a2a_path": "cp_pack_lse_rank -> NCCL all-to-all x2 -> cp_lse_combine_rank",
                     "hbm_peak_GB/s": peak, "hbm_peak_source": peak_source(peak_kind)},
        "cpu_baseline": None, "breakdown": None, "per_config": None,
    }
    if wl.name == "ulysses":
        line["ulysses_exchange"] = measure_ulysses_exchange(wl, dev, stream, K, Wm, barrier, world)
    if rank == 0:
        print(json.dumps(line), flush=True)
    torch.cuda.synchronize()
    if pull is not None:
        pull.close()
    return 0


def rank_max_calls(fn, stream, reps, world, dev):
    """Each of `reps` calls timed on its own (events around it, a barrier of the
    group before it), then, call by call, the slowest rank's time (ms)."""
    import torch
    import torch.distributed as dist
    for i in range(3):
        fn(i)
    torch.cuda.synchronize()
    ms = []
    for i in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        dist.barrier()
        a.record(stream)
        fn(i)
        b.record(stream)
        torch.cuda.synchronize()
        ms.append(a.elapsed_time(b))
    return reduce_max(ms, world, dev)


def all_to_all_4d_nccl(x, scatter_dim, gather_dim, world, out_shape):
    """The NCCL all-to-all of the Ulysses layout that the load/store exchange
    must match byte for byte: torch reshapes around all_to_all_single
    (seq->head: scatter_dim 2, gather_dim 1; head->seq: the inverse)."""
    import torch
    import torch.distributed as dist
    B, A1, A2, D = x.shape
    if scatter_dim == 2:            # [B, S/W, H, D] -> send [W, B, S/W, H/W, D]
        send = x.reshape(B, A1, world, A2 // world, D).permute(2, 0, 1, 3, 4).contiguous()
    else:                           # [B, S, H/W, D] -> send [W, B, S/W, H/W, D]
        send = x.reshape(B, world, A1 // world, A2, D).permute(1, 0, 2, 3, 4).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv.view(torch.uint8), send.view(torch.uint8))
    if gather_dim == 1:             # [W, B, S/W, Hc, D] -> [B, S, Hc, D]
        return recv.permute(1, 0, 2, 3, 4).reshape(out_shape)
    return recv.permute(1, 2, 0, 3, 4).reshape(out_shape)   # -> [B, S/W, H, D]


def measure_ulysses_exchange(wl, dev, stream, K, Wm, barrier, world):
    """The Ulysses transforms across the N GPUs: q/k/v (B = 3) seq->head and o
    (B = 1) head->seq by load/store over NVLink (UlyssesPullExchange), against
    the NCCL all_to_all_4D; both must agree bit for bit."""
    import torch
    import torch.distributed as dist
    from lse_pack_stable_b200.exchange import PeerMapError, UlyssesPullExchange

    rank = dist.get_rank()
    S, H, D = wl.T, wl.H, wl.D
    Bq, Bo = wl.ulysses_B
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float16
    try:
        ex = UlyssesPullExchange(Bq, Bo, S, H, D, tdt, dev)
    except PeerMapError as e:       # raised on every rank alike
        return {"unavailable": str(e)}
    wlr = synth.Workload(**{**wl.__dict__, "W": world})
    ex.seq.view(torch.int16).copy_(torch.from_numpy(
        synth.ulysses_seq_block(wlr, rank).view(np.int16)))
    ex.head.view(torch.int16).copy_(torch.from_numpy(
        synth.ulysses_head_block(wlr, rank).view(np.int16)))
    y = torch.empty((Bq, S, H // world, D), dtype=tdt, device=dev)
    z = torch.empty((Bo, S // world, H, D), dtype=tdt, device=dev)
    ex.seq2head(out=y)
    ex.head2seq(out=z)
    y_ref = all_to_all_4d_nccl(ex.seq, 2, 1, world, y.shape)
    z_ref = all_to_all_4d_nccl(ex.head, 1, 2, world, z.shape)
    torch.cuda.synchronize()
    same = torch.tensor([float(torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
                               and torch.equal(z.view(torch.int16), z_ref.view(torch.int16)))],
                        device=dev)
    dist.all_reduce(same, op=dist.ReduceOp.MIN)
    t = {}
    t["seq2head_pull"] = time_back_to_back(lambda i: ex.seq2head(out=y), stream, K, Wm, barrier)
    t["head2seq_pull"] = time_back_to_back(lambda i: ex.head2seq(out=z), stream, K, Wm, barrier)
    t["seq2head_nccl"] = time_back_to_back(
        lambda i: all_to_all_4d_nccl(ex.seq, 2, 1, world, y.shape), stream, K, Wm, barrier)
    t["head2seq_nccl"] = time_back_to_back(
        lambda i: all_to_all_4d_nccl(ex.head, 1, 2, world, z.shape), stream, K, Wm, barrier)
    names = list(t)
    ms = dict(zip(names, reduce_max([t[n] for n in names], world, dev)))
    torch.cuda.synchronize()
    ex.close()
    return {"pull_equals_nccl": bool(same.item() == 1.0),
            **{n + "_us": round(ms[n] / K * 1e3, 3) for n in names},
            "bytes_per_rank": {"seq2head": ex.seq.numel() * ex.seq.element_size(),
                               "head2seq": ex.head.numel() * ex.head.element_size()},
            "note": "q/k/v [3, S/W, H, D] seq->head and o [1, S, H/W, D] head->seq per rank; "
                    "NCCL: all_to_all_single between torch reshapes"}


def measure_e2e(cp, wl, inp, stream, dev, K, Wm, barrier, world):
    """Same metric, end to end through the public API with host buffers: every
    step copies its inputs from pinned host memory to the device, runs the
    fused call, and copies its outputs back to pinned host memory. Consecutive
    steps are pipelined on two streams over two device buffer sets, so step
    i+1's upload overlaps step i's download on the full-duplex host link."""
    import torch
    sets = list(inp.sets)
    if len(sets) < 2:
        # a second device buffer set, so that step i+1's upload overlaps step i
        sets.append(tuple(torch.empty_like(t) for t in sets[0]))
    o_h, m_h, s_h = inp.o_h, inp.m_h, inp.s_h
    nb = 2
    up = torch.cuda.Stream(dev)              # host -> device
    work = torch.cuda.Stream(dev)            # kernel, then device -> host
    ho = [torch.empty(sets[0][3].shape, dtype=torch.int16, pin_memory=True) for _ in range(nb)]
    hl = [torch.empty(sets[0][4].shape, dtype=torch.float32, pin_memory=True) for _ in range(nb)]
    h2d = o_h.numel() * 2 + m_h.numel() * 4 + s_h.numel() * 4
    d2h = ho[0].numel() * 2 + hl[0].numel() * 4
    loaded = [torch.cuda.Event() for _ in range(nb)]
    consumed = [torch.cuda.Event() for _ in range(nb)]
    fetched = [torch.cuda.Event() for _ in range(nb)]

    def one(i):
        k = i % nb
        oi, mi, si, out, ol = sets[k]
        with torch.cuda.stream(up):
            if i >= nb:
                up.wait_event(consumed[k])    # the kernel of step i-nb has read this set
            oi.view(torch.int16).copy_(o_h, non_blocking=True)
            mi.copy_(m_h, non_blocking=True)
            si.copy_(s_h, non_blocking=True)
            loaded[k].record(up)
        with torch.cuda.stream(work):
            work.wait_event(loaded[k])
            if i >= nb:
                work.wait_event(fetched[k])   # step i-nb's outputs have left this set
            cp.cp_pack_permute_combine_fused(oi, mi, si, out=out, out_lse=ol, stream=work)
            consumed[k].record(work)
            ho[k].copy_(out.view(torch.int16), non_blocking=True)
            hl[k].copy_(ol, non_blocking=True)
            fetched[k].record(work)

    ke = max(3, min(K, 50))
    for i in range(max(3, min(Wm, 5))):
        one(i)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    a.record(up)
    for i in range(ke):
        one(i)
    work.wait_stream(up)
    b.record(work)
    torch.cuda.synchronize()
    barrier()
    ms = reduce_max([a.elapsed_time(b) / ke], world, dev)[0]
    return {"value": round(job_throughput(world, wl.fused_bytes(), 1, ms), 3), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 4),
            "steps": ke, "note": "GB/s of the kernel's algorithmic bytes; each step uploads its "
                                 "inputs and downloads its outputs (pinned host memory), steps "
                                 "pipelined on two streams; bound by the host link"}


# --------------------------------------------------------------------------------------------
# the Before/After comparison of the DCP pull request, with its paired protocol

def paired_ab(base, cand, stream, warmup=10, blocks=8, samples=5, null_blocks=4):
    """Paired, interleaved A/B of two callables in a fixed order.

    The protocol of the DCP pull request ("Performance evidence"): warm-up
    iterations of both arms; `blocks` paired blocks, each timing `samples`
    event-bracketed calls of the baseline and then `samples` of the candidate;
    baseline-only null-control blocks (baseline against itself, same shape)
    before and after; no samples added afterwards. A block's effect is the
    relative improvement of the candidate's median over the baseline's. The
    noise floor is the median absolute effect of the null-control blocks. The
    rule fixed before measuring: positive if at least 75 % of the paired blocks
    favour the candidate and the median paired improvement exceeds
    max(1 %, 2 x noise floor); a regression under the mirror-image rule;
    otherwise neutral."""
    import torch

    def timed(fn, k):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(samples)]
        hold_device(stream, 2.0)
        for i in range(samples):
            ev[i][0].record(stream)
            fn(k * samples + i)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in ev]

    def block(a_fn, b_fn, k):
        ta = statistics.median(timed(a_fn, k))
        tb = statistics.median(timed(b_fn, k))
        return ta, tb, (ta - tb) / ta

    for i in range(warmup):
        base(i)
        cand(i)
    torch.cuda.synchronize()
    pre = [block(base, base, k) for k in range(null_blocks)]
    main = [block(base, cand, k) for k in range(blocks)]
    post = [block(base, base, k) for k in range(null_blocks)]
    rec = {"baseline_median_us": round(1e3 * statistics.median(a for a, _, _ in main), 3),
           "candidate_median_us": round(1e3 * statistics.median(b for _, b, _ in main), 3)}
    rec.update(ab_decision([e for _, _, e in main], [e for _, _, e in pre + post]))
    rec["protocol"] = ("%d warm-ups; %d paired blocks x %d samples per arm, baseline first; "
                       "%d + %d baseline-only null-control blocks before and after"
                       % (warmup, blocks, samples, null_blocks, null_blocks))
    return rec


def ab_decision(effects, null_effects):
    """The decision rule of the paired A/B. `effects` are the paired blocks'
    relative improvements of the candidate (positive: candidate faster),
    `null_effects` those of the baseline-only null-control blocks."""
    blocks = len(effects)
    noise = statistics.median(abs(e) for e in null_effects)
    effect = statistics.median(effects)
    favour = sum(1 for e in effects if e > 0)
    thresh = max(0.01, 2 * noise)
    if favour >= 0.75 * blocks and effect > thresh:
        verdict = "positive"
    elif blocks - favour >= 0.75 * blocks and -effect > thresh:
        verdict = "regression"
    else:
        verdict = "neutral"
    return {"paired_median_effect": round(effect, 5),
            "blocks_favouring_candidate": "%d/%d" % (favour, blocks),
            "noise_floor": round(noise, 5), "threshold": round(thresh, 5), "verdict": verdict}


def measure_breakdown(cp, wl, sets, stream, dev, peak):
    """Per-kernel times of the unfused path (and the Ulysses transforms on the
    Ulysses workload), each against its own algorithmic bytes, with the
    Before/After A/B of the pack. Inputs rotate over the device sets as in the
    timed region. Each figure is the median (p10, p90 beside it) of 20
    separately event-bracketed launches."""
    import torch
    W, T, H, D, Hc = wl.W, wl.T, wl.H, wl.D, wl.Hc
    tdt = sets[0][0].dtype
    n = len(sets)
    # two packet buffers alternate (L2 rotation) unless one alone exceeds L2 many times
    nb = 2 if W * T * H * D * 2 < 2e9 else 1
    pk = [(torch.empty((W, W, T, Hc, D), dtype=tdt, device=dev),
           torch.empty((W, W, T, Hc), dtype=torch.float32, device=dev)) for _ in range(nb)]
    rv = [(torch.empty_like(pk[0][0]), torch.empty_like(pk[0][1])) for _ in range(nb)]
    res = {}

    def rec(name, fn, nbytes, reps=20, hold_ms=None):
        res[name] = launch_stats(time_launches(fn, stream, reps, hold_ms=hold_ms), nbytes, peak)

    def pack(i):
        cp.cp_pack_lse(*sets[i % n][:3], pkt_o=pk[i % nb][0], pkt_lse=pk[i % nb][1], stream=stream)
    rec("pack", pack, wl.pack_bytes())
    if T % W == 0:
        # the token-chunk packet (scatter_dim = 0) in the same buffers, viewed [W][W][T/W][H]
        tpk = [(p[0].view(W, W, T // W, H, D), p[1].view(W, W, T // W, H)) for p in pk]

        def pack_tokens(i):
            cp.cp_pack_lse(*sets[i % n][:3], scatter_dim=0, pkt_o=tpk[i % nb][0],
                           pkt_lse=tpk[i % nb][1], stream=stream)
        rec("pack_token_chunks", pack_tokens, wl.pack_bytes())
        del tpk
    rows = W * T * H
    # the Before pipeline of the DCP pull request: materialize LSE, then pack from it
    lse_buf = torch.empty((W, T, H), dtype=torch.float32, device=dev)

    def legacy(i):
        oi, mi, si = sets[i % n][:3]
        cp.cp_lse_materialize(mi, si, lse=lse_buf, stream=stream)
        cp.cp_pack_from_lse(oi, lse_buf, pkt_o=pk[i % nb][0], pkt_lse=pk[i % nb][1], stream=stream)
    legacy_bytes = rows * (8 + 4) + rows * (2 * D * 2 + 4 + 4)
    rec("legacy_pack", legacy, legacy_bytes)
    res["legacy_over_pack"] = round(res["legacy_pack"]["us"] / res["pack"]["us"], 3)
    res["legacy_ab"] = paired_ab(legacy, pack, stream)
    del lse_buf

    def perm(i):
        cp.cp_a2a_local_permute(pk[i % nb][0], W, recv=rv[i % nb][0], stream=stream)
        cp.cp_a2a_local_permute(pk[i % nb][1], W, recv=rv[i % nb][1], stream=stream)
    rec("permute", perm, 2 * rows * (D * 2 + 4))
    outs = [(torch.empty((W, T, Hc, D), dtype=tdt, device=dev),
             torch.empty((W, T, Hc), dtype=torch.float32, device=dev)) for _ in range(nb)]
    rec("combine", lambda i: cp.cp_lse_combine(*rv[i % nb], out=outs[i % nb][0],
                                               out_lse=outs[i % nb][1], stream=stream),
        wl.combine_bytes())
    res["unfused_total_us"] = round(res["pack"]["us"] + res["permute"]["us"] + res["combine"]["us"], 2)
    del pk, rv, outs
    if T % W == 0:
        # the fused exchange of token chunks (same bytes, output in source order)
        touts = [(torch.empty((W, T // W, H, D), dtype=tdt, device=dev),
                  torch.empty((W, T // W, H), dtype=torch.float32, device=dev)) for _ in range(nb)]
        rec("fused_token_chunks",
            lambda i: cp.cp_pack_permute_combine_fused(*sets[i % n][:3], out=touts[i % nb][0],
                                                       out_lse=touts[i % nb][1], scatter_dim=0,
                                                       stream=stream),
            wl.fused_bytes())
        del touts
    # the pull kernel of the exchange across GPUs, here reading the W planes of
    # this GPU's own input (HBM, not NVLink): every destination at once, one
    # launch each on its own stream, as the W GPUs of a real exchange read every
    # rank's memory concurrently
    import ctypes
    pstreams = [torch.cuda.Stream(dev) for _ in range(W)]
    forked, joined = torch.cuda.Event(), [torch.cuda.Event() for _ in range(W)]
    pull_args = []
    for st in sets:
        oi, mi, si, out, ol = st
        tabs = [(ctypes.c_void_p * W)(*[t[r].data_ptr() for r in range(W)]) for t in (oi, mi, si)]
        pull_args.append([(tabs[0], cp._strides_plane(oi[0]), tabs[1], cp._strides_plane(mi[0]),
                           tabs[2], cp._strides_plane(si[0]), W, T, H, D, cp._dtype(oi), 1, j,
                           out[j].data_ptr(), ol[j].data_ptr(), pstreams[j].cuda_stream)
                          for j in range(W)])

    def pull_all(i):
        forked.record(stream)
        for j, args in enumerate(pull_args[i % n]):
            pstreams[j].wait_event(forked)
            st_ = cp._lib.cp_pull_combine(*args)
            if st_ != 0:
                raise cp.CplseError(st_, cp.last_error())
            joined[j].record(pstreams[j])
        for ev in joined:
            stream.wait_event(ev)
    rec("pull_all_destinations", pull_all, wl.fused_bytes(), hold_ms=max(2.0, 0.1 * 20 * W))
    res["pull_all_destinations"]["note"] = (
        "one-GPU stand-in for the exchange across GPUs: W destination kernels on W streams, each "
        "filling the GPU and reading one head chunk of every row from this GPU's HBM; across N "
        "GPUs each destination reads (N-1)/N of its bytes over NVLink, which bounds it there")
    del pull_args, pstreams
    # context for the fused share at this size: a plain device-to-device copy
    # moving the fused kernel's byte count (half read, half written), timed the
    # same way, its source rotating over the same sets
    half = wl.fused_bytes() // 32 * 16
    srcs = [s[0].reshape(-1).view(torch.uint8)[:half] for s in sets]
    dsts = [torch.empty(half, dtype=torch.uint8, device=dev) for _ in range(nb)]
    rec("copy_same_bytes", lambda i: dsts[i % nb].copy_(srcs[i % n]), 2 * half)
    del srcs, dsts
    if wl.name == "ulysses":
        S_l = T // W
        xs = [torch.empty((W, 3, S_l, H, D), dtype=tdt, device=dev).normal_() for _ in range(2)]
        ys = [torch.empty((W, 3, T, Hc, D), dtype=tdt, device=dev) for _ in range(2)]
        rec("ulysses_seq2head", lambda i: cp.ulysses_seq2head(xs[i % 2], out=ys[i % 2],
                                                              stream=stream),
            2 * xs[0].numel() * 2)
        # the load/store exchange across GPUs: every destination at once, one
        # launch each on its own stream, from the W planes of this GPU
        ustreams = [torch.cuda.Stream(dev) for _ in range(W)]
        ufork, ujoin = torch.cuda.Event(), [torch.cuda.Event() for _ in range(W)]
        uargs = []
        for x, y in zip(xs, ys):
            tab = (ctypes.c_void_p * W)(*[x[r].data_ptr() for r in range(W)])
            uargs.append([(tab, y[j].data_ptr(), W, 3, S_l, H, D, 2, j, ustreams[j].cuda_stream)
                          for j in range(W)])

        def uly_pull_all(i):
            ufork.record(stream)
            for j, args in enumerate(uargs[i % 2]):
                ustreams[j].wait_event(ufork)
                st_ = cp._lib.ulysses_seq2head_pull(*args)
                if st_ != 0:
                    raise cp.CplseError(st_, cp.last_error())
                ujoin[j].record(ustreams[j])
            for ev in ujoin:
                stream.wait_event(ev)
        rec("ulysses_seq2head_pull_all_destinations", uly_pull_all, 2 * xs[0].numel() * 2,
            hold_ms=max(2.0, 0.1 * 20 * W))
        del xs, ys, uargs, ustreams
        hs = [torch.empty((W, 1, T, Hc, D), dtype=tdt, device=dev).normal_() for _ in range(2)]
        gs = [torch.empty((W, 1, S_l, H, D), dtype=tdt, device=dev) for _ in range(2)]
        rec("ulysses_head2seq", lambda i: cp.ulysses_head2seq(hs[i % 2], out=gs[i % 2],
                                                              stream=stream),
            2 * hs[0].numel() * 2)
        del hs, gs
    torch.cuda.synchronize()
    return res


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
