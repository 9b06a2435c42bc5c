"""Benchmark of the DCP exchange hot path on B200: fused pack -> all-to-all ->
stable log-sum-exp combine, through the C-ABI of libcplse.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config decode] [--impl ours|reference]

One step = one call of cp_pack_permute_combine_fused over one batch: the whole
DCP path (LSE formation, head-chunk pack, the W x W block exchange, combine)
in one pass. `value` is the effective HBM throughput of that step, algorithmic
bytes W*T*H*(2D+8) + T*H*(2D+4) per call over the device time, summed over
ranks (each rank runs its own independent batch: weak scaling, no collective
on the data path). The breakdown times the unfused kernels and, for the
Ulysses workload, the layout transforms, outside the timed region.

--impl reference times the float64 CPU oracle (rank 0 only) on a bounded
sample of the same workload, on the host cores.

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import datetime
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
KERNEL_SOURCES = ["lse_pack_stable_b200/csrc/rowcombine_async.cuh",
                  "lse_pack_stable_b200/csrc/rowcombine_async.cu",
                  "lse_pack_stable_b200/csrc/rowcombine.cuh", "lse_pack_stable_b200/csrc/common.cuh"]


def parse():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", default="decode", choices=sorted(synth.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-breakdown", action="store_true")
    return ap.parse_args()


def env_rank():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def config_block(wl: synth.Workload, world: int, extra=None):
    c = {"workload": "%s: W=%d simulated ranks, T=%d, H=%d, D=%d, %s payload, fp32 max/sum"
                     % (wl.name, wl.W, wl.T, wl.H, wl.D, wl.dtype),
         "W": wl.W, "T": wl.T, "H": wl.H, "D": wl.D, "payload_dtype": wl.dtype,
         "global_batch": world, "parallelism": "replicas%d" % world,
         "bytes_per_call": wl.fused_bytes()}
    if extra:
        c.update(extra)
    return c


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


def kernel_source_hash():
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(config: str):
    """DRAM bytes per launch of the fused kernel from the committed ncu summary,
    if it was taken on the current kernel source (else None)."""
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


# --------------------------------------------------------------------------------------------
# clocks during the timed region (NVML)

class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, index: int, period_s: float = 0.01):
        self.samples, self.reasons, self.ok = [], set(), False
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = str(e)
            self.max_mhz = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                mask = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if mask & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()

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


def run_reference(args):
    rank, _, world = env_rank()
    if rank != 0:
        return 0
    wl = synth.CONFIGS[args.config]
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
        "data": "synthetic (seeded counter-based generator, the workload's shapes and distributions)",
        "config": config_block(wl, world), "impl": "reference",
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------------------------
# GPU arm

def run_ours(args):
    import torch
    import torch.distributed as dist

    import lse_pack_stable_b200 as cp

    rank, local_rank, world = env_rank()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    wl0 = synth.CONFIGS[args.config]
    wl = synth.Workload(**{**wl0.__dict__, "seed": wl0.seed + 1000 * rank})
    W, T, H, D, Hc = wl.W, wl.T, wl.H, wl.D, wl.Hc
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float16

    # ---- inputs: generated on the host block by block into pinned memory (the
    # end-to-end leg copies from there), uploaded once; extra device copies
    # rotate so that every step reads cold HBM
    o_h = torch.empty((W, T, H, D), dtype=torch.int16, pin_memory=True)
    m_h = torch.empty((W, T, H), dtype=torch.float32, pin_memory=True)
    s_h = torch.empty((W, T, H), dtype=torch.float32, pin_memory=True)
    tb = max(1, (256 << 20) // (H * D * 2))
    for r in range(W):
        for t0 in range(0, T, tb):
            t1 = min(T, t0 + tb)
            o_h[r, t0:t1].numpy()[...] = synth.o_block(wl, r, t0, t1).view(np.int16)
        mr, sr = synth.stats_block(wl, r)
        m_h[r].numpy()[...] = mr
        s_h[r].numpy()[...] = sr
    in_bytes = o_h.numel() * 2 + m_h.numel() * 4 + s_h.numel() * 4
    out_bytes = T * H * D * 2 + T * H * 4
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    nsets = max(2, math.ceil(3 * l2 / (in_bytes + out_bytes)) + 1)
    nsets = min(nsets, max(2, int(40e9 // (in_bytes + out_bytes))))
    o_d = o_h.to(dev).view(tdt)
    m_d = m_h.to(dev)
    s_d = s_h.to(dev)
    sets = []
    for i in range(nsets):
        oi = o_d if i == 0 else o_d.clone()
        mi = m_d if i == 0 else m_d.clone()
        si = s_d if i == 0 else s_d.clone()
        out = torch.empty((W, T, Hc, D), dtype=tdt, device=dev)
        ol = torch.empty((W, T, Hc), dtype=torch.float32, device=dev)
        sets.append((oi, mi, si, out, ol))
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream

    # pre-marshalled C-ABI arguments: the timed loop is one ctypes call per step
    def cargs(oi, mi, si, out, ol):
        return (oi.data_ptr(), cp._strides3(oi), mi.data_ptr(), cp._strides3(mi), si.data_ptr(),
                cp._strides3(si), W, T, H, D, cp._dtype(oi), 1, out.data_ptr(), ol.data_ptr(), sh)
    call_args = [cargs(*st) for st in sets]
    fused = cp._lib.cp_pack_permute_combine_fused

    def step(i):
        st = fused(*call_args[i % nsets])
        if st != 0:
            raise cp.CplseError(st, cp.last_error())

    bytes_per_call = wl.fused_bytes()
    K, Wm = max(1, args.steps), max(3, args.warmup)

    def barrier():
        if world > 1:
            dist.barrier()

    for i in range(Wm):
        step(i)
    torch.cuda.synchronize()

    # every 8th launch is bracketed by events (its duration is the kernel's);
    # the others run back to back, as a user's stream would
    sample_every = 8
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(0, K, sample_every)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clocks:
        barrier()
        torch.cuda.synchronize()
        t_start.record(stream)
        for i in range(K):
            if i % sample_every == 0:
                ev[i // sample_every][0].record(stream)
                step(i)
                ev[i // sample_every][1].record(stream)
            else:
                step(i)
        t_end.record(stream)
        torch.cuda.synchronize()
        barrier()
    total_ms = t_start.elapsed_time(t_end)
    launch_ms = [a.elapsed_time(b) for a, b in ev]
    mean_launch_ms = sum(launch_ms) / len(launch_ms)
    total_ms, mean_launch_ms = reduce_max([total_ms, mean_launch_ms], world, dev)
    ms_per_step = total_ms / K
    value = job_throughput(world, bytes_per_call, K, total_ms)

    peak, peak_kind = measured_peak()
    achieved = bytes_per_call / (mean_launch_ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": recorded_traffic(args.config),
                "peak_source": peak_kind + " (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                else "fallback 6.65 TB/s", "kernel": ("rowcombine_kernel (register-staged, fused mode)" if W > 8
                           else "rowcombine_async_kernel (shared-memory-staged, fused mode)"),
                "algorithmic_bytes_per_launch": bytes_per_call,
                "us_per_launch": round(mean_launch_ms * 1e3, 3),
                "launches_timed": len(launch_ms),
                "us_per_launch_p10_p50_p90": [round(1e3 * np.percentile(launch_ms, q), 3)
                                              for q in (10, 50, 90)]}

    # ---- end to end through the C-ABI with host buffers (pinned), N GPUs
    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(cp, wl, o_h, m_h, s_h, sets, stream, dev, K, Wm, barrier, world,
                          dist, tdt)

    breakdown = None
    if not args.no_breakdown:
        breakdown = measure_breakdown(cp, wl, sets, stream, dev, peak, tdt)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        host = (o_h.numpy().view(np.uint16), m_h.numpy(), s_h.numpy())
        gbs, _, sample, cores = time_oracle(wl, 15.0, *host)
        gbs1, _, sample1, _ = time_oracle_threads(wl, 5.0, 1, *host)
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": sample,
               "single_thread": {"value": round(gbs1, 4), "unit": "GB/s", "cores": 1,
                                 "sample": sample1}}

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": Wm, "ms_per_step": round(ms_per_step, 5),
        "us_per_call": round(ms_per_step * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded counter-based generator, the workload's shapes and distributions)",
        "config": config_block(wl, world, {
            "l2": "inputs and outputs rotate over %d device sets (%.0f MB each, %.0f MB total > "
                  "3x the %.0f MB L2)" % (nsets, (in_bytes + out_bytes) / 1e6,
                                          nsets * (in_bytes + out_bytes) / 1e6, l2 / 1e6)}),
        "roofline": roofline, "clocks": clocks.summary(), "gpu_launches": K,
        "e2e": e2e, "cpu_baseline": cpu, "breakdown": breakdown,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def measure_e2e(cp, wl, o_h, m_h, s_h, sets, stream, dev, K, Wm, barrier, world, dist, tdt):
    """Same metric, end to end through the public API with host buffers: every
    step copies its inputs from pinned host memory to the device, runs the
    fused call, and copies its outputs back to pinned host memory. Consecutive
    steps are pipelined on two streams over two device buffer sets, so step
    i+1's upload overlaps step i's download on the full-duplex host link."""
    import torch
    nb = min(2, len(sets))
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


def _time(fn, stream, reps=20):
    """Median device time of one call: back-to-back calls, each bracketed by
    events on the launching stream, one synchronisation at the end."""
    import torch
    for i in range(3):
        fn(i)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    for i in range(reps):
        ev[i][0].record(stream)
        fn(i)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in ev)


def measure_breakdown(cp, wl, sets, stream, dev, peak, tdt):
    """Per-kernel times of the unfused path (and the Ulysses transforms on the
    Ulysses workload), each against its own algorithmic bytes. Inputs rotate
    over the device sets as in the timed region."""
    import torch
    W, T, H, D, Hc = wl.W, wl.T, wl.H, wl.D, wl.Hc
    n = len(sets)
    # two packet buffers alternate (L2 rotation) unless one alone exceeds L2 many times
    nb = 2 if W * T * H * D * 2 < 2e9 else 1
    pk = [(torch.empty((W, W, T, Hc, D), dtype=tdt, device=dev),
           torch.empty((W, W, T, Hc), dtype=torch.float32, device=dev)) for _ in range(nb)]
    rv = [(torch.empty_like(pk[0][0]), torch.empty_like(pk[0][1])) for _ in range(nb)]
    res = {}

    def rec(name, ms, nbytes):
        gbs = nbytes / (ms * 1e-3) / 1e9
        res[name] = {"us": round(ms * 1e3, 2), "bytes": nbytes, "GB/s": round(gbs, 1),
                     "frac": round(gbs / peak, 4)}

    rec("pack", _time(lambda i: cp.cp_pack_lse(*sets[i % n][:3], pkt_o=pk[i % nb][0],
                                               pkt_lse=pk[i % nb][1], stream=stream), stream),
        wl.pack_bytes())
    rows = W * T * H
    # the Before pipeline of the DCP pull request: materialize LSE, then pack from it
    lse_buf = torch.empty((W, T, H), dtype=torch.float32, device=dev)

    def legacy(i):
        oi, mi, si = sets[i % n][:3]
        cp.cp_lse_materialize(mi, si, lse=lse_buf, stream=stream)
        cp.cp_pack_from_lse(oi, lse_buf, pkt_o=pk[i % nb][0], pkt_lse=pk[i % nb][1], stream=stream)
    legacy_bytes = rows * (8 + 4) + rows * (2 * D * 2 + 4 + 4)
    rec("legacy_pack", _time(legacy, stream), legacy_bytes)
    res["legacy_over_pack"] = round(res["legacy_pack"]["us"] / res["pack"]["us"], 3)
    del lse_buf

    def perm(i):
        cp.cp_a2a_local_permute(pk[i % nb][0], W, recv=rv[i % nb][0], stream=stream)
        cp.cp_a2a_local_permute(pk[i % nb][1], W, recv=rv[i % nb][1], stream=stream)
    rec("permute", _time(perm, stream), 2 * rows * (D * 2 + 4))
    outs = [(torch.empty((W, T, Hc, D), dtype=tdt, device=dev),
             torch.empty((W, T, Hc), dtype=torch.float32, device=dev)) for _ in range(nb)]
    rec("combine", _time(lambda i: cp.cp_lse_combine(*rv[i % nb], out=outs[i % nb][0],
                                                     out_lse=outs[i % nb][1], stream=stream),
                         stream), wl.combine_bytes())
    unfused_us = res["pack"]["us"] + res["permute"]["us"] + res["combine"]["us"]
    res["unfused_total_us"] = round(unfused_us, 2)
    del pk, rv, outs
    if T % W == 0:
        # the fused exchange of token chunks (same bytes, output in source order)
        touts = [(torch.empty((W, T // W, H, D), dtype=tdt, device=dev),
                  torch.empty((W, T // W, H), dtype=torch.float32, device=dev)) for _ in range(nb)]
        rec("fused_token_chunks",
            _time(lambda i: cp.cp_pack_permute_combine_fused(*sets[i % n][:3], out=touts[i % nb][0],
                                                             out_lse=touts[i % nb][1], scatter_dim=0,
                                                             stream=stream), stream),
            wl.fused_bytes())
        del touts
    # context for the fused share at this size: a plain device-to-device copy
    # moving the fused kernel's byte count (half read, half written), timed the
    # same way, its source rotating over the same sets
    half = wl.fused_bytes() // 32 * 16
    srcs = [s[0].reshape(-1).view(torch.uint8)[:half] for s in sets]
    dsts = [torch.empty(half, dtype=torch.uint8, device=dev) for _ in range(nb)]
    rec("copy_same_bytes", _time(lambda i: dsts[i % nb].copy_(srcs[i % n]), stream), 2 * half)
    del srcs, dsts
    if wl.name == "ulysses":
        S_l = T // W
        xs = [torch.empty((W, 3, S_l, H, D), dtype=tdt, device=dev).normal_() for _ in range(2)]
        ys = [torch.empty((W, 3, T, Hc, D), dtype=tdt, device=dev) for _ in range(2)]
        nb = 2 * xs[0].numel() * 2
        rec("ulysses_seq2head", _time(lambda i: cp.ulysses_seq2head(xs[i % 2], out=ys[i % 2],
                                                                    stream=stream), stream), nb)
        hs = [torch.empty((W, 1, T, Hc, D), dtype=tdt, device=dev).normal_() for _ in range(2)]
        gs = [torch.empty((W, 1, S_l, H, D), dtype=tdt, device=dev) for _ in range(2)]
        nb = 2 * hs[0].numel() * 2
        rec("ulysses_head2seq", _time(lambda i: cp.ulysses_head2seq(hs[i % 2], out=gs[i % 2],
                                                                    stream=stream), stream), nb)
    torch.cuda.synchronize()
    return res


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
