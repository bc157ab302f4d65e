#!/usr/bin/env python
"""Benchmark of the B200 attention forward pass.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {b200,reference}]
                    [--workload NAME]

One step = one attention forward pass (the whole hot path: one kernel launch)
over the workload's batch, inputs resident in HBM.  Prints ONE JSON line on
rank 0.  Multi-GPU (under torchrun): every rank runs its own copy of the
workload (independent batches, no collective on the data path, weak
scaling); the time is the max over ranks.

``--impl reference`` times the CPU oracle (fp64 plain definition) on the
host cores instead, on bounded row samples of the same workload.

``--workload`` also takes the general problems of ``inputs.GENERAL_WORKLOADS``
(a query block against a key/value cache, split keys, a packed
variable-length batch); their line reports the same metric from the exact
number of visible (query, key) pairs, with the roofline bound chosen by
arithmetic intensity.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from tiled_attention_forward_sm_b200.inputs import (BENCH_WORKLOAD,  # noqa: E402
                                                    GENERAL_WORKLOADS, KMEANS_WORKLOADS,
                                                    WORKLOADS, bf16_bits, make_general_inputs,
                                                    make_kmeans_inputs, make_workload_inputs)

METRIC = "attention fwd TFLOPS (bf16, d=128) and % of B200 dense BF16 peak, 1 GPU"
UNIT = "TFLOPS"
FALLBACK_PEAK = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
DATASHEET_BF16_TFLOPS = 2250.0
PROFILE_FILE = os.path.join(ROOT, "profiles", "attn_fwd_b2h32n8192d128_causal.txt")
PAIR_PROFILE_FILE = os.path.join(ROOT, "profiles", "attn_fwd_pair_b2h32n8192d128_causal.txt")
KERNEL_SOURCES = [os.path.join(ROOT, "tiled_attention_forward_sm_b200", "csrc", f)
                  for f in ("attn_fwd_kernel.cuh", "ptx.cuh", "attn_fwd.cu")]
PAIR_SOURCES = KERNEL_SOURCES + [os.path.join(ROOT, "tiled_attention_forward_sm_b200", "csrc", f)
                                 for f in ("attn_fwd_pair_kernel.cuh", "pair.cu")]
CLOCK_QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def kernel_sha(sources=None) -> str:
    h = hashlib.sha256()
    for p in sources or KERNEL_SOURCES:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAK), "fallback"


def load_traffic(workload_name: str, profile_file: str = PROFILE_FILE, sources=None):
    """dram read+write bytes per launch from the committed ncu summary of the
    bench workload, if it was taken on the current kernel sources; else None."""
    if workload_name != BENCH_WORKLOAD or not os.path.exists(profile_file):
        return None
    fields = {}
    with open(profile_file) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                fields[k.strip()] = v.strip()
    if fields.get("kernel_sha") != kernel_sha(sources):
        return None
    try:
        return int(fields["dram_read_write_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ----------------------------------------------------------------- clocks ---
_REASON_BITS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
                0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}


_NVML_SAMPLER = r"""
import os, sys, time, pynvml
pynvml.nvmlInit()
h = pynvml.nvmlDeviceGetHandleByUUID(sys.argv[1])
period, path = float(sys.argv[2]), sys.argv[3]
get = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
    pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
drv = pynvml.nvmlSystemGetDriverVersion()
drv = drv.decode() if isinstance(drv, bytes) else drv
smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
with open(path, "w", buffering=1) as f:
    f.write(f"ready,{smax},{drv}\n")
    while not os.path.exists(path + ".stop"):
        f.write(f"{pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)},"
                f"{pynvml.nvmlDeviceGetPowerUsage(h)},{get(h)}\n")
        time.sleep(period)
"""


class ClockSampler:
    """SM clock, power and clock-event reasons sampled every ``period_s``
    while the GPU works, by read-only NVML queries in a child process (the
    timed region of a short run lasts tens of milliseconds: too short for
    nvidia-smi's 100 ms period, and a thread of this process would wait on
    the interpreter lock).  Falls back to nvidia-smi when NVML cannot be
    used.  Nothing here changes a GPU setting."""

    def __init__(self, dev: torch.device, period_s: float = 0.001):
        self.dev = dev
        self.period = period_s
        self._proc = None
        self._path = None
        self._file = None
        self._kind = None
        self.sm_max = None
        self.driver = None
        self.source = None

    def _tmp_path(self, stem):
        out = os.environ.get("ATTN_BENCH_CLOCKS_DIR") or tempfile.gettempdir()
        os.makedirs(out, exist_ok=True)
        return os.path.join(out, f"{stem}_gpu{self.dev.index}_{os.getpid()}.csv")

    def _start_nvml(self) -> bool:
        props = torch.cuda.get_device_properties(self.dev)
        self._path = self._tmp_path("clocks_nvml")
        for p in (self._path, self._path + ".stop"):
            if os.path.exists(p):
                os.remove(p)
        self._proc = subprocess.Popen(
            [sys.executable, "-c", _NVML_SAMPLER, "GPU-" + str(props.uuid), str(self.period),
             self._path], stdin=subprocess.DEVNULL, stdout=subprocess.DEVNULL,
            stderr=subprocess.DEVNULL)
        t0 = time.time()
        while time.time() - t0 < 20:  # wait until it samples
            if self._proc.poll() is not None:
                return False
            if os.path.exists(self._path):
                with open(self._path) as f:
                    head = f.readline()
                if head.startswith("ready,") and head.endswith("\n"):
                    _, smax, drv = head.strip().split(",", 2)
                    self.sm_max, self.driver = float(smax), drv
                    self._kind = "nvml"
                    self.source = f"nvml in a child process, {self.period * 1e3:g} ms"
                    return True
            time.sleep(0.01)
        return False

    def start(self):
        try:
            if self._start_nvml():
                return
        except Exception:
            pass
        self._kill()
        # fallback: nvidia-smi at its 100 ms period, raw rows in a temp file
        self._path = self._tmp_path("clocks_smi")
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        ids = [x.strip() for x in vis.split(",")] if vis else []
        smi_id = ids[self.dev.index] if len(ids) > self.dev.index else str(self.dev.index)
        try:
            self._file = open(self._path, "w")
            self._proc = subprocess.Popen(
                ["nvidia-smi", f"--id={smi_id}", f"--query-gpu={CLOCK_QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self._file, stderr=subprocess.DEVNULL)
            self._kind = "smi"
            self.source = "nvidia-smi, 100 ms"
        except (OSError, FileNotFoundError):
            self._kill()

    def _kill(self):
        if self._proc is not None and self._proc.poll() is None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
        self._proc = None
        if self._file is not None:
            self._file.close()
            self._file = None

    def _read(self):
        rows = []
        if self._kind == "nvml":
            with open(self._path) as f:
                for line in f.read().splitlines()[1:]:
                    parts = line.split(",")
                    if len(parts) == 3:
                        rows.append((float(parts[0]), float(parts[1]) / 1000.0, int(parts[2])))
            return rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        bit = {v: k for k, v in _REASON_BITS.items()}
        with open(self._path) as f:
            for line in f:
                r = [x.strip() for x in line.split(",")]
                if len(r) < 9 or not r[1].replace(".", "").isdigit():
                    continue
                if r[2].replace(".", "").isdigit():
                    self.sm_max = float(r[2])
                bits = 0
                for i, n in enumerate(names):
                    if r[5 + i] == "Active":
                        bits |= bit[n]
                pw = float(r[3]) if r[3].replace(".", "").isdigit() else float("nan")
                rows.append((float(r[1]), pw, bits))
        return rows

    def stop(self):
        if self._proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock source"],
                    "samples": 0, "source": None}
        if self._kind == "nvml":
            open(self._path + ".stop", "w").close()
            try:
                self._proc.wait(timeout=10)
            except subprocess.TimeoutExpired:
                pass
        self._kill()
        samples = self._read()
        if not os.environ.get("ATTN_BENCH_CLOCKS_DIR"):
            for p in (self._path, self._path + ".stop"):
                if os.path.exists(p):
                    os.remove(p)
        if not samples:
            return {"sm_mhz": None, "sm_max_mhz": self.sm_max, "reasons": [], "samples": 0,
                    "source": self.source}
        sm = [x[0] for x in samples]
        load = [x for x in samples if not (x[2] & 0x1)] or samples  # drop GPU-idle samples
        reasons = sorted({n for x in samples for b, n in _REASON_BITS.items() if x[2] & b})
        return {"sm_mhz": statistics.median(x[0] for x in load),
                "sm_min_mhz": min(sm), "sm_max_mhz": self.sm_max,
                "reasons": reasons, "samples": len(samples), "samples_under_load": len(load),
                "power_w_max": max((x[1] for x in samples), default=None),
                "source": self.source}


# ------------------------------------------------------------ distributed ---
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ---------------------------------------------------------- CPU baseline ---
def oracle_sample_rows(w, n_rows: int, seed: int):
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(w.rows, size=min(n_rows, w.rows), replace=False)).astype(np.int64)


def row_flops(w, rows) -> float:
    """Metric FLOPs attributable to the listed rows: 4*d per visible key
    (the 4*N^2*d total, halved under the mask, is the sum over rows)."""
    i = rows % w.N
    keys = (i + 1) if w.causal else np.full_like(i, w.N)
    return float(4.0 * w.d * keys.astype(np.float64).sum())


def time_oracle(w, bits, target_s: float, seed: int = 123):
    """Run the oracle on growing seeded row batches until about target_s of
    CPU work; return (TFLOPS, rows, seconds, threads, last batch) where the
    last batch is (rows, O, LSE) of the oracle's final call."""
    import oracle  # CPU baseline leg only
    qb, kb, vb = bits
    total_rows, total_t, total_f = 0, 0.0, 0.0
    batch = 1024
    k = 0
    last = None
    while total_t < target_s and total_rows < w.rows:
        rows = oracle_sample_rows(w, batch, seed + k)
        t0 = time.perf_counter()
        o_ref, lse_ref = oracle.attn_ref(qb, kb, vb, w.causal, w.scale, rows=rows)
        dt = time.perf_counter() - t0
        total_t += dt
        total_f += row_flops(w, rows)
        total_rows += len(rows)
        last = (rows, o_ref, lse_ref)
        k += 1
        if dt < 0.5 * target_s:
            batch = min(batch * 2, 65536)
    return total_f / total_t / 1e12, total_rows, total_t, oracle.max_threads(), last


def parity_of_rows(o, lse, w, last):
    """Largest |O - O_oracle| and |LSE - LSE_oracle| over the oracle rows of
    the CPU-baseline leg, against the GPU result of the last timed step, with
    the parity tolerance (|dO| <= 2e-2 + 1e-2 |O|, |dLSE| <= 1e-3)."""
    rows, o_ref, lse_ref = last
    idx = torch.from_numpy(rows).to(o.device)
    o_g = o.reshape(-1, w.d).index_select(0, idx).double().cpu().numpy()
    l_g = lse.reshape(-1).index_select(0, idx).double().cpu().numpy()
    d_o = np.abs(o_g - o_ref)
    d_l = np.abs(l_g - lse_ref)
    ok = bool((d_o <= 2e-2 + 1e-2 * np.abs(o_ref)).all() and (d_l <= 1e-3).all())
    return {"rows": int(len(rows)), "max_abs_dO": float(d_o.max()),
            "max_abs_dLSE": float(d_l.max()), "pass": ok}


def versions(lib, sampler=None) -> dict:
    v = int(lib.attn_version())
    return {"torch": torch.__version__, "cuda_runtime": torch.version.cuda,
            "driver": getattr(sampler, "driver", None),
            "library": f"{v >> 16}.{(v >> 8) & 255}.{v & 255}",
            "device": torch.cuda.get_device_name()}


L2_BYTES = 126e6


class L2Flush:
    """Timing hygiene for inputs that fit in L2 (126 MB): a write of 256 MB
    between timed steps evicts them, so every step reads its inputs from
    HBM.  The write runs between the step's events, outside the timed
    interval.  For inputs larger than L2 it does nothing."""

    def __init__(self, input_bytes: float, dev):
        self.input_bytes = float(input_bytes)
        self.active = self.input_bytes < L2_BYTES
        self.buf = (torch.empty(int(2 * 128 * 2**20) // 4, dtype=torch.int32, device=dev)
                    if self.active else None)
        self.n = 0

    def __call__(self):
        if self.active:
            self.n += 1
            self.buf.fill_(self.n)

    def note(self) -> str:
        mb = self.input_bytes / 1e6
        if self.active:
            return (f"inputs {mb:.1f} MB fit in L2 (126 MB): L2 flushed between timed steps "
                    "by a 256 MB write outside each step's events")
        return f"inputs larger than L2: {mb:.0f} MB vs 126 MB; no flush"


def timed_steps(step, steps: int, stream, dev, flush=None):
    """Run ``steps`` steps on the launching stream, synchronised on both
    sides.  Without a flush: one event before each step and one after the
    last (back-to-back steps).  With an L2 flush: the flush runs before each
    step, outside that step's pair of events, and the total is the sum of
    the steps.  Returns the total milliseconds and the per-step list."""
    torch.cuda.synchronize(dev)
    if flush is not None and flush.active:
        ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        for i in range(steps):
            flush()
            ev0[i].record(stream)
            step()
            ev1[i].record(stream)
        torch.cuda.synchronize(dev)
        per = [ev0[i].elapsed_time(ev1[i]) for i in range(steps)]
        return sum(per), per
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    for i in range(steps):
        ev[i].record(stream)
        step()
    ev[steps].record(stream)
    torch.cuda.synchronize(dev)
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]
    return ev[0].elapsed_time(ev[steps]), per


# ------------------------------------------------------------- GPU arm -----
def run_b200(args, w):
    import tiled_attention_forward_sm_b200 as tab
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
        pg = True

    q_h, k_h, v_h = make_workload_inputs(w)
    q, k, v = (t.to(dev) for t in (q_h, k_h, v_h))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    pair = args.kernel == "pair"
    # the timed step calls the C ABI directly (the library's boundary), with
    # the arguments marshalled once
    import ctypes
    tuned = (args.exp2_poly_pairs, args.kv_stages, args.rescale_tau) != (None, None, None)
    if pair and tuned:
        raise SystemExit("the tuning options apply to attn_fwd, not to the pair kernel")
    cargs = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), w.B, w.H,
             w.N, w.d, int(w.causal), ctypes.c_float(w.scale))
    if tuned:
        opts = tab.AttnOpts(-1 if args.exp2_poly_pairs is None else args.exp2_poly_pairs,
                            0 if args.kv_stages is None else args.kv_stages,
                            -1.0 if args.rescale_tau is None else args.rescale_tau)
        fn = tab.library().attn_fwd_ex
        cargs = cargs + (ctypes.byref(opts), stream.cuda_stream)
    else:
        fn = tab.library().attn_fwd_pair if pair else tab.library().attn_fwd
        cargs = cargs + (stream.cuda_stream,)

    def step():
        rc = fn(*cargs)
        if rc != 0:
            raise SystemExit(f"attn_fwd returned {rc}: {tab.strerror(rc)}")

    sampler = ClockSampler(dev)
    for _ in range(args.warmup):
        step()
    flush = L2Flush(3 * w.rows * w.d * 2, dev)
    torch.cuda.synchronize(dev)
    sampler.start()
    if pg:
        torch.distributed.barrier()
    ms_total, per_step = timed_steps(step, args.steps, stream, dev, flush)
    clocks = sampler.stop()
    if pg:
        torch.distributed.barrier()
    status = tab.last_device_error(stream)
    if status != 0:
        raise SystemExit(f"device status {status}: {tab.strerror(status)}")

    # end to end: host buffers through the C ABI host entry point (the pair
    # kernel: pinned copies in and out around attn_fwd_pair on the stream)
    q_p, k_p, v_p = (t.pin_memory() for t in (q_h, k_h, v_h))
    o_p = torch.empty_like(q_p).pin_memory()
    lse_p = torch.empty((w.B, w.H, w.N), dtype=torch.float32).pin_memory()
    e2e_steps = max(1, min(args.steps, args.e2e_steps))

    def e2e_step():
        if not pair:
            tab.attn_fwd_host(q_p, k_p, v_p, o_p, lse_p, q, k, v, o, lse, w.causal, w.scale,
                              stream)
            return
        for dst, src in ((q, q_p), (k, k_p), (v, v_p)):
            dst.copy_(src, non_blocking=True)
        step()
        o_p.copy_(o, non_blocking=True)
        lse_p.copy_(lse, non_blocking=True)

    if args.no_e2e:
        e2e_ms = float("nan")
    else:
        for _ in range(min(args.warmup, 3)):
            e2e_step()
        if pg:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        f1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = f0.elapsed_time(f1) / e2e_steps

    t = torch.tensor([ms_total, e2e_ms], dtype=torch.float64, device=dev)
    if pg:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    ms_total, e2e_ms = float(t[0]), float(t[1])
    if pg:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return None

    ms_step = ms_total / args.steps
    if clocks.get("sm_mhz"):
        # clock-independent size of a step: device cycles at the sampled clock
        clocks["kcycles_per_step"] = round(ms_step * clocks["sm_mhz"], 1)
    value = world * w.flops / (ms_step * 1e-3) / 1e12
    e2e_value = world * w.flops / (e2e_ms * 1e-3) / 1e12
    peaks, peak_kind = load_peaks()
    peak = float(peaks["bf16_tflops"])
    achieved = w.flops / (ms_step * 1e-3) / 1e12  # per launch, this GPU
    tb = w.rows * w.d * 2
    sources = PAIR_SOURCES if pair else KERNEL_SOURCES
    traffic = load_traffic(w.name, PAIR_PROFILE_FILE if pair else PROFILE_FILE, sources)
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "us_per_step": round(ms_step * 1e3, 2),
        "step_ms": {"min": round(min(per_step), 4), "median": round(statistics.median(per_step), 4),
                    "max": round(max(per_step), 4)},
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 Q/K/V, see inputs.py)",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                   "causal": w.causal, "scale": w.scale, "q_std": w.q_std,
                   "flops_per_step": w.flops,
                   "l2": flush.note(),
                   "parallelism": f"replica x{world} (independent batches)",
                   "kernel": "cta_pair (attn_fwd_pair)" if pair else "one_cta (attn_fwd)",
                   "tuning": None if not tuned else {
                       "exp2_poly_pairs": args.exp2_poly_pairs, "kv_stages": args.kv_stages,
                       "rescale_tau": args.rescale_tau}},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "peak_source": f"{peak_kind} bf16 burst (MEASURED_PEAKS.json)"
                     if peak_kind == "measured" else "fallback 1.59 PFLOP/s",
                     "frac_of_sustained": round(achieved / float(peaks.get(
                         "bf16_tflops_sustained", FALLBACK_PEAK["bf16_tflops_sustained"])), 4),
                     "frac_of_datasheet_2250": round(achieved / DATASHEET_BF16_TFLOPS, 4),
                     "traffic": traffic,
                     "algorithmic_bytes": 4 * tb + w.rows * 4},
        "e2e": None if args.no_e2e else {
            "value": round(e2e_value, 2), "unit": UNIT,
            "h2d_bytes_per_step": 3 * tb, "d2h_bytes_per_step": tb + w.rows * 4,
            "steps": e2e_steps, "ms_per_step": round(e2e_ms, 4),
            "api": ("attn_fwd_pair_into between pinned-host copies" if pair else
                    "attn_fwd_host (pinned host buffers, copies in the timed region)")},
        "gpu_launches": args.steps,
        "clocks": clocks,
        "kernel_sha": kernel_sha(sources),
        "versions": versions(tab.library(), sampler),
    }
    if world == 1 and not args.no_cpu_baseline:
        bits = (bf16_bits(q_h), bf16_bits(k_h), bf16_bits(v_h))
        tf, nrows, secs, cores, last = time_oracle(w, bits, args.cpu_seconds)
        line["cpu_baseline"] = {
            "value": round(tf, 6), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{nrows} row evaluations in seeded batches of distinct rows (a row "
                      f"may recur across batches) out of {w.rows} rows ({secs:.1f} s); "
                      "TFLOPS from the rows' exact share of the metric FLOPs"}
        # the timed step's output, against the oracle rows the leg computed
        line["parity"] = parity_of_rows(o, lse, w, last)
    return line


# ------------------------------------------- general entry points (GPU) ---
def visible_pairs(w) -> int:
    """(query, key) pairs the mask lets through, summed over heads: the
    queries are the last positions of their key sequence under the mask."""
    def per_seq(nq: int, nk: int) -> int:
        if not w.causal:
            return nq * nk
        delta = nk - nq
        i = np.arange(nq, dtype=np.int64)
        return int(np.clip(i + delta + 1, 0, nk).sum())
    if w.kind == "varlen":
        return w.H * sum(per_seq(a, b) for a, b in zip(w.lens_q, w.lens_k))
    return w.B * w.H * per_seq(w.N_q, w.N_k)


def run_general(args, w):
    import ctypes
    import tiled_attention_forward_sm_b200 as tab
    world, rank, local = dist_env()
    if world > 1:
        raise SystemExit("general workloads run on one GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    q_h, k_h, v_h = make_general_inputs(w)
    q, k, v = (t.to(dev) for t in (q_h, k_h, v_h))
    stream = torch.cuda.current_stream(dev)
    lib = tab.library()
    sh = stream.cuda_stream
    launches = 1
    if w.kind == "varlen":
        lens_q = np.array(w.lens_q, dtype=np.int32)
        lens_k = np.array(w.lens_k, dtype=np.int32)
        cu_q = torch.from_numpy(np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)).to(dev)
        cu_k = torch.from_numpy(np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)).to(dev)
        o = torch.empty_like(q)
        lse = torch.empty((w.H, q.shape[0]), dtype=torch.float32, device=dev)

        def step():
            rc = lib.attn_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                     lse.data_ptr(), cu_q.data_ptr(), cu_k.data_ptr(), w.B, w.H,
                                     w.H_kv, w.N_q, w.N_k, int(q.shape[0]), int(k.shape[0]),
                                     w.d, int(w.causal), ctypes.c_float(w.scale), sh)
            assert rc == 0, rc
    elif w.kind == "chunk":
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.H, w.N_q), dtype=torch.float32, device=dev)

        def step():
            rc = lib.attn_fwd_chunk(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                    lse.data_ptr(), w.B, w.H, w.H_kv, w.N_q, w.N_k, w.d,
                                    int(w.causal), w.N_k - w.N_q, ctypes.c_float(w.scale), 0, sh)
            assert rc == 0, rc
    else:
        slices = tab.splitkv_slices(w.N_k, w.n_splits)
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.H, w.N_q), dtype=torch.float32, device=dev)
        rows = w.B * w.H * w.N_q
        ws_o = torch.empty((max(slices, 1), rows, w.d), dtype=torch.float32, device=dev)
        ws_l = torch.empty((max(slices, 1), rows), dtype=torch.float32, device=dev)
        launches = 2 if slices > 1 else 1

        def step():
            rc = lib.attn_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                      lse.data_ptr(), w.B, w.H, w.H_kv, w.N_q, w.N_k, w.d,
                                      int(w.causal), w.N_k - w.N_q, ctypes.c_float(w.scale),
                                      w.n_splits, ws_o.data_ptr(), ws_l.data_ptr(), sh)
            assert rc == 0, rc

    sampler = ClockSampler(dev)
    for _ in range(args.warmup):
        step()
    flush = L2Flush(2 * (q.numel() + k.numel() + v.numel()), dev)
    torch.cuda.synchronize(dev)
    sampler.start()
    ms_step = timed_steps(step, args.steps, stream, dev, flush)[0] / args.steps
    clocks = sampler.stop()
    status = tab.last_device_error(stream)
    if status != 0:
        raise SystemExit(f"device status {status}: {tab.strerror(status)}")
    flops = 4.0 * w.d * visible_pairs(w)
    bytes_alg = 2 * (q.numel() + k.numel() + v.numel() + o.numel()) + 4 * lse.numel()
    peaks, peak_kind = load_peaks()
    tflops = flops / (ms_step * 1e-3) / 1e12
    gbs = bytes_alg / (ms_step * 1e-3) / 1e9
    ridge = float(peaks["bf16_tflops"]) * 1e12 / (float(peaks["hbm_gbs"]) * 1e9)
    if flops / bytes_alg >= ridge:
        roof = {"bound": "tensor", "achieved": round(tflops, 2), "peak": float(peaks["bf16_tflops"]),
                "unit": "TFLOP/s", "frac": round(tflops / float(peaks["bf16_tflops"]), 4)}
    else:
        roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": float(peaks["hbm_gbs"]),
                "unit": "GB/s", "frac": round(gbs / float(peaks["hbm_gbs"]), 4)}
    roof.update({"traffic": None, "algorithmic_bytes": bytes_alg,
                 "arithmetic_intensity": round(flops / bytes_alg, 1),
                 "peak_source": f"{peak_kind} (MEASURED_PEAKS.json)"})
    cfg = {k_: getattr(w, k_) for k_ in ("name", "kind", "B", "H", "H_kv", "N_q", "N_k", "d",
                                          "causal", "n_splits")}
    cfg["workload"] = cfg.pop("name")
    if w.kind == "varlen":
        cfg["lens"] = list(w.lens_q)
    cfg.update({"flops_per_step": flops, "l2": flush.note()})
    return {
        "metric": METRIC, "value": round(tflops, 2), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 Q/K/V, see inputs.py)", "config": cfg,
        "roofline": roof,
        "e2e": None, "gpu_launches": launches * args.steps, "clocks": clocks,
        "kernel_sha": kernel_sha(),
    }


# ----------------------------------------------------------- FP8 path -----
FP8_SUFFIX = "_fp8"


def run_fp8(args, w):
    """The FP8 attention on a square workload's shapes: the attention alone
    (the line's value) and the bf16 -> E4M3 conversion of Q, K and V^T that
    feeds it (conversion_ms, and the metric with the conversion included)."""
    import tiled_attention_forward_sm_b200 as tab
    world, rank, local = dist_env()
    if world > 1:
        raise SystemExit("FP8 workloads run on one GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    q_h, k_h, v_h = make_workload_inputs(w)
    q, k, v = (t.to(dev) for t in (q_h, k_h, v_h))
    stream = torch.cuda.current_stream(dev)
    lib = tab.library()
    q8 = torch.empty(q.shape, dtype=torch.uint8, device=dev)
    k8 = torch.empty_like(q8)
    vt8 = torch.empty((w.B, w.H, w.d, w.N), dtype=torch.uint8, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    sh = stream.cuda_stream
    BH = w.B * w.H
    import ctypes

    def convert():
        for src, dst, tr in ((q, q8, 0), (k, k8, 0), (v, vt8, 1)):
            rc = lib.attn_quantize_e4m3(src.data_ptr(), dst.data_ptr(), BH, w.N, w.d,
                                        ctypes.c_float(1.0), tr, sh)
            assert rc == 0, rc

    def attend():
        rc = lib.attn_fwd_fp8(q8.data_ptr(), k8.data_ptr(), vt8.data_ptr(), o.data_ptr(),
                              lse.data_ptr(), w.B, w.H, w.N, w.d, int(w.causal),
                              ctypes.c_float(w.scale), ctypes.c_float(1.0), ctypes.c_float(1.0),
                              ctypes.c_float(1.0), sh)
        assert rc == 0, rc

    def timed(fn, steps, flush):
        for _ in range(args.warmup):
            fn()
        return timed_steps(fn, steps, stream, dev, flush)[0] / steps

    flush_attn = L2Flush(3 * w.rows * w.d, dev)       # E4M3 Q, K, V^T
    flush_conv = L2Flush(3 * w.rows * w.d * 2, dev)   # their bf16 sources
    convert()
    sampler = ClockSampler(dev)
    sampler.start()
    ms_attn = timed(attend, args.steps, flush_attn)
    clocks = sampler.stop()
    ms_conv = timed(convert, max(1, args.steps // 4), flush_conv)
    status = tab.last_device_error(stream)
    if status != 0:
        raise SystemExit(f"device status {status}: {tab.strerror(status)}")
    tflops = w.flops / (ms_attn * 1e-3) / 1e12
    peaks, peak_kind = load_peaks()
    conv_bytes = 3 * w.rows * w.d * 3  # 2 bytes read, 1 written per element
    return {
        "metric": METRIC.replace("(bf16, d=128)", "(FP8 E4M3 operands, d=128)"),
        "value": round(tflops, 2), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_attn, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
        "data": "synthetic (the square workload's seeded bf16 inputs, converted to E4M3)",
        "config": {"workload": w.name + FP8_SUFFIX, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                   "causal": w.causal, "flops_per_step": w.flops,
                   "descales": [1.0, 1.0, 1.0],
                   "l2": flush_attn.note()},
        "roofline": {"bound": "tensor", "achieved": round(tflops, 2),
                     "peak": 2.0 * float(peaks["bf16_tflops"]), "unit": "TFLOP/s",
                     "frac": round(tflops / (2.0 * float(peaks["bf16_tflops"])), 4),
                     "peak_source": f"{peak_kind} bf16 burst x 2 (the nominal fp8:bf16 ratio)",
                     "traffic": None},
        "conversion": {"ms": round(ms_conv, 4), "launches": 3,
                       "gbs": round(conv_bytes / (ms_conv * 1e-3) / 1e9, 1),
                       "hbm_frac": round(conv_bytes / (ms_conv * 1e-3) / 1e9 /
                                         float(peaks["hbm_gbs"]), 4),
                       "tflops_with_conversion": round(w.flops / ((ms_attn + ms_conv) * 1e-3)
                                                       / 1e12, 2)},
        "e2e": None, "gpu_launches": args.steps, "clocks": clocks, "kernel_sha": kernel_sha(),
    }


# ----------------------------------------------------------- FP4 path -----
FP4_SUFFIX = "_fp4"


def run_fp4(args, w):
    """The 4-bit (NVFP4) attention on a square workload's shapes: the
    attention alone (the line's value) and the bf16 -> NVFP4 conversion of
    Q, K and V^T that feeds it (conversion_ms, and the metric with the
    conversion included)."""
    import ctypes
    import tiled_attention_forward_sm_b200 as tab
    world, rank, local = dist_env()
    if world > 1:
        raise SystemExit("FP4 workloads run on one GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    q_h, k_h, v_h = make_workload_inputs(w)
    q, k, v = (t.to(dev) for t in (q_h, k_h, v_h))
    stream = torch.cuda.current_stream(dev)
    lib = tab.library()
    sh = stream.cuda_stream
    BH = w.B * w.H
    T = (w.N + 127) // 128
    qc = torch.empty((w.B, w.H, w.N, 64), dtype=torch.uint8, device=dev)
    kc = torch.empty_like(qc)
    vc = torch.empty((w.B, w.H, 128, w.N // 2), dtype=torch.uint8, device=dev)
    qs, ks, vs = (torch.empty((BH, T, 2, 512), dtype=torch.uint8, device=dev) for _ in range(3))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)

    def convert():
        for src, c, sc, tr in ((q, qc, qs, 0), (k, kc, ks, 0), (v, vc, vs, 1)):
            rc = lib.attn_quantize_nvfp4(src.data_ptr(), c.data_ptr(), sc.data_ptr(), BH, w.N,
                                         w.d, ctypes.c_float(1.0), tr, sh)
            assert rc == 0, rc

    cargs = (qc.data_ptr(), qs.data_ptr(), kc.data_ptr(), ks.data_ptr(), vc.data_ptr(),
             vs.data_ptr(), o.data_ptr(), lse.data_ptr(), w.B, w.H, w.N, w.d, int(w.causal),
             ctypes.c_float(w.scale), ctypes.c_float(1.0), ctypes.c_float(1.0),
             ctypes.c_float(1.0), sh)

    def attend():
        rc = lib.attn_fwd_fp4(*cargs)
        assert rc == 0, rc

    def timed(fn, steps, flush):
        for _ in range(args.warmup):
            fn()
        return timed_steps(fn, steps, stream, dev, flush)[0] / steps

    # E2M1 codes (half a byte per element) and their E4M3 scales
    flush_attn = L2Flush(3 * (w.rows * w.d // 2 + BH * T * 1024), dev)
    flush_conv = L2Flush(3 * w.rows * w.d * 2, dev)   # the bf16 sources
    convert()
    sampler = ClockSampler(dev)
    sampler.start()
    ms_attn = timed(attend, args.steps, flush_attn)
    clocks = sampler.stop()
    ms_conv = timed(convert, max(1, args.steps // 4), flush_conv)
    status = tab.last_device_error(stream)
    if status != 0:
        raise SystemExit(f"device status {status}: {tab.strerror(status)}")
    tflops = w.flops / (ms_attn * 1e-3) / 1e12
    peaks, peak_kind = load_peaks()
    # per element: 2 bytes read, half a byte of codes and 1/16 byte of scale written
    conv_bytes = 3 * w.rows * w.d * (2 + 0.5 + 1 / 16)
    if clocks.get("sm_mhz"):
        clocks["kcycles_per_step"] = round(ms_attn * clocks["sm_mhz"], 1)
    return {
        "metric": METRIC.replace("(bf16, d=128)", "(NVFP4 operands, d=128)"),
        "value": round(tflops, 2), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_attn, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4",
        "data": "synthetic (the square workload's seeded bf16 inputs, converted to NVFP4)",
        "config": {"workload": w.name + FP4_SUFFIX, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                   "causal": w.causal, "flops_per_step": w.flops, "descales": [1.0, 1.0, 1.0],
                   "l2": flush_attn.note()},
        "roofline": {"bound": "tensor", "achieved": round(tflops, 2),
                     "peak": 4.0 * float(peaks["bf16_tflops"]), "unit": "TFLOP/s",
                     "frac": round(tflops / (4.0 * float(peaks["bf16_tflops"])), 4),
                     "peak_source": f"{peak_kind} bf16 burst x 4 (the nominal fp4:bf16 ratio)",
                     "traffic": None},
        "conversion": {"ms": round(ms_conv, 4), "launches": 3,
                       "gbs": round(conv_bytes / (ms_conv * 1e-3) / 1e9, 1),
                       "hbm_frac": round(conv_bytes / (ms_conv * 1e-3) / 1e9 /
                                         float(peaks["hbm_gbs"]), 4),
                       "tflops_with_conversion": round(w.flops / ((ms_attn + ms_conv) * 1e-3)
                                                       / 1e12, 2)},
        "e2e": None, "gpu_launches": args.steps, "clocks": clocks, "kernel_sha": kernel_sha(),
    }


# ------------------------------------------------- k-means assignment -----
def run_kmeans(args, w):
    import ctypes
    import tiled_attention_forward_sm_b200 as tab
    world, rank, local = dist_env()
    if world > 1:
        raise SystemExit("k-means workloads run on one GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    x_h, c_h = make_kmeans_inputs(w)
    x, c = x_h.to(dev), c_h.to(dev)
    lib = tab.library()
    ws = torch.empty(int(lib.attn_kmeans_workspace_floats(w.N, w.K)), dtype=torch.float32,
                     device=dev)
    assign = torch.empty(w.N, dtype=torch.int32, device=dev)
    best = torch.empty(w.N, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    # centroid norms + assignment; a point-norm launch too when the points
    # fill more than four rounds of 256-point work items over the SMs
    n_sms = torch.cuda.get_device_properties(dev).multi_processor_count
    launches_per_step = 3 if (w.N + 255) // 256 > 4 * n_sms else 2

    def step():
        rc = lib.attn_kmeans_assign(x.data_ptr(), c.data_ptr(), ws.data_ptr(), assign.data_ptr(),
                                    best.data_ptr(), w.N, w.K, w.d, stream.cuda_stream)
        assert rc == 0, rc

    sampler = ClockSampler(dev)
    for _ in range(args.warmup):
        step()
    flush = L2Flush(2 * (x.numel() + c.numel()), dev)
    torch.cuda.synchronize(dev)
    sampler.start()
    ms_step = timed_steps(step, args.steps, stream, dev, flush)[0] / args.steps
    clocks = sampler.stop()
    status = tab.last_device_error(stream)
    if status != 0:
        raise SystemExit(f"device status {status}: {tab.strerror(status)}")
    bytes_alg = 2 * (x.numel() + c.numel()) + 8 * w.N
    tflops = w.flops / (ms_step * 1e-3) / 1e12
    peaks, peak_kind = load_peaks()
    return {
        "metric": "k-means assignment TFLOPS (2*N*K*d point-centroid products, bf16)",
        "value": round(tflops, 2), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded centroids and points around them, see inputs.py)",
        "config": {"workload": w.name, "N": w.N, "K": w.K, "d": w.d, "flops_per_step": w.flops,
                   "l2": flush.note()},
        "roofline": {"bound": "tensor", "achieved": round(tflops, 2),
                     "peak": float(peaks["bf16_tflops"]), "unit": "TFLOP/s",
                     "frac": round(tflops / float(peaks["bf16_tflops"]), 4), "traffic": None,
                     "algorithmic_bytes": bytes_alg,
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json)"},
        "e2e": None, "gpu_launches": launches_per_step * args.steps, "clocks": clocks,
        "kernel_sha": kernel_sha(),
    }


# ------------------------------------------------------- reference arm -----
def run_reference(args, w):
    world, rank, _ = dist_env()
    if rank != 0:
        return None
    import oracle
    q_h, k_h, v_h = make_workload_inputs(w)
    bits = (bf16_bits(q_h), bf16_bits(k_h), bf16_bits(v_h))
    qb, kb, vb = bits
    # each step: a bounded row sample, sized so the whole run stays ~1 minute
    t0 = time.perf_counter()
    probe_rows = oracle_sample_rows(w, 256, 999)
    oracle.attn_ref(qb, kb, vb, w.causal, w.scale, rows=probe_rows)
    per_flop = (time.perf_counter() - t0) / row_flops(w, probe_rows)
    budget = 60.0 / max(1, args.steps + args.warmup)
    avg_row = row_flops(w, oracle_sample_rows(w, 4096, 5)) / 4096
    n_rows = int(max(64, min(w.rows, budget / (per_flop * avg_row))))
    for s in range(args.warmup):
        oracle.attn_ref(qb, kb, vb, w.causal, w.scale, rows=oracle_sample_rows(w, n_rows, 10_000 + s))
    flops, secs = 0.0, 0.0
    for s in range(args.steps):
        rows = oracle_sample_rows(w, n_rows, 20_000 + s)
        t0 = time.perf_counter()
        oracle.attn_ref(qb, kb, vb, w.causal, w.scale, rows=rows)
        secs += time.perf_counter() - t0
        flops += row_flops(w, rows)
    value = flops / secs / 1e12
    cores = oracle.max_threads()
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * secs / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                   "causal": w.causal, "scale": w.scale, "q_std": w.q_std},
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cores,
                         "kind": "oracle",
                         "sample": f"{n_rows} seeded random rows per step of {w.rows}"},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def run_copy_rates(args, w):
    """Plain pinned-memory copy rates for the bytes the e2e leg moves per step
    (Q, K, V in; O and LSE out): the floor under the e2e figure on this machine.
    Host-to-device and device-to-host alone, then both at once on two
    streams; CUDA events on the current stream, after warm-up."""
    world, rank, local = dist_env()
    if world > 1:
        raise SystemExit("--copy-rates runs on one GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    n_in = 3 * w.rows * w.d * 2
    n_out = w.rows * w.d * 2 + w.rows * 4
    h_in = torch.empty(n_in, dtype=torch.uint8, pin_memory=True)
    d_in = torch.empty(n_in, dtype=torch.uint8, device=dev)
    h_out = torch.empty(n_out, dtype=torch.uint8, pin_memory=True)
    d_out = torch.empty(n_out, dtype=torch.uint8, device=dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    cur = torch.cuda.current_stream(dev)

    def both():
        ev = torch.cuda.Event()
        ev.record(cur)
        s_in.wait_event(ev)
        s_out.wait_event(ev)
        with torch.cuda.stream(s_in):
            d_in.copy_(h_in, non_blocking=True)
        with torch.cuda.stream(s_out):
            h_out.copy_(d_out, non_blocking=True)
        cur.wait_stream(s_in)
        cur.wait_stream(s_out)

    def ms(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(cur)
        for _ in range(args.steps):
            fn()
        e1.record(cur)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / args.steps

    t_in = ms(lambda: d_in.copy_(h_in, non_blocking=True))
    t_out = ms(lambda: h_out.copy_(d_out, non_blocking=True))
    t_both = ms(both)
    return {"copy_rates": {"workload": w.name, "h2d_bytes": n_in, "d2h_bytes": n_out,
                           "h2d_ms": round(t_in, 4), "h2d_GBps": round(n_in / t_in / 1e6, 1),
                           "d2h_ms": round(t_out, 4), "d2h_GBps": round(n_out / t_out / 1e6, 1),
                           "both_ms": round(t_both, 4),
                           "metric_at_both_ms": round(w.flops / t_both / 1e9, 2),
                           "unit": "TFLOPS", "steps": args.steps, "warmup": args.warmup}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--workload", default=BENCH_WORKLOAD,
                    choices=sorted(WORKLOADS) + sorted(GENERAL_WORKLOADS) +
                    sorted(KMEANS_WORKLOADS) +
                    sorted(n + FP8_SUFFIX for n, w_ in WORKLOADS.items() if w_.d == 128) +
                    sorted(n + FP4_SUFFIX for n, w_ in WORKLOADS.items() if w_.d == 128))
    ap.add_argument("--kernel", choices=["one_cta", "pair"], default="one_cta",
                    help="bf16 workloads at d=128: attn_fwd (one CTA per SM) or attn_fwd_pair "
                         "(clusters of two CTAs sharing each product)")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end (host buffers) measurement")
    ap.add_argument("--exp2-poly-pairs", type=int, default=None,
                    help="attn_fwd_ex option: exponential pairs of every 4 on the FMA polynomial")
    ap.add_argument("--kv-stages", type=int, default=None,
                    help="attn_fwd_ex option: K/V ring depth (2..5 at d = 128)")
    ap.add_argument("--rescale-tau", type=float, default=None,
                    help="attn_fwd_ex option: lazy-rescale threshold (0..16, log2 units)")
    ap.add_argument("--copy-rates", action="store_true",
                    help="print the pinned host<->device copy rates for the workload's e2e bytes "
                         "instead of timing the attention")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = dist_env()[0]
    if args.gpus != world:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE is {world}: launch N > 1 ranks with "
                 f"python -m torch.distributed.run --nproc-per-node N bench.py --gpus N")
    if args.copy_rates:
        line = run_copy_rates(args, WORKLOADS[args.workload])
    elif args.workload.endswith(FP4_SUFFIX):
        if args.impl == "reference":
            ap.error("--impl reference times the bf16 workloads only")
        line = run_fp4(args, WORKLOADS[args.workload[: -len(FP4_SUFFIX)]])
    elif args.workload.endswith(FP8_SUFFIX):
        if args.impl == "reference":
            ap.error("--impl reference times the bf16 workloads only")
        line = run_fp8(args, WORKLOADS[args.workload[: -len(FP8_SUFFIX)]])
    elif args.workload in KMEANS_WORKLOADS:
        if args.impl == "reference":
            ap.error("--impl reference times the attention workloads only")
        line = run_kmeans(args, KMEANS_WORKLOADS[args.workload])
    elif args.workload in GENERAL_WORKLOADS:
        if args.impl == "reference":
            ap.error("--impl reference times the square workloads only")
        line = run_general(args, GENERAL_WORKLOADS[args.workload])
    else:
        w = WORKLOADS[args.workload]
        line = run_reference(args, w) if args.impl == "reference" else run_b200(args, w)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
