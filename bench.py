#!/usr/bin/env python3
"""Benchmark: dfx_decode throughput on the 70B-shaped layer stream.

Workload: 24 BF16 tensors of 8192 x 28672 (5.64 B weights, 11.3 GB raw), values
N(0, 1/8192) with 0.05 % N(0, 0.5^2) outliers, each encoded with its own code
book by dfx_encode.  All 24 containers stay resident in HBM; one step decodes
them one after another into a single reused 470 MB BF16 buffer on one stream.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line on rank 0.  `value` is decoded BF16 GB/s over all ranks
(each rank decodes its own 24 tensors: weak scaling, no collective on the data
path).  Timing: CUDA events on the decode stream, W untimed steps first, a
barrier and a device synchronise on both sides, max over ranks.  Every
container (~0.32 GB) and the output buffer exceed the 126 MB L2, so no flush is
needed between steps.

The line also reports, on rank 0: `e2e` (pinned host containers through H2D, decode
and D2H), `offload` (weights streamed from pinned host memory, raw against
compressed), `layer_batch` (a Llama-3-8B-shaped layer as 7 launches and as one
batched launch), `decode_into_gemm` (a weight restored ahead of its GEMM), `tans`
(the tANS exponent coder on 4 of the tensors against the Huffman figures) and
`cpu_baseline` (the oracle, one host core).

`--impl reference` times the CPU oracle (single-threaded C) decoding a 16 M
weight sample with the same value distribution; it is the slow reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import shutil
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "dfx_decode BF16 GB/s & % of HBM roofline; bits/weight; bit-exact vs oracle"
UNIT = "GB/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
WORKLOAD = "70B-shaped layer stream: 24 x BF16[8192, 28672], N(0, 1/8192) + 0.05% N(0, 0.5^2) outliers"
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_dram_traffic.txt")
DECODE_SOURCES = [os.path.join(ROOT, "lossless_entropy_coded_exponent_b200", "csrc", f)
                  for f in ("decode.cu", "decode_pipeline.cuh", "huffman_reader.cuh", "huffman_tables.cuh", "bulk.cuh", "dfx_common.cuh")]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--tensors", type=int, default=24)
    ap.add_argument("--chunk-symbols", type=int, default=128)
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-layer-batch", action="store_true", help="skip the multi-tensor (Llama-3-8B layer) decode measurement")
    ap.add_argument("--no-tans", action="store_true", help="skip the tANS exponent coder comparison")
    ap.add_argument("--no-config-table", action="store_true",
                    help="skip the per-configuration decode table and the pinned oracle table")
    return ap.parse_args()


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            v = float(json.load(fh)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def host_cpu() -> str:
    """Model name and logical CPU count of this host (the oracle runs on one of them)."""
    model = "unknown CPU"
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return f"{model}, {os.cpu_count()} logical CPUs"


def decode_source_hash() -> str:
    h = hashlib.sha256()
    for p in DECODE_SOURCES:
        with open(p, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def ncu_traffic_per_launch(n_weights: int):
    """DRAM bytes per decode launch from the committed ncu summary, scaled to this
    launch's weights; None when the kernel source changed since the capture."""
    try:
        fields = {}
        with open(TRAFFIC_FILE) as fh:
            for line in fh:
                if ":" in line and not line.startswith("#"):
                    k, v = line.split(":", 1)
                    fields[k.strip()] = v.strip()
        if fields.get("decode_source_sha256") != decode_source_hash():
            return None
        return float(fields["dram_bytes_per_weight"]) * n_weights
    except Exception:
        return None


CLOCK_CHILD = r"""
import json, select, sys
import pynvml
pynvml.nvmlInit()
bus, index, period = sys.argv[1], int(sys.argv[2]), float(sys.argv[3])
h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode()) if bus != "-" else pynvml.nvmlDeviceGetHandleByIndex(index)
mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
clk, reasons, side = [], 0, []


def probe():  # memory clock, GPU and HBM temperature, board power; None where NVML has no answer
    out = []
    for f in (lambda: pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_MEM),
              lambda: pynvml.nvmlDeviceGetTemperature(h, pynvml.NVML_TEMPERATURE_GPU),
              lambda: pynvml.nvmlDeviceGetFieldValues(h, [pynvml.NVML_FI_DEV_MEMORY_TEMP])[0].value.uiVal,
              lambda: pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0):
        try:
            out.append(f())
        except Exception:
            out.append(None)
    return out


print("ready", flush=True)
while not select.select([sys.stdin], [], [], period)[0]:
    clk.append(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
    reasons |= pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
    if len(clk) % 5 == 1:
        side.append(probe())
print(json.dumps({"clk": clk, "max": mx, "reasons": reasons, "side": side}), flush=True)
"""


def tenths(launch_ms):
    """Mean microseconds per launch in each tenth of the timed steps, in order: how the
    launch time moves over the run (the 1 kW part lowers its clock under the power cap)."""
    k = len(launch_ms)
    if k < 10:
        return [round(1e3 * v, 1) for v in launch_ms]
    return [round(1e3 * statistics.mean(launch_ms[k * i // 10:k * (i + 1) // 10]), 1) for i in range(10)]


class ClockSampler:
    """Samples SM clock and clock-event reasons while running, through NVML in a child
    interpreter (so the launch loop of this one cannot starve it); stops when its stdin
    closes."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples, self.reasons, self.max_mhz, self.side = [], set(), None, []
        self.period = period_s
        self.device_index = device_index
        self.error = None
        self._proc = None

    @staticmethod
    def _bus_id(device_index):
        try:
            import torch

            props = torch.cuda.get_device_properties(device_index)
            return "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
        except Exception:
            return "-"

    def __enter__(self):
        try:
            self._proc = subprocess.Popen(
                [sys.executable, "-c", CLOCK_CHILD, self._bus_id(self.device_index), str(self.device_index),
                 str(self.period)], stdin=subprocess.PIPE, stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
            if self._proc.stdout.readline().strip() != "ready":  # sampling has started
                raise RuntimeError(self._proc.stderr.read()[-300:])
        except Exception as e:
            self.error = repr(e)
            if self._proc is not None:
                self._proc.kill()
            self._proc = None
        return self

    def __exit__(self, *exc):
        if self._proc is None:
            return
        try:
            out, _ = self._proc.communicate(input="", timeout=30)  # closes stdin: the child reports and exits
            d = json.loads(out.strip().splitlines()[-1])
            self.samples, self.max_mhz, self.side = d["clk"], d["max"], d.get("side", [])
            for bit, name in self.REASONS.items():
                if d["reasons"] & bit:
                    self.reasons.add(name)
        except Exception as e:
            self.error = repr(e)
            self._proc.kill()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0,
                    "error": self.error or "no samples"}
        out = {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
               "reasons": sorted(self.reasons), "samples": len(self.samples)}
        # memory clock (median), GPU and HBM temperature and board power at the first and the
        # last of the side samples (every fifth clock sample): a memory-bound kernel that slows
        # down while the SM clock holds points at the memory side
        for i, key in enumerate(("mem_mhz", "gpu_temp_c", "hbm_temp_c", "power_w")):
            vals = [r[i] for r in self.side if r[i] is not None]
            if not vals:
                continue
            out[key] = statistics.median(vals) if key == "mem_mhz" else {"first": vals[0], "last": vals[-1]}
        return out


def dist_setup(args):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# ------------------------------------------------------------------------ reference arm

def run_reference(args, world, rank):
    """The CPU oracle decoding a bounded sample of the workload, single-threaded."""
    if rank != 0:
        return None
    import numpy as np

    import oracle
    from lossless_entropy_coded_exponent_b200 import inputs

    n = 8192 * 2048
    w = inputs.layer70b_sample(n, seed=500)
    c = oracle.encode(w, K=args.chunk_symbols)
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        out = oracle.decode(c)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    assert np.array_equal(out, w)
    t = sum(times)
    value = 2.0 * n * len(times) / t / 1e9
    sample = f"one 8192x2048 BF16 tensor ({n} weights) of the same distribution, decoded per step"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u32", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": sample, "chunk_symbols": args.chunk_symbols},
            "bits_per_weight": 8.0 * c.size / n,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "host": host_cpu(), "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    return line


# ------------------------------------------------------------------------ our arm

def run_ours(args, world, rank, local):
    import numpy as np
    import torch

    import lossless_entropy_coded_exponent_b200 as dfx
    from lossless_entropy_coded_exponent_b200 import inputs

    dfx.lib()  # fail loudly if libdfx.so is missing
    dev = torch.device("cuda", local)
    rows, cols = inputs.LAYER70B_SHAPE
    n = rows * cols
    T = args.tensors
    K = args.chunk_symbols
    # the containers are written once, before the decoding starts: a decode may read its
    # container while the decode before it finishes (DFX_DECODE_EARLY_READ)
    plan = dfx.dfx_plan(n, chunk_symbols=K, decode_flags=dfx.DFX_DECODE_EARLY_READ)
    stream = torch.cuda.Stream(device=dev)

    # ---- set-up: generate, encode, keep every container and every input resident
    xs, comps, sizes = [], [], []
    scratch = torch.empty(plan.max_compressed_bytes, dtype=torch.uint8, device=dev)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=dev)
    enc_start = torch.cuda.Event(enable_timing=True)
    enc_end = torch.cuda.Event(enable_timing=True)
    enc_ms = []
    with torch.cuda.stream(stream):
        for i in range(T):
            x = inputs.layer70b_tensor_cuda(i, seed_base=500 + 1000 * rank, device=dev)
            enc_start.record(stream)
            size = dfx.dfx_encode(plan, x, scratch, scratch.numel(), ws, ws.numel(), want_size=False, stream=stream)
            enc_end.record(stream)
            stream.synchronize()
            enc_ms.append(enc_start.elapsed_time(enc_end))
            size = int(scratch[24:32].cpu().numpy().view(np.uint64)[0])
            comps.append(scratch[:size].clone())
            sizes.append(size)
            xs.append(x)
    stream.synchronize()
    if dfx.dfx_device_status(plan, stream=stream):
        raise RuntimeError("encode reported a device error")
    del scratch, ws
    out = torch.empty(n, dtype=torch.int16, device=dev)

    # ---- warm-up
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            for i in range(T):
                dfx.dfx_decode(plan, comps[i], sizes[i], out, stream=stream)
    stream.synchronize()

    # ---- timed region: K steps x T decodes back to back, one event per step boundary (an
    # event between two launches would keep the next decode from starting while the
    # previous one finishes; the decode kernels are launched as programmatic dependents)
    events = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        with torch.cuda.stream(stream):
            events[0].record(stream)
            for e in range(1, args.steps + 1):
                for i in range(T):
                    dfx.dfx_decode(plan, comps[i], sizes[i], out, stream=stream)
                events[e].record(stream)
        stream.synchronize()
    torch.cuda.synchronize(dev)
    barrier(world)
    launch_ms = [events[j].elapsed_time(events[j + 1]) / T for j in range(len(events) - 1)]  # per launch, by step
    total_ms = events[0].elapsed_time(events[-1])
    total_ms_max = max_over_ranks(total_ms, world)
    status = dfx.dfx_device_status(plan, stream=stream)

    # ---- verification: every tensor decodes back to its input, bit for bit
    roundtrip_ok = status == 0
    with torch.cuda.stream(stream):
        for i in range(T):
            dfx.dfx_decode(plan, comps[i], sizes[i], out, stream=stream)
            stream.synchronize()
            roundtrip_ok &= bool(torch.equal(out, xs[i]))
    roundtrip_ok &= dfx.dfx_device_status(plan, stream=stream) == 0

    decoded_bytes = 2.0 * n * T * args.steps
    value = sum_over_ranks(decoded_bytes, world) / (total_ms_max * 1e-3) / 1e9
    comp_total = float(sum(sizes))
    bits_per_weight = 8.0 * comp_total / (n * T)
    algo_bytes_per_launch = comp_total / T + 2.0 * n
    mean_launch_ms = statistics.mean(launch_ms)
    achieved = algo_bytes_per_launch / (mean_launch_ms * 1e-3) / 1e9
    peak, peak_kind = measured_hbm_peak()
    traffic = ncu_traffic_per_launch(n)

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "u32", "data": "synthetic",
            "config": {"workload": WORKLOAD, "tensors": T, "weights_per_tensor": n, "chunk_symbols": K,
                       "group_chunks": 32, "max_len": 24,
                       "l2": "no flush: each container (~0.32 GB) and the 0.47 GB output exceed the 126 MB L2",
                       "parallelism": f"replicas x{world} (independent tensors per GPU, no collective)"},
            "bits_per_weight": bits_per_weight,
            "hbm_roofline_frac_of_nominal_8TBs": achieved / NOMINAL_HBM_GBS,
            "bit_exact_roundtrip": bool(roundtrip_ok),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic, "peak_kind": peak_kind,
                         "algorithmic_bytes_per_launch": algo_bytes_per_launch,
                         "mean_launch_us": 1e3 * mean_launch_ms, "kernel": f"k_decode<HuffmanCoder, {K}>",
                         # per-step means: the first steps against the last show the effect of the
                         # power cap over the timed region
                         "launch_us_by_step": {"first": 1e3 * launch_ms[0], "last": 1e3 * launch_ms[-1],
                                               "min": 1e3 * min(launch_ms), "max": 1e3 * max(launch_ms),
                                               "by_tenth": tenths(launch_ms)}},
            "gpu_launches": args.steps * T,
            "clocks": clocks.summary(),
            "encode": {"unit": "GB/s", "value": 2.0 * n / (statistics.median(enc_ms) * 1e-3) / 1e9,
                       "median_ms_per_tensor": statistics.median(enc_ms),
                       "note": "dfx_encode (histogram, code book, chunk lengths, group scan, pack), BF16 bytes read / time"}}

    # ---- end to end through the C ABI with host buffers
    if not args.no_e2e:
        line["e2e"] = run_e2e(args, plan, comps, sizes, n, dev, world)
        if rank == 0:
            line["offload"] = run_offload(plan, comps, sizes, xs, n, dev)
    # ---- several tensors per launch: a Llama-3-8B-shaped layer
    if not args.no_layer_batch and rank == 0:
        line["layer_batch"] = run_layer_batch(args, dev, stream)
    # ---- decode feeding its consumer: slices through an L2-sized buffer into a GEMM
    if not args.no_layer_batch and rank == 0:
        line["decode_into_gemm"] = run_decode_into_gemm(args, dev)
    # ---- the other exponent coder (tANS) on the same tensors and launch configuration
    if not args.no_tans and rank == 0:
        line["tans"] = run_tans_compare(args, dev, stream, xs, sizes, 1e3 * mean_launch_ms, n)
        line["tans2"] = run_tans_compare(args, dev, stream, xs, sizes, 1e3 * mean_launch_ms, n, states=2)
    # ---- the smaller configurations, with and without an L2 flush
    if not args.no_config_table and rank == 0:
        line["config_table"] = run_config_table(args, dev, stream)
    # ---- oracle on the host: rank 0 at N=1 only
    if not args.no_cpu_baseline and rank == 0 and world == 1:
        line["cpu_baseline"], line["bit_exact_vs_oracle"] = run_cpu_baseline(xs[0], comps[0], K)
        if not args.no_config_table:
            line["cpu_baseline_table"] = run_oracle_table()
    plan.free()
    return line


CONFIG_TABLE = [
    # name, generator (inputs module, seeded), note
    ("cfg1 1024x1024 N(0, 0.02^2)", "small_gaussian", ()),
    ("cfg2 length 1000003", "gaussian", (1_000_003, 0.02, 23)),
    ("cfg2 all-zero 65536", "edge:all_zero", ()),
    ("cfg2 uniform 16-bit patterns 2^20", "edge:uniform_exponents", ()),
    ("cfg2 +-0/subnormal/+-Inf/NaN mix 2^20", "edge:special_mix", ()),
    ("cfg2 Fibonacci counts (24-bit limit)", "edge:fibonacci_clamp", ()),
    ("cfg3 4096x4096 + 0.1% N(0, 1) outliers", "projection_with_outliers", ()),
    ("cfg4 Llama-3-8B layer gate_proj 14336x4096", "llama3_8b_layer_tensor", (4,)),
    ("cfg4 Llama-3-8B layer k_proj 1024x4096", "llama3_8b_layer_tensor", (2,)),
]


def config_input(spec):
    """The seeded BF16 input (as uint16) of one row of CONFIG_TABLE."""
    from lossless_entropy_coded_exponent_b200 import inputs

    gen, args = spec[1], spec[2]
    if gen.startswith("edge:"):
        return inputs.edge_cases()[gen[5:]]
    return getattr(inputs, gen)(*args)


def run_config_table(args, dev, stream, reps=20, flush_mib=512):
    """Decode of each smaller configuration on the GPU (container from dfx_encode, checked
    against the input): median launch time back to back (inputs partly L2-resident) and
    with the L2 flushed before every launch (a 512 MiB buffer written between launches,
    outside the timed region), as decoded BF16 GB/s and as algorithmic GB/s (container +
    2n) against the measured HBM peak."""
    import numpy as np
    import torch

    import lossless_entropy_coded_exponent_b200 as dfx

    peak, peak_kind = measured_hbm_peak()
    flush = torch.empty(flush_mib << 20, dtype=torch.uint8, device=dev)
    rows = []
    for spec in CONFIG_TABLE:
        w = config_input(spec)
        n = int(w.size)
        x = torch.from_numpy(np.ascontiguousarray(w).view(np.int16)).to(dev)
        with dfx.dfx_plan(n, chunk_symbols=args.chunk_symbols) as plan:
            out = torch.empty(plan.max_compressed_bytes, dtype=torch.uint8, device=dev)
            ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=dev)
            size = dfx.dfx_encode(plan, x, out, out.numel(), ws, ws.numel(), want_size=True, stream=stream)
            comp = out[:size].clone()
            del out, ws
            y = torch.empty_like(x)

            def timed(flushed):
                ts = []
                with torch.cuda.stream(stream):
                    for r in range(reps + 3):
                        if flushed:
                            flush.fill_(r & 0xFF)
                        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                        e0.record(stream)
                        dfx.dfx_decode(plan, comp, size, y, stream=stream)
                        e1.record(stream)
                        ts.append((e0, e1))
                stream.synchronize()
                return statistics.median(a.elapsed_time(b) for a, b in ts[3:]) * 1e3

            warm_us, flushed_us = timed(False), timed(True)
            exact = bool(torch.equal(y, x)) and dfx.dfx_device_status(plan, stream=stream) == 0
        algo = float(size) + 2.0 * n
        rows.append({"config": spec[0], "weights": n, "bits_per_weight": 8.0 * size / max(n, 1),
                     "decode_us": warm_us, "decode_us_l2_flushed": flushed_us,
                     "bf16_gbs": 2.0 * n / (warm_us * 1e-6) / 1e9, "bf16_gbs_l2_flushed": 2.0 * n / (flushed_us * 1e-6) / 1e9,
                     "frac_of_measured": algo / (warm_us * 1e-6) / 1e9 / peak,
                     "frac_of_measured_l2_flushed": algo / (flushed_us * 1e-6) / 1e9 / peak, "bit_exact": exact})
        del x, y, comp
    del flush
    return {"peak_gbs": peak, "peak_kind": peak_kind, "reps": reps, "rows": rows,
            "note": "median launch time; 'l2_flushed' writes a 512 MiB buffer before every launch; these tensors "
                    "(at most 59 M weights) are small enough that launch and table-build costs weigh"}


ORACLE_CHILD = r"""
import json, os, sys, time
sys.path.insert(0, sys.argv[1])
core = int(sys.argv[2])
os.sched_setaffinity(0, {core})
import bench, oracle
oracle.lib()
out = []
for spec in bench.CONFIG_TABLE:
    w = bench.config_input(spec)
    t0 = time.perf_counter(); c = oracle.encode(w, K=128); t1 = time.perf_counter()
    d = oracle.decode(c); t2 = time.perf_counter()
    ok = bool((d == w).all())
    out.append({"config": spec[0], "weights": int(w.size), "encode_weights_per_s": w.size / max(t1 - t0, 1e-9),
                "decode_weights_per_s": w.size / max(t2 - t1, 1e-9), "decode_bf16_gbs": 2.0 * w.size / max(t2 - t1, 1e-9) / 1e9,
                "round_trip": ok})
print(json.dumps({"core": core, "rows": out}))
"""


def run_oracle_table():
    """The oracle (single-threaded C) encoding and decoding every row of CONFIG_TABLE in a
    child process pinned to one host core (sched_setaffinity, the same effect as
    taskset -c): weights/s per config, as the benchmark's CPU-baseline plan asks."""
    core = sorted(os.sched_getaffinity(0))[-1]
    r = subprocess.run([sys.executable, "-c", ORACLE_CHILD, ROOT, str(core)], capture_output=True, text=True,
                       timeout=600)
    if r.returncode != 0:
        return {"error": r.stderr[-500:]}
    res = json.loads(r.stdout.strip().splitlines()[-1])
    res.update({"cores": 1, "host": host_cpu(), "kind": "oracle", "pinned": f"sched_setaffinity to core {core}"})
    return res


def run_tans_compare(args, dev, stream, xs, huff_sizes, huff_launch_us, n, tensors=4, reps=10, states=1):
    """The tANS exponent coder (4096 states; one state per chunk, or with states = 2 two
    interleaved states) on the first `tensors` tensors of the workload, with the same
    chunk size and launch configuration: bits/weight, encode time and decode time per
    launch (CUDA events, launches back to back into the reused output buffer), next to
    the Huffman coder's numbers on the same tensors."""
    import numpy as np
    import torch

    import lossless_entropy_coded_exponent_b200 as dfx

    T = min(tensors, len(xs))
    K = args.chunk_symbols
    coder = dfx.DFX_CODER_TANS2 if states == 2 else dfx.DFX_CODER_TANS
    plan = dfx.dfx_plan(n, chunk_symbols=K, coder=coder, decode_flags=dfx.DFX_DECODE_EARLY_READ)
    try:
        scratch = torch.empty(plan.max_compressed_bytes, dtype=torch.uint8, device=dev)
        ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=dev)
        comps, sizes, enc_ms = [], [], []
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            for i in range(T):
                e0.record(stream)
                dfx.dfx_encode(plan, xs[i], scratch, scratch.numel(), ws, ws.numel(), stream=stream)
                e1.record(stream)
                stream.synchronize()
                enc_ms.append(e0.elapsed_time(e1))
                size = int(scratch[24:32].cpu().numpy().view(np.uint64)[0])
                comps.append(scratch[:size].clone())
                sizes.append(size)
        del scratch, ws
        out = torch.empty(n, dtype=torch.int16, device=dev)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
        with torch.cuda.stream(stream):  # as the main measurement: events at step boundaries only
            for _ in range(3):
                for i in range(T):
                    dfx.dfx_decode(plan, comps[i], sizes[i], out, stream=stream)
            ev[0].record(stream)
            for k in range(1, reps + 1):
                for i in range(T):
                    dfx.dfx_decode(plan, comps[i], sizes[i], out, stream=stream)
                ev[k].record(stream)
        stream.synchronize()
        launch_us = [1e3 * ev[j].elapsed_time(ev[j + 1]) / T for j in range(len(ev) - 1)]
        exact = dfx.dfx_device_status(plan, stream=stream) == 0
        with torch.cuda.stream(stream):
            for i in range(T):
                out.fill_(-1)
                dfx.dfx_decode(plan, comps[i], sizes[i], out, stream=stream)
                stream.synchronize()
                exact &= bool(torch.equal(out, xs[i]))
        exact &= dfx.dfx_device_status(plan, stream=stream) == 0
        mean_us = statistics.mean(launch_us)
        algo = float(sum(sizes)) / T + 2.0 * n
        achieved = algo / (mean_us * 1e-6) / 1e9
        peak, peak_kind = measured_hbm_peak()
        return {"coder": "tANS, 4096 states" + (", two interleaved states per chunk" if states == 2 else ""),
                "tensors": T, "chunk_symbols": K,
                "bits_per_weight": 8.0 * sum(sizes) / (n * T),
                "huffman_bits_per_weight": 8.0 * sum(huff_sizes[:T]) / (n * T),
                "decode_mean_launch_us": mean_us, "huffman_mean_launch_us": huff_launch_us,
                "decode_bf16_gbs": 2.0 * n / (mean_us * 1e-6) / 1e9,
                "decode_algorithmic_gbs": achieved, "decode_frac_of_measured": achieved / peak, "peak_kind": peak_kind,
                "encode_median_ms_per_tensor": statistics.median(enc_ms), "bit_exact": bool(exact),
                "kernel": f"k_decode<TansCoder<{states}>, {K}>",
                "note": f"{reps} x {T} launches back to back after 3 x {T} warm-up; the Huffman figures are "
                        "the main measurement's (same shape, K and grid)"}
    finally:
        plan.free()


def run_layer_batch(args, dev, stream):
    """The seven projections of a Llama-3-8B-shaped layer (218 M weights, tensors of 4 M
    to 59 M weights): per layer, seven dfx_decode launches against one dfx_decode_batch."""
    import torch

    import lossless_entropy_coded_exponent_b200 as dfx
    from lossless_entropy_coded_exponent_b200 import inputs

    L = len(inputs.LLAMA3_8B_LAYER)
    with torch.cuda.stream(stream):  # everything below is ordered on this one stream
        xs = [inputs.llama3_8b_layer_tensor_cuda(i, device=dev) for i in range(L)]
    plans = [dfx.dfx_plan(x.numel(), chunk_symbols=args.chunk_symbols, decode_flags=dfx.DFX_DECODE_EARLY_READ)
             for x in xs]
    try:
        comps, sizes = [], []
        with torch.cuda.stream(stream):
            for x, p in zip(xs, plans):
                out = torch.empty(p.max_compressed_bytes, dtype=torch.uint8, device=dev)
                ws = torch.empty(p.workspace_bytes, dtype=torch.uint8, device=dev)
                size = dfx.dfx_encode(p, x, out, out.numel(), ws, ws.numel(), want_size=True, stream=stream)
                comps.append(out[:size].clone())
                sizes.append(size)
            outs = [torch.empty_like(x) for x in xs]
        stream.synchronize()  # the containers are complete before any decode starts

        def separate():
            for i in range(L):
                dfx.dfx_decode(plans[i], comps[i], sizes[i], outs[i], stream=stream)

        def batch():
            dfx.dfx_decode_batch(plans, comps, sizes, outs, stream=stream)

        def time_it(fn, reps=20, warm=3):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
            with torch.cuda.stream(stream):
                for _ in range(warm):
                    fn()
                ev[0].record(stream)
                for r in range(reps):
                    fn()
                    ev[r + 1].record(stream)
            stream.synchronize()
            return statistics.median(ev[r].elapsed_time(ev[r + 1]) for r in range(reps)) * 1e3

        sep_us, bat_us = time_it(separate), time_it(batch)
        with torch.cuda.stream(stream):
            for o in outs:
                o.fill_(-1)
            batch()
        stream.synchronize()
        exact = all(torch.equal(o, x) for o, x in zip(outs, xs)) and all(dfx.dfx_device_status(p) == 0 for p in plans)
        n = sum(x.numel() for x in xs)
        algo = float(sum(sizes)) + 2.0 * n
        peak, peak_kind = measured_hbm_peak()
        return {"workload": "Llama-3-8B-shaped layer: q, o 4096x4096; k, v 1024x4096; gate, up 14336x4096; "
                            "down 4096x14336; N(0, 1/fan_in)", "tensors": L, "weights": n,
                "separate_us": sep_us, "batch_us": bat_us, "batch_algorithmic_gbs": algo / (bat_us * 1e-6) / 1e9,
                "batch_frac_of_measured": algo / (bat_us * 1e-6) / 1e9 / peak, "peak_kind": peak_kind,
                "bit_exact": bool(exact), "note": "median per layer over 20 reps; no L2 flush (0.5 GB of "
                "containers and outputs per layer exceed the 126 MB L2)"}
    finally:
        for p in plans:
            p.free()


def run_decode_into_gemm(args, dev, tokens=16, slice_rows=3584):
    """Y = X W^T for the gate projection of the Llama-3-8B-shaped layer (W 14336x4096
    BF16, X 16x4096), four ways, each replayed from a CUDA graph: W resident as BF16;
    W decoded whole into HBM, then the GEMM; W decoded 3584 rows at a time
    (dfx_decode_range) into two 29 MB buffers that stay in L2, each slice's GEMM (a
    torch/cuBLAS matmul on a second stream) overlapping the next slice's decode; and
    dfx_decode_gemm, one kernel that decodes W into shared-memory tiles and multiplies
    them on the tensor cores (W never written to HBM)."""
    import torch

    import lossless_entropy_coded_exponent_b200 as dfx
    from lossless_entropy_coded_exponent_b200 import inputs

    rows, cols = 14336, 4096
    n_slices = rows // slice_rows
    side = torch.cuda.Stream(device=dev)
    # weights written once and decoded for every product: the decodes may read their
    # container while the kernel before them finishes (both decoding paths alike)
    plan = dfx.dfx_plan(rows * cols, chunk_symbols=args.chunk_symbols, decode_flags=dfx.DFX_DECODE_EARLY_READ)
    try:
        assert dfx.group_elements(plan) == cols, "one group per row needs chunk_symbols = 128"
        w = inputs.llama3_8b_layer_tensor_cuda(4, device=dev)  # gate_proj
        x = (torch.randn(tokens, cols, device=dev, generator=torch.Generator(device=dev).manual_seed(7)) * 0.5
             ).to(torch.bfloat16)
        out = torch.empty(plan.max_compressed_bytes, dtype=torch.uint8, device=dev)
        ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=dev)
        size = dfx.dfx_encode(plan, w, out, out.numel(), ws, ws.numel(), want_size=True)
        comp = out[:size].clone()
        del out, ws
        wb = w.view(torch.bfloat16).view(rows, cols)
        full = torch.empty(rows * cols, dtype=torch.int16, device=dev)
        bufs = [torch.empty(slice_rows * cols, dtype=torch.int16, device=dev) for _ in range(2)]
        y = torch.empty(tokens, rows, dtype=torch.bfloat16, device=dev)
        ys = [torch.empty(tokens, slice_rows, dtype=torch.bfloat16, device=dev) for _ in range(n_slices)]
        yf = torch.empty(tokens, rows, dtype=torch.float32, device=dev)
        torch.cuda.synchronize(dev)

        def resident():
            torch.matmul(x, wb.t(), out=y)

        def whole():
            s = torch.cuda.current_stream()
            dfx.dfx_decode(plan, comp, size, full, stream=s)
            torch.matmul(x, full.view(torch.bfloat16).view(rows, cols).t(), out=y)

        def sliced():
            s = torch.cuda.current_stream()
            side.wait_stream(s)
            freed = [None, None]
            for i in range(n_slices):
                b = i % 2
                if freed[b] is not None:
                    s.wait_event(freed[b])
                dfx.dfx_decode_range(plan, comp, size, i * slice_rows, slice_rows, bufs[b], stream=s)
                ready = torch.cuda.Event()
                ready.record(s)
                side.wait_event(ready)
                with torch.cuda.stream(side):
                    torch.matmul(x, bufs[b].view(torch.bfloat16).view(slice_rows, cols).t(), out=ys[i])
                freed[b] = torch.cuda.Event()
                freed[b].record(side)
            s.wait_stream(side)

        def fused():
            dfx.dfx_decode_gemm(plan, comp, size, rows, cols, x, tokens, yf, stream=torch.cuda.current_stream())

        def graph_time(fn, reps=20):
            cap = torch.cuda.Stream(device=dev)
            with torch.cuda.stream(cap):
                fn()  # once outside capture (library set-up, cuBLAS handles)
            torch.cuda.synchronize(dev)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                fn()
            for _ in range(3):
                g.replay()
            torch.cuda.synchronize(dev)
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            ev[0].record()
            for _ in range(reps):
                g.replay()
            ev[1].record()
            torch.cuda.synchronize(dev)
            del g
            return ev[0].elapsed_time(ev[1]) * 1e3 / reps

        t_res, t_whole, t_sliced = graph_time(resident), graph_time(whole), graph_time(sliced)
        t_fused = graph_time(fused)
        # the fused product against an FP32 product of the same BF16 values
        y32 = x.float() @ wb.float().t()
        fused_rel = float((yf - y32).abs().max() / y32.abs().max())
        w_check = torch.empty(rows * cols, dtype=torch.int16, device=dev)
        dfx.dfx_decode_gemm(plan, comp, size, rows, cols, x, tokens, yf, w_check)
        fused_exact = bool(torch.equal(w_check, w.view(-1))) and dfx.dfx_device_status(plan) == 0
        del w_check
        y_ref = x @ wb.t()
        exact = all(torch.equal(bufs[(n_slices - 2 + k) % 2].view(slice_rows, cols),
                                w.view(rows, cols)[(n_slices - 2 + k) * slice_rows:(n_slices - 1 + k) * slice_rows])
                    for k in range(2)) and dfx.dfx_device_status(plan) == 0
        diff = float((torch.cat(ys, dim=1).float() - y_ref.float()).abs().max())
        return {"workload": f"Y = X W^T, W 14336x4096 BF16 (gate projection of the Llama-3-8B-shaped layer), "
                            f"X {tokens}x4096", "resident_bf16_us": t_res, "decode_whole_then_gemm_us": t_whole,
                "decode_slices_into_gemm_us": t_sliced, "fused_decode_gemm_us": t_fused,
                "fused_decoded_w_bit_exact": fused_exact, "fused_y_max_rel_diff_vs_fp32_gemm": fused_rel,
                "fused_container_gbs": size / t_fused / 1e3,
                "fused_frac_of_measured": size / t_fused / 1e3 / measured_hbm_peak()[0],
                "slice_rows": slice_rows,
                "container_mb": size / 1e6, "bf16_mb": 2 * rows * cols / 1e6,
                "decoded_slices_bit_exact": bool(exact), "y_max_abs_diff_vs_resident_gemm": diff,
                "note": "per product, CUDA-graph replays, mean over 20; the sliced path keeps the decoded weights "
                        "in two 29 MB buffers that stay in the 126 MB L2, so HBM sees the container instead of "
                        "the BF16 matrix; it is slower here because every slice launch builds its tables again "
                        "and the decoder is bound by instruction issue, not by its HBM writes"}
    finally:
        plan.free()


def run_offload(plan, comps, sizes, xs, n, dev, tensors=4, slices=8):
    """Weights kept in pinned host memory and brought to the GPU: raw BF16 copied over
    the host link, against the containers streamed with dfx_decode_host (copies of a
    tensor's slices overlapped with their decoding, two staging buffers)."""
    import torch

    import lossless_entropy_coded_exponent_b200 as dfx

    T = min(tensors, len(comps))
    host_c = [comps[i].cpu().pin_memory() for i in range(T)]
    host_x = [xs[i].cpu().pin_memory() for i in range(T)]
    cap = max(sizes[:T])
    staging = [torch.empty(cap, dtype=torch.uint8, device=dev) for _ in range(2)]
    out = torch.empty(n, dtype=torch.int16, device=dev)
    s_copy, s_dec = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def raw():
        with torch.cuda.stream(s_copy):
            for i in range(T):
                out.copy_(host_x[i], non_blocking=True)
        s_copy.synchronize()

    def compressed():
        for i in range(T):
            s_copy.wait_stream(s_dec)  # staging[i % 2] was read by the decode two tensors back
            dfx.dfx_decode_host(plan, host_c[i], sizes[i], staging[i % 2], cap, out, slices=slices,
                                copy_stream=s_copy, decode_stream=s_dec)
        s_dec.synchronize()

    def wall(fn, reps=3):
        fn()
        best = float("inf")
        for _ in range(reps):
            t0 = time.perf_counter()
            fn()
            best = min(best, time.perf_counter() - t0)
        return best

    dfx.dfx_device_status(plan)  # start from a clear status word
    t_raw, t_comp = wall(raw), wall(compressed)
    equal = bool(torch.equal(out, xs[T - 1]))
    status = dfx.dfx_device_status(plan, stream=s_dec)
    exact = equal and status == 0
    return {"tensors": T, "bf16_bytes_per_tensor": 2 * n, "container_bytes_per_tensor": float(sum(sizes[:T])) / T,
            "raw_bf16_h2d_gbs": 2.0 * n * T / t_raw / 1e9, "compressed_stream_gbs": 2.0 * n * T / t_comp / 1e9,
            "speedup": t_raw / t_comp, "bit_exact": exact, "last_tensor_equal": equal, "device_status": status,
            "slices_per_tensor": slices,
            "note": "GB/s of BF16 delivered to the device from pinned host memory (best of 3, host wall clock "
                    "around a synchronised pass over the tensors)"}


def run_e2e(args, plan, comps, sizes, n, dev, world):
    """Containers in pinned host memory; per tensor: H2D copy, dfx_decode, D2H
    copy of the BF16 result, on three streams so copies overlap decoding."""
    import torch

    import lossless_entropy_coded_exponent_b200 as dfx

    T = len(comps)
    host_c = [c.cpu().pin_memory() for c in comps]
    host_out = torch.empty(n, dtype=torch.int16).pin_memory()
    cap = max(sizes)
    dev_c = [torch.empty(cap, dtype=torch.uint8, device=dev) for _ in range(2)]
    dev_o = [torch.empty(n, dtype=torch.int16, device=dev) for _ in range(2)]
    s_in, s_dec, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))

    # per double-buffer slot, the last decode that read dev_c[b] and the last copy that
    # read dev_o[b], carried across steps: a slot is refilled only after both
    dec_done, d2h_done = [None, None], [None, None]

    def one_step():
        for i in range(T):
            b = i % 2
            if dec_done[b] is not None:
                s_in.wait_event(dec_done[b])
            with torch.cuda.stream(s_in):
                dev_c[b][: sizes[i]].copy_(host_c[i], non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(s_in)
            s_dec.wait_event(ev)
            if d2h_done[b] is not None:
                s_dec.wait_event(d2h_done[b])
            dfx.dfx_decode(plan, dev_c[b], sizes[i], dev_o[b], stream=s_dec)
            dec_done[b] = torch.cuda.Event()
            dec_done[b].record(s_dec)
            s_out.wait_event(dec_done[b])
            with torch.cuda.stream(s_out):
                host_out.copy_(dev_o[b], non_blocking=True)
            d2h_done[b] = torch.cuda.Event()
            d2h_done[b].record(s_out)
        return d2h_done[(T - 1) % 2]

    last = one_step()  # warm-up
    last.synchronize()
    torch.cuda.synchronize(dev)
    barrier(world)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    s_dec.wait_event(start)
    s_out.wait_event(start)
    for _ in range(args.e2e_steps):
        last = one_step()
    s_out.wait_event(last)
    end.record(s_out)
    end.synchronize()
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(start.elapsed_time(end), world)
    barrier(world)
    status = dfx.dfx_device_status(plan, stream=s_dec)
    value = sum_over_ranks(2.0 * n * T * args.e2e_steps, world) / (ms * 1e-3) / 1e9
    return {"value": value, "unit": UNIT, "h2d_bytes_per_step": int(sum(sizes)), "d2h_bytes_per_step": int(2 * n * T),
            "ms_per_step": ms / args.e2e_steps, "steps": args.e2e_steps, "device_status": status,
            "note": "pinned host containers -> H2D -> dfx_decode -> D2H of the BF16 result, copies overlapped"}


def run_cpu_baseline(x0, comp0, K):
    """The oracle (single-threaded C) on tensor 0 of the stream: encode it, compare
    the bytes with the GPU container, then time its decode."""
    import numpy as np

    import oracle

    w = x0.cpu().numpy().view(np.uint16)
    ref = oracle.encode(w, K=K)
    gpu = comp0.cpu().numpy()
    exact = bool(ref.size == gpu.size and np.array_equal(ref, gpu))
    t0 = time.perf_counter()
    dec = oracle.decode(ref)
    dt = time.perf_counter() - t0
    exact &= bool(np.array_equal(dec, w))
    return ({"value": 2.0 * w.size / dt / 1e9, "unit": UNIT, "cores": 1, "host": host_cpu(), "kind": "oracle",
             "sample": f"tensor 0 of the stream ({w.size} weights), one oracle decode, single thread"}, exact)


def main():
    args = parse_args()
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        line = run_reference(args, world, rank)
    else:
        line = run_ours(args, world, rank, local)
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
