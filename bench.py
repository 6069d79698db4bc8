#!/usr/bin/env python
"""Benchmark: DF11 decompression of BF16 weights on B200.

A step is one pass of the whole decode path over one stream: one kernel launch
that rebuilds every matrix of a Llama-3.1-8B-shaped transformer block
(218,112,000 BF16 weights, one shared code table) from its DF11 stream, with
the compressed arrays already resident in HBM.  The workload's inputs and
output (~726 MB per step) exceed the 126 MB L2, so no flush is needed between
steps; smaller configurations write a buffer of twice the L2 size before each
step and time each step on its own.  Every timed output is compared bit for
bit with the original weights.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config c3]
  python bench.py --impl reference ...   # the CPU oracle on the host cores

Under torchrun (N > 1) every rank decompresses its own block (other seeds):
independent streams, no data-path collective ("weak" scaling); the timed
region is bracketed by barriers and the slowest rank's time is reported.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import platform
import re
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decompressed BF16 GB/s on 1 B200 (bit-exact), % of HBM roofline"
METRIC_U8 = "decompressed 8-bit symbols GB/s on 1 B200 (bit-exact), % of HBM roofline"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 2**20  # B200 L2 capacity
LEAD_CYCLES = 200_000    # ~0.1 ms device-side wait before a timed region
KERNEL_SOURCE = os.path.join(ROOT, "lossless_entropy_coded_dfloat11_b200", "csrc", "df11_decode.cu")
# committed ncu summaries giving the decode kernel's DRAM bytes per launch, by workload
TRAFFIC_FILES = {"c3": os.path.join(ROOT, "profiles", "decode_kernel_llama8b_block.txt"),
                 "c5": os.path.join(ROOT, "profiles", "decode_kernel_u8_llama8b_block.txt")}

CONFIGS = {
    "c1": "matrix_1k: one 1024x1024 BF16 matrix, N(0, 0.02)",
    "c2": "matrix_outliers: one 14336x4096 BF16 matrix, N(0, 0.02), 0.1% Laplace(0, 0.5) outliers, 0.01% zeros",
    "c3": "llama3.1-8b-block: q/o 4096x4096, k/v 1024x4096, gate/up 14336x4096, down 4096x14336, "
          "2 RMSNorm 4096; 218,112,000 BF16 weights, one table, one launch",
    "c4": "8 llama3.1-70b-blocks: hidden 8192, intermediate 28672, kv 1024x8192; 855,654,400 weights "
          "per block, each block one launch into one reused buffer",
    "c5": "llama3.1-8b-block quantized per tensor to uint8 (asymmetric, round to nearest); 218,112,000 "
          "8-bit symbols coded whole with one table, no side array, one launch",
    "edge_one_value": "edge sweep, n = 2^26+13: 99.9% of exponents one value (1-bit code), sign+mantissa "
                      "a uniform byte",
    "edge_uniform": "edge sweep, n = 2^26+13: exponents uniform over 0..254 (the stream expands), "
                    "sign+mantissa a uniform byte",
    "edge_zipf": "edge sweep, n = 2^26+13: exponents Zipf(s=1.2) over 255 ranks mapped by a seeded "
                 "permutation, sign+mantissa a uniform byte",
}
U8_CONFIGS = {"c5"}


# --------------------------------------------------------------------------- #
# helpers shared with the CPU tests                                           #
# --------------------------------------------------------------------------- #
def aggregate(per_rank_elapsed_ms: list[float], bytes_per_rank_step: int, steps: int) -> dict:
    """Whole-job throughput: all ranks' bytes over the slowest rank's time."""
    t = max(per_rank_elapsed_ms)
    total = bytes_per_rank_step * steps * len(per_rank_elapsed_ms)
    return {"ms": t, "gbs": total / (t * 1e-3) / 1e9, "ms_per_step": t / steps}


def max_over_ranks(value: float, device) -> float:
    """The largest value over all ranks (the slowest rank's time); a no-op
    without a process group.  `device` is where the reduction tensor lives:
    the rank's GPU under NCCL, the CPU under gloo."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def min_over_ranks(flag: bool, device) -> bool:
    """True only if every rank reports True."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return flag
    t = torch.tensor([1 if flag else 0], device=device, dtype=torch.int32)
    dist.all_reduce(t, op=dist.ReduceOp.MIN)
    return bool(t.item())


def rank_seed_offset(rank: int) -> int:
    """Each rank draws its own block (seeds shifted by 1000 per rank)."""
    return 1000 * rank


def measured_peak_gbs() -> tuple[float, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def recorded_traffic(config: str = "c3") -> float | None:
    """DRAM bytes per launch from the committed ncu summary of this workload,
    only while the kernel source still matches the one that was profiled."""
    try:
        text = open(TRAFFIC_FILES[config]).read()
    except (KeyError, OSError):
        return None
    m_sha = re.search(r"kernel_source_sha256:\s*([0-9a-f]{64})", text)
    m_tr = re.search(r"traffic_bytes_per_launch_full_size:\s*([0-9.eE+]+)", text)
    if not m_sha or not m_tr:
        return None
    sha = hashlib.sha256(open(KERNEL_SOURCE, "rb").read()).hexdigest()
    return float(m_tr.group(1)) if sha == m_sha.group(1) else None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, interval_s: float = 0.005):
        self.interval = interval_s
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self.handle = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = self._handle(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception:  # NVML missing: no clock record
            self.handle = None

    def _handle(self, idx):
        import torch
        p = self.nvml
        props = torch.cuda.get_device_properties(idx)
        bus = getattr(props, "pci_bus_id", None)
        if bus is not None:
            try:
                busid = "%08X:%02X:%02X.0" % (getattr(props, "pci_domain_id", 0), bus,
                                               getattr(props, "pci_device_id", 0))
                return p.nvmlDeviceGetHandleByPciBusId(busid)
            except Exception:
                pass
        return p.nvmlDeviceGetHandleByIndex(idx)

    def _run(self):
        p = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append(p.nvmlDeviceGetClockInfo(self.handle, p.NVML_CLOCK_SM))
                self.reasons |= int(p.nvmlDeviceGetCurrentClocksEventReasons(self.handle))
            except Exception:
                pass
            time.sleep(self.interval)

    def __enter__(self):
        if self.handle is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def record(self) -> dict | None:
        if self.handle is None or not self.samples:
            return None
        s = sorted(self.samples)
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": s[len(s) // 2], "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(s)}


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


# --------------------------------------------------------------------------- #
# workloads                                                                   #
# --------------------------------------------------------------------------- #
EDGE_N = 2 ** 26 + 13  # the edge sweep's largest size


def make_workloads(config: str, rank: int, device: str):
    from lossless_entropy_coded_dfloat11_b200 import inputs as I
    off = rank_seed_offset(rank)
    if config.startswith("edge_"):
        dist = config[len("edge_"):]
        w = I.edge_case(EDGE_N, dist, 500 + len(I.EDGE_SIZES) - 1 + off)
        return [I.Workload(w.name, w.names, [t.to(device) for t in w.tensors])]
    if config == "c1":
        return [I.Workload("matrix_1k", ["w"], [I.gaussian((1024, 1024), 0.02, 1 + off, device=device)])]
    if config == "c2":
        return [I.matrix_outliers(seed=2 + off, device=device)]
    if config == "c3":
        return [I.llama_block(I.LLAMA_8B, seed_base=3 + off, device=device)]
    if config == "c4":
        return [I.llama_block(I.LLAMA_70B, seed_base=100 + 16 * b + off, device=device) for b in range(8)]
    if config == "c5":
        return [I.llama_block_u8(I.LLAMA_8B, seed_base=3 + off, device=device)]
    raise ValueError(config)


def reference_sample(config: str, n_target: int):
    """Host-side sample for the CPU oracle: the first n_target elements of the
    workload's concatenated matrices, drawn with the CPU generator."""
    import numpy as np
    from lossless_entropy_coded_dfloat11_b200 import inputs as I
    if config == "c5":
        # the oracle codes byte v as the exponent field of the BF16 pattern v << 7
        w = I.llama_block_u8(I.LLAMA_8B, seed_base=3)
        v = np.concatenate([t.reshape(-1).numpy() for t in w.tensors])[:n_target]
        return v.astype(np.uint16) << 7
    if config == "c4":
        cfg, base = I.LLAMA_70B, 100
    elif config == "c3":
        cfg, base = I.LLAMA_8B, 3
    else:
        w = I.matrix_1k() if config == "c1" else I.matrix_outliers()
        return w.flat_u16()[:n_target]
    parts, have = [], 0
    for k, (name, shape) in enumerate(I.block_shapes(**cfg)):
        if have >= n_target:
            break
        if len(shape) == 1:
            t = I.gaussian(shape, 0.05, base + k, mean=1.0)
        else:
            t = I.gaussian(shape, 1.0 / (shape[1] ** 0.5), base + k)
        parts.append(t.reshape(-1).view(__import__("torch").int16).numpy().view(np.uint16)[: n_target - have])
        have += parts[-1].size
    return np.concatenate(parts)


def time_oracle_decode(x, steps: int, warmup: int):
    """Oracle (single-threaded C, as it stands) decode of a fixed sample."""
    import numpy as np
    import oracle
    s = oracle.encode(x)
    for _ in range(warmup):
        oracle.decode(s)
    t0 = time.perf_counter()
    for _ in range(steps):
        y = oracle.decode(s)
    dt = time.perf_counter() - t0
    assert np.array_equal(y, x), "oracle round trip failed"
    return dt, s


def time_oracle_decode_parallel(s, x, threads: int):
    """The oracle's windowed decoder on `threads` host threads, one range of
    thread blocks per task: ranges decode independently through their Gaps and
    block offsets, the format's own parallel structure (the C oracle runs
    without the interpreter lock).  Returns (seconds for one full decode, the
    decoded elements), checked against x."""
    import numpy as np
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    parts = max(1, min(int(s.n_blocks), 8 * threads))
    bounds = [int(s.n_blocks) * k // parts for k in range(parts + 1)]

    def run(pool):
        return list(pool.map(lambda k: oracle.decode_windowed(s, bounds[k], bounds[k + 1]), range(parts)))

    with ThreadPoolExecutor(threads) as pool:
        run(pool)
        t0 = time.perf_counter()
        outs = run(pool)
        dt = time.perf_counter() - t0
    y = np.concatenate(outs)
    assert np.array_equal(y, x), "parallel oracle decode failed"
    return dt, y


# --------------------------------------------------------------------------- #
# arms                                                                        #
# --------------------------------------------------------------------------- #
def run_reference(args, rank: int, world: int) -> None:
    if rank != 0:
        return
    n_sample = args.ref_sample
    x = reference_sample(args.config, n_sample)
    dt, s = time_oracle_decode(x, args.steps, args.warmup)
    esize = 1 if args.config in U8_CONFIGS else 2  # output bytes per element
    value = esize * x.size * args.steps / dt / 1e9
    line = {
        "impl": "reference", "metric": METRIC_U8 if esize == 1 else METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u8" if esize == 1 else "bf16",
        "data": "synthetic",
        "config": {"workload": CONFIGS[args.config], "reference_sample_elements": int(x.size)},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"oracle bit-serial decode of the first {x.size} elements of the "
                                   f"workload per step, single thread on {cpu_model()} "
                                   f"({os.cpu_count()} host cores present)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def time_compress(df11, w, repeats: int, u8: bool = False, chunks: bool = False) -> dict:
    """Wall-clock time of the public compress call on device-resident BF16
    tensors (histogram kernel with per-range counts, host code build, encode
    kernel with the decode tables built on the host meanwhile and uploaded
    after it), synchronised on both sides; the median of `repeats` calls
    after one untimed call."""
    import torch
    times = []
    for r in range(repeats + 1):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        cs = (df11.compress_u8 if u8 else df11.compress_chunked if chunks else df11.compress)(w.tensors, names=w.names)
        torch.cuda.synchronize()
        if r:
            times.append(time.perf_counter() - t0)
        del cs
    t = sorted(times)[len(times) // 2]
    in_bytes = sum(x.numel() * x.element_size() for x in w.tensors)
    return {"value": in_bytes / t / 1e9, "unit": "GB/s of uint8 input" if u8 else "GB/s of BF16 input",
            "ms": t * 1e3,
            "repeats": repeats, "elements": sum(x.numel() for x in w.tensors),
            "what": f"df11.{'compress_u8' if u8 else 'compress'} on device-resident "
                    f"{'uint8' if u8 else 'BF16'} tensors: histogram kernel (per-range counts), host "
                    "package-merge, encode kernel (decode tables built on the host meanwhile, uploaded "
                    "after it); median wall clock, synchronised"}


def step_stats(per_step_ms: list[float]) -> dict:
    """Median, min and max of per-step device times (CUDA events)."""
    v = sorted(per_step_ms)
    return {"median": v[len(v) // 2], "min": v[0], "max": v[-1], "n": len(v)}


# how the per-step statistics of back-to-back workloads are taken
PER_STEP_SOURCE = ("a second pass of the same steps right after the timed one, with an event between "
                   "consecutive steps: such an event keeps each launch from overlapping the previous one "
                   "(~3 us per launch here), so the total comes from a pass with events at its ends only")


def time_steps(step, steps: int, warmup: int, stream, flush=None) -> tuple[float, list[float]]:
    """Run `warmup` untimed steps, then time `steps` steps on the launching
    stream.  Without `flush` the steps run back to back: the total is the span
    between an event before the first step and one after the last, and the
    per-step times come from a second pass of the same steps with an event
    between consecutive steps (PER_STEP_SOURCE).  With `flush`, a write of the
    flush buffer (larger than L2) precedes every step and only the steps,
    each between its own pair of events, are summed."""
    import torch
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if flush is None:
        # a short device-side wait ahead of the first event lets the host queue
        # the first launches before the GPU reaches it, so the first step does
        # not include the host's launch latency (the GPU would otherwise idle
        # between the event and the kernel)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda._sleep(LEAD_CYCLES)
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        total = e0.elapsed_time(e1)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        torch.cuda._sleep(LEAD_CYCLES)
        ev[0].record(stream)
        for i in range(steps):
            step()
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
        per = [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]
        return total, per
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i, (e0, e1) in enumerate(evs):
        flush.fill_(i & 0xFF)
        e0.record(stream)
        step()
        e1.record(stream)
    torch.cuda.synchronize()
    per = [e0.elapsed_time(e1) for e0, e1 in evs]
    return sum(per), per


class Prepared:
    """One workload compressed on this GPU, with its decode step and a
    whole-output bit-exactness check to run after the timed region."""

    def __init__(self, df11, config: str, rank: int, dev, chunks: bool = False, compress_repeats: int = 0,
                 options=None):
        import torch
        self.config = config
        self.options = options
        self.u8 = config in U8_CONFIGS
        self.chunks = chunks
        self.esize = 1 if self.u8 else 2
        self.compress = None
        compress = df11.compress_u8 if self.u8 else df11.compress_chunked if chunks else df11.compress
        self.decode = df11.decompress_u8 if self.u8 else df11.decompress_chunked if chunks else df11.decompress
        self.streams, self.originals, self.seeds = [], [], []
        bits = (lambda t: t) if self.u8 else (lambda t: t.view(torch.int16))
        self.bits = bits
        for w in make_workloads(config, rank, "cuda"):
            if self.compress is None and compress_repeats:
                self.compress = time_compress(df11, w, compress_repeats, self.u8, chunks)
            self.streams.append(compress(w.tensors, names=w.names))
            if config == "c4":  # 6.9B weights: regenerate each block for the check instead of keeping it
                self.originals.append(None)
            else:
                self.originals.append(bits(torch.cat([t.reshape(-1) for t in w.tensors])))
            del w
        torch.cuda.synchronize()
        self.n_max = max(cs.n_elems for cs in self.streams)
        self.out = torch.empty(max(self.n_max, 16), dtype=torch.uint8 if self.u8 else torch.bfloat16, device=dev)
        self.out_bytes = sum(self.esize * cs.n_elems for cs in self.streams)
        self.alg_bytes = sum(cs.read_bytes() + self.esize * cs.n_elems for cs in self.streams)
        self.elements = sum(cs.n_elems for cs in self.streams)

    def step(self, stream):
        if self.options is None:
            for cs in self.streams:
                self.decode(cs, out=self.out[: cs.n_elems], stream=stream)
        else:
            for cs in self.streams:
                self.decode(cs, out=self.out[: cs.n_elems], stream=stream, options=self.options)

    def check(self, rank: int, stream) -> tuple[bool, str]:
        """Decode every stream once more and compare every element with the
        original weights (C4: the block regenerated on the device from its
        seeds, since the eight blocks are not kept)."""
        import torch
        from lossless_entropy_coded_dfloat11_b200 import inputs as I
        ok = True
        for b, (cs, orig) in enumerate(zip(self.streams, self.originals)):
            if self.options is None:
                got = self.decode(cs, out=self.out[: cs.n_elems], stream=stream)
            else:
                got = self.decode(cs, out=self.out[: cs.n_elems], stream=stream, options=self.options)
            if orig is None:
                w = I.llama_block(I.LLAMA_70B, seed_base=100 + 16 * b + rank_seed_offset(rank), device="cuda")
                orig = self.bits(torch.cat([t.reshape(-1) for t in w.tensors]))
                del w
            ok &= bool(torch.equal(self.bits(got), orig))
        torch.cuda.synchronize()
        scope = (f"every element of every block ({len(self.streams)} blocks, each decoded again after the timed "
                 "region and compared with the block regenerated on the device)" if self.config == "c4" else
                 "every element of the output, decoded again after the timed region")
        return ok, scope


def measure(pw: Prepared, steps: int, warmup: int, stream, dev, world: int) -> dict:
    """Time one prepared workload and check it; the record every workload
    line carries."""
    import torch
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if pw.alg_bytes < 2 * L2_BYTES else None
    elapsed, per = time_steps(lambda: pw.step(stream), steps, warmup, stream, flush)
    flushed = flush is not None
    del flush
    elapsed = max_over_ranks(elapsed, dev)
    exact, scope = pw.check(0, stream)
    exact = min_over_ranks(exact, dev)
    agg = aggregate([elapsed] * world, pw.out_bytes, steps)
    peak, peak_kind = measured_peak_gbs()
    launches = len(pw.streams)
    launch_ms = elapsed / (steps * launches)
    achieved = (pw.alg_bytes / launches) / (launch_ms * 1e-3) / 1e9
    cs0 = pw.streams[0]
    return {
        "workload": CONFIGS[pw.config], "metric": METRIC_U8 if pw.u8 else METRIC, "value": agg["gbs"],
        "unit": UNIT, "ms_per_step": agg["ms_per_step"], "per_step_ms": step_stats(per),
        "per_step_source": "each step between its own pair of events" if flushed else PER_STEP_SOURCE,
        "elements_per_step": pw.elements, "elements_per_s": agg["gbs"] * 1e9 / pw.esize,
        "launches_per_step": launches, "bit_exact": exact, "bit_exact_scope": scope,
        "compression_ratio": sum(c.compressed_bytes() for c in pw.streams) / pw.out_bytes,
        "threads_per_block": None if pw.chunks else cs0.threads_per_block,
        "decode_kernel": None if pw.chunks else cs0.kernel_info(pw.u8, pw.options),
        "l2": ("no flush: compressed input + output per step exceed the 126 MB L2" if pw.alg_bytes >= 2 * L2_BYTES
               else f"flushed: a {2 * L2_BYTES >> 20} MiB buffer is written before each step; per-step CUDA "
                    "events time the decode alone"),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_kind": f"{peak_kind} (copy bandwidth)",
                     "algorithmic_bytes_per_launch": pw.alg_bytes / launches,
                     "frac_of_8000_nominal": achieved / 8000.0},
        "_elapsed_ms": elapsed,
    }


# the workloads measured besides the headline one in a default run; the
# last three are the C3 block again, through the independent-chunk container
# (an ablation of the gap layout), through the pages' 8-bit first-level table
# (an ablation of the 12-bit one), and with early staging (each launch stages
# its tables and first loads while the previous one finishes: the previous
# launch, a decode of the same stream, writes none of its arrays)
EXTRA_CONFIGS = ["c4", "c2", "c1", "c5", "edge_one_value", "edge_uniform", "edge_zipf", "c3_chunks", "c3_peek8",
                 "c3_early"]
EXTRA_VARIANTS = {"c3_chunks": ("c3", dict(chunks=True)), "c3_peek8": ("c3", dict(peek_bits=8)),
                  "c3_early": ("c3", dict(early_staging=True))}


def run_native(args, rank: int, world: int, local_rank: int) -> None:
    import numpy as np
    import torch
    import torch.distributed as dist
    import lossless_entropy_coded_dfloat11_b200 as df11

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    df11.load_library()
    chunks = args.layout == "chunks"  # independent-chunk variant of the container
    if chunks and args.config in U8_CONFIGS:
        raise SystemExit("--layout chunks takes BF16 configurations")
    stream = torch.cuda.current_stream()

    # ---- the headline workload, built and compressed on this GPU ----------
    opts = df11.decode_options(peek_bits=args.peek_bits) if args.peek_bits else None
    pw = Prepared(df11, args.config, rank, dev, chunks, 0 if args.no_compress else args.compress_repeats, opts)
    for _ in range(args.warmup):
        pw.step(stream)
    torch.cuda.synchronize()

    # ---- timed region -------------------------------------------------------
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if pw.alg_bytes < 2 * L2_BYTES else None
    with sampler:
        elapsed, per_step = time_steps(lambda: pw.step(stream), args.steps, 0, stream, flush)
    if world > 1:
        dist.barrier()
    flushed = flush is not None
    del flush
    exact, exact_scope = pw.check(rank, stream)
    per_rank = [max_over_ranks(elapsed, dev)] * world
    exact = min_over_ranks(exact, dev)
    agg = aggregate(per_rank, pw.out_bytes, args.steps)

    # ---- end to end: host buffers through the public API --------------------
    e2e = None
    if not args.no_e2e and len(pw.streams) == 1 and not chunks:
        hs = df11.HostStream(pw.streams[0])
        for _ in range(2):
            hs.run(stream)
        torch.cuda.synchronize()
        k = args.e2e_steps
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(k):
            res = hs.run(stream)
        e1.record(stream)
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1), dev)
        e2e_exact = min_over_ranks(bool(torch.equal(pw.bits(res), pw.originals[0].cpu())), dev)
        e2e = {"value": pw.esize * pw.streams[0].n_elems * k * world / (ems * 1e-3) / 1e9, "unit": UNIT,
               "h2d_bytes_per_step": hs.h2d_bytes(), "d2h_bytes_per_step": hs.d2h_bytes(),
               "steps": k, "bit_exact": e2e_exact}
        del hs

    # ---- CPU baseline (oracle, rank 0, one GPU) ----------------------------
    cpu = cpu_parallel = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not chunks:
        n_sample = min(args.cpu_sample, pw.streams[0].n_elems)
        if pw.originals[0] is not None:
            x = pw.originals[0][:n_sample].cpu().numpy()
            # the oracle codes byte v as the exponent field of the BF16 pattern v << 7
            x = x.astype(np.uint16) << 7 if pw.u8 else x.view(np.uint16)
        else:
            x = reference_sample(args.config, n_sample)
        dt, sx = time_oracle_decode(x, 1, 0)
        cpu = {"value": pw.esize * x.size / dt / 1e9, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"first {x.size} elements of the workload, oracle bit-serial decode, one "
                         f"thread on {cpu_model()} ({os.cpu_count()} host cores present)",
               "seconds": dt}
        threads = os.cpu_count() or 1
        dtp, _ = time_oracle_decode_parallel(sx, x, threads)
        cpu_parallel = {"value": pw.esize * x.size / dtp / 1e9, "unit": UNIT, "cores": threads,
                        "kind": "oracle windowed decode, ranges of thread blocks on host threads",
                        "sample": cpu["sample"].split(", oracle")[0], "seconds": dtp}

    # ---- headline record ----------------------------------------------------
    peak, peak_kind = measured_peak_gbs()
    launches = len(pw.streams)
    launch_ms = per_rank[0] / (args.steps * launches)
    achieved = (pw.alg_bytes / launches) / (launch_ms * 1e-3) / 1e9
    traffic = recorded_traffic(args.config) if not chunks else None
    cs0 = pw.streams[0]
    line = {
        "metric": METRIC_U8 if pw.u8 else METRIC, "value": agg["gbs"], "unit": UNIT, "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": agg["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "u8" if pw.u8 else "bf16", "data": "synthetic",
        "config": {"workload": CONFIGS[args.config], "elements_per_step": pw.elements,
                   "threads_per_block": None if chunks else cs0.threads_per_block,
                   "layout": (f"independent chunks of {df11.IND_CHUNK} elements (start-bit table), no gaps or scan"
                              if chunks else "gaps + thread-block offsets"),
                   "launches_per_step": launches,
                   "decode_kernel": None if chunks else cs0.kernel_info(pw.u8, opts),
                   "l2": ("no flush: compressed input + output per step exceed the 126 MB L2"
                          if pw.alg_bytes >= 2 * L2_BYTES else
                          f"flushed: a {2 * L2_BYTES >> 20} MiB buffer is written before each step; "
                          "per-step CUDA events time the decode alone"),
                   "parallelism": f"replicas x{world} (independent streams per rank)"},
        "per_step_ms": step_stats(per_step),
        "per_step_source": "each step between its own pair of events" if flushed else PER_STEP_SOURCE,
        "bit_exact": exact, "bit_exact_scope": exact_scope,
        "elements_per_s": agg["gbs"] * 1e9 / pw.esize,
        "compression_ratio": sum(c.compressed_bytes() for c in pw.streams) / pw.out_bytes,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_kind": f"{peak_kind} (copy bandwidth)",
                     "algorithmic_bytes_per_launch": pw.alg_bytes / launches,
                     "frac_of_8000_nominal": achieved / 8000.0},
        "cpu_baseline": cpu,
        "cpu_parallel": cpu_parallel,
        "e2e": e2e,
        "gpu_launches": args.steps * launches,
        "compress": pw.compress,
        "clocks": sampler.record(),
    }
    del pw
    torch.cuda.empty_cache()

    # ---- every other workload, each timed the same way ----------------------
    if world == 1 and not args.headline_only and not chunks and not args.peek_bits:
        extra = {}
        for c in EXTRA_CONFIGS:
            if c == args.config:
                continue
            base, var = EXTRA_VARIANTS.get(c, (c, {}))
            opts = (df11.decode_options(peek_bits=var.get("peek_bits", 0), early_staging=var.get("early_staging", False))
                    if "peek_bits" in var or "early_staging" in var else None)
            # the 8-bit-symbol workload also times its own compress call
            # (compress_u8), the other extras share the headline's codec
            repeats = args.compress_repeats if base in U8_CONFIGS and not var and not args.no_compress else 0
            other = Prepared(df11, base, rank, dev, chunks=var.get("chunks", False), compress_repeats=repeats,
                             options=opts)
            rec = measure(other, args.steps, args.warmup, stream, dev, world)
            if other.compress is not None:
                rec["compress"] = other.compress
            if var:
                rec["variant"] = ("independent chunks of 64 elements (start-bit table), no gaps or scan"
                                  if var.get("chunks") else
                                  "early staging: tables and first loads of each launch staged while the "
                                  "previous launch (a decode of the same stream) finishes"
                                  if var.get("early_staging") else
                                  f"first-level table of {var['peek_bits']} bits held in 16 shared-memory copies")
            rec["gpu_launches"] = args.steps * rec["launches_per_step"]  # in its own timed region
            rec.pop("_elapsed_ms")
            extra[c] = rec
            del other
            torch.cuda.empty_cache()
        line["workloads"] = extra
    line["when"] = datetime.datetime.now(datetime.timezone.utc).isoformat(timespec="seconds")
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_pipeline(args, local_rank: int) -> None:
    """Decompress-into-consumer: Llama-3.1-70B-shaped blocks, each block's
    matrices multiplied by a [tokens, in] BF16 activation (torch matmul) as
    the consumer.  Times, per block: the consumer alone, the decode alone,
    decode then consumer on one stream, and BlockPrefetcher (next block
    decoded on a side stream, optionally on capped SMs).  Prints one JSON
    line."""
    import torch
    import lossless_entropy_coded_dfloat11_b200 as df11
    from lossless_entropy_coded_dfloat11_b200 import inputs as I

    torch.cuda.set_device(local_rank)
    df11.load_library()
    streams = []
    for b in range(args.pipeline_blocks):
        w = I.llama_block(I.LLAMA_70B, seed_base=100 + 16 * b, device="cuda")
        streams.append(df11.compress(w.tensors, names=w.names))
        del w
    n_max = max(cs.n_elems for cs in streams)
    buf = torch.empty(n_max, dtype=torch.bfloat16, device="cuda")
    act = torch.randn(args.tokens, I.LLAMA_70B["intermediate"], device="cuda").to(torch.bfloat16)
    stream = torch.cuda.current_stream()

    def consume(views):
        for v in views:
            if v.dim() == 2:
                torch.matmul(act[:, : v.shape[1]], v.t())

    def timed_on(st, fn, reps=None):
        """Median over `reps` passes (each over every block) of the ms per
        block, events on stream `st` around each pass."""
        reps = reps or args.pipeline_reps
        with torch.cuda.stream(st):
            fn()
            torch.cuda.synchronize()
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
            for e0, e1 in evs:
                e0.record(st)
                fn()
                e1.record(st)
        torch.cuda.synchronize()
        per = sorted(e0.elapsed_time(e1) / len(streams) for e0, e1 in evs)
        return per[len(per) // 2]

    def timed(fn, reps=None):
        return timed_on(stream, fn, reps)

    first = streams[0].views(df11.decompress(streams[0], out=buf[: streams[0].n_elems]))
    res = {"consumer_only": timed(lambda: [consume(first) for _ in streams]),
           "decode_only": timed(lambda: [df11.decompress(cs, out=buf[: cs.n_elems]) for cs in streams])}

    def serial():
        for cs in streams:
            consume(cs.views(df11.decompress(cs, out=buf[: cs.n_elems])))
    res["serial"] = timed(serial)
    for cap in [None] + args.pipeline_sms:
        pf = df11.BlockPrefetcher(streams, max_sms=cap)
        res["prefetch_all_sms" if cap is None else f"prefetch_{cap}_sms"] = timed(
            lambda: [consume(views) for _, views in pf])
    # many small CTAs that queue behind the consumer's kernels and take the
    # SMs those leave idle (cuBLAS's B200 GEMMs run 128 CTAs of up to 226 KB
    # of shared memory: one per SM on 128 of the 148 SMs)
    for ctas, warps in args.pipeline_shapes:
        pf = df11.BlockPrefetcher(streams, options=df11.decode_options(ctas=ctas, max_warps_per_cta=warps))
        res[f"prefetch_{ctas}x{warps}w"] = timed(lambda: [consume(views) for _, views in pf])
    # the consumer on a high-priority stream and the decode on the lowest: when
    # an SM frees up, the block scheduler hands it to the consumer's CTAs
    # first, so the decode's CTAs take what the consumer leaves idle
    hi = torch.cuda.Stream(priority=-100)
    lo = torch.cuda.Stream(priority=0)
    for ctas, warps in [(0, 0)] + list(args.pipeline_shapes):
        opts = df11.decode_options(ctas=ctas, max_warps_per_cta=warps) if ctas else None
        pf = df11.BlockPrefetcher(streams, options=opts, decode_stream=lo)
        key = "prefetch_prio_all_sms" if not ctas else f"prefetch_prio_{ctas}x{warps}w"
        res[key] = timed_on(hi, lambda: [consume(views) for _, views in pf])
    # split: part of the next block on the SMs the consumer leaves idle, the
    # rest after the consumer (consumer on the high-priority stream)
    for frac in args.pipeline_split:
        pf = df11.BlockPrefetcher(streams, decode_stream=lo, split=frac, side_sms=args.side_sms)
        res[f"prefetch_split_{frac:g}_on_{args.side_sms}_sms"] = timed_on(hi, lambda: [consume(views) for _, views in pf])
    res["serial_hi_stream"] = timed_on(hi, serial)
    res["serial_again"] = timed(serial)  # drift check: serial timed first and last
    best = min(v for k, v in res.items() if k.startswith("prefetch"))
    serial_ms = min(res["serial"], res["serial_again"])
    hidden = (serial_ms - best) / min(res["decode_only"], res["consumer_only"])
    flops = 2 * args.tokens * sum(cs.n_elems for cs in streams) / len(streams)
    line = {"metric": "decompress-into-consumer, ms per transformer block", "unit": "ms",
            "higher_is_better": False, "n_gpus": 1, "data": "synthetic",
            "config": {"workload": "llama3.1-70b-blocks (855,654,400 weights each), consumer: "
                                   f"[{args.tokens}, in] x [in, out] BF16 matmul per matrix",
                       "blocks": len(streams), "tokens": args.tokens},
            "ms_per_block": res, "best_prefetch_ms": best,
            "decode_hidden_frac": hidden,
            "consumer_tflops": flops / (res["consumer_only"] * 1e-3) / 1e12,
            "when": datetime.datetime.now(datetime.timezone.utc).isoformat(timespec="seconds")}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--config", choices=sorted(CONFIGS), default="c3")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-sample", type=int, default=218_112_000,
                    help="elements the CPU baseline decodes (bounded sample)")
    ap.add_argument("--ref-sample", type=int, default=1_000_000,
                    help="elements per step in the reference arm")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-compress", action="store_true", help="skip timing the compress call")
    ap.add_argument("--peek-bits", type=int, default=0,
                    help="first-level table width of the timed decode: 12 (default), or 8, 9, 10 for a "
                         "narrow table in 16 shared-memory copies (BF16 configurations)")
    ap.add_argument("--headline-only", action="store_true",
                    help="time the --config workload only, not the other workloads")
    ap.add_argument("--layout", choices=["gaps", "chunks"], default="gaps",
                    help="chunks: the independent-chunk variant of the container (an ablation)")
    ap.add_argument("--compress-repeats", type=int, default=11)
    ap.add_argument("--pipeline", action="store_true",
                    help="time decompress-into-consumer (BlockPrefetcher) instead of the decode alone")
    ap.add_argument("--pipeline-blocks", type=int, default=4)
    ap.add_argument("--pipeline-split", type=float, nargs="*", default=[0.2, 0.3, 0.4],
                    help="fractions of the next block decoded beside the consumer (split prefetch)")
    ap.add_argument("--side-sms", type=int, default=20, help="SMs of the overlapped decode (split prefetch)")
    ap.add_argument("--pipeline-reps", type=int, default=9,
                    help="passes per pipeline variant; the median pass is reported")
    ap.add_argument("--tokens", type=int, default=1024, help="consumer activation rows (--pipeline)")
    ap.add_argument("--pipeline-sms", type=int, nargs="*", default=[16, 32, 64])
    ap.add_argument("--pipeline-shapes", type=lambda v: tuple(int(x) for x in v.split("x")), nargs="*",
                    default=[(1184, 4), (4736, 4), (9472, 2)],
                    help="CTAsxWARPS launch shapes of the prefetched decode (many small CTAs)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("at least 3 warm-up steps")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.pipeline:
        if world == 1:
            run_pipeline(args, local_rank)
        return
    if world > 1:
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_native(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
