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
def make_workloads(config: str, rank: int, device: str):
    from lossless_entropy_coded_dfloat11_b200 import inputs as I
    off = rank_seed_offset(rank)
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


def time_oracle_decode_parallel(s, x, threads: int) -> float:
    """The oracle's windowed decoder on `threads` host threads, one range of
    thread blocks per task: ranges decode independently through their Gaps and
    block offsets, the format's own parallel structure (the C oracle runs
    without the interpreter lock).  Returns seconds for one full decode,
    checked against x."""
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
    assert np.array_equal(np.concatenate(outs), x), "parallel oracle decode failed"
    return dt


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
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u8",
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
    tensors (histogram kernel, host code build, table upload, bit-pack
    kernels), synchronised on both sides; the median of `repeats` calls after
    one untimed call."""
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
                    f"{'uint8' if u8 else 'BF16'} tensors: histogram kernel, host package-merge and "
                    "table build, bit-pack kernels; median wall clock, synchronised"}


def run_native(args, rank: int, world: int, local_rank: int) -> None:
    import numpy as np
    import torch
    import torch.distributed as dist
    import lossless_entropy_coded_dfloat11_b200 as df11

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    df11.load_library()

    # ---- build the compressed workload on this GPU ------------------------
    workloads = make_workloads(args.config, rank, "cuda")
    u8 = args.config in U8_CONFIGS  # 8-bit symbols: uint8 out, no side array
    chunks = args.layout == "chunks"  # independent-chunk variant of the container
    if chunks and u8:
        raise SystemExit("--layout chunks takes BF16 configurations")
    esize = 1 if u8 else 2          # output bytes per element
    bits16 = (lambda t: t) if u8 else (lambda t: t.view(torch.int16))
    streams, originals = [], []
    compress = None
    for w in workloads:
        if compress is None and not args.no_compress:
            compress = time_compress(df11, w, args.compress_repeats, u8, chunks)
        cs = (df11.compress_u8 if u8 else df11.compress_chunked if chunks else df11.compress)(
            w.tensors, names=w.names)
        streams.append(cs)
        originals.append(bits16(torch.cat([t.reshape(-1) for t in w.tensors]))
                         if len(workloads) == 1 else None)
        if len(workloads) > 1:
            # keep a fingerprint per block instead of all 6.9B weights
            originals[-1] = [t.reshape(-1).view(torch.int16)[:: 4093].clone() for t in w.tensors]
        del w
    torch.cuda.synchronize()
    n_max = max(cs.n_elems for cs in streams)
    out = torch.empty(max(n_max, 16), dtype=torch.uint8 if u8 else torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    out_bytes = sum(esize * cs.n_elems for cs in streams)
    alg_bytes = sum(cs.read_bytes() + esize * cs.n_elems for cs in streams)
    launches_per_step = len(streams)
    decode = df11.decompress_u8 if u8 else df11.decompress_chunked if chunks else df11.decompress

    def step():
        for cs in streams:
            decode(cs, out=out[: cs.n_elems], stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---- timed region -------------------------------------------------------
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank)
    # a step whose bytes could stay in L2 is preceded by a write of a buffer
    # twice the L2 size and timed on its own
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if alg_bytes < 2 * L2_BYTES else None
    with sampler:
        if flush is None:
            ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ev0.record(stream)
            for _ in range(args.steps):
                step()
            ev1.record(stream)
            torch.cuda.synchronize()
            elapsed = ev0.elapsed_time(ev1)
        else:
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            for i, (e0, e1) in enumerate(evs):
                flush.fill_(i & 0xFF)
                e0.record(stream)
                step()
                e1.record(stream)
            torch.cuda.synchronize()
            elapsed = sum(e0.elapsed_time(e1) for e0, e1 in evs)
    if world > 1:
        dist.barrier()

    # ---- bit-exact check of the last step's output --------------------------
    exact = True
    if len(streams) == 1:
        exact = bool(torch.equal(bits16(out[: streams[0].n_elems]), originals[0]))
    else:
        for cs, fp in zip(streams, originals):
            step_out = decode(cs, out=out[: cs.n_elems], stream=stream)
            for v, f in zip(cs.views(step_out), fp):
                exact &= bool(torch.equal(v.reshape(-1).view(torch.int16)[:: 4093], f))
    torch.cuda.synchronize()

    per_rank = [max_over_ranks(elapsed, dev)] * world
    exact = min_over_ranks(exact, dev)
    agg = aggregate(per_rank, out_bytes, args.steps)

    # ---- end to end: host buffers through the public API --------------------
    e2e = None
    if not args.no_e2e and len(streams) == 1 and not chunks:
        hs = df11.HostStream(streams[0])
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
        e2e_exact = bool(torch.equal(bits16(res), originals[0].cpu()))
        e2e = {"value": esize * streams[0].n_elems * k * world / (ems * 1e-3) / 1e9, "unit": UNIT,
               "h2d_bytes_per_step": hs.h2d_bytes(), "d2h_bytes_per_step": hs.d2h_bytes(),
               "steps": k, "bit_exact": e2e_exact}
        del hs

    # ---- CPU baseline (oracle, rank 0, one GPU) ----------------------------
    cpu = cpu_parallel = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not chunks:
        n_sample = min(args.cpu_sample, streams[0].n_elems)
        if len(streams) == 1:
            x = originals[0][:n_sample].cpu().numpy()
            # the oracle codes byte v as the exponent field of the BF16 pattern v << 7
            x = x.astype(np.uint16) << 7 if u8 else x.view(np.uint16)
        else:
            x = reference_sample(args.config, n_sample)
        dt, sx = time_oracle_decode(x, 1, 0)
        cpu = {"value": esize * x.size / dt / 1e9, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"first {x.size} elements of the workload, oracle bit-serial decode, one "
                         f"thread on {cpu_model()} ({os.cpu_count()} host cores present)",
               "seconds": dt}
        threads = os.cpu_count() or 1
        dtp = time_oracle_decode_parallel(sx, x, threads)
        cpu_parallel = {"value": esize * x.size / dtp / 1e9, "unit": UNIT, "cores": threads,
                        "kind": "oracle windowed decode, ranges of thread blocks on host threads",
                        "sample": cpu["sample"].split(", oracle")[0], "seconds": dtp}

    if rank != 0:
        return
    peak, peak_kind = measured_peak_gbs()
    launch_ms = elapsed / (args.steps * launches_per_step)
    achieved = (alg_bytes / launches_per_step) / (launch_ms * 1e-3) / 1e9
    traffic = recorded_traffic(args.config) if not chunks else None
    cs0 = streams[0]
    line = {
        "metric": METRIC_U8 if u8 else METRIC, "value": agg["gbs"], "unit": UNIT, "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": agg["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "u8", "data": "synthetic",
        "config": {"workload": CONFIGS[args.config], "elements_per_step": sum(c.n_elems for c in streams),
                   "threads_per_block": None if chunks else cs0.threads_per_block,
                   "layout": (f"independent chunks of {df11.IND_CHUNK} elements (start-bit table), no gaps or scan"
                              if chunks else "gaps + thread-block offsets"),
                   "launches_per_step": launches_per_step,
                   "l2": ("no flush: compressed input + output per step exceed the 126 MB L2"
                          if flush is None else
                          f"flushed: a {2 * L2_BYTES >> 20} MiB buffer is written before each step; "
                          "per-step CUDA events time the decode alone"),
                   "parallelism": f"replicas x{world} (independent streams per rank)"},
        "bit_exact": exact,
        "elements_per_s": agg["gbs"] * 1e9 / esize,
        "compression_ratio": sum(c.compressed_bytes() for c in streams) / out_bytes,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_kind": f"{peak_kind} (copy bandwidth)",
                     "algorithmic_bytes_per_launch": alg_bytes / launches_per_step,
                     "frac_of_8000_nominal": achieved / 8000.0},
        "cpu_baseline": cpu,
        "cpu_parallel": cpu_parallel,
        "e2e": e2e,
        "gpu_launches": args.steps * launches_per_step,
        "compress": compress,
        "clocks": sampler.record(),
        "when": datetime.datetime.now(datetime.timezone.utc).isoformat(timespec="seconds"),
    }
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

    def timed(fn, reps=3):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / (reps * len(streams))

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
    best = min(v for k, v in res.items() if k.startswith("prefetch"))
    hidden = (res["serial"] - best) / min(res["decode_only"], res["consumer_only"])
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
    ap.add_argument("--layout", choices=["gaps", "chunks"], default="gaps",
                    help="chunks: the independent-chunk variant of the container (an ablation)")
    ap.add_argument("--compress-repeats", type=int, default=5)
    ap.add_argument("--pipeline", action="store_true",
                    help="time decompress-into-consumer (BlockPrefetcher) instead of the decode alone")
    ap.add_argument("--pipeline-blocks", type=int, default=4)
    ap.add_argument("--tokens", type=int, default=1024, help="consumer activation rows (--pipeline)")
    ap.add_argument("--pipeline-sms", type=int, nargs="*", default=[16, 32, 64])
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
