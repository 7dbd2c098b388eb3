"""Benchmark of the MXFP8 hot path on B200.

One step = one pass of the MXFP8 path over one batch: rowwise quantize of a
bf16 activation [16384, 7168] (Student-t(3) * 0.5, 1 % zero groups, 0.5 %
groups scaled by 2^-120, seed 2) with compact and 128x4-swizzled scales, then
dequantize back to bf16. The metric is algorithmic HBM bytes (read + written)
per second; the input (235 MB) is larger than the 126 MB L2, so no flush is
needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mxq|reference]
    python -m torch.distributed.run --nproc-per-node N bench.py --gpus N ...

Timing: the K steps run back to back between two CUDA events (nothing
recorded between kernels). The roofline's per-kernel time comes from a
separate loop of back-to-back launches of each kernel alone. Before the
headline line, one line per remaining workload (planted 256x1024, linear
weight 4096x4096, 64 stacked experts, NVFP4 8192x8192) gives its median
kernel time and a bit-exact check against the oracle on sampled rows.

Multi-GPU: every rank quantizes its own batch (rows are independent, so the
path shards with no exchange); value = bytes of all ranks / max over ranks of
the device-timed region ("scaling": "weak").

``--impl reference`` times the CPU oracle (test infrastructure) on the host's
cores (row chunks on threads, each running the single-threaded oracle) on a
bounded sample of the same workload. ``--suite`` prints one extra JSON line
per workload kernel (documentation beside the headline line).
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "MXFP8 quantize GB/s (read+write) and % of B200 HBM peak, bit-exact"
SPEC_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
SAMPLE_EVERY = 16
M_ROWS, N_COLS = 16384, 7168


# ------------------------------------------------------------------ bytes

def mxfp8_quant_bytes(M, N, in_bytes=2, swizzled=True):
    E = M * N
    S = N // 32
    swz = ((M + 127) // 128 * 128) * ((S + 3) // 4 * 4) if swizzled else 0
    return E * in_bytes + E + E // 32 + swz


def mxfp8_dequant_bytes(M, N, out_bytes=2):
    E = M * N
    return E + E // 32 + E * out_bytes


def mxfp4_quant_bytes(M, N, in_bytes=2, swizzled=False):
    E = M * N
    S = N // 32
    swz = ((M + 127) // 128 * 128) * ((S + 3) // 4 * 4) if swizzled else 0
    return E * in_bytes + E // 2 + E // 32 + swz


def mxfp4_dequant_bytes(M, N, out_bytes=2):
    E = M * N
    return E // 2 + E // 32 + E * out_bytes


def fake_quant_bytes(M, N, in_bytes=2, out_bytes=2):
    return M * N * (in_bytes + out_bytes)


def nvfp4_quant_bytes(M, N, in_bytes=2, two_pass=True):
    E = M * N
    return E * in_bytes * (2 if two_pass else 1) + E // 2 + E // 16 + 4


# ------------------------------------------------------------------ peaks

def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def tensor_peak(sustained=False):
    """fp8 dense peak: the measured bf16 figure times the nominal fp8 / bf16
    ratio of 2; the burst figure for a kernel timed alone, the sustained one
    (seconds of back-to-back GEMMs under the power cap) when asked."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    try:
        with open(p) as f:
            return 2.0 * float(json.load(f)[key]), f"measured {key} x 2"
    except Exception:
        return 2.0 * (1400.0 if sustained else 1590.0), "fallback bf16 x 2"


KERNEL_SOURCES = {"mx_quant_kernel": ("common.cuh", "mx_rowwise.cu"),
                  "mx_dequant_kernel": ("common.cuh", "mx_rowwise.cu"),
                  "mx_fake_quant_kernel": ("common.cuh", "mx_rowwise.cu"),
                  "mx_swizzle_experts_kernel": ("common.cuh", "mx_rowwise.cu"),
                  "mxfp8_colwise_kernel": ("common.cuh", "colwise.cu"),
                  "nvfp4_amax_kernel": ("common.cuh", "nvfp4.cu"),
                  "nvfp4_quant_kernel": ("common.cuh", "nvfp4.cu"),
                  "nvfp4_dequant_kernel": ("common.cuh", "nvfp4.cu")}


def kernel_source_sha(kernel):
    """Hash of the source files a kernel is built from."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "nvfp4_block_scaled_sm_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources (else None)."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[kernel]
        if rec.get("source_sha") == kernel_source_sha(kernel):
            return int(rec["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device: torch.device):
        self.samples, self.reasons, self.err = [], 0, None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception as e:  # NVML unavailable: report, do not guess
            self.err = f"nvml: {e}"
            self.h = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= self._reasons_fn(self.h)
            except Exception as e:
                self.err = str(e)
                return
            time.sleep(0.0005)

    def __enter__(self):
        if self.h is not None:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.h is not None:
            self._stop.set()
            self.t.join()

    def summary(self):
        if self.h is None or not self.samples:
            return {"error": self.err or "no samples"}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": float(self.max_mhz),
                "samples": len(self.samples), "reasons": names}


# ------------------------------------------------------------ distributed

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and not (world == 1 and args.gpus == 1):
        if world == 1:
            raise SystemExit(f"--gpus {args.gpus} needs torchrun with {args.gpus} processes")
        raise SystemExit(f"WORLD_SIZE={world} but --gpus {args.gpus}")
    return world, rank, local


def reduce_max(value: float, world: int, device) -> float:
    """Max of a per-rank float over all ranks (identity for one rank)."""
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------ CPU oracle

def host_threads(cap: int = 64) -> int:
    """Host cores this process may run on (capped)."""
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return max(1, min(cap, n))


def oracle_round_trip(x: np.ndarray):
    """Oracle MXFP8 quantize + swizzle + dequantize of the rows x (one
    single-threaded call of each)."""
    import oracle
    q, s = oracle.mxfp8_quantize(x)
    z = oracle.swizzle_scales(s)
    y = oracle.mxfp8_dequantize(q, s, out="bf16")
    return q, s, z, y


def pmap(fn, items, threads: int):
    """[fn(i) for i in items] on `threads` host threads. The oracle's C calls
    release the interpreter lock (ctypes), so each thread runs the unchanged
    single-threaded oracle on its own item."""
    from concurrent.futures import ThreadPoolExecutor
    items = list(items)
    if threads == 1:
        return [fn(i) for i in items]
    with ThreadPoolExecutor(threads) as ex:
        return list(ex.map(fn, items))


def oracle_rows_parallel(fn, x: np.ndarray, threads: int, chunk: int = 128):
    """fn over consecutive row chunks of x on `threads` host threads; results
    in row order."""
    parts = [np.ascontiguousarray(x[i:i + chunk]) for i in range(0, x.shape[0], chunk)]
    return pmap(fn, parts, threads)


def calibrate_row_seconds(x: np.ndarray, rows: int = 64) -> float:
    """Single-thread oracle round-trip seconds per row of x."""
    import oracle
    oracle.build()
    t0 = time.perf_counter()
    oracle_round_trip(np.ascontiguousarray(x[:rows]))
    return (time.perf_counter() - t0) / rows


def cpu_baseline(x_full: np.ndarray, target_s: float = 12.0):
    """The oracle round trip on all host cores (row chunks on threads) over
    the first rows of the workload, as many as fit in about target_s.
    Returns (cpu_baseline dict, rows, concatenated oracle outputs)."""
    threads = host_threads()
    t_row = calibrate_row_seconds(x_full)
    rows = int(min(x_full.shape[0], max(128, target_s * threads / max(t_row, 1e-9))))
    rows = rows // 128 * 128 or min(128, x_full.shape[0])
    x = x_full[:rows]
    t0 = time.perf_counter()
    res = oracle_rows_parallel(oracle_round_trip, x, threads)
    el = time.perf_counter() - t0
    outs = tuple(np.concatenate([r[i] for r in res]) for i in range(4))
    nbytes = mxfp8_quant_bytes(rows, N_COLS) + mxfp8_dequant_bytes(rows, N_COLS)
    return ({"value": nbytes / el / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
             "sample": f"first {rows} of {M_ROWS} rows of the activation workload, quantize "
                       f"(+swizzle) + dequantize, scalar C oracle on {threads} threads "
                       f"(128-row chunks), one pass of {el:.1f} s"},
            rows, outs)


def cpu_baseline_single_thread_planted(min_seconds: float = 1.0):
    """The oracle on one core over the small planted workload (256x1024)."""
    x = W.planted()
    passes, t0 = 0, time.perf_counter()
    while True:
        oracle_round_trip(x)
        passes += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    nbytes = mxfp8_quant_bytes(256, 1024) + mxfp8_dequant_bytes(256, 1024)
    return {"value": nbytes * passes / el / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"planted 256x1024, quantize (+swizzle) + dequantize, {passes} passes, "
                      "one thread"}


def run_reference(args):
    world, rank, _ = dist_setup(args)
    if rank != 0:
        return
    x_all = W.activation(M=M_ROWS, N=N_COLS)
    input_sha = hashlib.sha256(x_all.tobytes()).hexdigest()[:16]
    threads = host_threads()
    t_row = calibrate_row_seconds(x_all)
    budget = 120.0
    rows = int(max(128, min(M_ROWS, budget / max(1, args.steps + args.warmup) * threads / t_row)))
    rows = min(M_ROWS, rows // 128 * 128 or 128)
    x = x_all[:rows]
    for _ in range(args.warmup):
        oracle_rows_parallel(oracle_round_trip, x, threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_rows_parallel(oracle_round_trip, x, threads)
    el = time.perf_counter() - t0
    nbytes = (mxfp8_quant_bytes(rows, N_COLS) + mxfp8_dequant_bytes(rows, N_COLS)) * args.steps
    value = nbytes / el / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_block(world, input_sha),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": f"first {rows} of {M_ROWS} rows per step of the "
                                       f"{M_ROWS}x{N_COLS} activation workload, scalar C oracle "
                                       f"on {threads} threads (128-row chunks)"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_block(world, input_sha=None):
    c = {"workload": f"MXFP8 rowwise quantize (+128x4 swizzled scales) + dequantize round "
                        f"trip of a bf16 activation {M_ROWS}x{N_COLS}, Student-t(df=3)*0.5, 1% "
                        f"zero groups, 0.5% groups x2^-120, seed 2",
            "shape": [M_ROWS, N_COLS], "input_dtype": "bf16", "group": 32,
            "outputs": "e4m3 u8 [M,N], e8m0 u8 [M,N/32], swizzled e8m0, bf16 [M,N]",
            "l2": "inputs larger than L2 (235 MB bf16 input per step), no flush",
            "parallelism": f"replicas x{world} (rows independent, no exchange)"}
    if input_sha:
        c["input_sha256_rank0"] = input_sha
    return c


# -------------------------------------------------------------------- main

def events_loop(stream, fn, n: int) -> float:
    """Device milliseconds of n back-to-back calls of fn() on `stream`, with
    nothing recorded between them (events only before the first and after
    the last)."""
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(n):
        fn()
    b.record(stream)
    while not b.query():
        time.sleep(0.0002)
    torch.cuda.synchronize()
    return a.elapsed_time(b)


def e2e_chunks(M: int, first: int = 512, cap: int = 2048):
    """Row bounds of the end-to-end pipeline's chunks: `first` rows, then
    doubling up to `cap` (all multiples of 128 but the last). The download of
    the outputs is the longer direction on the host link; a small first chunk
    starts it early (measured 94.4 GB/s against 91.9 with eight equal chunks,
    and 90 with sixteen)."""
    bounds, r, c = [0], 0, first
    while r < M:
        c = min(c, cap, M - r)
        r += c
        bounds.append(r)
        c *= 2
    return bounds


def e2e_pipelined(mxq, x_h, outs_h, bounds, device):
    """One end-to-end step through the public Python API: the pinned host
    input goes to the device in row chunks (rows bounds[i] .. bounds[i+1]) on
    one stream, each chunk is quantized (+ swizzled scales) and dequantized on
    a second stream as soon as it has arrived, and its outputs go back to
    pinned host memory on a third, so uploads, kernels and downloads of
    different chunks overlap. Chunks start at multiples of 128 rows, so each
    chunk's swizzled scales are one contiguous slice of the full layout.
    Returns the device milliseconds of the step (events on the caller's
    stream around all three streams)."""
    q_h, s_h, z_h, y_h = outs_h
    M, N = x_h.shape
    Sp = (N // 32 + 3) // 4 * 4
    main = torch.cuda.current_stream(device)
    up, comp, down = e2e_pipelined.streams
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    for st in (up, comp, down):
        st.wait_event(e0)
    x_d = e2e_pipelined.x_d
    keep = []
    for r0, r1 in zip(bounds[:-1], bounds[1:]):
        with torch.cuda.stream(up):
            x_d[r0:r1].copy_(x_h[r0:r1], non_blocking=True)
            arrived = torch.cuda.Event()
            arrived.record(up)
        with torch.cuda.stream(comp):
            comp.wait_event(arrived)
            q, s, z = mxq.mxfp8_quantize(x_d[r0:r1], swizzled=True)
            y = mxq.mxfp8_dequantize(q, s, torch.bfloat16)
            done = torch.cuda.Event()
            done.record(comp)
        with torch.cuda.stream(down):
            down.wait_event(done)
            q_h[r0:r1].copy_(q, non_blocking=True)
            s_h[r0:r1].copy_(s, non_blocking=True)
            z_h[r0 * Sp:r0 * Sp + z.numel()].copy_(z, non_blocking=True)
            y_h[r0:r1].copy_(y, non_blocking=True)
        keep.append((q, s, z, y))
    fin = torch.cuda.Event()
    fin.record(down)
    main.wait_event(fin)
    e1.record(main)
    e1.synchronize()                     # the chunk outputs in `keep` are free after this
    del keep
    return e0.elapsed_time(e1)


def sample_rows(M: int, n: int, seed: int) -> np.ndarray:
    """First, last and n seeded random rows of M (sorted, unique)."""
    rng = np.random.default_rng(seed)
    rows = set(range(min(M, 64))) | set(range(max(0, M - 64), M))
    rows |= set(int(r) for r in rng.integers(0, M, n))
    return np.array(sorted(rows))


def config_lines(mxq, device, flush):
    """One bounded line per remaining workload of the statement of the
    problem: median device time over repeated launches, algorithmic bytes,
    GB/s, fractions of the measured and spec HBM peaks, and a bit-exact
    check of the timed launch's outputs against the oracle on sampled rows
    (all rows for the small workloads)."""
    import oracle
    peak, kind = hbm_peak()
    threads = host_threads()
    lines = []

    def check(st):
        if st:
            raise mxq.MxqError("bench", st, mxq.lib.mxq_status_string(st).decode())

    def bf(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)

    def line(cfg, name, nbytes, t_ms, exact, checked, extra=None):
        med = t_ms
        d = {"config_line": cfg, "workload": name, "median_us": med * 1e3, "bytes": nbytes,
             "gbs": nbytes / med / 1e6, "frac_of_" + kind: nbytes / med / 1e6 / peak,
             "frac_of_spec_8tbs": nbytes / med / 1e6 / SPEC_HBM_GBS,
             "bit_exact_vs_oracle": bool(exact), "checked": checked}
        if extra:
            d.update(extra)
        lines.append(d)
        print(json.dumps(d), flush=True)

    # 1: planted 256x1024, quantize (+swizzle) and dequantize, L2 flushed
    x = W.planted()
    xd = bf(x)
    tq = time_kernel(lambda: mxq.mxfp8_quantize(xd, swizzled=True), 50, flush)[0]
    q, s, z = mxq.mxfp8_quantize(xd, swizzled=True)
    td = time_kernel(lambda: mxq.mxfp8_dequantize(q, s), 50, flush)[0]
    y = mxq.mxfp8_dequantize(q, s)
    qo, so, zo, yo = oracle_round_trip(x)
    ok = (np.array_equal(q.cpu().numpy(), qo) and np.array_equal(s.cpu().numpy(), so)
          and np.array_equal(z.cpu().numpy(), zo)
          and np.array_equal(y.view(torch.int16).cpu().numpy().view(np.uint16), yo))
    line(1, "MXFP8 quantize (+swizzle) + dequantize, planted bf16 256x1024 (L2 flushed, "
            "launch-bound)", mxfp8_quant_bytes(256, 1024) + mxfp8_dequant_bytes(256, 1024),
         tq + td, ok, "all rows, all outputs",
         {"quantize_us": tq * 1e3, "dequantize_us": td * 1e3,
          "cpu_baseline_single_thread": cpu_baseline_single_thread_planted()})

    # 2: linear weight 4096x4096, quantize; 8 rotating input/output sets (> 2x L2),
    # back-to-back launches
    L, sp = mxq.lib, ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    stream = torch.cuda.current_stream(device)
    V = lambda t: ctypes.c_void_p(t.data_ptr())
    x = W.linear_weight()
    xs = [bf(x) for _ in range(8)]
    outs = [mxq.mxfp8_quantize(t) for t in xs]
    P = [[V(t) for t in (xs[i], outs[i][0], outs[i][1])] for i in range(8)]
    k = [0]

    def rot():
        p = P[k[0] % 8]
        k[0] += 1
        check(L.mxfp8_quantize(p[0], 0, 4096, 4096, 4096, p[1], p[2], None, sp))

    for _ in range(8):
        rot()
    t = events_loop(stream, rot, 96) / 96
    qo, so = zip(*oracle_rows_parallel(oracle.mxfp8_quantize, x, threads, 256))
    ok = (np.array_equal(outs[0][0].cpu().numpy(), np.concatenate(qo))
          and np.array_equal(outs[0][1].cpu().numpy(), np.concatenate(so)))
    line(2, "MXFP8 quantize, linear weight bf16 4096x4096 (8 rotating input/output sets, "
            "back-to-back launches)", mxfp8_quant_bytes(4096, 4096, swizzled=False), t, ok,
         "all rows")
    del xs, outs, P
    torch.cuda.empty_cache()

    # 4: 64 experts 2048x7168 stacked, one grouped launch (compact outputs), and
    # with the per-expert swizzled scales (a second, gather launch)
    E, R, Nn = 64, 2048, 7168
    x = W.experts()
    xd = bf(x)
    del x
    off = (torch.arange(E + 1, dtype=torch.int64) * R).to(device)
    q = torch.empty((E * R, Nn), dtype=torch.uint8, device=device)
    s = torch.empty((E * R, Nn // 32), dtype=torch.uint8, device=device)
    z = torch.empty(E * R * (Nn // 32), dtype=torch.uint8, device=device)
    grouped = lambda: check(L.mxfp8_quantize_grouped(V(xd), 0, E, V(off), E * R, Nn, V(q), V(s), sp))
    grouped_swz = lambda: check(L.mxfp8_quantize_grouped_swizzled(
        V(xd), 0, E, V(off), E * R, Nn, V(q), V(s), V(z), z.numel(), sp))
    for _ in range(3):
        grouped_swz()
    t_swz = events_loop(stream, grouped_swz, 10) / 10
    for _ in range(3):
        grouped()
    t = events_loop(stream, grouped, 10) / 10
    grouped_swz()
    picks = [0, 9, 21, 30, 42, 51, 58, 63]
    xh = {e: xd[e].view(torch.int16).cpu().numpy().view(np.uint16) for e in picks}
    res = pmap(lambda e: oracle.mxfp8_quantize(xh[e]), picks, threads)
    blk = R * (Nn // 32)
    ok = True
    qv, sv = q.view(E, R, Nn), s.view(E, R, Nn // 32)
    for e, (qo, so) in zip(picks, res):
        ok &= np.array_equal(qv[e].cpu().numpy(), qo) and np.array_equal(sv[e].cpu().numpy(), so)
        ok &= np.array_equal(z[e * blk:(e + 1) * blk].cpu().numpy(), oracle.swizzle_scales(so))
    line(4, "grouped MXFP8 quantize, 64 stacked experts bf16 2048x7168, one launch "
            "(back-to-back launches)", mxfp8_quant_bytes(E * R, Nn, swizzled=False), t, ok,
         f"experts {picks}: codes, scales and per-expert swizzled scales",
         {"with_per_expert_swizzled_scales_us": t_swz * 1e3,
          "with_per_expert_swizzled_scales_gbs": mxfp8_quant_bytes(E * R, Nn) / t_swz / 1e6})
    del xd, q, s, z, qv, sv
    torch.cuda.empty_cache()

    # 5: NVFP4 two passes, 8192x8192 (and the block pass alone, given the scale)
    x = W.nvfp4_tensor()
    xd = bf(x)
    ws = torch.empty(mxq.nvfp4_workspace_bytes(), dtype=torch.uint8, device=device)
    p = torch.empty((8192, 4096), dtype=torch.uint8, device=device)
    b = torch.empty((8192, 512), dtype=torch.uint8, device=device)
    g = torch.empty((), dtype=torch.float32, device=device)
    gg = torch.empty((), dtype=torch.float32, device=device)
    two = lambda: check(L.nvfp4_quantize(V(xd), 0, 8192, 8192, 8192, V(p), V(b), V(g), None, 0,
                                         V(ws), ws.numel(), sp))
    given = lambda: check(L.nvfp4_quantize(V(xd), 0, 8192, 8192, 8192, V(p), V(b), V(gg), None, 1,
                                           None, 0, sp))
    for _ in range(3):
        two()
    t = events_loop(stream, two, 30) / 30
    gg.copy_(g)
    for _ in range(3):
        given()
    tg = events_loop(stream, given, 30) / 30
    two()
    go = oracle.nvfp4_global_amax(x) / np.float32(2688.0)
    rows = sample_rows(8192, 512, 5)
    res = oracle_rows_parallel(lambda xr: oracle.nvfp4_quantize(xr, float(go))[:2],
                               x[rows], threads, 64)
    po, bo = np.concatenate([r[0] for r in res]), np.concatenate([r[1] for r in res])
    ok = (np.float32(g.item()) == np.float32(go)
          and np.array_equal(p.cpu().numpy()[rows], po) and np.array_equal(b.cpu().numpy()[rows], bo))
    single = nvfp4_quant_bytes(8192, 8192, two_pass=False)
    line(5, "NVFP4 two-level quantize (amax pass + block pass), bf16 8192x8192 (back-to-back "
            "launches)", nvfp4_quant_bytes(8192, 8192), t, ok,
         f"global scale and {rows.size} sampled rows",
         {"single_read_bytes": single, "gbs_single_read_count": single / t / 1e6,
          "block_pass_given_scale_us": tg * 1e3, "block_pass_gbs": single / tg / 1e6,
          "block_pass_frac_of_" + kind: single / tg / 1e6 / peak})
    del xd, p, b
    torch.cuda.empty_cache()
    return lines


def run(args):
    world, rank, local = dist_setup(args)
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    import nvfp4_block_scaled_sm_b200 as mxq
    L = mxq.lib

    xb = W.activation(seed=2 + 1000 * rank, M=M_ROWS, N=N_COLS)
    input_sha = hashlib.sha256(xb.tobytes()).hexdigest()[:16] if rank == 0 else None
    x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to(device)
    M, N = M_ROWS, N_COLS
    S = N // 32
    q = torch.empty((M, N), dtype=torch.uint8, device=device)
    s = torch.empty((M, S), dtype=torch.uint8, device=device)
    swz = torch.empty(mxq.swizzled_scale_bytes(M, S), dtype=torch.uint8, device=device)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream(device)
    sp = ctypes.c_void_p(stream.cuda_stream)
    P = [ctypes.c_void_p(t.data_ptr()) for t in (x, q, s, swz, y)]

    def quant():
        st = L.mxfp8_quantize(P[0], 0, M, N, N, P[1], P[2], P[3], sp)
        if st:
            raise mxq.MxqError("mxfp8_quantize", st, L.mxq_status_string(st).decode())

    def dequant():
        st = L.mxfp8_dequantize(P[1], P[2], M, N, P[4], 0, sp)
        if st:
            raise mxq.MxqError("mxfp8_dequantize", st, L.mxq_status_string(st).decode())

    def step():
        quant()
        dequant()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)

    # the timed region: K steps back to back, events only around all of them
    K = args.steps
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(device) as clk:
        elapsed_ms = events_loop(stream, step, K)
    if world > 1:
        torch.distributed.barrier()
    max_ms = reduce_max(elapsed_ms, world, device)

    # outputs of the timed region's last step, kept for the oracle check
    q_out, s_out = q.cpu().numpy(), s.cpu().numpy()
    z_out = swz.cpu().numpy()
    y_out = y.view(torch.int16).cpu().numpy().view(np.uint16)

    # per-kernel device time for the roofline: R launches of one kernel back
    # to back between two events (every launch rewrites the same outputs),
    # after three untimed ones, so that the write-back of the other kernel's
    # dirty lines left in L2 does not land in the loop
    R = max(50, min(200, K))
    with ClockSampler(device) as clk_k:
        for _ in range(3):
            quant()
        q_ms = events_loop(stream, quant, R) / R
        for _ in range(3):
            dequant()
        d_ms = events_loop(stream, dequant, R) / R
    q_ms = reduce_max(q_ms, world, device)
    d_ms = reduce_max(d_ms, world, device)

    # end to end through the public API: pinned host input -> device, quantize
    # (+ swizzled scales), dequantize, every output -> pinned host, each step,
    # with uploads, kernels and downloads of row chunks overlapped on 3 streams
    e2e_steps = max(3, min(K, 10))
    bounds = e2e_chunks(M)
    x_h = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).pin_memory()
    outs_h = (torch.empty(q.shape, dtype=q.dtype).pin_memory(),
              torch.empty(s.shape, dtype=s.dtype).pin_memory(),
              torch.empty(swz.shape, dtype=swz.dtype).pin_memory(),
              torch.empty(y.shape, dtype=y.dtype).pin_memory())
    e2e_pipelined.streams = tuple(torch.cuda.Stream(device) for _ in range(3))
    e2e_pipelined.x_d = torch.empty_like(x)
    e2e_pipelined(mxq, x_h, outs_h, bounds, device)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    e2e_ms = [e2e_pipelined(mxq, x_h, outs_h, bounds, device) for _ in range(e2e_steps)]
    e2e_ms = reduce_max(statistics.fmean(e2e_ms), world, device)
    e2e_same = (np.array_equal(outs_h[0].numpy(), q_out) and np.array_equal(outs_h[1].numpy(), s_out)
                and np.array_equal(outs_h[2].numpy(), z_out)
                and np.array_equal(outs_h[3].view(torch.int16).numpy().view(np.uint16), y_out))

    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return

    extra = []
    flush = torch.empty(64 * 2**20, dtype=torch.float32, device=device)  # 256 MB > L2
    if not args.headline_only:
        extra = config_lines(mxq, device, flush)

    qb, db = mxfp8_quant_bytes(M, N), mxfp8_dequant_bytes(M, N)
    step_bytes = qb + db
    value = step_bytes * K * world / (max_ms / 1e3) / 1e9
    peak, peak_kind = hbm_peak()
    kernels = {
        "mx_quant_kernel": {"avg_us": q_ms * 1e3, "bytes": qb, "gbs": qb / (q_ms / 1e3) / 1e9},
        "mx_dequant_kernel": {"avg_us": d_ms * 1e3, "bytes": db, "gbs": db / (d_ms / 1e3) / 1e9},
    }
    for k in kernels.values():
        k["frac_of_" + peak_kind] = k["gbs"] / peak
        k["frac_of_spec_8tbs"] = k["gbs"] / SPEC_HBM_GBS
    # the roofline is the quantize's: the kernel the metric names. The two
    # kernels share the step about evenly; both are in `breakdown`, each with
    # its share of the step's kernel time.
    dom = "mx_quant_kernel"
    for k in kernels.values():
        k["share_of_step"] = k["avg_us"] / sum(v["avg_us"] for v in kernels.values())
    h2d = x.numel() * 2
    d2h = q.numel() + s.numel() + swz.numel() + y.numel() * 2
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": max_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": config_block(world, input_sha),
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": kernels[dom]["gbs"], "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": kernels[dom]["gbs"] / peak,
                     "frac_basis": f"{peak_kind} copy bandwidth ({peak:.1f} GB/s); the statement "
                                   "of the problem's 80 % target is against the 8 TB/s spec: "
                                   "frac_of_spec_8tbs",
                     "frac_of_spec_8tbs": kernels[dom]["gbs"] / SPEC_HBM_GBS,
                     "spec_80pct_target_met": kernels[dom]["gbs"] >= 0.8 * SPEC_HBM_GBS,
                     "algorithmic_bytes_per_launch": kernels[dom]["bytes"],
                     "traffic": recorded_traffic(dom),
                     "timing": f"{R} back-to-back launches of each kernel between two events, "
                               "after 3 untimed ones",
                     "kernel_choice": "the kernel the metric names; it and the dequantize share "
                                      "the step about evenly (breakdown.share_of_step)"},
        "breakdown": kernels,
        "e2e": {"value": step_bytes * world / (e2e_ms / 1e3) / 1e9, "unit": "GB/s",
                "ms_per_step": e2e_ms, "steps": e2e_steps,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "pipeline": f"{len(bounds) - 1} row chunks ({bounds[1]} rows first, doubling to "
                            "2048); upload, kernels and download on three streams", "outputs_equal_device_run": bool(e2e_same)},
        "gpu_launches": 2 * K,
        "clocks": clk.summary(),
        "clocks_kernel_loops": clk_k.summary(),
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"], rows, (qo, so, zo, yo) = cpu_baseline(xb)
        Sp = (S + 3) // 4 * 4
        line["verified_bit_exact_first_rows"] = {
            "rows": rows,
            "equal_to_oracle": bool(np.array_equal(q_out[:rows], qo)
                                    and np.array_equal(s_out[:rows], so)
                                    and np.array_equal(z_out[:rows * Sp], zo)
                                    and np.array_equal(y_out[:rows], yo))}
    if extra:
        line["configs"] = {str(d["config_line"]): {"gbs": round(d["gbs"], 1),
                                                    "median_us": round(d["median_us"], 2),
                                                    "frac_of_" + peak_kind: round(d["frac_of_" + peak_kind], 3),
                                                    "bit_exact": d["bit_exact_vs_oracle"]}
                           for d in extra}
    print(json.dumps(line), flush=True)
    if args.suite:
        run_suite(device)


# ------------------------------------------------------------------ suite

def _flush_l2(buf):
    buf.add_(1)


def time_kernel(fn, iters, flush_buf=None, poll=False):
    """Device time (ms) per call of fn(). Without flush_buf: five loops of
    `iters` back-to-back calls, events only around each loop; returns the
    median, lowest and highest per-call average of the loops. With flush_buf
    (small workloads): L2 flushed before each call by a write larger than L2,
    events around each call alone; returns median, p10 and p90. poll: wait
    for the last event by polling, so that a clock-sampling thread runs while
    the GPU works."""
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    if flush_buf is None:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(5)]
        for a, b in evs:
            a.record()
            for _ in range(iters):
                fn()
            b.record()
    else:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(iters)]
        for a, b in evs:
            _flush_l2(flush_buf)
            a.record()
            fn()
            b.record()
    if poll:
        while not evs[-1][1].query():
            time.sleep(0.0002)
    torch.cuda.synchronize()
    if flush_buf is None:
        t = sorted(a.elapsed_time(b) / iters for a, b in evs)
        return t[2], t[0], t[-1]
    t = sorted(a.elapsed_time(b) for a, b in evs)
    return t[len(t) // 2], t[len(t) // 10], t[(len(t) * 9) // 10]


def run_suite(device, only=None):
    """One JSON line per workload kernel: device time per launch of repeated
    back-to-back launches (L2 flushed before each launch for the 50 MB workload
    and smaller, which are timed one launch at a time; the others
    exceed L2), algorithmic bytes, GB/s and fraction of the HBM peak."""
    import ctypes

    import nvfp4_block_scaled_sm_b200 as mxq
    peak, kind = hbm_peak()
    flush = torch.empty(64 * 2**20, dtype=torch.float32, device=device)  # 256 MB > L2

    def emit(name, nbytes, t):
        med, p10, p90 = t
        print(json.dumps({"suite": name, "median_us": med * 1e3, "p10_us": p10 * 1e3,
                          "p90_us": p90 * 1e3, "bytes": nbytes, "gbs": nbytes / med / 1e6,
                          "frac_of_" + kind: nbytes / med / 1e6 / peak,
                          "frac_of_spec_8tbs": nbytes / med / 1e6 / SPEC_HBM_GBS}), flush=True)

    def bf(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)

    def planted():
        x = bf(W.planted())
        emit("mxfp8_quantize planted 256x1024 (L2-flushed, launch-bound)",
             mxfp8_quant_bytes(256, 1024, swizzled=False),
             time_kernel(lambda: mxq.mxfp8_quantize(x), 50, flush))
        q, s = mxq.mxfp8_quantize(x)
        emit("mxfp8_dequantize->bf16 planted 256x1024 (L2-flushed, launch-bound)",
             mxfp8_dequant_bytes(256, 1024), time_kernel(lambda: mxq.mxfp8_dequantize(q, s), 50, flush))

    def linear_weight():
        x = bf(W.linear_weight())
        emit("mxfp8_quantize linear_weight 4096x4096 (L2 flushed by a 256 MB write)",
             mxfp8_quant_bytes(4096, 4096, swizzled=False),
             time_kernel(lambda: mxq.mxfp8_quantize(x), 50, flush))
        # rotating inputs and outputs: 8 sets of 34 MB in, 17 MB out (> 2x L2),
        # so no launch finds its input in L2 and no flush's dirty lines compete
        xs = [x.clone() for _ in range(8)]
        qs = [torch.empty((4096, 4096), dtype=torch.uint8, device=device) for _ in range(8)]
        ss = [torch.empty((4096, 128), dtype=torch.uint8, device=device) for _ in range(8)]
        L = mxq.lib
        sp = ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
        P = [[ctypes.c_void_p(t.data_ptr()) for t in (xs[i], qs[i], ss[i])] for i in range(8)]
        k = [0]

        def rotating():
            p = P[k[0] % 8]
            k[0] += 1
            L.mxfp8_quantize(p[0], 0, 4096, 4096, 4096, p[1], p[2], None, sp)

        emit("mxfp8_quantize linear_weight 4096x4096 (8 rotating input/output sets)",
             mxfp8_quant_bytes(4096, 4096, swizzled=False), time_kernel(rotating, 48))
        # eight such weights: one C-ABI call each, against one grouped launch
        # over the stacked eight (rotating between two stacks, 2 x 268 MB > L2)
        stacks = [torch.stack(xs), torch.stack(xs).clone()]
        del xs, qs, ss, P
        q8 = torch.empty((8 * 4096, 4096), dtype=torch.uint8, device=device)
        s8 = torch.empty((8 * 4096, 128), dtype=torch.uint8, device=device)
        off8 = (torch.arange(9, dtype=torch.int64) * 4096).to(device)
        V = lambda t: ctypes.c_void_p(t.data_ptr())
        k[0] = 0

        def eight_calls():
            st = stacks[k[0] % 2]
            k[0] += 1
            for i in range(8):
                L.mxfp8_quantize(V(st[i]), 0, 4096, 4096, 4096, V(q8[4096 * i:]), V(s8[4096 * i:]),
                                 None, sp)

        def one_grouped():
            st = stacks[k[0] % 2]
            k[0] += 1
            L.mxfp8_quantize_grouped(V(st), 0, 8, V(off8), 8 * 4096, 4096, V(q8), V(s8), sp)

        eight = 8 * mxfp8_quant_bytes(4096, 4096, swizzled=False)
        emit("8 x mxfp8_quantize linear_weight 4096x4096, one call each", eight,
             time_kernel(eight_calls, 10))
        emit("mxfp8_quantize_grouped of the 8 stacked linear weights 8x4096x4096, one launch",
             eight, time_kernel(one_grouped, 10))

    def activation():
        x = bf(W.activation())
        emit("mxfp8_quantize activation 16384x7168",
             mxfp8_quant_bytes(M_ROWS, N_COLS, swizzled=False),
             time_kernel(lambda: mxq.mxfp8_quantize(x), 30))
        emit("mxfp8_quantize+swizzle activation 16384x7168", mxfp8_quant_bytes(M_ROWS, N_COLS),
             time_kernel(lambda: mxq.mxfp8_quantize(x, swizzled=True), 30))
        q, s = mxq.mxfp8_quantize(x)
        emit("mxfp8_dequantize->bf16 activation 16384x7168", mxfp8_dequant_bytes(M_ROWS, N_COLS),
             time_kernel(lambda: mxq.mxfp8_dequantize(q, s), 30))
        emit("mxfp8_dequantize->fp32 activation 16384x7168",
             mxfp8_dequant_bytes(M_ROWS, N_COLS, 4),
             time_kernel(lambda: mxq.mxfp8_dequantize(q, s, torch.float32), 30))
        emit("mxfp8_quantize_columnwise activation 16384x7168",
             mxfp8_quant_bytes(M_ROWS, N_COLS, swizzled=False),
             time_kernel(lambda: mxq.mxfp8_quantize_columnwise(x), 30))
        emit("mxfp8_quantize rowwise+columnwise (one read) activation 16384x7168",
             2 * mxfp8_quant_bytes(M_ROWS, N_COLS, swizzled=False) - 2 * M_ROWS * N_COLS,
             time_kernel(lambda: mxq.mxfp8_quantize_columnwise(x, rowwise=True), 30))
        xf = x.float()
        emit("mxfp8_quantize fp32-input activation 16384x7168",
             mxfp8_quant_bytes(M_ROWS, N_COLS, in_bytes=4, swizzled=False),
             time_kernel(lambda: mxq.mxfp8_quantize(xf), 30))

    def mxfp4_activation():
        x = bf(W.activation())
        emit("mxfp4_quantize activation 16384x7168", mxfp4_quant_bytes(M_ROWS, N_COLS),
             time_kernel(lambda: mxq.mxfp4_quantize(x), 30))
        p, s = mxq.mxfp4_quantize(x)
        emit("mxfp4_dequantize->bf16 activation 16384x7168", mxfp4_dequant_bytes(M_ROWS, N_COLS),
             time_kernel(lambda: mxq.mxfp4_dequantize(p, s), 30))

    def fake_activation():
        x = bf(W.activation())
        for fmt in ("mxfp8", "mxfp4"):
            emit(f"mx_fake_quantize {fmt} bf16->bf16 activation 16384x7168",
                 fake_quant_bytes(M_ROWS, N_COLS),
                 time_kernel(lambda: mxq.mx_fake_quantize(x, fmt), 30))

    def gemm():
        xa = bf(W.activation())
        xb = bf(W.linear_weight(seed=111, M=7168, N=7168))
        qa, _, za = mxq.mxfp8_quantize(xa, swizzled=True)
        qb, _, zb = mxq.mxfp8_quantize(xb, swizzled=True)
        del xa, xb
        flops = 2 * M_ROWS * 7168 * N_COLS
        with ClockSampler(device) as clk:
            t = time_kernel(lambda: mxq.mxfp8_gemm(qa, za, qb, zb), 20, poll=True)
        med, p10, p90 = t
        bf16_peak = tensor_peak()
        sus_peak = tensor_peak(sustained=True)
        print(json.dumps({"suite": "mxfp8_gemm activation 16384x7168 x weight 7168x7168 -> bf16",
                          "median_us": med * 1e3, "p10_us": p10 * 1e3, "p90_us": p90 * 1e3,
                          "tflops": flops / med / 1e9,
                          "frac_of_fp8_peak": flops / med / 1e9 / bf16_peak[0],
                          "fp8_peak_tflops": bf16_peak[0], "peak_kind": bf16_peak[1],
                          "frac_of_fp8_sustained": flops / med / 1e9 / sus_peak[0],
                          "fp8_sustained_tflops": sus_peak[0], "clocks": clk.summary()}), flush=True)
        # context: NVIDIA's library MX GEMM (through torch) on the same codes and scales
        F = torch.nn.functional
        try:
            lib_mm = lambda: F.scaled_mm(
                qa.view(torch.float8_e4m3fn), qb.view(torch.float8_e4m3fn).t(),
                za.view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                zb.view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                output_dtype=torch.bfloat16)
            with ClockSampler(device) as clk:
                med, p10, p90 = time_kernel(lib_mm, 20, poll=True)
            print(json.dumps({"suite": "library MX GEMM (torch scaled_mm, same operands), for context",
                              "median_us": med * 1e3, "p10_us": p10 * 1e3, "p90_us": p90 * 1e3,
                              "tflops": flops / med / 1e9,
                              "frac_of_fp8_peak": flops / med / 1e9 / bf16_peak[0],
                              "frac_of_fp8_sustained": flops / med / 1e9 / sus_peak[0],
                              "clocks": clk.summary()}), flush=True)
            # the two one after the other, in alternating rounds, so that both
            # see the same power and clock state (a GEMM this size drives the
            # GPU into its power cap within a few launches)
            def loop(fn, n=10):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                for _ in range(n):
                    fn()
                b.record()
                b.synchronize()
                return a.elapsed_time(b) / n
            ours_mm = lambda: mxq.mxfp8_gemm(qa, za, qb, zb)
            rounds = []
            with ClockSampler(device) as clk:
                for _ in range(6):
                    rounds.append((loop(ours_mm), loop(lib_mm)))
            ours_t = sorted(r[0] for r in rounds)
            lib_t = sorted(r[1] for r in rounds)
            ratios = [r[0] / r[1] for r in rounds]
            print(json.dumps({"suite": "mxfp8_gemm against the library MX GEMM, alternating rounds of 10 launches",
                              "median_us": ours_t[3] * 1e3, "library_median_us": lib_t[3] * 1e3,
                              "time_ratio_median": sorted(ratios)[3],
                              "time_ratio_per_round": [round(x, 3) for x in ratios],
                              "clocks": clk.summary()}), flush=True)
        except Exception as e:  # not every torch build exposes the MX recipe
            print(json.dumps({"suite": "library MX GEMM (torch scaled_mm)", "unavailable": str(e)[:200]}),
                  flush=True)

    def experts():
        x = bf(W.experts())
        emit("mxfp8_quantize_grouped experts 64x2048x7168",
             mxfp8_quant_bytes(64 * 2048, 7168, swizzled=False),
             time_kernel(lambda: mxq.mxfp8_quantize_grouped(x), 10))
        emit("mxfp4_quantize_grouped experts 64x2048x7168",
             mxfp4_quant_bytes(64 * 2048, 7168),
             time_kernel(lambda: mxq.mxfp4_quantize_grouped(x), 10))
        ws = torch.empty(int(mxq.lib.mxq_nvfp4_sliced_workspace_bytes(128)), dtype=torch.uint8,
                         device=device)
        for per_half in (False, True):
            rows = [1024] * 128 if per_half else [2048] * 64
            emit(f"nvfp4_quantize_sliced (two passes, {'per gate/up half' if per_half else 'per expert'})"
                 " experts 64x2048x7168", nvfp4_quant_bytes(64 * 2048, 7168),
                 time_kernel(lambda: mxq.nvfp4_quantize_sliced(x, rows, workspace=ws), 10))

    def nvfp4():
        x = bf(W.nvfp4_tensor())
        emit("nvfp4_quantize (two passes) nvfp4_tensor 8192x8192", nvfp4_quant_bytes(8192, 8192),
             time_kernel(lambda: mxq.nvfp4_quantize(x), 30))
        p, b, g = mxq.nvfp4_quantize(x)
        emit("nvfp4_quantize (given scale, one pass) nvfp4_tensor 8192x8192",
             nvfp4_quant_bytes(8192, 8192, two_pass=False),
             time_kernel(lambda: mxq.nvfp4_quantize(x, global_scale=g), 30))
        emit("nvfp4_dequantize->bf16 8192x8192", 8192 * 8192 // 2 + 8192 * 512 + 8192 * 8192 * 2,
             time_kernel(lambda: mxq.nvfp4_dequantize(p, b, g), 30))

    for name, fn in (("planted", planted), ("gemm", gemm), ("linear_weight", linear_weight),
                     ("activation", activation),
                     ("mxfp4 activation", mxfp4_activation), ("fake activation", fake_activation),
                     ("experts", experts), ("nvfp4", nvfp4)):
        if only is None or only in name:
            fn()
            torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["mxq", "reference"], default="mxq")
    ap.add_argument("--suite", action="store_true", help="also time every workload kernel")
    ap.add_argument("--suite-only", default=None,
                    help="time only the workload kernels whose workload name contains this")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the lines of the other workloads")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.suite_only is not None:
        torch.cuda.set_device(0)
        run_suite(torch.device("cuda", 0), args.suite_only)
    else:
        run(args)


if __name__ == "__main__":
    main()
