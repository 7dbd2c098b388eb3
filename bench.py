"""Benchmark of the MXFP8 hot path on B200.

One step = one pass of the MXFP8 path over one batch: rowwise quantize of a
bf16 activation [16384, 7168] (Student-t(3) * 0.5, 1 % zero groups, 0.5 %
groups scaled by 2^-120, seed 2) with compact and 128x4-swizzled scales, then
dequantize back to bf16. The metric is algorithmic HBM bytes (read + written)
per second; the input (235 MB) is larger than the 126 MB L2, so no flush is
needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mxq|reference]
    python -m torch.distributed.run --nproc-per-node N bench.py --gpus N ...

Multi-GPU: every rank quantizes its own batch (rows are independent, so the
path shards with no exchange); value = bytes of all ranks / max over ranks of
the device-timed region ("scaling": "weak").

``--impl reference`` times the CPU oracle (test infrastructure) on host cores
on a bounded sample of the same workload. ``--suite`` prints one extra JSON
line per workload kernel (documentation, not the default line).
"""
from __future__ import annotations

import argparse
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

def time_oracle_round_trip(x: np.ndarray, min_seconds: float):
    """Oracle MXFP8 quantize + swizzle + dequantize of the rows `x`, repeated
    until min_seconds have elapsed; returns (seconds per pass, passes,
    (qweight, scale, dequantized bf16 bits))."""
    import oracle
    oracle.build()
    passes, t0 = 0, time.perf_counter()
    while True:
        q, s = oracle.mxfp8_quantize(x)
        oracle.swizzle_scales(s)
        y = oracle.mxfp8_dequantize(q, s, out="bf16")
        passes += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            return el / passes, passes, (q, s, y)


def cpu_baseline(x_full: np.ndarray, rows: int = 2048, min_seconds: float = 12.0):
    """The oracle timed on the first `rows` rows; also returns its outputs."""
    x = np.ascontiguousarray(x_full[:rows])
    sec, passes, outs = time_oracle_round_trip(x, min_seconds)
    nbytes = mxfp8_quant_bytes(rows, N_COLS) + mxfp8_dequant_bytes(rows, N_COLS)
    return {"value": nbytes / sec / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"first {rows} of {M_ROWS} rows of the activation workload, quantize "
                      f"(+swizzle) + dequantize, {passes} passes, single-threaded scalar C"}, outs


def run_reference(args):
    world, rank, _ = dist_setup(args)
    if rank != 0:
        return
    x_all = W.activation(M=M_ROWS, N=N_COLS)
    input_sha = hashlib.sha256(x_all.tobytes()).hexdigest()[:16]
    t_row, _, _ = time_oracle_round_trip(np.ascontiguousarray(x_all[:64]), 0.5)
    t_row /= 64
    budget = 150.0
    rows = int(max(1, min(M_ROWS, budget / max(1, args.steps + args.warmup) / t_row)))
    x = np.ascontiguousarray(x_all[:rows])
    import oracle
    for _ in range(args.warmup):
        q, s = oracle.mxfp8_quantize(x)
        oracle.swizzle_scales(s)
        oracle.mxfp8_dequantize(q, s, out="bf16")
    t0 = time.perf_counter()
    for _ in range(args.steps):
        q, s = oracle.mxfp8_quantize(x)
        oracle.swizzle_scales(s)
        oracle.mxfp8_dequantize(q, s, out="bf16")
    el = time.perf_counter() - t0
    nbytes = (mxfp8_quant_bytes(rows, N_COLS) + mxfp8_dequant_bytes(rows, N_COLS)) * args.steps
    value = nbytes / el / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": config_block(world, input_sha),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": f"first {rows} rows per step of the {M_ROWS}x{N_COLS} "
                                       "activation workload, single-threaded scalar C"},
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
    import ctypes

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

    def step():
        st = L.mxfp8_quantize(P[0], 0, M, N, N, P[1], P[2], P[3], sp)
        if st:
            raise mxq.MxqError("mxfp8_quantize", st, L.mxq_status_string(st).decode())
        st = L.mxfp8_dequantize(P[1], P[2], M, N, P[4], 0, sp)
        if st:
            raise mxq.MxqError("mxfp8_dequantize", st, L.mxq_status_string(st).decode())

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)

    K = args.steps
    # Per-kernel durations come from events around the two kernels of every
    # SAMPLE_EVERY-th step only: an event recorded between two kernels ends
    # their programmatic overlap, so events on every step would slow the step.
    # A short run samples more often (every step at K < 16) so that the
    # average still rests on about eight launches or more.
    every = min(SAMPLE_EVERY, max(1, K // 8))
    sampled = [k for k in range(K) if k % every == every - 1] or [K - 1]
    ev = {k: [torch.cuda.Event(enable_timing=True) for _ in range(3)] for k in sampled}
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(device) as clk:
        t_start.record(stream)
        for k in range(K):
            e = ev.get(k)
            if e:
                e[0].record(stream)
            L.mxfp8_quantize(P[0], 0, M, N, N, P[1], P[2], P[3], sp)
            if e:
                e[1].record(stream)
            L.mxfp8_dequantize(P[1], P[2], M, N, P[4], 0, sp)
            if e:
                e[2].record(stream)
        t_end.record(stream)
        # wait by polling so that the sampler thread gets the interpreter while
        # the GPU works through the queued steps
        while not t_end.query():
            time.sleep(0.0002)
        torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    q_ms = [ev[k][0].elapsed_time(ev[k][1]) for k in sampled]
    d_ms = [ev[k][1].elapsed_time(ev[k][2]) for k in sampled]
    max_ms = reduce_max(elapsed_ms, world, device)

    # outputs of the timed region's last step, kept for the CPU-baseline leg's check
    n_check = 2048
    q_last = q[:n_check].cpu().numpy()
    s_last = s[:n_check].cpu().numpy()
    y_last = y[:n_check].view(torch.int16).cpu().numpy().view(np.uint16)

    # end-to-end through the public API: pinned host input -> device, quantize,
    # dequantize, all outputs -> pinned host, every step
    e2e_steps = max(1, min(K, 10))
    x_h = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).pin_memory()
    q_h = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    s_h = torch.empty(s.shape, dtype=s.dtype).pin_memory()
    z_h = torch.empty(swz.shape, dtype=swz.dtype).pin_memory()
    y_h = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    x_d = torch.empty_like(x)

    def e2e_step():
        x_d.copy_(x_h, non_blocking=True)
        qq, ss, zz = mxq.mxfp8_quantize(x_d, swizzled=True)
        yy = mxq.mxfp8_dequantize(qq, ss, torch.bfloat16)
        q_h.copy_(qq, non_blocking=True)
        s_h.copy_(ss, non_blocking=True)
        z_h.copy_(zz, non_blocking=True)
        y_h.copy_(yy, non_blocking=True)
        torch.cuda.current_stream(device).synchronize()

    e2e_step()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = reduce_max(e0.elapsed_time(e1) / e2e_steps, world, device)

    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return

    qb, db = mxfp8_quant_bytes(M, N), mxfp8_dequant_bytes(M, N)
    step_bytes = qb + db
    value = step_bytes * K * world / (max_ms / 1e3) / 1e9
    peak, peak_kind = hbm_peak()
    q_avg, d_avg = statistics.fmean(q_ms), statistics.fmean(d_ms)
    kernels = {
        "mx_quant_kernel": {"avg_us": q_avg * 1e3, "bytes": qb, "gbs": qb / (q_avg / 1e3) / 1e9},
        "mx_dequant_kernel": {"avg_us": d_avg * 1e3, "bytes": db, "gbs": db / (d_avg / 1e3) / 1e9},
    }
    for k in kernels.values():
        k["frac_of_measured"] = k["gbs"] / peak
        k["frac_of_spec_8tbs"] = k["gbs"] / SPEC_HBM_GBS
    dom = max(kernels, key=lambda k: kernels[k]["avg_us"])
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
                     "frac_of_spec_8tbs": kernels[dom]["gbs"] / SPEC_HBM_GBS,
                     "algorithmic_bytes_per_launch": kernels[dom]["bytes"],
                     "traffic": recorded_traffic(dom)},
        "breakdown": kernels,
        "e2e": {"value": step_bytes * world / (e2e_ms / 1e3) / 1e9, "unit": "GB/s",
                "ms_per_step": e2e_ms, "steps": e2e_steps,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": 2 * K,
        "kernel_time_sampling": f"events around both kernels on every {every}th step "
                                f"({len(sampled)} of {K} steps)",
        "clocks": clk.summary(),
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"], (qo, so, yo) = cpu_baseline(xb, n_check)
        line["verified_bit_exact_first_rows"] = {
            "rows": n_check,
            "equal_to_oracle": bool(np.array_equal(q_last, qo) and np.array_equal(s_last, so)
                                    and np.array_equal(y_last, yo))}
    print(json.dumps(line), flush=True)
    if args.suite:
        run_suite(device)


# ------------------------------------------------------------------ suite

def _flush_l2(buf):
    buf.add_(1)


def time_kernel(fn, iters, flush_buf=None, poll=False):
    """Median device time (ms) of fn() over iters launches, L2 flushed between
    launches when flush_buf is given (the flush is outside the timed span).
    poll: wait for the last event by polling, so that a clock-sampling thread
    runs while the GPU works."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(iters)]
    for _ in range(3):
        fn()
    for a, b in evs:
        if flush_buf is not None:
            _flush_l2(flush_buf)
        a.record()
        fn()
        b.record()
    if poll:
        while not evs[-1][1].query():
            time.sleep(0.0002)
    torch.cuda.synchronize()
    t = sorted(a.elapsed_time(b) for a, b in evs)
    return t[len(t) // 2], t[len(t) // 10], t[(len(t) * 9) // 10]


def run_suite(device, only=None):
    """One JSON line per workload kernel: median device time over repeated
    launches (L2 flushed between launches for the 50 MB workload, the others
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
