"""Benchmark of the INT4 weight-only path on B200.

One step is one pass of the whole path over one weight matrix
W [28672, 8192] (bf16, heavy-tailed Student-t(3) * 0.02 with 1% all-zero
groups, group 128):

  quantize  W -> packed [28672, 4096] uint8 + scales [28672, 64] fp16
  unpack    packed -> int8 [28672, 8192]
  decode    y = x @ dequant(W)^T with x [1, 8192] bf16         (M = 1)
  prefill   y = x @ dequant(W)^T with x [8192, 8192] bf16      (M = 8192)

Every kernel is timed with CUDA events on the stream it runs on, and L2 is
flushed before each kernel, outside its events (a 256 MiB write, then a
256 MiB read of another buffer, so no dirty lines are written back during the
timed kernel).  The
headline ``value`` is the decode throughput on packed-weight bytes
(N * ceil(K/2) / time); the other rows are reported under ``rows``.

Launch: ``python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]``
(under torchrun for N > 1: every rank runs the same step on its own GPU,
"replicas only"; value is the sum over ranks with the max time over ranks).
``--impl reference`` times the CPU oracle on a bounded sample on this host.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

N_W, K_W, GROUP = 28672, 8192, 128
M_DECODE, M_PREFILL = 1, 8192
METRIC = "int4_matmul decode GB/s & prefill TFLOP/s vs B200 roofline; quantize GB/s"
WORKLOAD = ("W[28672,8192] bf16 g128: quantize+unpack, decode M=1 (32 calls back to back over "
            "32 copies of the packed weights, as consecutive layers), prefill M=8192")
# Weight copies the decode row streams back to back (32 x 117 MB, far more
# than L2), as consecutive layers of a decode step: the row's per-call time is
# then close to the steady state of a decode loop, with the start of the
# first call and the end of the last spread over 32 calls.
DECODE_COPIES = 32
# Layers per read-back of y in the end-to-end step.
E2E_READBACK = 8


# DRAM traffic per launch of each kernel (dram__bytes_read.sum +
# dram__bytes_write.sum) from the ncu captures summarized under profiles/.  A
# figure holds only for the kernel source it was taken on, so each carries the
# sha256 of that source file and is reported as null once the file changes.
KERNEL_TRAFFIC = {
    # kernel: (bytes per launch, source file, sha256 of the source at capture)
    "prefill": (812_040_000 + 919_400_000, "dequant_gemm_int4_b200/csrc/matmul_prefill.cu",
                "fb5b9e91a3e50e847a3e16ee33705d4b1cf935874397d6e856b9fded9b268250"),
    "decode": (125_570_000 + 3_240_000, "dequant_gemm_int4_b200/csrc/matmul_decode.cu",
               "7a09f42f7ba224b046786c6639e561bd7ffffb659138712f3b01fa51b6273e55"),
    "quantize": (469_856_256 + 104_254_208, "dequant_gemm_int4_b200/csrc/quantize.cu",
                 "24a51fde9c6ea1afd8a159345f565f16441d8a085e241e8e6d8d123c71573f57"),
    "unpack": (117_450_000 + 180_200_000, "dequant_gemm_int4_b200/csrc/unpack.cu",
               "51f56d9ff427ee0f35313e26571656e7ae1fe4ff8b53aaacec1ce407868e3cd8"),
}


def _traffic(kernel: str):
    import hashlib
    entry = KERNEL_TRAFFIC.get(kernel)
    if entry is None:
        return None
    nbytes, src, digest = entry
    try:
        with open(os.path.join(ROOT, src), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != digest:
                return None
    except OSError:
        return None
    return nbytes


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


def _row_units():
    Kp = (K_W + 1) // 2
    G = -(-K_W // GROUP)
    packed = N_W * Kp
    scales = 2 * N_W * G
    return {
        "quantize": {"bytes": N_W * K_W * 2 + packed + scales, "bound": "hbm"},
        "quantize_affine": {"bytes": N_W * K_W * 2 + packed + scales + N_W * G, "bound": "hbm"},
        "unpack": {"bytes": packed + N_W * K_W, "bound": "hbm"},
        "decode": {"bytes": packed, "bytes_total": packed + scales + M_DECODE * K_W * 2 + 4 * M_DECODE * N_W,
                   "bound": "hbm"},
        "prefill": {"flops": 2 * M_PREFILL * N_W * K_W, "bound": "tensor"},
    }


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
            return self
        # nvidia-smi can take a second to start on a fresh box: wait for its
        # first sample (or at most 3 s, in case it buffers its output), so
        # that a short timed region is still sampled.
        deadline = time.time() + 3.0
        while self.proc.poll() is None and time.time() < deadline and os.path.getsize(self.path) == 0:
            time.sleep(0.02)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


def _dist_setup(args):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "ours":
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device(f"cuda:{local}"))
    return world, rank, local


def _max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    # NCCL reduces device tensors; the gloo backend (CPU tests) host tensors.
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def cpu_baseline(rows: int = 8192):
    """Time the CPU oracle on bounded row samples of the same workload."""
    import numpy as np
    import torch

    import oracle
    from workloads import make_activations, make_weights

    threads = torch.get_num_threads()
    w = make_weights(rows, K_W, seed=5, device="cpu", dtype=torch.bfloat16, dist="student_t3",
                     zero_group_frac=0.01, group=GROUP).float().numpy()
    out = {}
    t0 = time.perf_counter()
    packed, scales, K = oracle.quantize_int4(w, GROUP)
    tq = time.perf_counter() - t0
    out["quantize_gbs"] = (rows * K_W * 2 + packed.nbytes + scales.nbytes) / tq / 1e9
    t0 = time.perf_counter()
    oracle.unpack_int4(packed, K)
    tu = time.perf_counter() - t0
    out["unpack_gbs"] = (packed.nbytes + rows * K_W) / tu / 1e9
    x1 = make_activations(1, K_W, seed=11, device="cpu").float().numpy()
    t0 = time.perf_counter()
    oracle.int4_matmul_ref(x1, packed, scales, K, GROUP)
    td = time.perf_counter() - t0
    out["decode_gbs"] = packed.nbytes / td / 1e9
    xm = make_activations(64, K_W, seed=12, device="cpu").float().numpy()
    t0 = time.perf_counter()
    oracle.int4_matmul_ref(xm, packed, scales, K, GROUP)
    tp = time.perf_counter() - t0
    out["prefill_tflops"] = 2 * 64 * rows * K_W / tp / 1e12
    out["seconds"] = tq + tu + td + tp
    out["threads"] = threads
    out["sample"] = (f"{rows} rows of W [{N_W},{K_W}] bf16 g{GROUP}: quantize, unpack, decode M=1, "
                     f"prefill M=64 slice (fp64 BLAS); throughput per the full-size byte/flop counts")
    return out


def run_reference(args):
    """The reference arm: the CPU oracle, timed on this host's cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import numpy as np  # noqa: F401
    times = []
    res = None
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        res = cpu_baseline(rows=2048)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    line = {
        "impl": "reference", "metric": METRIC, "value": res["decode_gbs"], "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.mean(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD + " (row sample)"},
        "rows": {k: res[k] for k in ("quantize_gbs", "unpack_gbs", "decode_gbs", "prefill_tflops")},
        "cpu_baseline": {"value": res["decode_gbs"], "unit": "GB/s", "cores": res["threads"],
                         "kind": "oracle", "sample": res["sample"]},
        "e2e": {"value": res["decode_gbs"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# Decode at the Llama-7B-shaped linears (group 128, bf16 x, M = 1, 4, 16): per
# shape and batch, calls back to back over rotating copies of the packed
# weights whose total exceeds 3x L2, so every call streams its weights from
# HBM.  The loop is timed twice: replayed from a CUDA graph (the kernels' own
# rate; launch gaps only) and launched call by call from the host.
DECODE_SHAPES = [(4096, 4096), (11008, 4096), (4096, 11008)]
DECODE_MS = (1, 4, 16)
PREFILL_SHAPES = [(8192, 8192), (28672, 8192)]
PREFILL_MS = (2048, 8192)


def decode_shape_rows(dev, peaks, reps: int = 10):
    import torch

    import dequant_gemm_int4_b200 as q4
    from workloads import make_activations, make_weights

    L = q4.lib()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    rows = {}
    for N, K in DECODE_SHAPES:
        w = make_weights(N, K, seed=3, device=dev, dtype=torch.float32)
        packed, scales, _ = q4.quantize_int4(w, GROUP)
        del w
        per_copy = packed.numel() + 2 * scales.numel()
        ncopy = max(2, -(-3 * l2 // per_copy))
        copies = [(packed.clone(), scales.clone()) for _ in range(ncopy)]
        for M in DECODE_MS:
            x = make_activations(M, K, seed=M, device=dev, dtype=torch.bfloat16)
            y = torch.empty((M, N), dtype=torch.float32, device=dev)
            nb = q4.matmul_workspace_size(torch.bfloat16, K, GROUP, M, N, dev)
            ws = torch.zeros(max(nb, 256), dtype=torch.uint8, device=dev)

            def run():
                sp = torch.cuda.current_stream(dev).cuda_stream
                for pk, sc in copies:
                    rc = L.int4_matmul_ws(x.data_ptr(), 1, pk.data_ptr(), sc.data_ptr(), K, GROUP,
                                          M, N, y.data_ptr(), ws.data_ptr(), ws.numel(), sp)
                    if rc != 0:
                        raise RuntimeError(f"INT4 library error {rc}: {L.int4_last_error()}")

            def timed(fn):
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                fn()
                torch.cuda.synchronize()
                e0.record()
                for _ in range(reps):
                    fn()
                e1.record()
                torch.cuda.synchronize()
                return e0.elapsed_time(e1) * 1e3 / (reps * ncopy)

            for _ in range(3):
                run()
            torch.cuda.synchronize()
            host_us = timed(run)
            graph_us = None
            try:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    run()
                graph_us = timed(g.replay)
                del g
            except RuntimeError:
                graph_us = None
            us = graph_us if graph_us is not None else host_us
            gbs = N * (K // 2) / (us * 1e-6) / 1e9
            rows[f"{N}x{K}_m{M}"] = {
                "us_per_call": us, "GB/s": gbs, "frac": gbs / peaks["hbm_gbs"],
                "timing": "cuda graph replay" if graph_us is not None else "host launched",
                "us_per_call_host_launched": host_us,
                "path": q4.matmul_select(torch.bfloat16, K, GROUP, M, N), "copies": ncopy}
        del copies
    return rows


def prefill_shape_rows(dev, peaks, reps: int = 3, windows: int = 5):
    """The configured prefill workloads W [8192, 8192] and [28672, 8192], group
    128, bf16 x at M = 2048 and 8192: per call, the median of `windows` event
    windows of `reps` back-to-back calls."""
    import statistics

    import torch

    import dequant_gemm_int4_b200 as q4
    from workloads import make_activations, make_weights

    L = q4.lib()
    rows = {}
    for N, K in PREFILL_SHAPES:
        w = make_weights(N, K, seed=4, device=dev, dtype=torch.float32)
        packed, scales, _ = q4.quantize_int4(w, GROUP)
        del w
        for M in PREFILL_MS:
            x = make_activations(M, K, seed=M, device=dev, dtype=torch.bfloat16)
            y = torch.empty((M, N), dtype=torch.float32, device=dev)
            nb = q4.matmul_workspace_size(torch.bfloat16, K, GROUP, M, N, dev)
            ws = torch.zeros(max(nb, 256), dtype=torch.uint8, device=dev)

            def run():
                sp = torch.cuda.current_stream(dev).cuda_stream
                rc = L.int4_matmul_ws(x.data_ptr(), 1, packed.data_ptr(), scales.data_ptr(), K, GROUP,
                                      M, N, y.data_ptr(), ws.data_ptr(), ws.numel(), sp)
                if rc != 0:
                    raise RuntimeError(f"INT4 library error {rc}: {L.int4_last_error()}")

            for _ in range(2):
                run()
            torch.cuda.synchronize()
            times = []
            for _ in range(windows):
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(reps):
                    run()
                e1.record()
                torch.cuda.synchronize()
                times.append(e0.elapsed_time(e1) / reps)
            ms = statistics.median(times)
            tf = 2.0 * M * N * K / (ms * 1e-3) / 1e12
            rows[f"{N}x{K}_m{M}"] = {"ms": ms, "TFLOP/s": tf, "frac": tf / peaks["bf16_tflops"],
                                     "path": q4.matmul_select(torch.bfloat16, K, GROUP, M, N)}
            del x, y
        del packed, scales
    return rows


DISTILGPT2_SHAPES = [(2304, 768), (3072, 768), (768, 3072)]
DISTILGPT2_GROUPS = (32, 64)
DISTILGPT2_M_PREFILL = 1024
BULK_QUANT = [((28672, 8192), (32, 64)), ((8192, 28673), (32, 64, 128))]
DECODE_GROUPS = (32, 64)


def _graph_us(fn, reps: int, calls: int) -> float:
    """Per-call device time of `fn` (calls launches) replayed from a CUDA graph."""
    import torch

    for _ in range(2):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    g.replay()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) * 1e3 / (reps * calls)


def config_rows(dev, peaks, flush_l2, reps: int = 5):
    """The other configured workloads, each timed on its own after the step:
    the distilgpt2-shaped linears (groups 32 and 64, fp16 x; M = 1 decode back
    to back over weight copies that exceed L2, from a CUDA graph, and M = 1024
    prefill back to back, its operands L2-resident), the bulk quantize and
    unpack at groups 32 and 64 and odd K (each call after an L2 flush, median
    of `reps`), and the group-32/64 decode kernel on W [28672, 8192] at M = 1."""
    import statistics

    import torch

    import dequant_gemm_int4_b200 as q4
    from workloads import make_activations, make_weights

    L = q4.lib()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    sp = lambda: torch.cuda.current_stream(dev).cuda_stream  # noqa: E731

    def call(rc):
        if rc != 0:
            raise RuntimeError(f"INT4 library error {rc}: {L.int4_last_error()}")

    def decode_us(x, copies, K, g, M, N, xcode):
        nb = q4.matmul_workspace_size(x.dtype, K, g, M, N, dev)
        ws = torch.zeros(max(nb, 256), dtype=torch.uint8, device=dev)
        y = torch.empty((M, N), dtype=torch.float32, device=dev)

        def run():
            for pk, sc in copies:
                call(L.int4_matmul_ws(x.data_ptr(), xcode, pk.data_ptr(), sc.data_ptr(), K, g, M, N,
                                      y.data_ptr(), ws.data_ptr(), ws.numel(), sp()))
        return _graph_us(run, 10, len(copies))

    def flushed_ms(fn):
        times = []
        for _ in range(reps):
            flush_l2()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        return statistics.median(times)

    out = {"distilgpt2": {}, "bulk_quantize": {}, "decode_groups": {}}
    f16 = q4.DTYPE_F16
    for N, K in DISTILGPT2_SHAPES:
        w = make_weights(N, K, seed=N + K, device=dev, dtype=torch.float32)
        for g in DISTILGPT2_GROUPS:
            packed, scales, _ = q4.quantize_int4(w, g)
            per_copy = packed.numel() + 2 * scales.numel()
            ncopy = max(2, -(-3 * l2 // per_copy))
            copies = [(packed, scales)] + [(packed.clone(), scales.clone()) for _ in range(ncopy - 1)]
            x1 = make_activations(1, K, seed=1, device=dev, dtype=torch.float16)
            us = decode_us(x1, copies, K, g, 1, N, f16)
            gbs = N * (K // 2) / (us * 1e-6) / 1e9
            del copies
            M = DISTILGPT2_M_PREFILL
            xp = make_activations(M, K, seed=2, device=dev, dtype=torch.float16)
            yp = torch.empty((M, N), dtype=torch.float32, device=dev)
            nb = q4.matmul_workspace_size(torch.float16, K, g, M, N, dev)
            wsp = torch.zeros(max(nb, 256), dtype=torch.uint8, device=dev)
            pus = _graph_us(lambda: call(L.int4_matmul_ws(xp.data_ptr(), f16, packed.data_ptr(),
                                                          scales.data_ptr(), K, g, M, N, yp.data_ptr(),
                                                          wsp.data_ptr(), wsp.numel(), sp())), 20, 1)
            tf = 2.0 * M * N * K / (pus * 1e-6) / 1e12
            out["distilgpt2"][f"{N}x{K}_g{g}"] = {
                "decode_m1_us": us, "decode_m1_GB/s": gbs, "decode_m1_frac": gbs / peaks["hbm_gbs"],
                "decode_copies": ncopy, "decode_path": q4.matmul_select(torch.float16, K, g, 1, N),
                f"prefill_m{M}_us": pus, f"prefill_m{M}_TFLOP/s": tf,
                f"prefill_m{M}_frac": tf / peaks["bf16_tflops"],
                "prefill_path": q4.matmul_select(torch.float16, K, g, M, N),
                "timing": "graph replay; decode over weight copies beyond L2, prefill operands L2-resident"}
            del packed, scales, xp, yp, wsp
        del w
    for (N, K), groups in BULK_QUANT:
        w = make_weights(N, K, seed=17, device=dev, dtype=torch.bfloat16, dist="student_t3",
                         zero_group_frac=0.01, group=32)
        Kp = (K + 1) // 2
        packed = torch.empty((N, Kp), dtype=torch.uint8, device=dev)
        unpacked = torch.empty((N, K), dtype=torch.int8, device=dev)
        for g in groups:
            G = -(-K // g)
            scales = torch.empty((N, G), dtype=torch.float16, device=dev)
            qms = flushed_ms(lambda: call(L.int4_quantize(w.data_ptr(), q4.DTYPE_BF16, N, K, g,
                                                          packed.data_ptr(), scales.data_ptr(), sp())))
            ums = flushed_ms(lambda: call(L.int4_unpack(packed.data_ptr(), K, N, unpacked.data_ptr(), sp())))
            qb = N * K * 2 + N * Kp + 2 * N * G
            ub = N * Kp + N * K
            out["bulk_quantize"][f"{N}x{K}_g{g}"] = {
                "quantize_ms": qms, "quantize_GB/s": qb / (qms * 1e-3) / 1e9,
                "quantize_frac": qb / (qms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                "unpack_ms": ums, "unpack_GB/s": ub / (ums * 1e-3) / 1e9,
                "unpack_frac": ub / (ums * 1e-3) / 1e9 / peaks["hbm_gbs"],
                "timing": "single call after an L2 flush, median"}
            del scales
        del w, packed, unpacked
    N, K = N_W, K_W
    w = make_weights(N, K, seed=5, device=dev, dtype=torch.bfloat16, dist="student_t3",
                     zero_group_frac=0.01, group=32)
    x = make_activations(1, K, seed=7, device=dev, dtype=torch.bfloat16)
    for g in DECODE_GROUPS:
        packed, scales, _ = q4.quantize_int4(w, g)
        per_copy = packed.numel() + 2 * scales.numel()
        ncopy = max(2, -(-3 * l2 // per_copy))
        copies = [(packed, scales)] + [(packed.clone(), scales.clone()) for _ in range(ncopy - 1)]
        us = decode_us(x, copies, K, g, 1, N, q4.DTYPE_BF16)
        gbs = N * (K // 2) / (us * 1e-6) / 1e9
        out["decode_groups"][f"{N}x{K}_g{g}_m1"] = {
            "us_per_call": us, "GB/s": gbs, "frac": gbs / peaks["hbm_gbs"], "copies": ncopy,
            "timing": "cuda graph replay over weight copies beyond L2"}
        del copies, packed, scales
    del w
    return out


def unfused_rows(dev, packed, scales, xd, xp, flush_l2, peaks, reps: int = 5):
    """The unfused design the fused matmul replaces, as context: the library's
    int4_dequantize to a bf16 w_hat [N, K], then a cuBLAS bf16 GEMM (torch)
    x @ w_hat^T with fp32 accumulation and bf16 output.  Timed per call with
    CUDA events after an L2 flush, the dequantization included."""
    import torch

    import dequant_gemm_int4_b200 as q4

    rows = {}
    for name, x in (("decode", xd), ("prefill", xp)):
        if x is None:
            continue
        M = x.shape[0]

        def once():
            w_hat = q4.dequantize_int4(packed, scales, K_W, GROUP, dtype=torch.bfloat16)
            return torch.matmul(x, w_hat.t())

        for _ in range(2):
            once()
        tot_ms, deq_ms = 0.0, 0.0
        for _ in range(reps):
            flush_l2()
            e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            e0.record()
            w_hat = q4.dequantize_int4(packed, scales, K_W, GROUP, dtype=torch.bfloat16)
            e1.record()
            torch.matmul(x, w_hat.t())
            e2.record()
            torch.cuda.synchronize()
            tot_ms += e0.elapsed_time(e2)
            deq_ms += e0.elapsed_time(e1)
            del w_hat
        tot_ms /= reps
        deq_ms /= reps
        row = {"ms": tot_ms, "dequantize_ms": deq_ms, "gemm_ms": tot_ms - deq_ms,
               "what": "int4_dequantize to bf16, then torch.matmul (cuBLAS) bf16 out"}
        if name == "decode":
            row["GB/s_on_packed_bytes"] = N_W * (K_W // 2) / (tot_ms * 1e-3) / 1e9
        else:
            row["TFLOP/s"] = 2 * M * N_W * K_W / (tot_ms * 1e-3) / 1e12
        deq_bytes = N_W * (K_W // 2) + 2 * N_W * (K_W // GROUP) + 2 * N_W * K_W
        row["dequantize_GB/s"] = deq_bytes / (deq_ms * 1e-3) / 1e9
        rows[name] = row
    return rows


def variant_rows(dev, w, xd, xp, flush_l2, peaks, reps: int = 5):
    """The asymmetric (zero-point) variant and the fused bias + ReLU epilogue
    on the bench's matrix, each timed per call with CUDA events after an L2
    flush: affine quantize (GB/s on its bytes: bf16 w in, packed codes, fp16
    scales and uint8 zero points out), affine decode M = 1 and prefill
    M = 8192, and the symmetric decode and prefill with bias + ReLU."""
    import torch

    import dequant_gemm_int4_b200 as q4

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        tot = 0.0
        for _ in range(reps):
            flush_l2()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            tot += e0.elapsed_time(e1)
        return tot / reps

    Kp, G = K_W // 2, K_W // GROUP
    packed_a, scales_a, zeros_a, _ = q4.quantize_int4_affine(w, GROUP)
    ms = timed(lambda: q4.quantize_int4_affine(w, GROUP))
    qbytes = N_W * K_W * 2 + N_W * Kp + 3 * N_W * G
    rows = {"affine_quantize": {"ms": ms, "GB/s": qbytes / (ms * 1e-3) / 1e9,
                                "frac": qbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}}
    packed, scales, _ = q4.quantize_int4(w, GROUP)
    bias = torch.randn(N_W, generator=torch.Generator().manual_seed(0)).to(dev)
    yd = torch.empty((xd.shape[0], N_W), dtype=torch.float32, device=dev)
    for name, kw, pk, sc in (("affine_decode", {"zeros": zeros_a}, packed_a, scales_a),
                             ("bias_relu_decode", {"bias": bias, "relu": True}, packed, scales)):
        ms = timed(lambda: q4.int4_matmul(xd, pk, sc, K_W, GROUP, out=yd, **kw))
        gbs = N_W * Kp / (ms * 1e-3) / 1e9
        rows[name] = {"ms": ms, "GB/s": gbs, "frac": gbs / peaks["hbm_gbs"],
                      "timing": "single call after an L2 flush (the launch inside the events)"}
    if xp is not None:
        yp = torch.empty((xp.shape[0], N_W), dtype=torch.float32, device=dev)
        for name, kw, pk, sc in (("affine_prefill", {"zeros": zeros_a}, packed_a, scales_a),
                                 ("bias_relu_prefill", {"bias": bias, "relu": True}, packed, scales)):
            ms = timed(lambda: q4.int4_matmul(xp, pk, sc, K_W, GROUP, out=yp, **kw))
            tf = 2 * xp.shape[0] * N_W * K_W / (ms * 1e-3) / 1e12
            rows[name] = {"ms": ms, "TFLOP/s": tf, "frac": tf / peaks["bf16_tflops"]}
    return rows


def run_ours(args):
    import torch

    import dequant_gemm_int4_b200 as q4
    from workloads import make_activations, make_weights

    world, rank, local = _dist_setup(args)
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    q4.lib()
    stream = torch.cuda.current_stream(dev)

    order = [args.only] if args.only else ["quantize", "unpack", "decode", "prefill"]
    # Buffers of the kernels that run (all of them for a full step).
    w = make_weights(N_W, K_W, seed=5, device=dev, dtype=torch.bfloat16, dist="student_t3",
                     zero_group_frac=0.01, group=GROUP)
    packed = torch.empty((N_W, K_W // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((N_W, K_W // GROUP), dtype=torch.float16, device=dev)
    xd = yd = xp = yp = unpacked = None
    dcopies = []
    if "decode" in order:
        xd = make_activations(M_DECODE, K_W, seed=7, device=dev, dtype=torch.bfloat16)
        yd = torch.empty((M_DECODE, N_W), dtype=torch.float32, device=dev)
        # Further copies of the packed weights (quantized from the same w, so
        # the same bytes at other addresses): the decode row's back-to-back
        # calls never find their weights in L2.
        for _ in range(DECODE_COPIES - 1):
            pc = torch.empty((N_W, K_W // 2), dtype=torch.uint8, device=dev)
            sc = torch.empty((N_W, K_W // GROUP), dtype=torch.float16, device=dev)
            dcopies.append((pc, sc))
    if "prefill" in order:
        xp = make_activations(M_PREFILL, K_W, seed=8, device=dev, dtype=torch.bfloat16)
        yp = torch.empty((M_PREFILL, N_W), dtype=torch.float32, device=dev)
    if "unpack" in order:
        unpacked = torch.empty((N_W, K_W), dtype=torch.int8, device=dev)
    zeros_q = (torch.empty((N_W, K_W // GROUP), dtype=torch.uint8, device=dev)
               if "quantize_affine" in order else None)
    # The decode matmul's workspace (zero-filled once; every call leaves it so).
    ws_bytes = q4.matmul_workspace_size(torch.bfloat16, K_W, GROUP, M_DECODE, N_W, dev)
    ws = torch.zeros(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    # The prefill's workspace (the K pieces of a last partial wave of tiles).
    wsp_bytes = q4.matmul_workspace_size(torch.bfloat16, K_W, GROUP, M_PREFILL, N_W, dev)
    wsp = torch.zeros(max(wsp_bytes, 256), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    def flush_l2():
        # Write 256 MiB, then read another 256 MiB: L2 ends up holding clean
        # lines of an unrelated buffer, so no write-back of dirty lines
        # overlaps the next timed kernel.
        flush.fill_(1)
        flush_rd.sum()
    L = q4.lib()
    # The stream of each launch: torch's current one, which is `stream`
    # except while a CUDA graph is being captured.
    sp = lambda: torch.cuda.current_stream(dev).cuda_stream  # noqa: E731

    def call(rc):
        if rc != 0:
            raise RuntimeError(f"INT4 library error {rc}: {L.int4_last_error()}")

    kernels = {
        "quantize": lambda: call(L.int4_quantize(w.data_ptr(), 1, N_W, K_W, GROUP, packed.data_ptr(),
                                                 scales.data_ptr(), sp())),
        "unpack": lambda: call(L.int4_unpack(packed.data_ptr(), K_W, N_W, unpacked.data_ptr(), sp())),
        "quantize_affine": lambda: call(L.int4_quantize_affine(w.data_ptr(), 1, N_W, K_W, GROUP, packed.data_ptr(),
                                                               scales.data_ptr(), zeros_q.data_ptr(), sp())),
        "decode": lambda: [call(L.int4_matmul_ws(xd.data_ptr(), 1, pk.data_ptr(), sc.data_ptr(), K_W,
                                                  GROUP, M_DECODE, N_W, yd.data_ptr(), ws.data_ptr(),
                                                  ws.numel(), sp()))
                           for pk, sc in [(packed, scales)] + dcopies],
        "decode_single": lambda: call(L.int4_matmul_ws(xd.data_ptr(), 1, packed.data_ptr(),
                                                       scales.data_ptr(), K_W, GROUP, M_DECODE, N_W,
                                                       yd.data_ptr(), ws.data_ptr(), ws.numel(), sp())),
        "prefill": lambda: call(L.int4_matmul_ws(xp.data_ptr(), 1, packed.data_ptr(), scales.data_ptr(),
                                                 K_W, GROUP, M_PREFILL, N_W, yp.data_ptr(), wsp.data_ptr(),
                                                 wsp.numel(), sp())),
    }
    for pc, sc in dcopies:
        call(L.int4_quantize(w.data_ptr(), 1, N_W, K_W, GROUP, pc.data_ptr(), sc.data_ptr(), sp()))
    if args.only and args.only not in ("quantize", "quantize_affine"):
        # The kernel reads packed weights: quantize them once, outside timing.
        kernels["quantize"]()
        torch.cuda.synchronize()
        w = None
    # Kernels of this library per row: one per call.  At M <= 2 the decode
    # matmul converts x inside its own launch and reduces the tiles it splits
    # across CTAs there too; the decode row makes DECODE_COPIES calls, and a
    # single call after it is timed on its own (decode_single).
    launches_per_step = {
        "quantize": 1, "quantize_affine": 1, "unpack": 1, "decode": DECODE_COPIES + 1,
        # the tensor-core kernel, plus the adding kernel when it splits K
        "prefill": 2 if wsp_bytes > 0 else 1,
    }

    # The decode row's back-to-back calls run as a CUDA graph, as a decode
    # loop would launch them: the kernels' own rate, not the Python binding's
    # launch cost.  (Their host-launched time is reported beside it.)
    decode_graph = None
    if "decode" in order:
        for _ in range(2):
            kernels["decode"]()
        torch.cuda.synchronize()
        decode_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(decode_graph):
            kernels["decode"]()
        torch.cuda.synchronize()
        host_decode = kernels["decode"]
        kernels["decode"] = decode_graph.replay

    timed = [n for n in order] + (["decode_single"] if "decode" in order else [])

    def step(events=None):
        for name in timed:
            flush_l2()
            if events is not None:
                events[name][0].record(stream)
            kernels[name]()
            if events is not None:
                events[name][1].record(stream)

    ev = [{n: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for n in timed} for _ in range(args.steps)]
    # The clock sampler runs from the first warm-up step to the end of the timed
    # steps (the GPU is busy throughout), so short timed regions still get samples.
    with ClockSampler(local) as clk:
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        _barrier(world)
        torch.cuda.synchronize()
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for i in range(args.steps):
            step(ev[i])
        t_end.record(stream)
        torch.cuda.synchronize()
    _barrier(world)
    clocks = clk.summary()
    per = {n: statistics.mean(e[n][0].elapsed_time(e[n][1]) for e in ev) for n in timed}
    per = {n: _max_over_ranks(v, world) for n, v in per.items()}
    step_ms = sum(per.values())  # every timed launch of a step
    single_ms = per.pop("decode_single", None)
    # The same back-to-back calls launched one by one from Python (after an
    # L2 flush, per call), for reference beside the graph replay.
    host_ms = None
    if "decode" in order:
        hts = []
        for _ in range(5):
            flush_l2()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            host_decode()
            e1.record(stream)
            torch.cuda.synchronize()
            hts.append(e0.elapsed_time(e1) / DECODE_COPIES)
        host_ms = _max_over_ranks(statistics.median(hts), world)
    if "decode" in per:
        per["decode"] /= DECODE_COPIES  # per call
    wall_ms = _max_over_ranks(t_start.elapsed_time(t_end), world)
    units = _row_units()
    peaks = _peaks()
    rows = {}
    for n in order:
        t = per[n] * 1e-3
        u = units[n]
        if u["bound"] == "hbm":
            ach = u["bytes"] / t / 1e9
            rows[n] = {"ms": per[n], "GB/s": ach * world, "frac": ach / peaks["hbm_gbs"]}
            if "bytes_total" in u:
                rows[n]["GB/s_total_bytes"] = u["bytes_total"] / t / 1e9 * world
        else:
            ach = u["flops"] / t / 1e12
            rows[n] = {"ms": per[n], "TFLOP/s": ach * world, "frac": ach / peaks["bf16_tflops"]}
        rows[n]["traffic"] = _traffic(n)
        rows[n]["path"] = (q4.matmul_select(torch.bfloat16, K_W, GROUP, M_DECODE if n == "decode" else M_PREFILL, N_W)
                           if n in ("decode", "prefill") else None)
        if n == "decode":
            rows[n]["calls_back_to_back"] = DECODE_COPIES
            rows[n]["launch"] = "CUDA graph of the back-to-back calls"
            rows[n]["host_launched_ms"] = host_ms
            rows[n]["single_call_ms"] = single_ms
            rows[n]["single_call_GB/s"] = u["bytes"] / (single_ms * 1e-3) / 1e9 * world
    dom = max(order, key=lambda n: per[n])
    du = units[dom]
    if du["bound"] == "hbm":
        roof = {"kernel": dom, "bound": "hbm", "achieved": du["bytes"] / (per[dom] * 1e-3) / 1e9,
                "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        roof = {"kernel": dom, "bound": "tensor", "achieved": du["flops"] / (per[dom] * 1e-3) / 1e12,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["peak_source"] = peaks["source"] + (" bf16 burst" if roof["bound"] == "tensor" else " copy")
    roof["traffic"] = _traffic(dom)

    shape_rows = None
    prefill_rows = None
    cfg_rows = None
    if not args.no_shapes and not args.only:
        shape_rows = decode_shape_rows(dev, peaks)
        prefill_rows = prefill_shape_rows(dev, peaks)
        cfg_rows = config_rows(dev, peaks, flush_l2)
    unfused = None
    if not args.no_unfused and not args.only:
        unfused = unfused_rows(dev, packed, scales, xd, xp, flush_l2, peaks)
    variants = None
    if not args.no_variants and not args.only and w is not None:
        variants = variant_rows(dev, w, xd, xp, flush_l2, peaks)

    # End to end through the public Python API, one step of the decode row:
    # pinned host x in, the DECODE_COPIES layer calls launched from Python
    # (no graph), every layer's y back to pinned host memory.  The ys are
    # read back on a copy stream, E2E_READBACK layers at a time as soon as
    # those calls end, so the reads overlap the next layers; the step ends
    # when the last read has landed.  A single call per step (x in, one call,
    # y out) is reported beside it.
    e2e = None
    if not args.no_e2e and not args.only:
        import dequant_gemm_int4_b200 as api
        layers = [(packed, scales)] + dcopies
        xh = xd.cpu().pin_memory()
        yh = torch.empty((len(layers), M_DECODE, N_W), dtype=torch.float32).pin_memory()
        ydev = torch.empty((len(layers), M_DECODE, N_W), dtype=torch.float32, device=dev)
        copy_stream = torch.cuda.Stream(dev)
        batches = [(b, min(b + E2E_READBACK, len(layers))) for b in range(0, len(layers), E2E_READBACK)]
        done = [torch.cuda.Event() for _ in batches]

        def e2e_step():
            xdev = xh.to(dev, non_blocking=True)
            for (b0, b1), ev in zip(batches, done):
                for i in range(b0, b1):
                    api.int4_matmul(xdev, layers[i][0], layers[i][1], K_W, GROUP, out=ydev[i])
                ev.record(stream)
                copy_stream.wait_event(ev)
                with torch.cuda.stream(copy_stream):
                    yh[b0:b1].copy_(ydev[b0:b1], non_blocking=True)
            stream.wait_stream(copy_stream)

        def single_step():
            y = api.int4_matmul(xh.to(dev, non_blocking=True), packed, scales, K_W, GROUP)
            yh[0].copy_(y, non_blocking=True)

        def time_e2e(fn):
            for _ in range(args.warmup):
                fn()
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            tot = 0.0
            for _ in range(args.steps):
                flush_l2()
                torch.cuda.synchronize()
                e0.record(stream)
                fn()
                e1.record(stream)
                torch.cuda.synchronize()
                tot += e0.elapsed_time(e1)
            return _max_over_ranks(tot / args.steps, world) * 1e-3

        t = time_e2e(e2e_step)
        t1 = time_e2e(single_step)
        ybytes = M_DECODE * N_W * 4
        e2e = {"value": units["decode"]["bytes"] * len(layers) / t / 1e9 * world, "unit": "GB/s",
               "h2d_bytes_per_step": xh.numel() * xh.element_size(),
               "d2h_bytes_per_step": ybytes * len(layers),
               "ms_per_step": t * 1e3, "calls_per_step": len(layers),
               "scope": ("decode row via the Python API: H2D of x, then int4_matmul over the "
                         f"{len(layers)} weight copies launched from Python, every y read back "
                         f"to pinned host memory on a copy stream, {E2E_READBACK} layers at a time"),
               "single_call": {"value": units["decode"]["bytes"] / t1 / 1e9 * world, "ms": t1 * 1e3,
                               "h2d_bytes": xh.numel() * xh.element_size(), "d2h_bytes": ybytes,
                               "scope": "H2D of x, one int4_matmul call, D2H of its y"}}
        del ydev

    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return 0

    cpu = None
    if world == 1 and not args.no_cpu_baseline and not args.only:
        cb = cpu_baseline()
        cpu = {"value": cb["decode_gbs"], "unit": "GB/s", "cores": cb["threads"], "kind": "oracle",
               "sample": cb["sample"], "rows": {k: cb[k] for k in ("quantize_gbs", "unpack_gbs",
                                                                    "decode_gbs", "prefill_tflops")}}
    line = {
        "metric": METRIC, "value": rows["decode"]["GB/s"] if "decode" in rows else None,
        "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "l2": "flushed before every row (256 MiB write, then 256 MiB read of another buffer); the decode row's back-to-back calls read distinct weight copies (3.9 GB > L2)",
                   "parallelism": f"replicas x{world}"},
        "rows": rows, "decode_llama7b": shape_rows, "prefill_shapes": prefill_rows, "configs": cfg_rows,
        "unfused": unfused, "variants": variants,
        "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks,
        "gpu_launches": args.steps * sum(launches_per_step[n] for n in order),
        "wall_ms_timed_region": wall_ms,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the affine-variant and bias+ReLU epilogue rows")
    ap.add_argument("--no-unfused", action="store_true",
                    help="skip the dequantize-then-GEMM comparison rows")
    ap.add_argument("--no-shapes", action="store_true",
                    help="skip the rows at the other configured shapes (Llama-7B decode, prefill, distilgpt2, bulk quantize, group-32/64 decode)")
    ap.add_argument("--only", choices=["quantize", "unpack", "decode", "prefill", "quantize_affine"],
                    default=None,
                    help="run one kernel of the step only (for profiling); no e2e or CPU baseline. "
                         "quantize_affine is the asymmetric variant's quantizer on the same W")
    ap.add_argument("--shape", default=None, metavar="N,K,M",
                    help="with --only: a smaller weight matrix N x K (and prefill batch M) for "
                         "profiler captures that must stay a few GB on the device")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.shape is not None:
        if not args.only:
            ap.error("--shape is for single-kernel profiling runs (--only)")
        global N_W, K_W, M_PREFILL
        N_W, K_W, M_PREFILL = (int(v) for v in args.shape.split(","))
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
