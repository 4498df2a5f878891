"""Benchmark of the int8 mixed-precision linear layer (LLM.int8()) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one whole int8_mixed_linear call (outlier detection, row
quantisation, outlier gather, int8 + fp16 tensor-core GEMM, dequantise and
merge) on one batch that is already resident in HBM.  The headline workload
is the largest single-GPU configuration, the 175B-shaped QKV projection at
prefill (T=4096, K=12288, N=36864, 0.1% outlier columns in every row,
alpha = 6), which is bound by the int8 tensor cores.  The same JSON line
carries, under "decode", the 175B-shaped fc1 at decode size (T=16, K=12288,
N=49152, 7 outlier columns), which is bound by HBM: the same steps and
warm-up, its own value, roofline, clocks and CPU baseline.  Three input sets
(X, Wq, sW, W16) are rotated so that every step reads operands that are not
in L2 (each set's weights alone are several times the 126 MB L2).

Under torchrun (N > 1) every rank runs its own independent batch (replicas;
the layer has no exchange step), the time is the max over ranks and the
value is the work of all ranks divided by that time ("scaling": "weak").
With --parallel column the ranks instead split one layer by weight columns
and all-gather Y over NCCL ("scaling": "strong": the job's work is fixed).

Prints one JSON line (rank 0).  --impl reference times the CPU oracle instead
(the reference arm for this method: it runs the plain CPU definition on a
bounded sample of the same workload).
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from int8_quantized_row_b200 import workloads as wl  # noqa: E402

DEFAULT_WORKLOAD = "b175_qkv_prefill_4096x12288x36864"
DECODE_WORKLOAD = "b175_fc1_decode_t16_12288x49152"
METRIC = "int8-mixed linear effective TOPS & weight GB/s; % of B200 int8/HBM roofline"
ROTATE = 3
PROFILES = os.path.join(ROOT, "profiles")
# A timed region shorter than this is a burst: the GEMM's roofline takes the
# burst GEMM peak (the sustained one was measured over seconds under the power cap).
BURST_WINDOW_S = 1.0
# Sources of each GEMM kernel, for keying its committed DRAM-traffic capture.
KERNEL_SOURCES = {
    "gemm_prefill_pair_kernel": ("gemm_prefill_pair.cuh", "device_common.cuh"),
    "gemm_decode_kernel": ("gemm_decode.cuh", "device_common.cuh"),
}


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--decode-workload", default=DECODE_WORKLOAD,
                    help="the HBM-bound point reported under \"decode\" in the same line ('none' to skip)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--rotate", type=int, default=ROTATE,
                    help="input sets rotated between steps (default 3: operands not in L2)")
    ap.add_argument("--sweep", action="store_true",
                    help="time every point of the 175B decoder-layer sweep in one process (one JSON line each; "
                         "not the one-line contract run)")
    ap.add_argument("--sweep-layers", default="qkv,out,fc1,fc2", help="layers of --sweep")
    ap.add_argument("--sweep-t", default="1,16,128,2048", help="batch sizes of --sweep")
    ap.add_argument("--chain", action="store_true",
                    help="time the 175B decoder layer's four projections (qkv, out, fc1, fc2) as one "
                         "int8_mixed_linear_chain call replayed from a CUDA graph (one JSON line; "
                         "not the one-line contract run)")
    ap.add_argument("--chain-t", type=int, default=16, help="tokens per projection for --chain")
    ap.add_argument("--parallel", default="replica", choices=["replica", "column"],
                    help="N>1 ranks: replica = an independent batch per GPU (weak scaling, the default); "
                         "column = one layer split by weight columns over the GPUs, Y all-gathered over NCCL "
                         "(strong scaling)")
    ap.add_argument("--codec", default="int8", choices=["int8", "int4"],
                    help="--sweep only: int8 = the LLM.int8() layer; int4 = the group-wise 4-bit weight codec "
                         "(int4_linear, T <= 64)")
    ap.add_argument("--variant", default="w16", choices=["w16", "wq"],
                    help="w16: int8_mixed_linear (fp16 weight resident for the outlier rows); "
                         "wq: int8_mixed_linear_wq (only Wq and sW resident)")
    return ap.parse_args(argv)


def all_configs():
    c = dict(wl.CONFIGS)
    c.update(wl.sweep_configs())
    return c


def work(cfg, n_out, variant="w16"):
    """Effective ops and algorithmic weight bytes of one call: Wq, sW and the
    outlier rows actually read (fp16 rows of W16, or int8 rows of Wq again
    for the Wq-only variant)."""
    T, K, N = cfg["T"], cfg["K"], cfg["N"]
    ops = 2.0 * T * K * N
    weight_bytes = K * N + 4 * N + (1 if variant == "wq" else 2) * n_out * N
    return ops, weight_bytes


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained"), src="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, src="fallback")


def tensor_peak(pk, region_s):
    """Dense int8 peak for a GEMM timed over a region of `region_s` seconds:
    the bf16 GEMM figure x 2 (B200's nominal dense int8 : bf16 ratio, 4.5 : 2.25
    POPS), the burst figure for a region under BURST_WINDOW_S, else the
    sustained one.  Returns (peak TOP/s, description)."""
    if region_s < BURST_WINDOW_S or not pk["bf16_tflops_sustained"]:
        return 2.0 * pk["bf16_tflops"], (f"{pk['src']} bf16 burst x 2 (dense int8 : bf16 nominal 4.5 : 2.25); "
                                         f"timed region {region_s * 1e3:.1f} ms < {BURST_WINDOW_S:.0f} s")
    return 2.0 * pk["bf16_tflops_sustained"], (f"{pk['src']} bf16 sustained x 2 (dense int8 : bf16 nominal "
                                               f"4.5 : 2.25); timed region {region_s:.2f} s")


def kernel_source_sha(kernel):
    """Hash of the sources of one GEMM kernel (its header and the PTX wrappers it uses)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "int8_quantized_row_b200", "csrc")
    for f in KERNEL_SOURCES[kernel]:
        h.update(f.encode())
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(workload, kernel):
    """DRAM bytes per launch of `kernel` on `workload` from a committed ncu
    capture, only while that kernel's sources are unchanged since the capture."""
    p = os.path.join(PROFILES, "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get("captures", {}).get(workload)
    if not d or d.get("kernel") != kernel or d.get("source_sha") != kernel_source_sha(kernel):
        return None
    return d.get("bytes_per_launch")


# ------------------------------------------------------------------ clocks

REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}


def summarise_clock_samples(samples, sm_max_mhz, source):
    """samples: (sm MHz, power W, clock-event reason bits) tuples taken under load."""
    reasons = set()
    for _, _, bits in samples:
        for nm, b in REASON_BITS.items():
            if bits & b:
                reasons.add(nm)
    sm = [s[0] for s in samples]
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": sm_max_mhz,
            "samples": len(sm), "power_w_max": max((s[1] for s in samples), default=None),
            "reasons": sorted(reasons), "source": source}


class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU, sampled on a
    background thread through NVML every `period_s` between start() and stop()
    (a timed region of a few milliseconds still gets samples); nvidia-smi at
    100 ms when NVML is unavailable."""

    def __init__(self, torch_device, period_s=0.001):
        self.period = period_s
        self.handle = None
        self.nvml = None
        self.samples = []
        self.stop_evt = threading.Event()
        self.thread = None
        self.smi = None
        self.index = getattr(torch_device, "index", None) or 0
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(torch_device)
            try:
                self.handle = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(props.uuid))
            except Exception:
                bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
                self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.nvml = pynvml
            self.sm_max = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
        except Exception:
            self.handle = None

    def _poll(self):
        n = self.nvml
        while not self.stop_evt.is_set():
            try:
                sm = n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM)
                pw = n.nvmlDeviceGetPowerUsage(self.handle) / 1000.0
                bits = n.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append((float(sm), pw, int(bits)))
            except Exception:
                return
            time.sleep(self.period)

    def start(self):
        self.samples = []
        self.stop_evt.clear()
        if self.handle is not None:
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        try:
            self.f = tempfile.TemporaryFile(mode="w+")
            self.smi = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={SMI_FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.index)],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.smi = None

    def stop(self):
        if self.thread is not None:
            self.stop_evt.set()
            self.thread.join()
            self.thread = None
            return summarise_clock_samples(self.samples, self.sm_max, f"NVML every {self.period * 1e3:g} ms")
        if self.smi is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "samples": 0, "reasons": ["no clock source"]}
        self.smi.terminate()
        try:
            self.smi.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.smi.kill()
        self.f.seek(0)
        return parse_clock_csv(self.f.read())


SMI_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def parse_clock_csv(text):
    """Median SM clock, max SM clock and the throttle reasons seen, from
    `nvidia-smi --query-gpu=<SMI_FIELDS> --format=csv,noheader,nounits` lines."""
    sm, smax, reasons = [], None, set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for line in text.splitlines():
        parts = [x.strip() for x in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            smax = float(parts[2])
        except ValueError:
            continue
        for nm, v in zip(names, parts[5:9]):
            if v.lower().startswith("active"):
                reasons.add(nm)
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
            "samples": len(sm), "reasons": sorted(reasons), "source": "nvidia-smi every 100 ms"}


# ------------------------------------------------------------------ distributed

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1 and args.impl == "ours":
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group(backend="nccl", timeout=timedelta(seconds=120))
        pg = dist
    return world, rank, local, pg


def barrier(pg, device=None):
    if pg is not None:
        if device is not None:
            pg.barrier(device_ids=[device])
        else:
            pg.barrier()


def max_over_ranks(pg, value, device):
    if pg is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ CPU oracle timing

def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _libgomp():
    import ctypes
    try:
        return ctypes.CDLL("libgomp.so.1")
    except OSError:
        return None


def cpu_threads():
    """Threads the oracle's OpenMP loops run with (OMP_NUM_THREADS, which
    torchrun sets to 1 per rank, else every core this process may use)."""
    gomp = _libgomp()
    if gomp is not None:
        return int(gomp.omp_get_max_threads())
    env = os.environ.get("OMP_NUM_THREADS", "").split(",")[0].strip()
    return int(env) if env.isdigit() and int(env) > 0 else host_cores()


def use_all_cores():
    """Let the oracle's OpenMP loops on this thread use every core this
    process may use (the reference arm runs on rank 0 alone)."""
    gomp = _libgomp()
    if gomp is not None:
        gomp.omp_set_num_threads(host_cores())


def oracle_sample(cfg, X, W, target_s=15.0, orc_state=None, variant="w16"):
    """Time the oracle on a bounded, seeded sample of the workload: a sub-batch
    of R rows of X (the whole method, outlier scan included, on those R
    tokens) against the first C columns of the weight (a column slice is the
    same sub-problem: column scales are per column).  Returns
    (TOPS, R, C, seconds, threads used, state, run)."""
    import oracle
    if orc_state is None:
        orc = oracle.default()
        Wq, sW = orc.quantize_weight_colwise(W)   # offline weight conversion: not timed
        orc_state = (orc, Wq, sW)
    orc, Wq, sW = orc_state
    T, N = cfg["T"], cfg["N"]
    threads = cpu_threads()
    rng = np.random.default_rng(1234)

    def run(R, C):
        rows = np.sort(rng.choice(T, size=R, replace=False))
        Xs = np.ascontiguousarray(X[rows])
        Wqs, sWs, Ws = (np.ascontiguousarray(Wq[:, :C]), np.ascontiguousarray(sW[:C]),
                        np.ascontiguousarray(W[:, :C]))
        t0 = time.perf_counter()
        orc.mixed_linear(Xs, Wqs, sWs, None if variant == "wq" else Ws, cfg["alpha"])
        return time.perf_counter() - t0

    R, C = min(T, threads), N
    dt = run(R, C)
    if dt < target_s:
        R = int(min(T, max(R, R * target_s / max(dt, 1e-9) // threads * threads)))
    else:
        R = 1
        C = int(max(16, (N * target_s / dt) // 16 * 16))     # one row runs on one thread
        C = min(C, N)
    dt = run(R, C)
    ops = 2.0 * R * cfg["K"] * C
    return ops / dt / 1e12, R, C, dt, min(R, threads), orc_state, run


def cpu_baseline(cfg, X, W, variant, target_s):
    tops, R, C, dt, cores, _, _ = oracle_sample(cfg, X, W, target_s=target_s, variant=variant)
    T, N = cfg["T"], cfg["N"]
    return {"value": tops, "unit": "TOPS", "cores": cores, "kind": "oracle",
            "sample": f"sub-batch of {R} of {T} rows x {C} of {N} columns ({dt:.1f} s, "
                      f"whole method incl. outlier scan); weight conversion untimed"}


def reference_line(args, name, cfg, world, seconds):
    """The oracle timed per step on a bounded sample of workload `name`."""
    X, W = wl.generate(cfg)
    T, K, N = cfg["T"], cfg["K"], cfg["N"]
    per_step = seconds / max(1, args.steps + args.warmup)
    _, R, C, _, cores, state, run = oracle_sample(cfg, X, W, target_s=min(per_step, 15.0), variant=args.variant)
    times = []
    for i in range(args.warmup + args.steps):
        dt = run(R, C)
        if i >= args.warmup:
            times.append(dt)
    total = sum(times)
    ops = 2.0 * R * K * C * len(times)
    value = ops / total / 1e12
    sample = (f"sub-batch of {R} of {T} rows x {C} of {N} columns per step (whole method incl. outlier "
              f"scan on the sub-batch); weight conversion untimed")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "i8",
        "data": "synthetic, seeded", "config": {"workload": name, "T": T, "K": K, "N": N,
                                                "alpha": cfg["alpha"], "variant": args.variant},
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_reference(args, world, rank):
    if rank != 0:
        return
    use_all_cores()                         # the other ranks do no work
    cfgs = all_configs()
    decode = args.decode_workload != "none"
    line = reference_line(args, args.workload, cfgs[args.workload], world, 80.0 if decode else 100.0)
    if decode:
        d = reference_line(args, args.decode_workload, cfgs[args.decode_workload], world, 20.0)
        line["decode"] = {k: d[k] for k in ("metric", "value", "unit", "ms_per_step", "config", "cpu_baseline",
                                            "e2e")}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm

def cublas_int8_tops(T, K, N, dev, iters=10):
    """cuBLAS int8 GEMM (torch._int_mm: int8 x int8 -> int32, no outlier part,
    no quantisation) on the same shape, as a burst: a measured int8 reference
    point, timed outside the benchmark's timed regions."""
    import torch
    if T <= 16:
        return None
    g = torch.Generator(device=dev).manual_seed(0)
    a = torch.randint(-127, 128, (T, K), dtype=torch.int8, device=dev, generator=g)
    b = torch.randint(-127, 128, (N, K), dtype=torch.int8, device=dev, generator=g).t()   # column-major B
    try:
        for _ in range(3):
            torch._int_mm(a, b)
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(iters):
            torch._int_mm(a, b)
        e.record()
        torch.cuda.synchronize()
        return 2.0 * T * K * N / (s.elapsed_time(e) / iters * 1e-3) / 1e12
    except RuntimeError:
        return None
    finally:
        del a, b
        torch.cuda.empty_cache()


def measure(args, name, cfg, world, rank, local, pg, with_cublas):
    """One workload on this rank: the timed steps, the GEMM-only pass, the
    end-to-end pass and the roofline.  Returns the fields of its JSON object."""
    import torch
    import int8_quantized_row_b200 as i8

    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    T, K, N, alpha = cfg["T"], cfg["K"], cfg["N"], cfg["alpha"]
    column = args.parallel == "column" and world > 1
    if column:
        from int8_quantized_row_b200 import column_parallel as cp
        ca, cb = cp.column_bounds(N, world, rank)
    else:
        ca, cb = 0, N
    NL = cb - ca                        # this rank's output columns

    # inputs: ROTATE independent sets, each seeded per (set, rank); with the
    # column split every rank draws the same layer and keeps its column block
    sets, host_x = [], []
    X0 = W0 = None
    nrot = max(1, args.rotate)
    for r in range(nrot):
        c = dict(cfg, seed=cfg["seed"] + (0 if column else 1000 * rank) + r)
        X, W = wl.generate(c)
        if column:
            W = np.ascontiguousarray(W[:, ca:cb])
        if r == 0:
            X0, W0 = X, W
        Xd = torch.from_numpy(X).to(dev)
        Wd = torch.from_numpy(W).to(dev)
        Wq, sW = i8.int8_quantize_weight_colwise(Wd)
        if args.variant == "wq":
            torch.cuda.synchronize()
            Wd = None                   # only Wq and sW stay resident
        sets.append((Xd, Wq, sW, Wd))
        host_x.append(torch.from_numpy(X).pin_memory())
    Y = torch.empty((T, NL), dtype=torch.float16, device=dev)
    Y_full = Y
    Y_host = torch.empty((T, N), dtype=torch.float16).pin_memory()
    if args.variant == "wq":
        ws = torch.empty(max(1, i8.int8_mixed_linear_wq_workspace_size(T, K, NL)), dtype=torch.uint8, device=dev)
    else:
        ws = i8.workspace(T, K, NL, dev)
    torch.cuda.synchronize()

    stats = i8.int8_outlier_stats(sets[0][0], alpha)
    n_out = int(stats[0].item())
    frac8 = float(stats[3].item())
    ops, wbytes = work(dict(cfg, N=NL), n_out, args.variant)       # this rank's share
    ops_job = 2.0 * T * K * N if column else world * ops               # the whole job's

    def step(i):
        nonlocal Y_full
        Xd, Wq, sW, Wd = sets[i % nrot]
        if Wd is None:
            i8.int8_mixed_linear_wq(Xd, Wq, sW, alpha, Y=Y, workspace_buf=ws)
        else:
            i8.int8_mixed_linear(Xd, Wq, sW, Wd, alpha, Y=Y, workspace_buf=ws)
        if column:
            Y_full = cp.gather_columns(Y, N, world, rank)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    clocks = ClockSampler(dev)
    launches0 = i8.int8_kernel_launch_count()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    barrier(pg, local)
    torch.cuda.synchronize()
    clocks.start()
    start.record(stream)
    for i in range(args.steps):
        step(i)
    end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier(pg, local)
    launches = i8.int8_kernel_launch_count() - launches0
    ms = start.elapsed_time(end)
    ms_max = max_over_ranks(pg, ms, dev)

    # The GEMM kernel's own duration, for the roofline: a second timed pass of
    # the same steps in which the library records CUDA events on this stream
    # right around each GEMM launch.  (It is a separate pass because an event
    # between the quantiser and the GEMM stops the GEMM from being launched as
    # a programmatic dependent, so the headline steps carry no such events.)
    gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in gev:
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize()
    for i in range(args.steps):
        i8.int8_time_next_gemm(gev[i][0], gev[i][1])
        step(i)
    torch.cuda.synchronize()
    gemm_ms = sum(a.elapsed_time(b) for a, b in gev) / args.steps
    status = i8.int8_read_and_clear_device_status()

    ms_step = ms_max / args.steps
    value = ops_job / (ms_step * 1e-3) / 1e12

    # end to end through the public API with host buffers: H2D of X, the call,
    # D2H of Y, every step, all inside the timed region
    for i in range(min(args.warmup, 3)):
        Xd = sets[i % nrot][0]
        Xd.copy_(host_x[i % nrot], non_blocking=True)
        step(i)
        Y_host[:, :Y_full.shape[1]].copy_(Y_full, non_blocking=True)
    torch.cuda.synchronize()
    e_steps = max(1, min(args.steps, 200))
    barrier(pg, local)
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(e_steps):
        Xd = sets[i % nrot][0]
        Xd.copy_(host_x[i % nrot], non_blocking=True)
        step(i)
        Y_host[:, :Y_full.shape[1]].copy_(Y_full, non_blocking=True)
    end.record(stream)
    torch.cuda.synchronize()
    barrier(pg, local)
    e_ms = max_over_ranks(pg, start.elapsed_time(end), dev) / e_steps
    e_value = ops_job / (e_ms * 1e-3) / 1e12

    pk = peaks()
    decode = T <= i8.DECODE_MAX_T
    if decode:
        kernel = "gemm_decode_kernel"
        achieved = (wbytes + 2 * T * K + 2 * T * N) / (gemm_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / pk["hbm_gbs"], "peak_src": f"{pk['src']} HBM copy bandwidth",
                "algorithmic_bytes_per_launch": wbytes + 2 * T * K + 2 * T * N}
    else:
        kernel = "gemm_prefill_pair_kernel"
        region_s = ms_step * args.steps * 1e-3          # the length of the GEMM-timing pass
        peak, src = tensor_peak(pk, region_s)
        achieved = ops / (gemm_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "peak_src": src, "algorithmic_ops_per_launch": ops}
        cub = cublas_int8_tops(T, K, NL, dev) if with_cublas else None
        if cub:
            roof["int8_cublas_measured"] = cub
            roof["frac_of_int8_cublas"] = achieved / cub
            roof["int8_cublas_note"] = ("torch._int_mm (cuBLAS int8 x int8 -> int32, no outlier part, no "
                                        "quantisation) on the same shape, 10 calls, timed in this process")
    roof["traffic"] = ncu_traffic(name, kernel) if args.variant == "w16" else None
    roof["kernel"] = kernel
    roof["kernel_ms"] = gemm_ms

    out = {
        "metric": METRIC, "value": value, "unit": "TOPS", "ms_per_step": ms_step,
        "config": {"workload": name, "T": T, "K": K, "N": N, "alpha": alpha, "outlier_cols": n_out,
                   "frac_8bit": frac8,
                   "parallelism": (f"column-parallel x{world}: weight columns split, Y all-gathered over NCCL"
                                   if column else f"replicas x{world}" if world > 1 else "single GPU"),
                   "l2": f"{nrot} rotating input sets" + (" (each step's operands not in L2)" if nrot >= 3 else
                                                          " (operands may be partly L2-resident)"),
                   "variant": ("wq-only: outlier rows dequantised from Wq, no fp16 weight resident"
                               if args.variant == "wq" else "w16: fp16 weight rows for the outliers"),
                   "resident_weight_bytes": K * NL + 4 * NL + (0 if args.variant == "wq" else 2 * K * NL)},
        "weight_gbs": world * wbytes / (ms_step * 1e-3) / 1e9,
        "roofline": roof,
        "e2e": {"value": e_value, "unit": "TOPS", "h2d_bytes_per_step": 2 * T * K,
                "d2h_bytes_per_step": 2 * T * N, "ms_per_step": e_ms},
        "gpu_launches": int(launches),
        "clocks": clk,
        "device_status": status,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(cfg, X0, W0, args.variant, 15.0 if not decode else 8.0)
    del sets, Y, Y_full, ws
    torch.cuda.empty_cache()
    return out


def run_ours(args, world, rank, local, pg):
    import torch
    torch.cuda.set_device(local)
    cfgs = all_configs()
    head = measure(args, args.workload, cfgs[args.workload], world, rank, local, pg, with_cublas=True)
    line = {
        "metric": METRIC, "value": head["value"], "unit": "TOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
        "scaling": "strong" if (args.parallel == "column" and world > 1) else "weak",
        "vs_baseline": None, "dtype": "i8", "data": "synthetic, seeded (N(0,1) activations with planted outlier "
        "columns, N(0,sigma) weights); no datasets or trained weights",
    }
    line.update({k: v for k, v in head.items() if k not in line})
    if args.decode_workload != "none":
        d = measure(args, args.decode_workload, cfgs[args.decode_workload], world, rank, local, pg,
                    with_cublas=False)
        line["decode"] = d
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def int4_bytes(T, K, N):
    """Algorithmic bytes of one int4_linear call: the packed codes (1/2 byte per
    weight) and the (s, lo) pairs (4 bytes per group of 64), X read, Y written."""
    return K * N // 2 + (K // 64) * N * 4 + 2 * T * K + 2 * T * N


def run_sweep_int4(args):
    """The 175B decoder-layer projections with the group-wise 4-bit weight codec
    (int4_linear): every layer's weight is drawn, packed once, and each T point
    is timed over whole calls and over the GEMM kernel alone.  The packed
    weights (76-302 MB) exceed L2, so every call streams them from HBM."""
    import torch
    import int8_quantized_row_b200 as i8
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    pk = peaks()
    want_t = sorted(int(t) for t in args.sweep_t.split(",") if int(t) <= i8.INT4_MAX_T)
    for layer, (K, N) in wl.SWEEP_LAYERS.items():
        if layer not in args.sweep_layers.split(","):
            continue
        W = torch.from_numpy(wl.make_w(K, N, 0.01)).to(dev)
        W4, S4 = i8.int4_quantize_weight_groupwise(W)
        del W
        ws = torch.empty(max(1, i8.int4_linear_workspace_size(max(want_t), K, N)), dtype=torch.uint8, device=dev)
        for T in want_t:
            X = torch.from_numpy(wl.make_x(T, K, 0, seed=T)).to(dev)
            Y = torch.empty((T, N), dtype=torch.float16, device=dev)

            def step():
                i8.int4_linear(X, W4, S4, N, Y=Y, workspace_buf=ws)
            steps = 200
            for _ in range(5):
                step()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(steps):
                step()
            b.record(stream)
            torch.cuda.synchronize()
            ms = a.elapsed_time(b) / steps
            gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
            for x, y in gev:
                x.record(stream)
                y.record(stream)
            torch.cuda.synchronize()
            for i in range(steps):
                i8.int8_time_next_gemm(gev[i][0], gev[i][1])
                step()
            torch.cuda.synchronize()
            gemm_ms = sum(x.elapsed_time(y) for x, y in gev) / steps
            nbytes = int4_bytes(T, K, N)
            line = {"workload": f"b175_int4_{layer}_t{T}_{K}x{N}", "codec": "int4 group-wise (64)", "T": T,
                    "K": K, "N": N, "ms_per_call": ms, "gemm_ms": gemm_ms,
                    "tops": 2.0 * T * K * N / (ms * 1e-3) / 1e12,
                    "weight_gbs": (K * N // 2 + (K // 64) * N * 4) / (ms * 1e-3) / 1e9,
                    "algorithmic_bytes": nbytes,
                    "gemm_frac_hbm": nbytes / (gemm_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                    "call_frac_hbm": nbytes / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                    "status": i8.int8_read_and_clear_device_status()}
            print(json.dumps(line), flush=True)
            del X, Y
        del W4, S4, ws
        torch.cuda.empty_cache()


def run_sweep(args):
    """The 175B decoder-layer sweep: each layer's weight is drawn and converted
    once, then every (T, outlier fraction, alpha) point is timed on it: whole
    calls with CUDA events, then the GEMM alone through int8_time_next_gemm.
    The weights (151-604 MB of int8) exceed L2, so steps stream them from HBM."""
    import torch
    import int8_quantized_row_b200 as i8
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    pk = peaks()
    cfgs = wl.sweep_configs()
    want_t = {int(t) for t in args.sweep_t.split(",")}
    for layer, (K, N) in wl.SWEEP_LAYERS.items():
        if layer not in args.sweep_layers.split(","):
            continue
        W = torch.from_numpy(wl.make_w(K, N, 0.01)).to(dev)
        Wq, sW = i8.int8_quantize_weight_colwise(W)
        Tmax = max(wl.SWEEP_T)
        if args.variant == "wq":
            W = None
            ws = torch.empty(max(1, i8.int8_mixed_linear_wq_workspace_size(Tmax, K, N)), dtype=torch.uint8, device=dev)
        else:
            ws = i8.workspace(Tmax, K, N, dev)
        Y = torch.empty((Tmax, N), dtype=torch.float16, device=dev)
        for name, cfg in cfgs.items():
            if not name.startswith(f"b175_sweep_{layer}_") or cfg["T"] not in want_t:
                continue
            T, alpha = cfg["T"], cfg["alpha"]
            X = torch.from_numpy(wl.make_x(T, K, cfg["n_out"], cfg["lo"], cfg["hi"], cfg["row_prob"], cfg["seed"])).to(dev)
            Yt = Y[:T]

            def step():
                if W is None:
                    i8.int8_mixed_linear_wq(X, Wq, sW, alpha, Y=Yt, workspace_buf=ws)
                else:
                    i8.int8_mixed_linear(X, Wq, sW, W, alpha, Y=Yt, workspace_buf=ws)
            steps = 40 if T >= 2048 else 200
            for _ in range(5):
                step()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(steps):
                step()
            b.record(stream)
            torch.cuda.synchronize()
            ms = a.elapsed_time(b) / steps
            gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
            for x, y in gev:            # torch only reports times of events it has seen recorded
                x.record(stream)
                y.record(stream)
            torch.cuda.synchronize()
            for i in range(steps):
                i8.int8_time_next_gemm(gev[i][0], gev[i][1])
                step()
            torch.cuda.synchronize()
            gemm_ms = sum(x.elapsed_time(y) for x, y in gev) / steps
            n_out = int(i8.int8_outlier_stats(X, alpha)[0].item())
            ops, wbytes = work(cfg, n_out, args.variant)
            line = {"workload": name, "T": T, "K": K, "N": N, "alpha": alpha, "outlier_cols": n_out,
                    "variant": args.variant, "ms_per_call": ms, "tops": ops / (ms * 1e-3) / 1e12,
                    "weight_gbs": wbytes / (ms * 1e-3) / 1e9, "gemm_ms": gemm_ms,
                    "status": i8.int8_read_and_clear_device_status()}
            if T <= i8.DECODE_MAX_T:
                io = 2 * T * K + 2 * T * N
                line["gemm_frac_hbm"] = (wbytes + io) / (gemm_ms * 1e-3) / 1e9 / pk["hbm_gbs"]
                line["call_frac_hbm"] = (wbytes + io) / (ms * 1e-3) / 1e9 / pk["hbm_gbs"]
            if T >= 128:
                peak, _ = tensor_peak(pk, ms * steps * 1e-3)
                line["gemm_frac_int8"] = ops / (gemm_ms * 1e-3) / 1e12 / peak
            print(json.dumps(line), flush=True)
            del X
        del W, Wq, sW, ws, Y
        torch.cuda.empty_cache()


def run_chain(args):
    """The 175B decoder layer's projections qkv, out, fc1 and fc2 (each with its
    own seeded input of 0.1 % outlier columns, alpha 6) as one
    int8_mixed_linear_chain call: sixteen launches, captured once into a CUDA
    graph and replayed.  The weights (1.8 GB of int8) exceed L2, so every
    replay streams them from HBM.  Each layer is also timed alone, eagerly."""
    import torch
    import int8_quantized_row_b200 as i8
    dev = torch.device("cuda", 0)
    pk = peaks()
    T, alpha, frac = args.chain_t, 6.0, 0.001
    layers, meta = [], []
    for seed, (name, (K, N)) in enumerate(wl.SWEEP_LAYERS.items()):
        W = torch.from_numpy(wl.make_w(K, N, 0.01)).to(dev)
        Wq, sW = i8.int8_quantize_weight_colwise(W)
        n_out = int(round(frac * K))
        X = torch.from_numpy(wl.make_x(T, K, n_out, 6.0, 60.0, 1.0, seed)).to(dev)
        layers.append((X, Wq, sW, None if args.variant == "wq" else W, alpha,
                       torch.empty((T, N), dtype=torch.float16, device=dev)))
        meta.append(dict(layer=name, K=K, N=N, outlier_cols=int(i8.int8_outlier_stats(X, alpha)[0].item())))
    ws = torch.empty(max(1, i8.int8_mixed_linear_chain_workspace_size(layers)), dtype=torch.uint8, device=dev)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        for _ in range(3):
            i8.int8_mixed_linear_chain(layers, workspace_buf=ws, stream=side)
        side.synchronize()
        n0 = i8.int8_kernel_launch_count()
        i8.int8_mixed_linear_chain(layers, workspace_buf=ws, stream=side)
        launches = i8.int8_kernel_launch_count() - n0        # the library's kernels in one chain
        side.synchronize()
        with torch.cuda.graph(graph, stream=side):
            i8.int8_mixed_linear_chain(layers, workspace_buf=ws, stream=side)
    stream = torch.cuda.current_stream()
    for _ in range(max(3, args.warmup)):
        graph.replay()
    torch.cuda.synchronize()
    steps = min(args.steps, 500)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        graph.replay()
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    # each layer alone, eager calls on the same workspace
    for m, (X, Wq, sW, W, al, Y) in zip(meta, layers):
        for _ in range(3):
            i8.int8_mixed_linear_chain([(X, Wq, sW, W, al, Y)], workspace_buf=ws)
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(steps):
            i8.int8_mixed_linear_chain([(X, Wq, sW, W, al, Y)], workspace_buf=ws)
        b.record(stream)
        torch.cuda.synchronize()
        m["ms_eager"] = a.elapsed_time(b) / steps
    ops = sum(2.0 * T * m["K"] * m["N"] for m in meta)
    wbytes = sum(m["K"] * m["N"] + 4 * m["N"] + (1 if args.variant == "wq" else 2) * m["outlier_cols"] * m["N"]
                 for m in meta)
    io_bytes = sum(2 * T * (m["K"] + m["N"]) for m in meta)
    line = {"metric": "175B decoder-layer projections (qkv, out, fc1, fc2) as one int8_mixed_linear_chain call, "
                      "CUDA-graph replay",
            "value": ops / (ms * 1e-3) / 1e12, "unit": "TOPS", "ms_per_chain": ms, "steps": steps,
            "T": T, "alpha": alpha, "variant": args.variant, "graph": True, "launches_per_chain": launches,
            "weight_bytes": wbytes, "weight_gbs": wbytes / (ms * 1e-3) / 1e9,
            "frac_hbm": (wbytes + io_bytes) / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
            "peak_hbm_gbs": pk["hbm_gbs"], "peak_src": pk["src"],
            "sum_of_eager_layer_ms": sum(m["ms_eager"] for m in meta), "layers": meta,
            "data": "synthetic, seeded", "status": i8.int8_read_and_clear_device_status()}
    del graph
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.sweep:
        run_sweep_int4(args) if args.codec == "int4" else run_sweep(args)
        return
    if args.chain:
        run_chain(args)
        return
    cfgs = all_configs()
    for w in (args.workload, args.decode_workload):
        if w != "none" and w not in cfgs:
            raise SystemExit(f"unknown workload {w}; known: {sorted(cfgs)[:8]} ...")
    world, rank, local, pg = dist_setup(args)
    if args.impl == "reference":
        run_reference(args, world, rank)   # rank 0 only; other ranks exit 0
        return
    run_ours(args, world, rank, local, pg)


if __name__ == "__main__":
    main()
