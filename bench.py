"""Benchmark of the fused rotate + quantize operator on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-cpu-baseline] [--no-e2e]

One step = one pass of the whole operator (rotation, scale, codes, packing) over one
batch: the largest workload, x bf16 [32768, 128, 112] with P1 [128,128], P2 [112,112]
random orthogonal, per-group E2M1 with E8M0 scales, dstTypeMax 10.0. Inputs (940 MB)
are larger than the 126 MB L2, so no flush is needed between steps; a smaller workload
(--workload) cycles through enough copies of its inputs and outputs to exceed twice the
L2. Under torchrun each
rank processes its own batch (weak scaling; tokens are independent, no collective on the
data path); the reported time is the max over ranks of the device time.

Prints one JSON line (rank 0). `--impl reference` times the CPU oracle instead, on a
bounded sample of the same workload, with the same metric.
"""

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from rotation_bit_quantization_token_b200.workloads import (  # noqa: E402
    BENCH_WORKLOAD, WORKLOADS, make_inputs)

METRIC = "tokens/s of fused rotate+quantize (HBM GB/s and roofline fraction alongside)"
UNIT = "tokens/s"
CSRC = os.path.join(ROOT, "rotation_bit_quantization_token_b200", "csrc")


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=BENCH_WORKLOAD, choices=sorted(WORKLOADS))
    p.add_argument("--kernel", default="auto", choices=["auto", "general", "tcgen05"])
    p.add_argument("--tokens", type=int, default=0,
                   help="override the token count (a smaller case of the same workload, "
                        "for profiling); 0 keeps the workload's own K")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-clocks", action="store_true")
    p.add_argument("--no-consumer", action="store_true",
                   help="skip the consumer FP4 x FP4 GEMM leg (timed apart from the step)")
    p.add_argument("--consumer-only", action="store_true",
                   help="time only the consumer GEMM leg and print its object (for profiling)")
    return p.parse_args(argv)


# ----------------------------------------------------------------------------------------
# host-side helpers (covered by CPU tests)
# ----------------------------------------------------------------------------------------

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def rank_seed(rank):
    """Each rank draws its own batch (weak scaling): seed 0 for rank 0, and so on."""
    return int(rank)


def max_over_ranks(value, world, device=None):
    """Max of a float over all ranks (all_reduce MAX); the identity for one rank."""
    if world <= 1:
        return float(value)
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), float(pk["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, "fallback"


KERNEL_SOURCES = {
    "tcgen05": ["fq_tc.cu", "fq_quant.cuh", "fq_internal.h"],
    "general": ["fq_general.cu", "fq_quant.cuh", "fq_internal.h"],
}


# GPU sleep queued ahead of the timed launches, per step: about 200 us at 2 GHz, several
# times the host's time to enqueue one step through the Python API
PRIME_CYCLES_PER_STEP = 400_000


def prime_stream(steps):
    """Queues a GPU sleep on the current stream, so that the launches enqueued after it wait
    until the host has enqueued them all (torch.cuda._sleep is torch's own spin kernel);
    False where this torch has no such call (the timing then holds the host's gaps)."""
    sleep = getattr(torch.cuda, "_sleep", None)
    if sleep is None:
        return False
    sleep(int(PRIME_CYCLES_PER_STEP * max(steps, 20)))
    return True


def kernel_source_hash(kernel="tcgen05"):
    """Hash of the source files of one kernel (a recorded DRAM-traffic figure is valid only
    for the source it was captured on)."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload, src_hash):
    """DRAM bytes per launch from a committed ncu summary, or None when the summary is
    missing or was taken on a different kernel source."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    try:
        with open(path) as f:
            for ln in f:
                ln = ln.strip()
                if not ln or ln.startswith("#"):
                    continue
                k, w, hsh, b = ln.split()[:4]
                if k == kernel and w == workload and hsh == src_hash:
                    return float(b)
    except OSError:
        pass
    return None


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.out = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        return parse_clock_samples(out)


def parse_clock_samples(text):
    sm, smax, reasons = [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for ln in (text or "").splitlines():
        f = [s.strip() for s in ln.split(",")]
        if len(f) < 9:
            continue
        try:
            sm.append(float(f[1]))
            smax.append(float(f[2]))
        except ValueError:
            continue
        for name, val in zip(names, f[5:9]):
            if val.lower().startswith("active"):
                reasons.add(name)
    if not sm:
        return None
    return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(smax)),
            "reasons": sorted(reasons), "samples": len(sm)}


def host_cores():
    """Cores this process may run on (its affinity mask) and the host's logical CPUs."""
    try:
        usable = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        usable = os.cpu_count() or 1
    return usable, os.cpu_count() or usable


def single_core_oracle_rate(w, seed, target_s=3.0):
    """The oracle's rate on one core (BLAS limited to one thread) on a small token sample
    of workload w, scaled to tokens/s. Returns (tokens/s, tokens timed, seconds)."""
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):
        r, n, dt, _ = bounded_oracle_sample(w, seed, target_s=target_s, max_tokens=512)
    return r, n, dt


def bounded_oracle_sample(w, seed, target_s=12.0, min_tokens=16, max_tokens=4096):
    """Times the CPU oracle on a bounded token sample of workload w (about target_s of
    work). Returns (tokens/s, tokens timed, seconds, threads)."""
    import oracle
    from threadpoolctl import threadpool_info
    x, P1, P2 = make_inputs(w.with_tokens(min(w.K, max_tokens)), seed=seed)
    xf = x.float().numpy().astype(np.float64)
    p1 = P1.float().numpy().astype(np.float64)
    p2 = P2.float().numpy().astype(np.float64)

    def run(n):
        t0 = time.perf_counter()
        if w.mode == "per_token":
            oracle.flat_quant_per_token(xf[:n], p1, p2, w.clip_ratio, w.out)
        else:
            oracle.flat_quant_mx(xf[:n], p1, p2, w.dst_type_max)
        return time.perf_counter() - t0

    n = min_tokens
    dt = run(n)
    while dt < target_s / 8 and n < xf.shape[0]:
        n = min(xf.shape[0], n * 4)
        dt = run(n)
    # final sample sized to about target_s of work (bounded by the tokens drawn)
    n_final = int(min(xf.shape[0], max(n, n * target_s / max(dt, 1e-9))))
    if n_final > n:
        n = n_final
        dt = run(n)
    threads = max([d.get("num_threads", 1) for d in threadpool_info()] or [1])
    return n / dt, n, dt, threads


FP4_PER_BF16 = 4.0  # nominal dense FP4 / bf16 tensor rate on B200 (9 / 2.25 PFLOP/s)


def consumer_gemm_leg(w, dev, steps, bf16_tflops, peak_src, O=4096):
    """Times fq_mx_matmul (the consumer contraction of two per-group outputs) on operands of
    the workload's row length L = M*N: activations [T, L] with T = min(K, 8192), weights
    [O, L], seeded random E2M1 codes and E8M0 bytes in [120, 133] drawn on the device. It is
    timed apart from the step (it is not part of the fused operator). Returns a dict with
    the time, TFLOP/s and the roofline against the FP4 dense peak, taken as the bf16 peak
    times the nominal FP4 / bf16 ratio."""
    import ctypes
    from rotation_bit_quantization_token_b200 import _lib
    lib = _lib.load()
    L = w.M * w.N
    T = min(w.K, 8192)
    g = torch.Generator(device=dev).manual_seed(0)
    S = 2 * (-(-L // 64))
    a = torch.randint(0, 256, (T, L // 2), dtype=torch.uint8, device=dev, generator=g)
    wt = torch.randint(0, 256, (O, L // 2), dtype=torch.uint8, device=dev, generator=g)
    sa = torch.randint(120, 134, (T, S), dtype=torch.uint8, device=dev, generator=g)
    sw = torch.randint(120, 134, (O, S), dtype=torch.uint8, device=dev, generator=g)
    C = torch.empty((T, O), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    vp = ctypes.c_void_p

    def call():
        st = lib.fq_mx_matmul(T, O, L, vp(a.data_ptr()), vp(sa.data_ptr()), vp(wt.data_ptr()),
                              vp(sw.data_ptr()), vp(C.data_ptr()), vp(status.data_ptr()),
                              vp(stream.cuda_stream))
        if st != 0:
            raise SystemExit(f"fq_mx_matmul failed: {st}")

    for _ in range(3):
        call()
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for e0, e1 in evs:
        e0.record(stream)
        call()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    if int(status.item()) != 0:
        raise SystemExit(f"fq_mx_matmul status {int(status.item())}")
    ms = float(np.mean([e0.elapsed_time(e1) for e0, e1 in evs]))
    tflops = 2.0 * T * O * L / (ms / 1e3) / 1e12
    peak = bf16_tflops * FP4_PER_BF16
    return {"op": "fq_mx_matmul", "shape": {"T": T, "O": O, "L": L}, "kernel_ms": ms,
            "value": tflops, "unit": "TFLOP/s", "launches": steps,
            "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
                         "frac": tflops / peak,
                         "peak_source": f"{peak_src} bf16 dense x {FP4_PER_BF16:g} (nominal FP4 / bf16 ratio)"},
            "data": "seeded random E2M1 codes, E8M0 bytes 120-133"}


# ----------------------------------------------------------------------------------------
# arms
# ----------------------------------------------------------------------------------------

def run_reference(args, rank, world):
    w = WORKLOADS[args.workload]
    if rank != 0:
        return 0
    # each step times the oracle on the same bounded sample of the workload; the sample
    # size is fixed by a sizing run before the warm-up, so every step does the same work,
    # about 2 s of it, less when many steps are asked for (the run stays near two minutes)
    import oracle
    from threadpoolctl import threadpool_info
    target_s = min(2.0, 120.0 / max(1, args.steps + args.warmup))
    _, n_tok, _, threads = bounded_oracle_sample(w, seed=0, target_s=target_s)
    x, P1, P2 = make_inputs(w.with_tokens(n_tok), seed=0)
    xf = x.float().numpy().astype(np.float64)
    p1 = P1.float().numpy().astype(np.float64)
    p2 = P2.float().numpy().astype(np.float64)

    def step():
        if w.mode == "per_token":
            oracle.flat_quant_per_token(xf, p1, p2, w.clip_ratio, w.out)
        else:
            oracle.flat_quant_mx(xf, p1, p2, w.dst_type_max)

    for _ in range(args.warmup):
        step()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        step()
        times.append(time.perf_counter() - t0)
    threads = max([d.get("num_threads", 1) for d in threadpool_info()] or [threads])
    ms_per_step = 1e3 * float(np.mean(times))
    value = n_tok / (ms_per_step / 1e3)
    usable, logical = host_cores()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "K": w.K, "M": w.M, "N": w.N,
                   "mode": w.mode, "dst_type_max": w.dst_type_max,
                   "clip_ratio": w.clip_ratio, "tokens_per_step_sample": n_tok,
                   "step": f"the oracle over {n_tok} of the workload's {w.K} tokens"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "nproc": logical, "usable_cores": usable,
                         "omp_num_threads": os.environ.get("OMP_NUM_THREADS"),
                         "sample": f"{n_tok} tokens of {w.name} per step "
                                   f"({ms_per_step / 1e3:.2f} s each), rate in tokens/s"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


L2_BYTES = 126 * 1024 * 1024


def buffer_copies(bytes_per_launch, l2_bytes=L2_BYTES):
    """How many copies of the inputs and outputs the timed loop cycles through, so that
    each launch touches memory no recent launch left in L2: 1 when one launch already
    moves more than twice the L2, else enough copies to exceed that."""
    if bytes_per_launch >= 2 * l2_bytes:
        return 1
    return int(-(-2 * l2_bytes // bytes_per_launch)) + 1


def run_ours(args, rank, world, local):
    import rotation_bit_quantization_token_b200 as fqlib
    from rotation_bit_quantization_token_b200 import FlatQuant, HostPipeline

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=dev)
    w = WORKLOADS[args.workload]
    if args.tokens:
        w = w.with_tokens(args.tokens)
    if args.consumer_only:
        hbm_gbs, bf16_tflops, peak_src = load_peaks()
        if rank == 0:
            print(json.dumps(consumer_gemm_leg(w, dev, max(1, args.steps), bf16_tflops, peak_src)),
                  flush=True)
        return 0
    # cpu baseline first (rank 0 at N = 1 only), while nothing runs on the GPU
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r, n, dt, threads = bounded_oracle_sample(w, seed=0)
        r1, n1, dt1 = single_core_oracle_rate(w, seed=0)
        usable, logical = host_cores()
        cpu = {"value": r, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"{n} tokens of {w.name} ({dt:.1f} s), scaled to tokens/s",
               "nproc": logical, "usable_cores": usable,
               "omp_num_threads": os.environ.get("OMP_NUM_THREADS"),
               "single_core": {"value": r1, "unit": UNIT,
                               "sample": f"{n1} tokens on one BLAS thread ({dt1:.1f} s)"}}

    x, P1, P2 = make_inputs(w, seed=rank_seed(rank))
    P1d, P2d = P1.to(dev), P2.to(dev)
    fq = FlatQuant(w.K, w.M, w.N, kernel=args.kernel)
    K, M, N = w.K, w.M, w.N
    copies = buffer_copies(w.bytes_per_token() * K)
    xds, outs, scales = [], [], []
    for _ in range(copies):
        xds.append(x.to(dev))
        if w.mode == "per_token":
            scales.append(torch.empty((K,), dtype=torch.float32, device=dev))
            outs.append(torch.empty((K, M, N // 8), dtype=torch.int32, device=dev) if w.out == "int32"
                        else torch.empty((K, M * N // 2), dtype=torch.uint8, device=dev))
        else:
            outs.append(torch.empty((K, M * N // 2), dtype=torch.uint8, device=dev))
            scales.append(torch.empty((K, -(-M * N // 64), 2), dtype=torch.uint8, device=dev))
    stream = torch.cuda.current_stream(dev)
    n_step = [0]

    def step():
        c = n_step[0] % copies
        n_step[0] += 1
        if w.mode == "per_token":
            fq.quantize_per_token(xds[c], P1d, P2d, w.clip_ratio, w.out, out=outs[c],
                                  quant_scale=scales[c], stream=stream)
        else:
            fq.quantize_mx(xds[c], P1d, P2d, w.dst_type_max, out=outs[c], scales=scales[c],
                           stream=stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    status = fq.device_status()
    if status:
        raise SystemExit(f"device status {status} after warm-up")

    clocks = ClockSampler(local) if not args.no_clocks else None
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(dev)
    if clocks:
        clocks.start()
        time.sleep(0.3)
    # CUDA events on the launching stream at the two ends of the timed region; the step is
    # one kernel launch, so the average launch duration is the region over the launches. The
    # timed launches queue up behind a short GPU sleep (outside the timed region), so that
    # the host has enqueued them all before the first one runs and they run back to back:
    # the events then time the device work, not the host's Python and ctypes time between
    # calls, which is longer than the kernel of the smaller workloads (events between the
    # launches would add their own gaps, about 2 us a launch). `queue_primed` records that
    # the sleep was still running when the last launch had been enqueued.
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    launches = 0
    primed = prime_stream(args.steps)
    t_start.record(stream)
    for i in range(args.steps):
        step()
        launches += fq.last_launch_count
    t_end.record(stream)
    queue_primed = primed and not t_start.query()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clock_info = clocks.stop() if clocks else None
    elapsed_ms = t_start.elapsed_time(t_end)
    kernel_ms = elapsed_ms / max(launches, 1)  # average launch duration
    elapsed_ms = max_over_ranks(elapsed_ms, world, dev)
    kernel_ms_max = max_over_ranks(kernel_ms, world, dev)
    status = fq.device_status()
    if status:
        raise SystemExit(f"device status {status} after timing")

    tokens_total = K * args.steps * world
    value = tokens_total / (elapsed_ms / 1e3)
    hbm_gbs, bf16_tflops, peak_src = load_peaks()
    bytes_per_launch = w.bytes_per_token() * K
    achieved = bytes_per_launch / (kernel_ms_max / 1e3) / 1e9
    kname = fq.last_kernel
    src_hash = kernel_source_hash(kname)
    traffic = recorded_traffic(kname, w.name, src_hash)

    # end to end through the public API: pinned host buffers, copies inside the region
    e2e = None
    if not args.no_e2e:
        pipe = HostPipeline(fq, w.mode, w.out if w.mode == "per_token" else "int4", dev)
        xh, P1h, P2h = x.pin_memory(), P1.pin_memory(), P2.pin_memory()
        oh, sh = pipe.host_outputs()
        e_steps = max(3, min(args.steps, 10))

        def e2e_step():
            pipe.run(xh, P1h, P2h, oh, sh, clip_ratio=w.clip_ratio, dst_type_max=w.dst_type_max,
                     stream=stream)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(e_steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks(a.elapsed_time(b), world, dev)
        e2e = {"value": K * e_steps * world / (e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": pipe.h2d_bytes(), "d2h_bytes_per_step": pipe.d2h_bytes(),
               "ms_per_step": e_ms / e_steps}

    consumer = None
    if rank == 0 and world == 1 and not args.no_consumer:
        consumer = consumer_gemm_leg(w, dev, max(3, min(args.steps, 10)), bf16_tflops, peak_src)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16-in/fp32-acc/e2m1-out"
            if w.mode == "mx" else "bf16-in/fp32-acc/int4-out",
            "data": "synthetic (seeded numpy PCG64; distribution of the workload)",
            "config": {"workload": w.name, "K": K, "M": M, "N": N, "mode": w.mode,
                       "dst_type_max": w.dst_type_max, "clip_ratio": w.clip_ratio,
                       "tokens_per_gpu_per_step": K,
                       "l2": "inputs larger than L2 (no flush)" if copies == 1 else
                       f"{copies} rotating input/output copies ({copies * bytes_per_launch / 1e6:.0f} MB, "
                       "more than twice the L2; no flush)",
                       "parallelism": f"dp{world} (token shards, no collective)",
                       "kernel": kname,
                       "queue_primed": queue_primed},
            "hbm_gbs": bytes_per_launch * world / (elapsed_ms / args.steps / 1e3) / 1e9,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                         "frac": achieved / hbm_gbs, "traffic": traffic,
                         "peak_source": peak_src + " (MEASURED_PEAKS.json hbm_gbs, copy)"
                         if peak_src == "measured" else "fallback 6.65 TB/s",
                         "algorithmic_bytes_per_launch": bytes_per_launch,
                         "kernel_ms": kernel_ms_max,
                         "tensor_frac": w.flops_per_token() * K / (kernel_ms_max / 1e3)
                         / (bf16_tflops * 1e12)},
            "gpu_launches": launches,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "clocks": clock_info,
            "consumer_gemm": consumer,
            "kernel_source": src_hash,
            "library": os.path.relpath(fqlib._lib.LIB_PATH, ROOT),
        }
        print(json.dumps(line), flush=True)
    fq.close()
    if world > 1:
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    rank, world, local = dist_env()
    if args.gpus != world and world > 1:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args, rank, world)
    return run_ours(args, rank, world, local)


if __name__ == "__main__":
    sys.exit(main())
