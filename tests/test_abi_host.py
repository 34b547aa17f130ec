"""Host-side tests that need no GPU: the C ABI library loads and exports every symbol of
include/fq.h, plan-phase validation returns the page's codes, the workloads are seeded
and shaped as stated, and bench.py's host logic (sharding, max over ranks, clock parsing)
works, including with two gloo ranks."""

import ctypes
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from rotation_bit_quantization_token_b200 import build as b
    b.build()
    from rotation_bit_quantization_token_b200 import _lib
    return _lib.load()


def test_every_declared_symbol_is_exported(lib):
    from rotation_bit_quantization_token_b200 import _lib
    names = _lib.declared_symbols()
    assert len(names) >= 11
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert hasattr(lib, n)


_C_PROGRAM = r"""
#include <stdio.h>
#include "fq.h"
int main(void) {
  fq_handle *h = 0;
  int bad = 0;
  /* calls that the library answers from its argument checks, before any CUDA call */
  bad |= fq_create(0, 4, 16, 16, FQ_BF16) != FQ_ERR_NULLPTR;
  bad |= fq_create(&h, 0, 16, 16, FQ_BF16) != FQ_ERR_INVALID;
  bad |= fq_quantize_mx(0, 0, 0, 0, 0.0, 0, 0, 0) != FQ_ERR_NULLPTR;
  bad |= fq_set_intermediate_rounding(0, 1) != FQ_ERR_NULLPTR;
  bad |= fq_destroy(0) != FQ_OK;
  printf("%s\n", fq_status_string(FQ_ERR_INVALID));
  return bad;
}
"""


def test_c_program_builds_and_calls_the_abi(lib, tmp_path):
    """The header is plain C: a C99 program (gcc -pedantic, no CUDA headers) includes it,
    links against libfq.so and gets the documented status codes back."""
    from rotation_bit_quantization_token_b200 import _lib
    src = tmp_path / "abi.c"
    src.write_text(_C_PROGRAM)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(_lib.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", libdir, "-lfq", f"-Wl,-rpath,{libdir}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert r.stdout.startswith("FQ_ERR_INVALID")


def test_library_is_built_for_sm100a_only():
    """The build compiles every source for sm_100a alone: one -gencode pair, compute_100a
    to sm_100a, for the objects and for the link (no PTX for other targets)."""
    from rotation_bit_quantization_token_b200 import build
    flags = build.NVCC_FLAGS
    pairs = [flags[i + 1] for i, f in enumerate(flags) if f == "-gencode"]
    assert pairs == ["arch=compute_100a,code=sm_100a"]
    assert not any(f.startswith("-arch") or f.startswith("--gpu-architecture") for f in flags)


def test_plan_validation_without_device(lib):
    from rotation_bit_quantization_token_b200 import _lib
    h = ctypes.c_void_p()
    assert lib.fq_create(None, 4, 16, 16, 0) == _lib.FQ_ERR_NULLPTR
    bad = [(0, 16, 16), (262145, 16, 16), (4, 0, 16), (4, 257, 16), (4, 16, 0), (4, 16, 257)]
    for K, M, N in bad:
        assert lib.fq_create(ctypes.byref(h), K, M, N, 0) == _lib.FQ_ERR_INVALID
    assert lib.fq_create(ctypes.byref(h), 4, 16, 16, 7) == _lib.FQ_ERR_INVALID
    # calls on a NULL handle
    assert lib.fq_quantize_mx(None, None, None, None, 0.0, None, None, None) == _lib.FQ_ERR_NULLPTR
    assert lib.fq_quantize_per_token(None, None, None, None, 1.0, 0, None, None, None) == _lib.FQ_ERR_NULLPTR
    assert lib.fq_destroy(None) == _lib.FQ_OK
    assert lib.fq_last_kernel(None) == 0
    assert lib.fq_set_intermediate_rounding(None, 1) == _lib.FQ_ERR_NULLPTR
    for code in (0, 161001, 161002, 161003, 161004, 161005):
        assert lib.fq_status_string(code).decode().startswith("FQ_")


def test_workloads_seeded_and_shaped():
    from rotation_bit_quantization_token_b200.workloads import WORKLOADS, make_inputs, draw_x
    w = WORKLOADS["per_token_int32_4096x64x64"].with_tokens(64)
    x1, P1, P2 = make_inputs(w, seed=0)
    x2, _, _ = make_inputs(w, seed=0)
    assert x1.dtype == torch.bfloat16 and tuple(x1.shape) == (64, 64, 64)
    assert torch.equal(x1, x2)
    # random orthogonal P, rounded to bf16: P P^T close to I
    p = P1.double().numpy()
    assert np.abs(p @ p.T - np.eye(64)).max() < 2e-2
    # outlier positions: ~1% of feature positions carry x20
    xs = np.abs(draw_x(w, 0)).reshape(64, -1).mean(axis=0)
    big = xs > 5 * np.median(xs)
    assert abs(int(big.sum()) - 41) <= 2
    w5 = WORKLOADS["mx_case3_32768x128x112"].with_tokens(16)
    x5 = np.abs(draw_x(w5, 0)).reshape(16, -1).mean(axis=0)
    assert int((x5 > 10 * np.median(x5)).sum()) == 8
    w3 = WORKLOADS["mx_case1_8192x64x128"].with_tokens(64)
    x3 = draw_x(w3, 0)
    assert 0.002 < float((np.abs(x3) > 6).mean()) < 0.01


def test_workload_byte_counts():
    from rotation_bit_quantization_token_b200.workloads import WORKLOADS
    w = WORKLOADS["mx_case3_32768x128x112"]
    assert w.bytes_per_token() == 28672 + 7168 + 448
    assert w.flops_per_token() == 2 * (128 * 112 * 112 + 128 * 128 * 112)
    w2 = WORKLOADS["per_token_int32_4096x64x64"]
    assert w2.bytes_per_token() == 8192 + 2048 + 4


def test_bench_host_helpers():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.rank_seed(3) == 3
    text = ("0, 1800, 1965, 700.5, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n"
            "0, 1900, 1965, 800.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n")
    c = bench.parse_clock_samples(text)
    assert c["sm_mhz"] == 1850.0 and c["sm_max_mhz"] == 1965.0 and c["reasons"] == ["sw_power_cap"]
    assert bench.parse_clock_samples("") is None
    hb, tf, src = bench.load_peaks()
    assert hb > 1000 and tf > 100
    assert len(bench.kernel_source_hash()) == 16
    assert bench.recorded_traffic("nope", "nope", "0") is None


def test_bench_reference_arm_json_contract():
    """`bench.py --impl reference` (the oracle timed on the host cores) prints one JSON line
    with the keys and types the launcher reads, on the same metric and workload as the
    CUDA arm. Runs on CPU: the reference arm needs no GPU."""
    import json
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True,
                       timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    for key, typ in [("metric", str), ("value", float), ("unit", str), ("n_gpus", int),
                     ("steps", int), ("warmup", int), ("ms_per_step", float),
                     ("higher_is_better", bool), ("scaling", str), ("dtype", str),
                     ("data", str), ("config", dict), ("cpu_baseline", dict), ("e2e", dict)]:
        assert isinstance(d[key], typ), (key, d.get(key))
    assert d["impl"] == "reference" and d["vs_baseline"] is None
    assert d["value"] > 0 and d["steps"] == 1 and d["n_gpus"] == 1
    assert d["config"]["workload"] == "mx_case3_32768x128x112"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    # it reports what it timed: the per-step time of its sample, not an extrapolation to
    # the whole workload, so the steps fit in the run
    n = d["config"]["tokens_per_step_sample"]
    assert 1 <= n <= d["config"]["K"]
    assert abs(d["value"] - n / (d["ms_per_step"] / 1e3)) <= 1e-6 * d["value"]
    assert d["cpu_baseline"]["nproc"] >= d["cpu_baseline"]["usable_cores"] >= 1


def test_bench_buffer_copies_exceed_l2():
    """Workloads smaller than twice the L2 cycle through enough copies to exceed it."""
    sys.path.insert(0, ROOT)
    import bench
    from rotation_bit_quantization_token_b200.workloads import WORKLOADS
    assert bench.buffer_copies(WORKLOADS["mx_case3_32768x128x112"].bytes_per_token() * 32768) == 1
    for name in WORKLOADS:
        b = WORKLOADS[name].bytes_per_token() * WORKLOADS[name].K
        c = bench.buffer_copies(b)
        assert c * b > 2 * bench.L2_BYTES
        assert c == 1 or (c - 1) * b <= 2 * bench.L2_BYTES + b


_GLOO_SCRIPT = r"""
import os, sys
sys.path.insert(0, {root!r})
import torch.distributed as dist
import bench
dist.init_process_group("gloo", rank=int(os.environ["RANK"]), world_size=int(os.environ["WORLD_SIZE"]))
r, w, l = bench.dist_env()
v = bench.max_over_ranks(10.0 + r, w)
assert v == 10.0 + (w - 1), v
assert bench.rank_seed(r) == r
print("ok", r, v)
dist.destroy_process_group()
"""


def test_bench_max_over_ranks_two_gloo_ranks(tmp_path):
    script = tmp_path / "gloo_ranks.py"
    script.write_text(_GLOO_SCRIPT.format(root=ROOT))
    procs = []
    port = 29500 + (os.getpid() % 1000)
    for r in range(2):
        env = dict(os.environ, RANK=str(r), WORLD_SIZE="2", LOCAL_RANK=str(r),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, str(script)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True))
    outs = [p.communicate(timeout=120)[0] for p in procs]
    for p, o in zip(procs, outs):
        assert p.returncode == 0, o
        assert "ok" in o


def test_output_buffer_checks_on_host():
    """Caller-supplied outputs are refused before any launch unless they sit on the
    input's device, are contiguous, hold exactly the bytes the kernel writes, and (for
    numeric outputs) have the right dtype; an undersized buffer would otherwise be
    overrun on the GPU. Checked here on CPU tensors, with the CPU as the device."""
    from rotation_bit_quantization_token_b200 import api

    cpu = torch.device("cpu")
    K, M, N = 3, 4, 16
    api._check_output("out", torch.empty((K, M * N // 2), dtype=torch.uint8), K * M * N // 2, cpu)
    api._check_output("out", torch.empty((K, M, N // 8), dtype=torch.int32), K * M * N // 2, cpu)
    api._check_output("scales", torch.empty((K, 1, 2), dtype=torch.uint8), api._scale_bytes(K, M, N), cpu)
    api._check_output("quant_scale", torch.empty(K, dtype=torch.float32), 4 * K, cpu, torch.float32)
    bad = [
        (torch.empty((K, M * N // 2 - 1), dtype=torch.uint8), K * M * N // 2, None, "bytes"),
        (torch.empty((M * N // 2, K), dtype=torch.uint8).t(), K * M * N // 2, None, "contiguous"),
        (torch.empty(K, dtype=torch.float16), 4 * K, torch.float32, "dtype"),
        ([0] * K, 4 * K, None, "Tensor"),
    ]
    for t, nbytes, dtype, word in bad:
        with pytest.raises((ValueError, TypeError), match=word):
            api._check_output("buf", t, nbytes, cpu, dtype)
    # scale tensor of an odd group count: [K, ceilDiv(M*N, 64), 2] includes the spare slot
    assert api._scale_bytes(2, 3, 32) == 2 * 2 * 2
