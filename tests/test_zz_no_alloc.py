"""fq_quantize_mx_static: the per-group entry point that allocates nothing.

Some callers cannot allocate device memory themselves (their memory belongs to another
allocator or a fixed budget, or a cudaMalloc would synchronize a latency-critical path).
This entry point keeps its only scratch, a status word, in a static device array of the
library. The test calls it through the C ABI twice in a row and checks that it writes the
same codes and scales as the allocating entry point (fq_quantize_mx through a handle),
which the parity tests hold to the oracle, and that fq_static_device_status reads the word
back as 0. A second test makes one launch's bounded wait run out (the process-wide
one-shot fq_static_debug_arm_stall; no fault, a 50 ms limit) and checks that the reader
reports it and that the next call is correct again. The file is collected last.
"""

import ctypes
import time

import pytest
import torch

from rotation_bit_quantization_token_b200 import FlatQuant, _lib
from rotation_bit_quantization_token_b200.workloads import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu


def _call_static(lib, x, P1, P2, D, out, sc):
    K, M, N = x.shape
    vp = ctypes.c_void_p
    dt = _lib.FQ_BF16 if x.dtype == torch.bfloat16 else _lib.FQ_FP16
    return lib.fq_quantize_mx_static(K, M, N, dt, vp(x.data_ptr()), vp(P1.data_ptr()),
                                     vp(P2.data_ptr()) if P2 is not None else vp(0), float(D),
                                     vp(out.data_ptr()), vp(sc.data_ptr()),
                                     vp(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("w", [
    WORKLOADS["mx_case3_32768x128x112"].with_tokens(371),   # tensor-core kernel
    WORKLOADS["mx_case2_16384x64x64"].with_tokens(741),     # tensor-core kernel, M = 64
    Workload("small", 37, 16, 16, "mx", "normal", dst_type_max=0.0),  # general kernel
], ids=lambda w: f"{w.K}x{w.M}x{w.N}")
def test_static_scratch_matches_allocating_entry_point(w):
    lib = _lib.load()
    dev = torch.device("cuda", 0)
    x, P1, P2 = (t.to(dev) for t in make_inputs(w, seed=3))
    ref_out, ref_sc = FlatQuant(w.K, w.M, w.N).quantize_mx(x, P1, P2, w.dst_type_max)
    torch.cuda.synchronize()
    for _ in range(2):  # two calls in a row share (and reuse) the static scratch
        out = torch.full_like(ref_out, 0xAB)
        sc = torch.full_like(ref_sc, 0xAB)
        assert _call_static(lib, x, P1, P2, w.dst_type_max, out, sc) == _lib.FQ_OK
        torch.cuda.synchronize()
        assert torch.equal(out, ref_out)
        assert torch.equal(sc, ref_sc)
        assert _static_status(lib) == (_lib.FQ_OK, 0)


def _static_status(lib):
    v = ctypes.c_uint32(0xFFFFFFFF)
    st = lib.fq_static_device_status(ctypes.byref(v))
    return st, int(v.value)


def test_static_path_reports_an_expired_wait():
    lib = _lib.load()
    dev = torch.device("cuda", 0)
    w = WORKLOADS["mx_case3_32768x128x112"].with_tokens(300)
    x, P1, P2 = (t.to(dev) for t in make_inputs(w, seed=7))
    ref_out, ref_sc = FlatQuant(w.K, w.M, w.N).quantize_mx(x, P1, P2, w.dst_type_max)
    out = torch.empty_like(ref_out)
    sc = torch.empty_like(ref_sc)
    torch.cuda.synchronize()
    assert _static_status(lib) == (_lib.FQ_OK, 0)
    assert lib.fq_static_debug_arm_stall(0.05) == _lib.FQ_OK
    t0 = time.monotonic()
    assert _call_static(lib, x, P1, P2, w.dst_type_max, out, sc) == _lib.FQ_OK
    torch.cuda.synchronize()
    elapsed = time.monotonic() - t0
    st, v = _static_status(lib)
    assert st == _lib.FQ_ERR_DEVICE_TIMEOUT and v != 0, (st, v)
    assert v & 2, f"stage A's wait for the x tile is not among the expired waits ({v:#x})"
    assert elapsed < 2.0
    assert _static_status(lib) == (_lib.FQ_OK, 0)  # the read cleared it
    # the hook is one-shot: the next call runs normally
    assert _call_static(lib, x, P1, P2, w.dst_type_max, out, sc) == _lib.FQ_OK
    torch.cuda.synchronize()
    assert _static_status(lib) == (_lib.FQ_OK, 0)
    assert torch.equal(out, ref_out) and torch.equal(sc, ref_sc)
    for bad in (0.0, -1.0, 11.0, float("nan")):
        assert lib.fq_static_debug_arm_stall(bad) == _lib.FQ_ERR_INVALID
    assert lib.fq_static_device_status(None) == _lib.FQ_ERR_NULLPTR


def test_static_entry_point_rejects_bad_arguments():
    lib = _lib.load()
    dev = torch.device("cuda", 0)
    x = torch.zeros((4, 16, 16), dtype=torch.bfloat16, device=dev)
    P = torch.eye(16, dtype=torch.bfloat16, device=dev)
    out = torch.empty((4, 128), dtype=torch.uint8, device=dev)
    sc = torch.empty((4, 4, 2), dtype=torch.uint8, device=dev)
    vp = ctypes.c_void_p
    s = vp(torch.cuda.current_stream().cuda_stream)
    args = (vp(x.data_ptr()), vp(P.data_ptr()), vp(P.data_ptr()))
    assert lib.fq_quantize_mx_static(4, 16, 16, 0, vp(0), args[1], args[2], 0.0,
                                     vp(out.data_ptr()), vp(sc.data_ptr()), s) == _lib.FQ_ERR_NULLPTR
    for K, M, N in [(0, 16, 16), (262145, 16, 16), (4, 257, 16), (4, 16, 15)]:
        assert lib.fq_quantize_mx_static(K, M, N, 0, *args, 0.0, vp(out.data_ptr()),
                                         vp(sc.data_ptr()), s) == _lib.FQ_ERR_INVALID
    assert lib.fq_quantize_mx_static(4, 16, 16, 0, *args, 5.0, vp(out.data_ptr()),
                                     vp(sc.data_ptr()), s) == _lib.FQ_ERR_INVALID
