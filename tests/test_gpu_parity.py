"""CUDA path vs the CPU oracle, element by element, through the C ABI (libfq.so).

Every test here needs a B200 (sm_100a). The tolerance is the one stated in
tests/parity_util.py. Sizes: each workload at a reduced token count that the oracle
finishes in seconds (several 128-row tiles plus a ragged tail), and at its full size in
the launch configuration bench.py times, compared on sampled tokens.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle
from parity_util import compare_mx, compare_per_token, rotate_close, unpack_nibbles
from rotation_bit_quantization_token_b200 import FlatQuant, FQError, HostPipeline, _lib
from rotation_bit_quantization_token_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

NAMES = list(WORKLOADS)


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def _kernels_for(w):
    ks = ["general"]
    probe = FlatQuant(w.K, w.M, w.N)
    try:
        probe.set_kernel("tcgen05")
        ks.append("tcgen05")
    except FQError:
        pass
    probe.close()
    return ks


def _run_and_compare(w, x, P1, P2, kernel, tokens=None):
    """Run the CUDA path on (x, P1, P2) and compare the listed tokens with the oracle."""
    dev = torch.device("cuda", 0)
    xd, P1d = x.to(dev), P1.to(dev)
    P2d = P2.to(dev) if P2 is not None else None
    fq = FlatQuant(w.K, w.M, w.N, x.dtype, kernel=kernel)
    idx = np.arange(w.K) if tokens is None else np.asarray(tokens)
    xs = _f64(x[torch.as_tensor(idx)])
    p1, p2 = _f64(P1), (_f64(P2) if P2 is not None else None)
    if w.mode == "per_token":
        out, qs = fq.quantize_per_token(xd, P1d, P2d, w.clip_ratio, w.out)
        torch.cuda.synchronize()
        assert fq.last_kernel == kernel
        out_b = out.cpu().numpy().reshape(w.K, -1).view(np.uint8)[idx]
        codes, rqs, v = oracle.per_token_quantize(oracle.rotate(xs, p1, p2), w.clip_ratio)
        stats = compare_per_token(out_b, qs.cpu().numpy()[idx], codes, rqs, v)
    else:
        out, sc = fq.quantize_mx(xd, P1d, P2d, w.dst_type_max)
        torch.cuda.synchronize()
        assert fq.last_kernel == kernel
        _, _, info = oracle.flat_quant_mx(xs, p1, p2, w.dst_type_max)
        stats = compare_mx(out.cpu().numpy()[idx], sc.cpu().numpy()[idx], info, w.dst_type_max)
    assert fq.device_status() == 0
    return stats


@pytest.mark.parametrize("name", NAMES)
def test_workload_reduced_all_kernels(name):
    w = WORKLOADS[name]
    # about 2.5 tiles of 128 rows per SM (148 SMs), so every CTA runs its pipeline over
    # several tiles, plus a ragged last tile when M = 64
    w = w.with_tokens(min(w.K, 741 if w.M <= 64 else 371))
    x, P1, P2 = make_inputs(w, seed=0)
    for kernel in _kernels_for(w):
        stats = _run_and_compare(w, x, P1, P2, kernel)
        print(name, kernel, stats)


@pytest.mark.parametrize("name", NAMES)
def test_workload_rotation_all_kernels(name):
    w = WORKLOADS[name]
    w = w.with_tokens(min(w.K, 64))
    x, P1, P2 = make_inputs(w, seed=0)
    ref = oracle.rotate(_f64(x), _f64(P1), _f64(P2))
    for kernel in _kernels_for(w):
        fq = FlatQuant(w.K, w.M, w.N, kernel=kernel)
        x2 = fq.debug_rotate(x.cuda(), P1.cuda(), P2.cuda()).cpu().numpy()
        worst = rotate_close(x2, ref)
        print(name, kernel, "max |dx''| / rms:", worst)
        assert worst < 1e-5


@pytest.mark.parametrize("name", NAMES)
def test_workload_full_size_sampled(name):
    """Full token count, the kernel AUTO picks (the one bench.py times), sampled tokens."""
    w = WORKLOADS[name]
    x, P1, P2 = make_inputs(w, seed=0)
    rng = np.random.default_rng(99)
    idx = np.unique(np.concatenate([np.arange(min(8, w.K)), np.arange(max(w.K - 8, 0), w.K),
                                    rng.integers(0, w.K, 48)]))
    kernel = "tcgen05" if "tcgen05" in _kernels_for(w) else "general"  # what AUTO picks
    stats = _run_and_compare(w, x, P1, P2, kernel, tokens=idx)
    print(name, kernel, stats)


def test_host_example_fp16_closed_form():
    """The page's complete example: ones fp16 [16,16,16], ones P1/P2, clipRatio 1, INT32.
    Every word is 0x77777777 and quantScale is fp32(256/7)."""
    dev = torch.device("cuda", 0)
    x = torch.ones((16, 16, 16), dtype=torch.float16, device=dev)
    P = torch.ones((16, 16), dtype=torch.float16, device=dev)
    fq = FlatQuant(16, 16, 16, torch.float16)
    out, qs = fq.quantize_per_token(x, P, P, 1.0, "int32")
    assert out.shape == (16, 16, 2)
    assert torch.all(out.cpu() == 2004318071)
    assert np.all(qs.cpu().numpy().view(np.uint32) == 0x42124925)


@pytest.mark.parametrize("shape", [(1, 16, 16), (3, 3, 14), (5, 1, 96), (4, 17, 2),
                                   (6, 48, 40), (3, 256, 256), (9, 64, 64), (5, 128, 112),
                                   (3, 32, 64), (7, 64, 80), (4, 32, 96), (3, 128, 128),
                                   (5, 128, 64), (6, 32, 128), (2, 64, 96), (4, 128, 80)])
@pytest.mark.parametrize("mode", ["per_token", "mx0", "mx6", "mx7", "mx10"])
def test_edge_shapes(shape, mode):
    K, M, N = shape
    from rotation_bit_quantization_token_b200.workloads import Workload
    if mode == "per_token":
        w = Workload("edge", K, M, N, "per_token", "normal", out="int4", clip_ratio=0.85)
    else:
        w = Workload("edge", K, M, N, "mx", "normal_outliers", dst_type_max=float(mode[2:]))
    x, P1, P2 = make_inputs(w, seed=K * 1000 + M * 10 + N)
    for kernel in _kernels_for(w):
        _run_and_compare(w, x, P1, P2, kernel)


@pytest.mark.parametrize("shape", [(741, 128, 80), (741, 128, 96), (1481, 64, 80),
                                   (2963, 32, 96), (1481, 64, 128)])
@pytest.mark.parametrize("mode", ["per_token", "mx6", "mx10"])
def test_multi_tile_other_widths(shape, mode):
    """The tensor-core widths no workload uses (N = 80, 96; M = 32 packing; N = 128 at
    M = 64), at about five 128-row tiles per SM plus a ragged tail, so every TMEM slot and
    ring stage is reused several times and, at N = 96, both stage-B issuer warps run."""
    K, M, N = shape
    from rotation_bit_quantization_token_b200.workloads import Workload
    if mode == "per_token":
        w = Workload("multi", K, M, N, "per_token", "normal", out="int4", clip_ratio=0.9)
    else:
        w = Workload("multi", K, M, N, "mx", "normal_outliers", dst_type_max=float(mode[2:]))
    x, P1, P2 = make_inputs(w, seed=K + M + N)
    kernels = _kernels_for(w)
    assert "tcgen05" in kernels
    _run_and_compare(w, x, P1, P2, "tcgen05")


@pytest.mark.parametrize("shape", [(5, 128, 112), (7, 64, 64), (3, 32, 96)])
@pytest.mark.parametrize("mode", ["per_token", "mx10"])
def test_fp16_inputs_tensor_core_shapes(shape, mode):
    # fp16 x, P1, P2 (the page's second input type) on the shapes the tensor-core kernel takes
    K, M, N = shape
    from rotation_bit_quantization_token_b200.workloads import Workload
    if mode == "per_token":
        w = Workload("fp16", K, M, N, "per_token", "normal", out="int4", clip_ratio=1.0)
    else:
        w = Workload("fp16", K, M, N, "mx", "normal_outliers", dst_type_max=10.0)
    x, P1, P2 = make_inputs(w, seed=11, dtype=torch.float16)
    assert x.dtype == torch.float16
    for kernel in _kernels_for(w):
        _run_and_compare(w, x, P1, P2, kernel)


@pytest.mark.parametrize("dst", [0.0, 6.0, 10.0])
def test_identity_rotation_is_plain_mx(dst):
    from rotation_bit_quantization_token_b200.workloads import Workload
    w = Workload("id", 33, 64, 64, "mx", "laplace_gain", dst_type_max=dst)
    x, _, _ = make_inputs(w, seed=5)
    I1 = torch.eye(64, dtype=torch.bfloat16)
    for kernel in _kernels_for(w):
        _run_and_compare(w, x, I1, I1, kernel)


def test_skip_right_multiply():
    from rotation_bit_quantization_token_b200.workloads import Workload
    for (M, N) in [(64, 64), (16, 16), (128, 112)]:
        w = Workload("skip", 19, M, N, "mx", "normal", dst_type_max=0.0)
        x, P1, _ = make_inputs(w, seed=6)
        for kernel in _kernels_for(w):
            _run_and_compare(w, x, P1, None, kernel)


def test_zero_input():
    dev = torch.device("cuda", 0)
    for (M, N) in [(16, 16), (64, 64), (128, 112)]:
        x = torch.zeros((5, M, N), dtype=torch.bfloat16, device=dev)
        P1 = torch.eye(M, dtype=torch.bfloat16, device=dev)
        P2 = torch.eye(N, dtype=torch.bfloat16, device=dev)
        fq = FlatQuant(5, M, N)
        for kernel in _kernels_for(fq):
            fq.set_kernel(kernel)
            out, qs = fq.quantize_per_token(x, P1, P2, 1.0)
            assert torch.all(out == 0) and torch.all(qs == 0)
            for d in (0.0, 6.0, 7.0, 10.0):
                out, sc = fq.quantize_mx(x, P1, P2, d)
                assert torch.all(out == 0) and torch.all(sc == 0)


def test_deterministic_and_int32_same_bytes():
    w = WORKLOADS["per_token_int32_4096x64x64"].with_tokens(300)
    x, P1, P2 = (t.cuda() for t in make_inputs(w, seed=1))
    fq = FlatQuant(w.K, w.M, w.N)
    for kernel in _kernels_for(w):
        fq.set_kernel(kernel)
        a, qa = fq.quantize_per_token(x, P1, P2, 0.9, "int32")
        b, qb = fq.quantize_per_token(x, P1, P2, 0.9, "int4")
        assert torch.equal(a.cpu().view(torch.uint8).reshape(w.K, -1), b.cpu())
        assert torch.equal(qa, qb)
        c, _ = fq.quantize_per_token(x, P1, P2, 0.9, "int32")
        assert torch.equal(a, c)
        m1 = fq.quantize_mx(x, P1, P2, 10.0)
        m2 = fq.quantize_mx(x, P1, P2, 10.0)
        assert torch.equal(m1[0], m2[0]) and torch.equal(m1[1], m2[1])


@pytest.mark.parametrize("name,K", [("mx_case3_32768x128x112", 512), ("per_token_int32_4096x64x64", 256)])
def test_host_pipeline_chunks_match_device_call(name, K):
    # the chunked three-stream pipeline from pinned host memory gives the bytes of one
    # device call, also on a second step that reuses its buffers
    w = WORKLOADS[name].with_tokens(K)
    x, P1, P2 = make_inputs(w, seed=5)
    fq = FlatQuant(w.K, w.M, w.N)
    xd, P1d, P2d = x.cuda(), P1.cuda(), P2.cuda()
    if w.mode == "mx":
        ref = fq.quantize_mx(xd, P1d, P2d, w.dst_type_max)
    else:
        ref = fq.quantize_per_token(xd, P1d, P2d, w.clip_ratio, w.out)
    for chunks in (8, 1):
        pipe = HostPipeline(fq, w.mode, w.out if w.mode == "per_token" else "int4", chunks=chunks)
        oh, sh = pipe.host_outputs()
        for _ in range(2):
            oh.zero_()
            sh.zero_()
            pipe.run(x.pin_memory(), P1.pin_memory(), P2.pin_memory(), oh, sh,
                     clip_ratio=w.clip_ratio, dst_type_max=w.dst_type_max)
            torch.cuda.synchronize()
            assert torch.equal(oh, ref[0].cpu()) and torch.equal(sh, ref[1].cpu())


@pytest.mark.parametrize("name", NAMES)
def test_full_size_repeatable(name):
    # ten launches at the full size give the same bytes: the pipeline's barriers leave no
    # room for a race to change the result from one run to the next
    w = WORKLOADS[name]
    x, P1, P2 = (t.cuda() for t in make_inputs(w, seed=3))
    fq = FlatQuant(w.K, w.M, w.N)
    if w.mode == "mx":
        run = lambda: fq.quantize_mx(x, P1, P2, w.dst_type_max)  # noqa: E731
    else:
        run = lambda: fq.quantize_per_token(x, P1, P2, w.clip_ratio, w.out)  # noqa: E731
    ref = [t.clone() for t in run()]
    for _ in range(10):
        out = run()
        assert torch.equal(out[0], ref[0]) and torch.equal(out[1], ref[1])
    torch.cuda.synchronize()
    assert fq.device_status() == 0


def test_invalid_arguments_return_page_codes():
    dev = torch.device("cuda", 0)
    lib = _lib.load()
    x = torch.zeros((4, 16, 16), dtype=torch.bfloat16, device=dev)
    P = torch.eye(16, dtype=torch.bfloat16, device=dev)
    fq = FlatQuant(4, 16, 16)
    for clip in (0.0, -0.5, 1.5, float("nan")):
        with pytest.raises(FQError) as e:
            fq.quantize_per_token(x, P, P, clip)
        assert e.value.status == _lib.FQ_ERR_INVALID
    for d in (5.9, 12.5, -1.0, 3.0):
        with pytest.raises(FQError) as e:
            fq.quantize_mx(x, P, P, d)
        assert e.value.status == _lib.FQ_ERR_INVALID
    out = torch.empty(4 * 16 * 8, dtype=torch.uint8, device=dev)
    qs = torch.empty(4, dtype=torch.float32, device=dev)
    vp = ctypes.c_void_p
    h = fq._h
    s = vp(torch.cuda.current_stream().cuda_stream)
    assert lib.fq_quantize_per_token(h, vp(0), vp(P.data_ptr()), vp(P.data_ptr()), 1.0, 0,
                                     vp(out.data_ptr()), vp(qs.data_ptr()), s) == _lib.FQ_ERR_NULLPTR
    assert lib.fq_quantize_per_token(h, vp(x.data_ptr()), vp(P.data_ptr()), vp(0), 1.0, 0,
                                     vp(out.data_ptr()), vp(qs.data_ptr()), s) == _lib.FQ_ERR_NULLPTR
    assert lib.fq_quantize_mx(h, vp(x.data_ptr()), vp(P.data_ptr()), vp(0), 0.0,
                              vp(out.data_ptr()), vp(0), s) == _lib.FQ_ERR_NULLPTR
    assert lib.fq_quantize_per_token(h, vp(x.data_ptr()), vp(P.data_ptr()), vp(P.data_ptr()), 1.0, 7,
                                     vp(out.data_ptr()), vp(qs.data_ptr()), s) == _lib.FQ_ERR_INVALID
    # N odd (INT4 / FP4) and N % 8 != 0 (INT32)
    x_odd = torch.zeros((2, 4, 5), dtype=torch.bfloat16, device=dev)
    fq_odd = FlatQuant(2, 4, 5)
    with pytest.raises(FQError):
        fq_odd.quantize_per_token(x_odd, P[:4, :4].contiguous(), torch.eye(5, dtype=torch.bfloat16, device=dev))
    x6 = torch.zeros((2, 4, 6), dtype=torch.bfloat16, device=dev)
    fq6 = FlatQuant(2, 4, 6)
    with pytest.raises(FQError):
        fq6.quantize_per_token(x6, P[:4, :4].contiguous(), torch.eye(6, dtype=torch.bfloat16, device=dev),
                               1.0, "int32")
    torch.cuda.synchronize()
