"""GPU parity of the consumer contraction fq_mx_matmul against oracle.consumer.mx_matmul.

The page ("aclnnFlatQuantV2 complete guide: from two-level matmul to FP4 E2M1 quantization
fusion", http://www.zwxr.cn/news/277566, "per-token mode" and its summary) says the
operator's FP4 codes and scales are emitted for later dequantization and low-precision
compute. The oracle's reading of that compute is C[t, o] = sum_i A_hat[t, i] W_hat[o, i] over
the flattened M*N axis, each operand dequantized as e2m1(code) * 2^(byte - 127) per group of
32. Operands here are drawn on the host (seeded codes and scale bytes, or the oracle's own
quantization of a workload), never by the CUDA path.

Every product of two E2M1 values and two powers of two is exact, so the only difference the
kernel may show is its float32 accumulation: |C - C_ref| <= L * 2^-24 * sum_i |A_hat W_hat|.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle
from rotation_bit_quantization_token_b200 import _lib
from rotation_bit_quantization_token_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def _operand(rng, rows, L, lo=118, hi=136):
    """Random packed E2M1 codes [rows, L/2] and scale bytes [rows, ceilDiv(L, 64), 2]; the spare
    slot of an odd group count is 0x7F, as the operator writes it."""
    codes = rng.integers(0, 256, size=(rows, L // 2), dtype=np.uint8)
    G = L // 32
    S = -(-L // 64)
    sc = np.full((rows, 2 * S), 0x7F, dtype=np.uint8)
    sc[:, :G] = rng.integers(lo, hi + 1, size=(rows, G), dtype=np.uint8)
    return codes, sc.reshape(rows, S, 2)


def _abs_ref(a, sa, w, sw, L):
    """sum_i |A_hat[t, i] W_hat[o, i]| (the scale of the accumulation error bound)."""
    ca = oracle.unpack_nibbles(a, L) & 7
    cw = oracle.unpack_nibbles(w, L) & 7
    a2 = np.zeros_like(a)
    w2 = np.zeros_like(w)
    a2[:] = oracle.pack_nibbles(ca)
    w2[:] = oracle.pack_nibbles(cw)
    return oracle.mx_matmul(a2, sa, w2, sw, L)


def _run(a, sa, w, sw, T, O, L, stream=None):
    lib = _lib.load()
    dev = torch.device("cuda", 0)
    ad, sad = torch.from_numpy(a).to(dev), torch.from_numpy(np.ascontiguousarray(sa)).to(dev)
    wd, swd = torch.from_numpy(w).to(dev), torch.from_numpy(np.ascontiguousarray(sw)).to(dev)
    C = torch.full((T, O), float("nan"), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    vp = ctypes.c_void_p
    st = lib.fq_mx_matmul(T, O, L, vp(ad.data_ptr()), vp(sad.data_ptr()), vp(wd.data_ptr()),
                          vp(swd.data_ptr()), vp(C.data_ptr()), vp(status.data_ptr()),
                          vp(torch.cuda.current_stream().cuda_stream))
    assert st == _lib.FQ_OK, st
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return C.cpu().numpy().astype(np.float64)


def _check(C, ref, bound, L):
    tol = L * 2.0 ** -24 * bound + 1e-300
    err = np.abs(C - ref)
    assert np.all(np.isfinite(C))
    assert np.all(err <= tol), f"worst {float((err / tol).max())} of the bound"
    return float((err / tol).max())


# L = 32, 96, 320: scale rows of 2, 4, 10 bytes (read word by word); 1536, 2560: rows of 48
# and 80 bytes, whose last 16-byte piece of a wide read lies past the row
SHAPES = [(300, 520, 8192), (129, 257, 14336), (1, 1, 32), (5, 3, 96), (77, 300, 320),
          (256, 512, 4096), (130, 17, 2048), (70, 260, 1536), (33, 40, 2560)]


@pytest.mark.parametrize("T,O,L", SHAPES, ids=[f"{t}x{o}x{l}" for t, o, l in SHAPES])
def test_mx_matmul_matches_oracle_random_operands(T, O, L):
    rng = np.random.default_rng([T, O, L])
    a, sa = _operand(rng, T, L)
    w, sw = _operand(rng, O, L)
    C = _run(a, sa, w, sw, T, O, L)
    ref = oracle.mx_matmul(a, sa, w, sw, L)
    worst = _check(C, ref, _abs_ref(a, sa, w, sw, L), L)
    print(T, O, L, "worst/bound", worst)


@pytest.mark.parametrize("name,T,O", [("mx_case1_8192x64x128", 136, 264), ("mx_case3_32768x128x112", 140, 300)])
def test_mx_matmul_on_operator_outputs(name, T, O):
    """Operands quantized by the oracle from the workload's own inputs (C3 / C5 shaped: L =
    8192 and 14336): activations from x, weights from a second draw of the same workload."""
    w_ = WORKLOADS[name]
    L = w_.M * w_.N
    f64 = lambda t: t.float().numpy().astype(np.float64)  # noqa: E731
    xa, P1, P2 = make_inputs(w_.with_tokens(T), seed=11)
    xw, _, _ = make_inputs(w_.with_tokens(O), seed=12)
    a, sa, _ = oracle.flat_quant_mx(f64(xa), f64(P1), f64(P2), w_.dst_type_max)
    w, sw, _ = oracle.flat_quant_mx(f64(xw), f64(P1), f64(P2), w_.dst_type_max)
    C = _run(a, sa, w, sw, T, O, L)
    ref = oracle.mx_matmul(a, sa, w, sw, L)
    _check(C, ref, _abs_ref(a, sa, w, sw, L), L)


def test_mx_matmul_one_hot_and_scale_shift():
    """A one-hot weight row (code 1.0 at element j, scale byte 127) returns column j of
    A_hat exactly; adding k to every scale byte of A multiplies C by 2^k exactly."""
    rng = np.random.default_rng(5)
    T, L = 140, 512
    a, sa = _operand(rng, T, L)
    cols = [0, 31, 32, 255, 256, 511]
    O = len(cols)
    codes = np.zeros((O, L), dtype=np.uint8)
    for o, j in enumerate(cols):
        codes[o, j] = 0x2  # E2M1 1.0
    w = oracle.pack_nibbles(codes)
    sw = np.full((O, L // 64, 2), 127, dtype=np.uint8)
    C = _run(a, sa, w, sw, T, O, L)
    a_hat = oracle.dequantize_mx(a, sa, 1, L).reshape(T, L)
    np.testing.assert_array_equal(C, a_hat[:, cols])
    sa2 = (sa.astype(np.int64) + 3).astype(np.uint8)
    C2 = _run(a, sa2, w, sw, T, O, L)
    np.testing.assert_array_equal(C2, C * 8.0)


def test_mx_matmul_rejects_bad_arguments():
    lib = _lib.load()
    dev = torch.device("cuda", 0)
    buf = torch.zeros(1 << 16, dtype=torch.uint8, device=dev)
    C = torch.zeros(64, dtype=torch.float32, device=dev)
    vp = ctypes.c_void_p
    p = vp(buf.data_ptr())
    s = vp(torch.cuda.current_stream().cuda_stream)
    assert lib.fq_mx_matmul(4, 4, 64, vp(0), p, p, p, vp(C.data_ptr()), vp(0), s) == _lib.FQ_ERR_NULLPTR
    for T, O, L in [(0, 4, 64), (4, 0, 64), (4, 4, 48), (4, 4, 0), (4, 4, 65568), (262145, 4, 64)]:
        assert lib.fq_mx_matmul(T, O, L, p, p, p, p, vp(C.data_ptr()), vp(0), s) == _lib.FQ_ERR_INVALID
    assert lib.fq_mx_matmul(4, 4, 64, vp(buf.data_ptr() + 8), p, p, p, vp(C.data_ptr()), vp(0), s) \
        == _lib.FQ_ERR_INVALID


def test_mx_matmul_full_size_sampled():
    """The consumer contraction at the size bench.py times (T = 8192, O = 4096, L = 14336:
    the row length of the 128x112 workload), operands drawn on the host; a sampled block of
    C (random rows and columns plus the first, the last and those beside tile edges) against
    the oracle's contraction of just those rows."""
    T, O, L = 8192, 4096, 14336
    rng = np.random.default_rng([T, O, L, 1])
    a, sa = _operand(rng, T, L, lo=120, hi=133)
    w, sw = _operand(rng, O, L, lo=120, hi=133)
    C = _run(a, sa, w, sw, T, O, L)
    ts = np.unique(np.concatenate([rng.choice(T, 20, replace=False), [0, 127, 128, T - 1]]))
    os_ = np.unique(np.concatenate([rng.choice(O, 20, replace=False), [0, 255, 256, O - 1]]))
    ref = oracle.mx_matmul(a[ts], sa[ts], w[os_], sw[os_], L)
    worst = _check(C[np.ix_(ts, os_)], ref, _abs_ref(a[ts], sa[ts], w[os_], sw[os_], L), L)
    print("full size sampled, worst/bound", worst)
