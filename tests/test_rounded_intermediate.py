"""Intermediate-rounding mode (fq_set_intermediate_rounding) against the oracle.

The page's "How it works" gives x' = x . kroneckerP2 and x'' = kroneckerP1 . x' without
saying whether x' is kept in the input type in between. The default path keeps it exact.
This mode stores it in the 16-bit input type. The oracle (`oracle.rotate_rounded`) defines
it from the page alone: x' = round16(exact x . P2), nearest with ties to even, and assumes
no summation order.

Two kinds of test:
* inputs on an integer grid (x = k / 8 with |k| <= 127, P2 = j / 16 with |j| <= 15), where
  every partial sum of x . P2 is a multiple of 2^-7 below 2^11 in magnitude (18 significant
  bits at most) and so exact in float32 in any order: the
  kernel's x' must then be the oracle's x' exactly, ties included, and x'' and the codes
  follow the tolerance of every other parity test;
* the seeded workloads, where a float32 sum may fall on the other side of a 16-bit rounding
  midpoint than the exact value: every x' element whose exact value lies within the
  worst-case float32 accumulation bound N * 2^-24 * sum_j |x_j P2_jn| of a midpoint is marked,
  and the x'' elements, groups and tokens it can move are exempt (at most 0.01% of the
  compared elements may differ at all).
The mode runs the general kernel only.
"""

import numpy as np
import pytest
import torch

import oracle
from parity_util import (compare_mx, compare_per_token, intermediate_rounding_taint,
                         rotate_close, token_taint_from)
from rotation_bit_quantization_token_b200 import FlatQuant, FQError, _lib
from rotation_bit_quantization_token_b200.workloads import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def _check(w, dtype, x, P1, P2, taint):
    """Runs the mode on the GPU and compares x'', codes and scales with the oracle. With
    taint, the values the inputs do not decide are exempt. Returns the comparison stats."""
    dev = torch.device("cuda", 0)
    xd, P1d, P2d = x.to(dev), P1.to(dev), P2.to(dev)
    tag = "bf16" if dtype == torch.bfloat16 else "fp16"
    xs, p1, p2 = _f64(x), _f64(P1), _f64(P2)
    fq = FlatQuant(w.K, w.M, w.N, dtype)
    fq.set_intermediate_rounding(True)
    ref = oracle.rotate_rounded(xs, p1, p2, tag)
    if taint:
        dev_x2, x1_taint = intermediate_rounding_taint(xs, p1, p2, tag)
    else:
        dev_x2, x1_taint = np.zeros_like(ref), np.zeros(ref.shape, dtype=bool)
    elem_taint = (dev_x2 > 0).reshape(w.K, -1)

    x2 = fq.debug_rotate(xd, P1d, P2d)
    torch.cuda.synchronize()
    assert fq.last_kernel == "general"
    rotate_close(x2.cpu().numpy(), ref, extra=dev_x2)
    assert not np.array_equal(ref, oracle.rotate(xs, p1, p2))

    if w.mode == "per_token":
        out, qs = fq.quantize_per_token(xd, P1d, P2d, w.clip_ratio, w.out)
        torch.cuda.synchronize()
        codes, rqs, v = oracle.per_token_quantize(ref, w.clip_ratio)
        tok = token_taint_from(dev_x2, ref) if taint else None
        stats = compare_per_token(out.cpu().numpy().reshape(w.K, -1).view(np.uint8), qs.cpu().numpy(),
                                  codes, rqs, v, elem_taint=elem_taint, token_taint=tok)
        stats["tokens_skipped"] = int(tok.sum()) if tok is not None else 0
    else:
        out, sc = fq.quantize_mx(xd, P1d, P2d, w.dst_type_max)
        torch.cuda.synchronize()
        _, _, info = oracle.flat_quant_mx(xs, p1, p2, w.dst_type_max, intermediate=tag)
        stats = compare_mx(out.cpu().numpy(), sc.cpu().numpy(), info, w.dst_type_max,
                           elem_taint=elem_taint)
    assert fq.last_kernel == "general"
    stats["x1_marked"] = int(x1_taint.sum())
    stats["x2_elements_marked"] = int(elem_taint.sum())

    # switched off again, the handle is back on the exact path
    fq.set_intermediate_rounding(False)
    x2e = fq.debug_rotate(xd, P1d, P2d)
    torch.cuda.synchronize()
    rotate_close(x2e.cpu().numpy(), oracle.rotate(xs, p1, p2))
    return stats


def _grid_inputs(K, M, N, dtype, seed):
    """x = k / 8 and P2 = j / 16 with integers |k| <= 127, |j| <= 15; P1 random orthogonal."""
    rng = np.random.default_rng([seed, 17])
    x = rng.integers(-127, 128, size=(K, M, N)) / 8.0
    P2 = rng.integers(-15, 16, size=(N, N)) / 16.0
    q, r = np.linalg.qr(rng.standard_normal((M, M)))
    P1 = q * np.sign(np.diag(r))[None, :]
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dtype)  # noqa: E731
    return t(x), t(P1), t(P2)


GRID = [
    (Workload("grid", 16, 16, 16, "per_token", "normal", out="int4", clip_ratio=1.0), torch.bfloat16),
    (Workload("grid", 40, 64, 64, "per_token", "normal", out="int32", clip_ratio=0.9), torch.bfloat16),
    (Workload("grid", 24, 64, 128, "mx", "normal", dst_type_max=0.0), torch.bfloat16),
    (Workload("grid", 24, 64, 64, "mx", "normal", dst_type_max=6.0), torch.bfloat16),
    (Workload("grid", 12, 128, 112, "mx", "normal", dst_type_max=10.0), torch.bfloat16),
    (Workload("grid", 24, 32, 96, "mx", "normal", dst_type_max=7.0), torch.float16),
    (Workload("grid", 24, 64, 64, "per_token", "normal", out="int4", clip_ratio=0.9), torch.float16),
]


@pytest.mark.parametrize("w,dtype", GRID, ids=[f"{w.K}x{w.M}x{w.N}-{w.mode}-{str(d)[6:]}" for w, d in GRID])
def test_rounded_intermediate_exact_on_integer_grid(w, dtype):
    x, P1, P2 = _grid_inputs(w.K, w.M, w.N, dtype, seed=w.K + w.M + w.N)
    stats = _check(w, dtype, x, P1, P2, taint=False)
    print(w.name, w.K, w.M, w.N, stats)


CASES = [
    (WORKLOADS["per_token_int32_4096x64x64"].with_tokens(96), torch.bfloat16),
    (WORKLOADS["mx_case1_8192x64x128"].with_tokens(48), torch.bfloat16),
    (WORKLOADS["mx_case2_16384x64x64"].with_tokens(96), torch.bfloat16),
    (WORKLOADS["mx_case3_32768x128x112"].with_tokens(40), torch.bfloat16),
    (WORKLOADS["per_token_int4_16x16x16"], torch.bfloat16),
    (Workload("fp16", 24, 32, 96, "mx", "normal_outliers", dst_type_max=6.0), torch.float16),
    (Workload("fp16", 24, 64, 64, "per_token", "normal", out="int4", clip_ratio=0.9), torch.float16),
]


@pytest.mark.parametrize("w,dtype", CASES, ids=[f"{w.name}-{str(d)[6:]}" for w, d in CASES])
def test_rounded_intermediate_matches_oracle(w, dtype):
    x, P1, P2 = make_inputs(w, seed=5, dtype=dtype)
    stats = _check(w, dtype, x, P1, P2, taint=True)
    print(w.name, stats)


def test_rounded_intermediate_is_general_kernel_only():
    dev = torch.device("cuda", 0)
    w = WORKLOADS["mx_case3_32768x128x112"].with_tokens(8)
    x, P1, P2 = (t.to(dev) for t in make_inputs(w, seed=2))
    fq = FlatQuant(w.K, w.M, w.N, kernel="tcgen05")
    fq.set_intermediate_rounding(True)
    with pytest.raises(FQError) as e:
        fq.quantize_mx(x, P1, P2, w.dst_type_max)
    assert e.value.status == _lib.FQ_ERR_UNSUPPORTED
    lib = _lib.load()
    assert lib.fq_set_intermediate_rounding(fq._h, 2) == _lib.FQ_ERR_INVALID
    fq.set_intermediate_rounding(False)
    fq.quantize_mx(x, P1, P2, w.dst_type_max)
    torch.cuda.synchronize()
    assert fq.last_kernel == "tcgen05"
