"""Intermediate-rounding mode (fq_set_intermediate_rounding) against the oracle.

The page's "How it works" gives x' = x . kroneckerP2 and x'' = kroneckerP1 . x' without
saying whether x' is kept in the input type in between. The default path keeps it exact.
This mode stores it in the 16-bit input type: each x' element is summed in float32 in index
order and rounded to nearest even. That is `oracle.rotate_rounded`, which the general
kernel reproduces bit for bit, so x' agrees exactly and x'' and the codes follow the same
tolerance as every other parity test. The mode runs the general kernel only.
"""

import numpy as np
import pytest
import torch

import oracle
from parity_util import compare_mx, compare_per_token, rotate_close
from rotation_bit_quantization_token_b200 import FlatQuant, FQError, _lib
from rotation_bit_quantization_token_b200.workloads import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


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
    dev = torch.device("cuda", 0)
    x, P1, P2 = make_inputs(w, seed=5, dtype=dtype)
    xd, P1d, P2d = x.to(dev), P1.to(dev), P2.to(dev)
    tag = "bf16" if dtype == torch.bfloat16 else "fp16"
    xs, p1, p2 = _f64(x), _f64(P1), _f64(P2)
    fq = FlatQuant(w.K, w.M, w.N, dtype)
    fq.set_intermediate_rounding(True)

    # x'': the rounded path, and different from the exact one
    x2 = fq.debug_rotate(xd, P1d, P2d)
    torch.cuda.synchronize()
    assert fq.last_kernel == "general"
    ref = oracle.rotate_rounded(xs, p1, p2, tag)
    rotate_close(x2.cpu().numpy(), ref)
    assert not np.array_equal(ref, oracle.rotate(xs, p1, p2))

    if w.mode == "per_token":
        out, qs = fq.quantize_per_token(xd, P1d, P2d, w.clip_ratio, w.out)
        torch.cuda.synchronize()
        codes, rqs, v = oracle.per_token_quantize(ref, w.clip_ratio)
        stats = compare_per_token(out.cpu().numpy().reshape(w.K, -1).view(np.uint8), qs.cpu().numpy(),
                                  codes, rqs, v)
    else:
        out, sc = fq.quantize_mx(xd, P1d, P2d, w.dst_type_max)
        torch.cuda.synchronize()
        _, _, info = oracle.flat_quant_mx(xs, p1, p2, w.dst_type_max, intermediate=tag)
        stats = compare_mx(out.cpu().numpy(), sc.cpu().numpy(), info, w.dst_type_max)
    assert fq.last_kernel == "general"
    print(w.name, tag, stats)

    # switched off again, the handle is back on the exact path
    fq.set_intermediate_rounding(False)
    x2e = fq.debug_rotate(xd, P1d, P2d)
    torch.cuda.synchronize()
    rotate_close(x2e.cpu().numpy(), oracle.rotate(xs, p1, p2))


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
