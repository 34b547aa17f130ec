"""The largest shapes the boundary accepts, on the GPU, against the oracle on sampled tokens.

fq_create accepts K up to 262144 and M, N up to 256 ([FQ] parameter table, as the boundary
restates it). At K = 262144 and M = N = 256 one x holds 17.2 G elements (34 GB of bf16), past
2^31, so every index of both kernels has to be 64-bit; the tensor-core kernel at 128 x 128
runs 262144 tiles of 128 rows per launch (a TMA row coordinate up to 33.5 M).

x is drawn on the device by torch's seeded generator (N(0, 1) in bf16): generating 34 GB on
the host would take minutes. Only the sampled tokens travel back, and the oracle sees exactly
those inputs. P1 and P2 come from the shared seeded generator. Tokens checked: the first
four, the last four and sixteen drawn at random, under the tolerance of tests/parity_util.py.
"""

import numpy as np
import pytest
import torch

import oracle
from parity_util import compare_mx, compare_per_token
from rotation_bit_quantization_token_b200 import FlatQuant
from rotation_bit_quantization_token_b200.workloads import (STREAM_P1, STREAM_P2, random_orthogonal,
                                                            to_bf16)

pytestmark = pytest.mark.gpu

KMAX = 262144


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def _device_x(K, M, N, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    return torch.randn((K, M, N), generator=g, device="cuda", dtype=torch.bfloat16)


@pytest.mark.parametrize("M,N,kernel,mode,arg", [
    (256, 256, "general", "mx", 10.0),
    (256, 256, "general", "per_token", ("int32", 0.9)),
    (128, 128, "tcgen05", "mx", 6.0),
    (128, 112, "tcgen05", "per_token", ("int4", 1.0)),
])
def test_largest_token_count_sampled(M, N, kernel, mode, arg):
    K = KMAX
    seed = M + N
    x = _device_x(K, M, N, seed)
    P1 = to_bf16(random_orthogonal(M, seed, STREAM_P1)).cuda()
    P2 = to_bf16(random_orthogonal(N, seed, STREAM_P2)).cuda()
    rng = np.random.default_rng(seed)
    idx = np.unique(np.concatenate([np.arange(4), np.arange(K - 4, K), rng.integers(0, K, 16)]))
    idx_t = torch.as_tensor(idx, device="cuda")
    xs, p1, p2 = _f64(x[idx_t]), _f64(P1), _f64(P2)
    fq = FlatQuant(K, M, N, torch.bfloat16, kernel=kernel)
    try:
        if mode == "mx":
            out, sc = fq.quantize_mx(x, P1, P2, arg)
            torch.cuda.synchronize()
            assert fq.last_kernel == kernel
            _, _, info = oracle.flat_quant_mx(xs, p1, p2, arg)
            stats = compare_mx(out[idx_t].cpu().numpy(), sc[idx_t].cpu().numpy(), info, arg)
        else:
            out_dtype, clip = arg
            out, qs = fq.quantize_per_token(x, P1, P2, clip, out_dtype)
            torch.cuda.synchronize()
            assert fq.last_kernel == kernel
            out_b = out[idx_t].cpu().numpy().reshape(len(idx), -1).view(np.uint8)
            codes, rqs, v = oracle.per_token_quantize(oracle.rotate(xs, p1, p2), clip)
            stats = compare_per_token(out_b, qs[idx_t].cpu().numpy(), codes, rqs, v)
        assert fq.device_status() == 0
        print(K, M, N, kernel, mode, stats)
    finally:
        fq.close()
        del x
        torch.cuda.empty_cache()
