"""Seeded synthetic workloads for the fused rotate + quantize operator.

Shared by the tests (oracle side and CUDA side) and by `bench.py`. This module holds
no arithmetic of the operator itself: it only draws random inputs, rounds them to the
16-bit input type and describes the five workloads.

Recipe (all streams are numpy PCG64, `default_rng([seed, stream])`; values are drawn in
float32/float64 and rounded to bfloat16 with round-to-nearest-even):

* stream 1: x; stream 2: P1; stream 3: P2; stream 4: outlier masks, gains, positions.
* P1, P2: Q of the QR factorisation of a standard Gaussian matrix (float64),
  with columns multiplied by sign(diag R) so that Q is Haar-distributed, then bf16.
* x distributions:
  - "normal": N(0, 1).
  - "student_t_cols": Student-t(nu=3) * 0.5, and 1% of the M*N feature positions
    (fixed for all tokens, ceil(0.01*M*N) of them) multiplied by 20.
  - "normal_outliers": N(0, 1), each element replaced with probability 0.005 by a draw
    from N(0, 30^2).
  - "laplace_gain": Laplace(0, 1) per element times a lognormal(0, 1) gain per token.
  - "normal_channels": N(0, 1), with 8 fixed feature positions (of M*N) multiplied by 50.
"""

from dataclasses import dataclass

import numpy as np
import torch

STREAM_X, STREAM_P1, STREAM_P2, STREAM_AUX = 1, 2, 3, 4


@dataclass(frozen=True)
class Workload:
    name: str
    K: int
    M: int
    N: int
    mode: str            # "per_token" or "mx"
    dist: str
    out: str = "fp4"     # "int4" / "int32" for per_token, "fp4" for mx
    clip_ratio: float = 1.0
    dst_type_max: float = 0.0

    @property
    def tokens(self):
        return self.K

    def in_bytes_per_token(self):
        return self.M * self.N * 2

    def out_bytes_per_token(self):
        return self.M * self.N // 2

    def scale_bytes_per_token(self):
        if self.mode == "per_token":
            return 4
        return -(-self.M * self.N // 64) * 2

    def bytes_per_token(self):
        """Algorithmic HBM bytes per token: bf16 x in, packed 4-bit codes out, scales out
        (P1 and P2 are read once per CTA and are not counted)."""
        return (self.in_bytes_per_token() + self.out_bytes_per_token()
                + self.scale_bytes_per_token())

    def flops_per_token(self):
        """Algorithmic flops of the two contractions, 2(M N^2 + M^2 N)."""
        return 2 * (self.M * self.N * self.N + self.M * self.M * self.N)

    def with_tokens(self, K):
        return Workload(self.name, K, self.M, self.N, self.mode, self.dist, self.out,
                        self.clip_ratio, self.dst_type_max)


WORKLOADS = {
    w.name: w for w in [
        Workload("per_token_int4_16x16x16", 16, 16, 16, "per_token", "normal",
                 out="int4", clip_ratio=1.0),
        Workload("per_token_int32_4096x64x64", 4096, 64, 64, "per_token",
                 "student_t_cols", out="int32", clip_ratio=0.9),
        Workload("mx_case1_8192x64x128", 8192, 64, 128, "mx", "normal_outliers",
                 dst_type_max=0.0),
        Workload("mx_case2_16384x64x64", 16384, 64, 64, "mx", "laplace_gain",
                 dst_type_max=6.0),
        Workload("mx_case3_32768x128x112", 32768, 128, 112, "mx", "normal_channels",
                 dst_type_max=10.0),
    ]
}

# The largest single-GPU workload; bench.py times this one.
BENCH_WORKLOAD = "mx_case3_32768x128x112"


def _rng(seed, stream):
    return np.random.default_rng([seed, stream])


def to_bf16(a):
    """Round a float array to bfloat16 (round-to-nearest-even); returns a CPU tensor."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def to_fp16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.float16)


def random_orthogonal(n, seed, stream):
    """Haar-random orthogonal [n, n] matrix in float64 (QR of a Gaussian, sign-fixed)."""
    g = _rng(seed, stream).standard_normal((n, n))
    q, r = np.linalg.qr(g)
    return q * np.sign(np.diag(r))[None, :]


def draw_x(w: Workload, seed=0):
    """Draw x [K, M, N] as float32 numpy following the workload's distribution."""
    K, M, N = w.K, w.M, w.N
    rx = _rng(seed, STREAM_X)
    ra = _rng(seed, STREAM_AUX)
    shape = (K, M, N)
    if w.dist == "normal":
        return rx.standard_normal(shape, dtype=np.float32)
    if w.dist == "student_t_cols":
        x = (rx.standard_t(3, size=shape) * 0.5).astype(np.float32)
        n_pos = -(-M * N // 100)
        pos = ra.choice(M * N, size=n_pos, replace=False)
        x.reshape(K, M * N)[:, pos] *= np.float32(20.0)
        return x
    if w.dist == "normal_outliers":
        x = rx.standard_normal(shape, dtype=np.float32)
        mask = ra.random(shape, dtype=np.float32) < np.float32(0.005)
        n_out = int(mask.sum())
        x[mask] = ra.standard_normal(n_out, dtype=np.float32) * np.float32(30.0)
        return x
    if w.dist == "laplace_gain":
        x = rx.laplace(0.0, 1.0, size=shape).astype(np.float32)
        gain = ra.lognormal(0.0, 1.0, size=K).astype(np.float32)
        x *= gain[:, None, None]
        return x
    if w.dist == "normal_channels":
        x = rx.standard_normal(shape, dtype=np.float32)
        pos = ra.choice(M * N, size=8, replace=False)
        x.reshape(K, M * N)[:, pos] *= np.float32(50.0)
        return x
    raise ValueError(f"unknown distribution {w.dist!r}")


def make_inputs(w: Workload, seed=0, dtype=torch.bfloat16):
    """Return (x [K,M,N], P1 [M,M], P2 [N,N]) as CPU tensors of the 16-bit input type."""
    conv = to_bf16 if dtype == torch.bfloat16 else to_fp16
    x = conv(draw_x(w, seed))
    P1 = conv(random_orthogonal(w.M, seed, STREAM_P1))
    P2 = conv(random_orthogonal(w.N, seed, STREAM_P2))
    return x, P1, P2
