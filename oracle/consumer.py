"""Plain CPU oracle for the consumers of the operator's outputs (test infrastructure).

TEST INFRASTRUCTURE ONLY, like the rest of `oracle/`: imported by `tests/` and by
nothing on the product path, with which it shares no code.

Page: "aclnnFlatQuantV2 complete guide: from two-level matmul to FP4 E2M1
quantization fusion" (http://www.zwxr.cn/news/277566). Its "per-token mode" says that
quantScale is emitted as its own FLOAT32 [K] tensor so that the low-precision data can be
dequantized later, and its summary calls the operator the tool for FP4 E2M1 compression
of weights and activations. The page defines neither step beyond that. The readings here
are the plainest ones its formulas allow:

* per-token dequantization is the inverse of "out = x'' / quantScale":
  x''_hat = code * quantScale;
* per-group dequantization is the inverse of the per-group encodings of cases 1-3. In every
  case an element is encoded as E2M1(x'' * R) with R = 2^-(byte - 127) (case 1: the E8M0
  byte is sharedExp + 127 and quantScale = 2^sharedExp; case 3: S_ue8m0 = 2^(E - 127)),
  so x''_hat = E2M1 value * 2^(byte - 127), with the byte of group g = i // 32 of the
  flattened token;
* the consumer contraction of two per-group-quantized operands (activations [T, L] and
  weights [O, L], both in the operator's output layout) is C[t, o] = sum_i A_hat[t, i] *
  W_hat[o, i], the reduction running over the flattened M*N axis that the groups of 32 tile.
  This is the product that a block-scaled FP4 tensor-core MMA computes. No kernel for it
  exists yet.

Every function is written from these definitions. The fp64 sums are exact for the
dyadic values involved as long as the exponents stay within the fp64 significand, which
the pins keep to.
"""

import numpy as np

from .flatquant import E2M1_GRID, GROUP


def unpack_nibbles(packed, L):
    """Inverse of the LSB-first packing: byte b holds element 2b in bits 0-3 and element
    2b + 1 in bits 4-7. Returns uint8 nibbles [..., L]."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out[..., :L]


def int4_value(nibbles):
    """Two's complement value of INT4 nibbles, in [-8, 7]."""
    n = np.asarray(nibbles, dtype=np.int64) & 0xF
    return np.where(n >= 8, n - 16, n)


def e2m1_value(nibbles):
    """Value of E2M1 codes: magnitude index in bits 0-2, sign in bit 3."""
    n = np.asarray(nibbles, dtype=np.uint8)
    mag = E2M1_GRID[n & 7]
    return np.where(n & 8, -mag, mag)


def group_bytes_from_layout(scales, L):
    """E8M0 byte of each group from the [T, ceilDiv(L, 64), 2] scale tensor (group g at
    [t, g // 2, g % 2]). Returns uint8 [T, ceilDiv(L, 32)]."""
    s = np.asarray(scales, dtype=np.uint8)
    T = s.shape[0]
    G = -(-L // GROUP)
    return s.reshape(T, -1)[:, :G]


def dequantize_per_token(out, quant_scale, M, N):
    """x''_hat [K, M, N] (float64) from per-token INT4 bytes (uint8 [K, M*N/2], or the same
    bytes as INT32 words) and the FLOAT32 quantScale [K]."""
    qs = np.asarray(quant_scale, dtype=np.float32).astype(np.float64)
    K = qs.shape[0]
    b = np.ascontiguousarray(out).view(np.uint8).reshape(K, -1)
    codes = int4_value(unpack_nibbles(b, M * N))
    return (codes * qs[:, None]).reshape(K, M, N)


def dequantize_mx(out_fp4, scales, M, N):
    """x''_hat [K, M, N] (float64) from per-group E2M1 codes (uint8 [K, M*N/2]) and E8M0
    bytes in the [K, ceilDiv(M*N, 64), 2] layout: code value * 2^(byte - 127) of its
    group."""
    L = M * N
    codes = unpack_nibbles(np.asarray(out_fp4, dtype=np.uint8).reshape(-1, L // 2), L)
    K = codes.shape[0]
    gb = group_bytes_from_layout(scales, L).astype(np.int64)
    per_elem = np.repeat(gb, GROUP, axis=1)[:, :L]
    return (e2m1_value(codes) * np.ldexp(1.0, per_elem - 127)).reshape(K, M, N)


def mx_matmul(a_fp4, a_scales, w_fp4, w_scales, L):
    """C [T, O] (float64) = A_hat . W_hat^T for per-group-quantized activations (codes
    [T, L/2], scales [T, ceilDiv(L, 64), 2]) and weights (codes [O, L/2], scales
    [O, ceilDiv(L, 64), 2]), both in the operator's output layout; the reduction runs over
    the L = M*N axis."""
    def dq(codes, scales):
        c = unpack_nibbles(np.asarray(codes, dtype=np.uint8).reshape(-1, L // 2), L)
        gb = group_bytes_from_layout(scales, L).astype(np.int64)
        return e2m1_value(c) * np.ldexp(1.0, np.repeat(gb, GROUP, axis=1)[:, :L] - 127)
    return dq(a_fp4, a_scales) @ dq(w_fp4, w_scales).T
