"""Bit-exact GPU pins of the rounding and exponent boundaries, with no exemption.

With P1 = I and P2 = I the rotation is exact (x'' = x: every product has one nonzero term,
and both kernels carry a bf16 value through exactly), so the quantizer sees exactly the
values placed in x. The tokens below put values ON the boundaries the page's rules decide
(page: "aclnnFlatQuantV2 complete guide: from two-level matmul to FP4 E2M1 quantization
fusion", http://www.zwxr.cn/news/277566):

* "per-group mode" E2M1 cast: the seven midpoints of the E2M1 grid (ties to the even code),
  saturation above 6, values that round to zero with a minus sign (a zero code is +0);
* case 1: group maxima at powers of two;
* case 2 (6.0 / 7.0): maxima at exactly 1.5 * 2^e and 1.75 * 2^e (the mantissa check is
  strict) and one bf16 step above and below;
* case 3 (8.0-12.0): maxima with amax / dstTypeMax exactly a power of two (no round-up)
  and one bf16 step either side;
* "per-token mode": half-integers of the scaled value (quantScale a power of two, so x''
  / quantScale is exact) and the clamp to [-8, 7] with clipRatio 0.9;
* every hand-worked group and token of tests/golden/hand_worked_groups.txt, whose bytes
  and codes were derived by hand from the page.

Codes and scale bytes must equal the oracle's bit for bit (and the golden values), on
both kernels, with no element or group exempt.
"""

import os

import numpy as np
import pytest
import torch

import oracle
from parity_util import unpack_nibbles
from rotation_bit_quantization_token_b200 import FlatQuant

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked_groups.txt")
MIDS = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]


def _bf16(v):
    return torch.tensor(np.asarray(v, dtype=np.float64), dtype=torch.float32).to(torch.bfloat16)


def _bf16_exact(v):
    """True when v is a bf16 value."""
    return float(_bf16([v]).double()[0]) == v


def _golden():
    mx, pt = [], []
    with open(GOLDEN) as f:
        for ln in f:
            if ln.startswith("#") or not ln.strip():
                continue
            parts = [p.strip() for p in ln.split("|")]
            vals = [float(t) for t in parts[2].split()]
            if parts[0] == "mx":
                mx.append((float(parts[1]), vals, int(parts[3]), [int(c, 16) for c in parts[4].split()]))
            else:
                pt.append((float(parts[1]), vals, float(parts[3]), [int(c) for c in parts[4].split()]))
    return mx, pt


def _boundary_groups(D, rng):
    """Groups of 32 values (bf16-exact) whose maxima or elements sit on the boundaries of
    the rule selected by dstTypeMax D."""
    groups = []
    for e in (-5, -1, 0, 3, 6):
        s = 2.0 ** e
        # midpoints (both signs) with amax 6 * 2^e: scale 2^e for every rule with D < 12
        g = [m * s for m in MIDS] + [-m * s for m in MIDS] + [6.0 * s, -0.25 * s, -0.2 * s, 0.2 * s]
        groups.append(g)
        # saturation and tiny negatives; amax 7.5 * 2^e
        groups.append([7.5 * s, -7.0 * s, 6.5 * s, -6.25 * s, -0.125 * s, -0.0625 * s, 0.0])
    for k in (-3, 0, 2, 5):
        p = 2.0 ** k
        if D in (0.0, 6.0, 7.0):
            for a in (1.0, 1.5, 1.5 * (1 + 2 ** -7), 1.5 * (1 - 2 ** -8), 1.75, 1.75 * (1 + 2 ** -7),
                      1.75 * (1 - 2 ** -8), 2.0 * (1 - 2 ** -8)):
                groups.append([a * p, -0.75 * a * p, 0.5 * a * p, 0.3 * p])
        else:
            for a in (D, D * (1 + 2 ** -7), D * (1 - 2 ** -8), D / 2, 0.75 * D):
                groups.append([-a * p, 0.5 * a * p, 0.25 * a * p, 0.1 * p])
    groups.append([0.0] * 4)
    out = []
    for g in groups:
        vals = [float(_bf16([v]).double()[0]) for v in g]
        full = np.zeros(32)
        full[:len(vals)] = vals
        rng.shuffle(full)
        out.append(full)
    return out


def _mx_tokens(K, M, N, D, rng):
    """x [K, M, N] filled, group by group, with the boundary groups and the golden groups
    of D (golden groups keep their leading positions so their codes can be read back)."""
    L = M * N
    G = L // 32
    golden = [(vals, byte, codes) for d, vals, byte, codes in _golden()[0] if d == D]
    bgroups = _boundary_groups(D, rng)
    flat = np.zeros((K, G * 32))
    placed = []  # (token, group, expected byte, expected codes)
    gi = 0
    for k in range(K):
        for g in range(G):
            if gi < len(golden):
                vals, byte, codes = golden[gi]
                flat[k, 32 * g:32 * g + len(vals)] = [float(_bf16([v]).double()[0]) for v in vals]
                placed.append((k, g, byte, codes, len(vals)))
            else:
                flat[k, 32 * g:32 * g + 32] = bgroups[(gi - len(golden)) % len(bgroups)]
            gi += 1
    x = flat[:, :L].reshape(K, M, N)
    assert all(_bf16_exact(v) for v in np.unique(x))
    return x, placed


def _pt_tokens(K, M, N, clip, rng):
    """Per-token tokens: amax = 7 * 2^k (quantScale 2^k at clip 1.0) with half-integer
    multiples of 2^k; at clip 0.9 the extremes +-amax land at +-7.78 (codes 7 and -8)."""
    L = M * N
    x = np.zeros((K, L))
    golden = [(vals, qs, codes) for c, vals, qs, codes in _golden()[1] if c == clip]
    placed = []
    for k in range(K):
        if k < len(golden):
            vals, qs, codes = golden[k]
            x[k, :len(vals)] = [float(_bf16([v]).double()[0]) for v in vals]
            placed.append((k, qs, codes, len(vals)))
            continue
        s = 2.0 ** int(rng.integers(-6, 7))
        halves = [(n + 0.5) * s for n in range(7)]
        vals = [7.0 * s, -7.0 * s] + halves + [-h for h in halves] + [0.25 * s, -0.25 * s, -0.125 * s]
        vals += list(np.round(rng.uniform(-6.9, 6.9, size=max(0, min(L, 64) - len(vals))) * 4) / 4 * s)
        v = np.zeros(L)
        v[:len(vals)] = vals[:L]
        rng.shuffle(v)
        x[k] = v
    return x.reshape(K, M, N), placed


SHAPES = [("tcgen05", 5, 128, 112), ("tcgen05", 7, 64, 64), ("tcgen05", 3, 32, 96), ("tcgen05", 4, 64, 128),
          ("general", 5, 128, 112), ("general", 16, 16, 16), ("general", 6, 8, 40)]


@pytest.mark.parametrize("kernel,K,M,N", SHAPES, ids=[f"{k}-{a}x{b}x{c}" for k, a, b, c in SHAPES])
@pytest.mark.parametrize("D", [0.0, 6.0, 7.0, 8.0, 10.0, 12.0])
def test_mx_boundaries_bit_exact(kernel, K, M, N, D):
    rng = np.random.default_rng([int(D * 10), K, M, N])
    x, placed = _mx_tokens(K, M, N, D, rng)
    dev = torch.device("cuda", 0)
    xd = _bf16(x).to(dev)
    P1 = torch.eye(M, dtype=torch.bfloat16, device=dev)
    P2 = torch.eye(N, dtype=torch.bfloat16, device=dev)
    fq = FlatQuant(K, M, N, kernel=kernel)
    out, sc = fq.quantize_mx(xd, P1, P2, D)
    torch.cuda.synchronize()
    assert fq.last_kernel == kernel
    ref_out, ref_sc, info = oracle.flat_quant_mx(x, np.eye(M), np.eye(N), D)
    np.testing.assert_array_equal(sc.cpu().numpy(), ref_sc)
    np.testing.assert_array_equal(out.cpu().numpy(), ref_out)
    # the golden groups: bytes and codes derived by hand from the page
    got_codes = unpack_nibbles(out.cpu().numpy())
    got_b = sc.cpu().numpy().reshape(K, -1)
    for k, g, byte, codes, n in placed:
        assert int(got_b[k, g]) == byte, (k, g)
        assert list(got_codes[k, 32 * g:32 * g + n]) == codes, (k, g)


PT_SHAPES = [("tcgen05", 6, 128, 112), ("tcgen05", 9, 64, 64), ("general", 16, 16, 16), ("general", 6, 64, 64)]


@pytest.mark.parametrize("kernel,K,M,N", PT_SHAPES, ids=[f"{k}-{a}x{b}x{c}" for k, a, b, c in PT_SHAPES])
@pytest.mark.parametrize("clip", [1.0, 0.9])
def test_per_token_boundaries_bit_exact(kernel, K, M, N, clip):
    rng = np.random.default_rng([int(clip * 10), K, M, N, 1])
    x, placed = _pt_tokens(K, M, N, clip, rng)
    dev = torch.device("cuda", 0)
    xd = _bf16(x).to(dev)
    P1 = torch.eye(M, dtype=torch.bfloat16, device=dev)
    P2 = torch.eye(N, dtype=torch.bfloat16, device=dev)
    fq = FlatQuant(K, M, N, kernel=kernel)
    out, qs = fq.quantize_per_token(xd, P1, P2, clip, "int4")
    torch.cuda.synchronize()
    assert fq.last_kernel == kernel
    ref_out, ref_qs, info = oracle.flat_quant_per_token(x, np.eye(M), np.eye(N), clip, "int4")
    np.testing.assert_array_equal(qs.cpu().numpy(), ref_qs)
    np.testing.assert_array_equal(out.cpu().numpy(), ref_out)
    got = unpack_nibbles(out.cpu().numpy()).astype(np.int64)
    got = np.where(got >= 8, got - 16, got)
    for k, q, codes, n in placed:
        assert abs(float(qs[k]) - q) <= 1e-6 * q
        assert list(got[k, :n]) == codes
    if clip == 1.0:
        # every non-golden token has quantScale exactly a power of two
        for k in range(len(placed), K):
            m, e = np.frexp(float(qs[k]))
            assert m == 0.5
