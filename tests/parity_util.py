"""Comparison of the CUDA outputs with the oracle under the stated tolerance.

Tolerance (bit-exact on codes and scale exponents, except near rounding boundaries):
  * an element is exempt when the oracle's value before rounding lies within 1e-5
    (relative) of a rounding boundary: k + 0.5 for INT4, the E2M1 midpoints 0.25, 0.75,
    1.25, 1.75, 2.5, 3.5, 5 for E2M1;
  * a group is exempt when its oracle absmax lies within 1e-5 (relative) of an exponent
    boundary of its rule (a power of two; for 6.0 / 7.0 also 1.5 / 1.75 times one; for
    the ratio rule, amax / dstTypeMax near a power of two);
  * exempt elements may differ by one code step, exempt groups by one exponent step (and
    then their codes are not compared); at most 0.01% of elements may differ at all.
  * the per-token float32 quantScale is compared to a relative 1e-6 (its only source of
    difference is the float32 rounding of x'' inside the kernel).
"""

import numpy as np

REL = 1e-5
MAX_MISMATCH_FRAC = 1e-4
E2M1_MIDS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def unpack_nibbles(b):
    b = np.asarray(b, dtype=np.uint8)
    out = np.empty(b.shape[:-1] + (b.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = b & 0xF
    out[..., 1::2] = b >> 4
    return out


def int4_exempt(v):
    v = np.asarray(v, dtype=np.float64)
    b = np.floor(v) + 0.5
    return np.abs(v - b) <= REL * np.abs(b)


def e2m1_exempt(v):
    a = np.abs(np.asarray(v, dtype=np.float64))
    d = np.abs(a[..., None] - E2M1_MIDS)
    return np.any(d <= REL * E2M1_MIDS, axis=-1)


def _near_pow2(a):
    a = np.asarray(a, dtype=np.float64)
    pos = a > 0
    s = np.where(pos, a, 1.0)
    m = s / np.exp2(np.floor(np.log2(s)))
    return pos & ((m <= 1 + REL) | (m >= 2 * (1 - REL)))


def group_exempt(amax, D):
    amax = np.asarray(amax, dtype=np.float64)
    if D == 0.0:
        return _near_pow2(amax)
    if D in (6.0, 7.0):
        pos = amax > 0
        s = np.where(pos, amax, 1.0)
        m = s / np.exp2(np.floor(np.log2(s)))
        t = D / 4.0
        return _near_pow2(amax) | (pos & (np.abs(m - t) <= REL * t))
    return _near_pow2(amax / D)


def compare_per_token(out_bytes, qs, ref_codes, ref_qs, ref_v, elem_taint=None, token_taint=None):
    """out_bytes: uint8 [K, M*N/2] from the GPU; ref_* from oracle.per_token_quantize.
    elem_taint [K, M*N] / token_taint [K] (optional) mark elements and whole tokens whose
    reference value is not decided by the inputs alone (see intermediate_rounding_taint):
    tainted elements are exempt, tainted tokens are skipped."""
    K = ref_codes.shape[0]
    keep = np.ones(K, dtype=bool) if token_taint is None else ~np.asarray(token_taint)
    got = unpack_nibbles(np.asarray(out_bytes).reshape(K, -1)).astype(np.int64)[keep]
    got = np.where(got >= 8, got - 16, got)
    want = ref_codes.reshape(K, -1).astype(np.int64)[keep]
    v = ref_v.reshape(K, -1)[keep]
    diff = got != want
    exempt = int4_exempt(v)
    if elem_taint is not None:
        exempt = exempt | np.asarray(elem_taint).reshape(K, -1)[keep]
    qs = np.asarray(qs)[keep]
    ref_qs = np.asarray(ref_qs)[keep]
    stats = {"elements": int(want.size), "mismatch": int(diff.sum()),
             "exempt_mismatch": int((diff & exempt).sum())}
    bad = diff & ~exempt
    assert not bad.any(), f"non-exempt INT4 mismatches: {int(bad.sum())} {stats}"
    assert np.all(np.abs(got - want)[diff] <= 1), "exempt INT4 codes differ by more than one"
    assert stats["mismatch"] <= MAX_MISMATCH_FRAC * want.size, stats
    # quantScale within 1e-6 relative (about 8 ulp) of the reference: it is the maximum of
    # the kernel's float32 x'', which carries the accumulation's rounding (up to 7 ulp seen).
    # For non-negative floats the difference of the bit patterns counts the ulps between them.
    qs32 = np.asarray(qs, dtype=np.float32).reshape(-1)
    rq32 = np.asarray(ref_qs, dtype=np.float32).reshape(-1)
    assert np.all(qs32 >= 0) and np.all(rq32 >= 0), "negative quantScale"
    ulps = np.abs(qs32.view(np.int32).astype(np.int64) - rq32.view(np.int32).astype(np.int64))
    rel = np.abs(qs32.astype(np.float64) - rq32) / np.maximum(rq32.astype(np.float64), 1e-30)
    stats["quant_scale_max_rel"] = float(rel.max()) if rel.size else 0.0
    stats["quant_scale_max_ulp"] = int(ulps.max()) if ulps.size else 0
    assert np.all(rel <= 1e-6), f"quantScale differs: max rel {rel.max()} ({ulps.max()} ulp)"
    return stats


def _e2m1_step(a_codes, b_codes):
    """Distance in code steps between two E2M1 codes on the signed number line."""
    def pos(c):
        mag = (c & 7).astype(np.int64)
        return np.where(c & 8, -mag, mag)
    return np.abs(pos(a_codes) - pos(b_codes))


def compare_mx(out_bytes, scales, ref_info, D, elem_taint=None):
    """out_bytes uint8 [K, M*N/2], scales uint8 [K, S, 2] from the GPU; ref_info from
    oracle.flat_quant_mx. elem_taint [K, M*N] (optional) marks elements whose reference
    value is not decided by the inputs alone: every group holding one is exempt, its
    byte and its codes (see intermediate_rounding_taint)."""
    ref_codes = ref_info["codes"]
    K, L = ref_codes.shape
    G = ref_info["group_bytes"].shape[1]
    got = unpack_nibbles(np.asarray(out_bytes).reshape(K, -1))[:, :L]
    got_b = np.asarray(scales).reshape(K, -1)
    want_b = ref_info["group_bytes"]
    # the spare slot of an odd group count is 0x7F (2^0)
    if got_b.shape[1] > G:
        assert np.all(got_b[:, G:] == 0x7F), "spare scale byte is not 0x7F"
    got_b = got_b[:, :G].astype(np.int64)
    gex = group_exempt(ref_info["amax"], D)
    if elem_taint is not None:
        t = np.zeros((K, G * 32), dtype=bool)
        t[:, :L] = np.asarray(elem_taint).reshape(K, -1)
        gex = gex | t.reshape(K, G, 32).any(axis=-1)
    bdiff = got_b != want_b.astype(np.int64)
    assert not (bdiff & ~gex).any(), \
        f"non-exempt E8M0 mismatches: {int((bdiff & ~gex).sum())}"
    assert np.all(np.abs(got_b - want_b)[bdiff] <= 1)
    # element codes, skipping groups whose exponent legitimately differs
    skip = np.repeat(bdiff, 32, axis=1)[:, :L]
    v = ref_info["v"].reshape(K, -1)[:, :L]
    diff = (got != ref_codes) & ~skip
    exempt = e2m1_exempt(v) | np.repeat(gex, 32, axis=1)[:, :L]
    bad = diff & ~exempt
    stats = {"elements": int(ref_codes.size), "groups": int(K * G),
             "scale_mismatch": int(bdiff.sum()), "mismatch": int(diff.sum()),
             "exempt_mismatch": int((diff & exempt).sum())}
    assert not bad.any(), f"non-exempt E2M1 mismatches: {int(bad.sum())} {stats}"
    assert np.all(_e2m1_step(got[diff], ref_codes[diff]) <= 1), "exempt E2M1 codes differ by more than one step"
    total = stats["mismatch"] + 32 * stats["scale_mismatch"]
    assert total <= MAX_MISMATCH_FRAC * ref_codes.size, stats
    return stats


def rotate_close(x2_gpu, x2_ref, extra=None):
    """x'' within 2e-3 relative: |d| <= 2e-3 * max(|ref|, 1e-3 * amax_token) (+ extra, an
    optional per-element allowance). Returns the largest error divided by the token's rms
    (a finer figure that is reported)."""
    K = x2_ref.shape[0]
    g = np.asarray(x2_gpu, dtype=np.float64).reshape(K, -1)
    r = np.asarray(x2_ref, dtype=np.float64).reshape(K, -1)
    amax = np.abs(r).max(axis=1, keepdims=True)
    tol = 2e-3 * np.maximum(np.abs(r), 1e-3 * amax)
    if extra is not None:
        tol = tol + np.asarray(extra, dtype=np.float64).reshape(K, -1)
    d = np.abs(g - r)
    assert np.all(d <= tol), f"x'' outside tolerance: worst {float((d / np.maximum(tol, 1e-300)).max())}"
    rms = np.sqrt((r * r).mean(axis=1, keepdims=True))
    return float((d / np.maximum(rms, 1e-300)).max())


# --------------------------------------------------------------------------------------
# intermediate-rounding mode: which reference values the inputs do not decide
# --------------------------------------------------------------------------------------

_P16 = {"bf16": (8, -126), "fp16": (11, -14)}


def _spacing16(a, dtype):
    """Spacing of 16-bit values around magnitudes a (the quantum of their binade)."""
    p, emin = _P16[dtype]
    a = np.asarray(a, dtype=np.float64)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    e = np.maximum(ex.astype(np.int64) - 1, emin)
    return np.ldexp(1.0, e - (p - 1))


def intermediate_rounding_taint(x, P1, P2, dtype):
    """In the intermediate-rounding mode x' = round16(x . P2). A kernel forms x . P2 in
    float32 in some order, so its sum can lie anywhere within N * 2^-24 * sum_j |x_j P2_jn|
    of the exact one; where a 16-bit rounding midpoint lies inside that bound, the kernel
    may round x' to the other neighbour, one 16-bit spacing away. Returns (dev [K, M, N]:
    the largest change of each x'' element that such roundings can cause, sum over m of
    |P1[r, m]| * spacing(x'[m, n]) for the x'[m, n] so marked; x1_taint [K, M, N]: the x'
    elements marked). Elements of x'' with dev > 0 are not decided by the inputs."""
    x = np.asarray(x, dtype=np.float64)
    P2 = np.asarray(P2, dtype=np.float64)
    N = P2.shape[0]
    v = np.matmul(x, P2)
    bound = N * 2.0 ** -24 * 1.01 * np.matmul(np.abs(x), np.abs(P2))
    a = np.abs(v)
    q = _spacing16(a, dtype)
    mid = (np.floor(a / q) + 0.5) * q
    lower_mid = (np.floor(a / q) - 0.5) * q  # the midpoint below, for values just above one
    taint = (np.abs(a - mid) <= bound) | (np.abs(a - lower_mid) <= bound)
    step = np.where(taint, 2.0 * q, 0.0)   # the binade may change at a power of two
    dev = np.matmul(np.abs(np.asarray(P1, dtype=np.float64)), step)
    return dev, taint


def token_taint_from(dev, x2_ref):
    """Tokens whose absolute maximum the tainted elements can change (their per-token
    scale, and so every code, is then not decided by the inputs)."""
    K = x2_ref.shape[0]
    d = np.asarray(dev).reshape(K, -1)
    r = np.abs(np.asarray(x2_ref, dtype=np.float64)).reshape(K, -1)
    amax = r.max(axis=1)
    return (d > 0).any(axis=1) & ((r + d).max(axis=1) >= amax - d.max(axis=1))
