"""Plain, slow, obviously-correct CPU oracle for the FlatQuantV2 fused operator.

TEST INFRASTRUCTURE ONLY. Imported by `tests/`, `__graft_entry__.smoke()` and the
CPU-baseline / reference legs of `bench.py`; never by the product path, with which
it shares no code, table or helper.

Everything below restates the page "aclnnFlatQuantV2 complete guide: from two-level
matmul to FP4 E2M1 quantization fusion" (http://www.zwxr.cn/news/277566):

* "How it works / two-level small matmul": x' = x . kroneckerP2 ([N,N] applied from
  the right), x'' = kroneckerP1 . x' ([M,M] applied from the left); shape stays
  [K, M, N].
* "per-token mode": quantScale[k] = max|x''[k]| / (7 / clipRatio) (FLOAT32, shape
  [K]); out = x'' / quantScale, as INT4 or INT4 packed eight per INT32.
* "per-group mode", case 1 (dstTypeMax = 0.0), case 2 (6.0 / 7.0) and case 3
  (8.0-12.0 and other values): groups of 32 consecutive elements of x'' reshaped to
  [K, M*N]; E8M0 shared exponents in a [K, ceilDiv(M*N, 64), 2] tensor; E2M1 codes.

Readings taken where the page is silent or garbled:

* x'' is formed in float64 with no intermediate rounding.
* Every step that turns a float into an integer (a code, an exponent) is taken in
  float32 on the float32 rounding of x'' -- the precision of the kernel's
  accumulator -- because the page names no other precision except the explicit
  FP32 of case 3.
* INT4 rounding is round-half-to-even with a clamp to [-8, 7].
* Nibble order is LSB-first: element 2b sits in bits 0-3 of byte b, element 2b+1 in
  bits 4-7, so the INT4 and the INT32 outputs are the same bytes.
* Case 1 reads "emax" as the largest exponent of E2M1 (2, since 4 = 2^2 is the top
  binade) and reduceMax as the group's largest magnitude:
  sharedExp = floor(log2(amax)) - 2, clamped to [-127, 127]; an all-zero group
  gets byte 0x00.
* Case 2 reads the mantissa check as "the significand's leading one (6.0) or two
  (7.0) fraction bits are 1 and the remaining fraction bits are not all zero", in
  which case the exponent is rounded up.
* E2M1 casts round to nearest with ties to the even code and saturate to +-6; every
  value whose magnitude rounds to zero encodes as +0 (0x0), so the format's two zero
  codes never both appear (the page gives no rule for the sign of a zero code, and a
  sign kept on values that round to zero would hinge on the last bit of x'').
* The spare byte of an odd group count (the scale tensor holds ceilDiv(M*N, 64) pairs) is
  0x7F, the scale 2^0: the page gives it no value.
"""

import numpy as np

# Magnitudes of E2M1 codes 0..7 (bit 3 is the sign): 1 sign, 2 exponent, 1 mantissa bit.
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)

GROUP = 32  # per-group mode: 32 consecutive elements share one E8M0 exponent


def e2m1_encode(v):
    """E2M1 cast of float values (page: per-group mode, "P_i = cast_to_dst_type(V_i /
    mxscale, round_mode)"): nearest grid magnitude, ties to the even code, values above
    6 saturate to 6, sign in bit 3 for nonzero magnitudes. Returns uint8 codes in [0, 15].

    Brute force: every value is compared with all eight grid magnitudes."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    dist = np.abs(a[..., None] - E2M1_GRID)
    nearest = dist == dist.min(axis=-1, keepdims=True)
    even_bonus = 2 - (np.arange(8) % 2)  # even codes win ties
    mag = np.argmax(nearest * even_bonus, axis=-1).astype(np.uint8)
    neg = ((v < 0) & (mag > 0)).astype(np.uint8)  # a zero magnitude is always +0 (0x0)
    return mag | (neg << 3)


def e2m1_decode(codes):
    """Value of each E2M1 code (sign bit 3, magnitude index bits 0-2)."""
    codes = np.asarray(codes, dtype=np.uint8)
    mag = E2M1_GRID[codes & 7]
    return np.where(codes & 8, -mag, mag)


def rotate(x, P1, P2):
    """Two-level small matmul (page: "How it works"): x' = x . P2, then x'' = P1 . x',
    per token, in float64 with no intermediate rounding.

    x: [K, M, N]; P1: [M, M]; P2: [N, N], or None / an empty [0, 0] array, which skips
    the right multiply (page: parameter table, kroneckerP2 "[0, 0] only in per-group
    mode")."""
    x = np.asarray(x, dtype=np.float64)
    P1 = np.asarray(P1, dtype=np.float64)
    if P2 is None or np.size(P2) == 0:
        x1 = x
    else:
        x1 = np.matmul(x, np.asarray(P2, dtype=np.float64))
    return np.matmul(P1, x1)


def round_to_16bit(v, dtype):
    """float32 values rounded to "bf16" or "fp16" (nearest, ties to even), returned as
    float64. bf16: the low 16 bits of the float32 encoding are dropped after adding
    0x7FFF plus the lowest kept bit (round half to even on the bit pattern; finite values
    only). fp16: numpy's float32 -> float16 cast, which rounds to nearest even."""
    v = np.asarray(v, dtype=np.float32)
    if dtype == "fp16":
        with np.errstate(over="ignore"):
            return v.astype(np.float16).astype(np.float64)
    bits = v.view(np.uint32).astype(np.uint64)
    bits = (bits + 0x7FFF + ((bits >> 16) & 1)) & 0xFFFF0000
    return bits.astype(np.uint32).view(np.float32).astype(np.float64)


# significant bits, smallest normal exponent and largest finite value of the 16-bit types
_FMT16 = {"bf16": (8, -126, (2.0 - 2.0 ** -7) * 2.0 ** 127),
          "fp16": (11, -14, 65504.0)}


def _quantum16(a, dtype):
    """Spacing of the 16-bit type's values around magnitudes a (float64 array, a >= 0):
    2^(e - (p - 1)) in the binade [2^e, 2^(e+1)), the subnormal spacing below 2^emin."""
    p, emin, _ = _FMT16[dtype]
    e = _floor_log2(np.where(a > 0, a, 1.0))
    e = np.maximum(e, emin)
    return np.ldexp(1.0, e - (p - 1))


def round_f64_to_16bit(v, dtype):
    """float64 values rounded directly (no float32 step) to the nearest "bf16" / "fp16"
    value, ties to the even significand; magnitudes at or beyond the midpoint between the
    largest finite value and the next power of two become infinite. Returned as float64.
    The division by the spacing is exact (a power of two) and numpy's rint rounds half to
    even."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    q = _quantum16(a, dtype)
    r = np.rint(a / q) * q
    _, _, top = _FMT16[dtype]
    r = np.where(r > top, np.inf, r)
    return np.copysign(r, v)


def _round_fraction_16bit(fr, dtype):
    """Exact rational fr rounded to the 16-bit type (nearest, ties to even): the
    definition itself, in integer arithmetic."""
    from fractions import Fraction
    if fr == 0:
        return 0.0
    p, emin, top = _FMT16[dtype]
    a = abs(fr)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1                                  # now 2^e <= a < 2^(e+1)
    q = Fraction(2) ** (max(e, emin) - (p - 1))
    k = a / q
    n = k.numerator // k.denominator            # floor
    rem = k - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    r = float(n * q) if n * q <= Fraction(top) else float("inf")
    return r if fr > 0 else -r


def round16_of_exact_product(x, P2, dtype):
    """x' = x . P2 with every element rounded once, from its exact value, to the 16-bit
    type (nearest, ties to even). x [..., M, N] and P2 [N, N] hold 16-bit values, so each
    product is exact in float64; the float64 matmul is within N * 2^-52 * (|x| . |P2|) of
    the exact sum, so its rounding is the rounding of the exact sum unless a rounding
    midpoint lies inside that bound. Those elements (rare) are summed exactly as rationals
    and rounded by definition."""
    from fractions import Fraction
    x = np.asarray(x, dtype=np.float64)
    P2 = np.asarray(P2, dtype=np.float64)
    N = P2.shape[0]
    v = np.matmul(x, P2)
    bound = (N * 2.0 ** -52) * 1.01 * np.matmul(np.abs(x), np.abs(P2))
    a = np.abs(v)
    q = _quantum16(a, dtype)
    mid = (np.floor(a / q) + 0.5) * q
    near = np.abs(a - mid) <= bound
    out = round_f64_to_16bit(v, dtype)
    for idx in zip(*np.nonzero(near)):
        row = x[idx[:-1]]
        col = P2[:, idx[-1]]
        exact = sum(Fraction(float(row[j])) * Fraction(float(col[j])) for j in range(N))
        out[idx] = _round_fraction_16bit(exact, dtype)
    return out


def rotate_rounded(x, P1, P2, dtype="bf16"):
    """Two-level small matmul with x' kept in the input type between the products: the
    intermediate-rounding reading of "How it works", whose formulas leave the precision of
    x' open. x' = x . P2 is formed exactly and each element is rounded once to the input
    type (nearest, ties to even); x'' = P1 . x' is then formed in float64 from the rounded
    values. No summation order is assumed for x'. P2 None or empty skips the right
    multiply (x' = x, already in the input type)."""
    x = np.asarray(x, dtype=np.float64)
    P1 = np.asarray(P1, dtype=np.float64)
    if P2 is None or np.size(P2) == 0:
        x1 = x
    else:
        x1 = round16_of_exact_product(x, P2, dtype)
    return np.matmul(P1, x1)


def per_token_quantize(x2, clip_ratio):
    """Per-token mode (page: "per-token mode"):
    quantScale[k] = max|x''[k]| / (7 / clipRatio) as FLOAT32, out = x'' / quantScale,
    rounded half-to-even and clamped to [-8, 7].

    Returns (codes int8 [K, M, N], quantScale float32 [K], v float32 [K, M, N]) where v is
    the value before rounding. A token whose x'' is all zero gets quantScale 0 and codes 0.
    """
    x2 = np.asarray(x2, dtype=np.float64)
    K = x2.shape[0]
    amax = np.abs(x2).reshape(K, -1).max(axis=1)
    qscale = (amax / (7.0 / clip_ratio)).astype(np.float32)
    x2_32 = x2.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = x2_32 / qscale.reshape((K,) + (1,) * (x2.ndim - 1))
    v = np.where(qscale.reshape((K,) + (1,) * (x2.ndim - 1)) == 0, np.float32(0), v)
    v = v.astype(np.float32)
    codes = np.clip(np.rint(v), -8, 7).astype(np.int8)
    return codes, qscale, v


def pack_nibbles(codes):
    """Pack 4-bit codes two per byte along the last axis, LSB-first (element 2b in bits
    0-3 of byte b, element 2b+1 in bits 4-7). Accepts INT4 codes in [-8, 7] (two's
    complement nibbles) or E2M1 codes in [0, 15]."""
    c = np.asarray(codes).astype(np.int64) & 0xF
    assert c.shape[-1] % 2 == 0, "the packed axis must have even length"
    lo = c[..., 0::2]
    hi = c[..., 1::2]
    return (lo | (hi << 4)).astype(np.uint8)


def mx_group_view(x2):
    """Per-group mode layout (page: case 1): reshape x'' [K, M, N] to [K, M*N] and split
    the second axis into groups of 32; a short last group is padded with zeros (page:
    case 3, "missing values count as 0"). Returns (groups [K, G, 32] float64, M*N)."""
    x2 = np.asarray(x2, dtype=np.float64)
    K = x2.shape[0]
    flat = x2.reshape(K, -1)
    L = flat.shape[1]
    G = -(-L // GROUP)
    padded = np.zeros((K, G * GROUP), dtype=np.float64)
    padded[:, :L] = flat
    return padded.reshape(K, G, GROUP), L


def _floor_log2(a):
    """floor(log2(a)) for a > 0, exact (from the binary exponent)."""
    _, ex = np.frexp(a)
    return ex.astype(np.int64) - 1


def mx_scale_exponent(amax32, dst_type_max):
    """Shared-exponent rule for one group, from its float32 absolute maximum.

    Returns (e8m0 byte uint8, R float64) where the group's elements are encoded as
    E2M1(x * R), R being an exact power of two.

    * dstTypeMax == 0.0 (page: case 1): sharedExp = floor(log2 amax) - emax with
      emax = 2 (E2M1's top binade), clamped to [-127, 127]; quantScale = 2^sharedExp;
      byte = sharedExp + 127; R = 1 / quantScale. An all-zero group has sharedExp -127.
    * dstTypeMax in {6.0, 7.0} (page: case 2): the exponent is ceil(log2 amax) - emax
      when the significand's leading one (6.0) or two (7.0) fraction bits are 1 and the
      remaining fraction bits are not all 0, otherwise floor(log2 amax) - emax.
    * any other dstTypeMax in [6, 12] (page: case 3): S = fp32(amax / dstTypeMax); take
      S's biased exponent E and mantissa field; E += 1 when S is normal, E < 254 and the
      mantissa field is nonzero; byte = E; R = 1 / fp32(2^(E - 127)).
    """
    amax32 = np.asarray(amax32, dtype=np.float32)
    D = float(dst_type_max)
    a64 = amax32.astype(np.float64)
    pos = a64 > 0
    safe = np.where(pos, a64, 1.0)
    if D == 0.0 or D in (6.0, 7.0):
        E = _floor_log2(safe)
        e = E - 2
        if D in (6.0, 7.0):
            frac = safe / np.ldexp(1.0, E) - 1.0  # fraction bits of the significand, [0, 1)
            lead = 0.5 if D == 6.0 else 0.75      # leading one / two fraction bits set
            lead_bits_set = frac >= lead
            rest_nonzero = frac != lead
            e = e + (lead_bits_set & rest_nonzero).astype(np.int64)
        e = np.where(pos, e, -127)
        e = np.clip(e, -127, 127)
        byte = (e + 127).astype(np.uint8)
        R = np.ldexp(1.0, -e)
        return byte, R
    # case 3: S in float32, exponent/mantissa fields of its IEEE-754 encoding
    S = (amax32 / np.float32(D)).astype(np.float32)
    bits = S.view(np.uint32).astype(np.int64)
    E = (bits >> 23) & 0xFF
    Mf = bits & 0x7FFFFF
    bump = (E >= 1) & (E < 254) & (Mf != 0)
    E = E + bump.astype(np.int64)
    byte = E.astype(np.uint8)
    s_ue8m0 = np.ldexp(1.0, E - 127).astype(np.float32)   # fp32(S_ue8m0)
    R = 1.0 / s_ue8m0.astype(np.float64)                   # exact power of two
    return byte, R


def mx_quantize(x2, dst_type_max):
    """Per-group mode quantizer (page: per-group mode, cases 1-3) on x'' [K, M, N].

    Returns (codes uint8 [K, M*N] E2M1 codes, group_bytes uint8 [K, G],
    v float32 [K, G, 32] values before the E2M1 rounding, amax float32 [K, G])."""
    groups, L = mx_group_view(x2)
    g32 = groups.astype(np.float32)
    amax = np.abs(g32).max(axis=-1)
    byte, R = mx_scale_exponent(amax, dst_type_max)
    v = (g32.astype(np.float64) * R[..., None]).astype(np.float32)
    codes = e2m1_encode(v).reshape(groups.shape[0], -1)[:, :L]
    return codes, byte, v, amax


def mx_scale_layout(group_bytes):
    """Place per-group E8M0 bytes in the page's [K, ceilDiv(M*N, 64), 2] scale tensor
    (group g at [k, g // 2, g % 2]); the spare slot of an odd group count holds 0x7F (2^0)."""
    group_bytes = np.asarray(group_bytes, dtype=np.uint8)
    K, G = group_bytes.shape
    out = np.full((K, -(-G // 2) * 2), 0x7F, dtype=np.uint8)
    out[:, :G] = group_bytes
    return out.reshape(K, -1, 2)


def flat_quant_per_token(x, P1, P2, clip_ratio, out_dtype="int4", intermediate=None):
    """Whole per-token path. Returns (out, quantScale, info):
    out is uint8 [K, M*N/2] for "int4" or int32 [K, M, N/8] for "int32" (same bytes).
    intermediate = "bf16" / "fp16" keeps x' in that type (rotate_rounded)."""
    x = np.asarray(x, dtype=np.float64)
    K, M, N = x.shape
    x2 = rotate(x, P1, P2) if intermediate is None else rotate_rounded(x, P1, P2, intermediate)
    codes, qscale, v = per_token_quantize(x2, clip_ratio)
    packed = pack_nibbles(codes.reshape(K, M * N))
    if out_dtype == "int32":
        out = np.ascontiguousarray(packed).view("<i4").reshape(K, M, N // 8)
    else:
        out = packed
    return out, qscale, {"x2": x2, "codes": codes, "v": v}


def flat_quant_mx(x, P1, P2, dst_type_max, intermediate=None):
    """Whole per-group path. Returns (out uint8 [K, M*N/2], scales uint8
    [K, ceilDiv(M*N, 64), 2], info). intermediate = "bf16" / "fp16" keeps x' in that
    type (rotate_rounded)."""
    x = np.asarray(x, dtype=np.float64)
    K, M, N = x.shape
    x2 = rotate(x, P1, P2) if intermediate is None else rotate_rounded(x, P1, P2, intermediate)
    codes, gbytes, v, amax = mx_quantize(x2, dst_type_max)
    out = pack_nibbles(codes)
    return out, mx_scale_layout(gbytes), {"x2": x2, "codes": codes, "v": v,
                                          "amax": amax, "group_bytes": gbytes}
