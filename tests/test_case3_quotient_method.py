"""Both kernels decide the case-3 byte ("per-group mode", case 3: S = amax / dstTypeMax in
FP32, then E += 1 when S is normal, E < 254 and its mantissa is nonzero) without dividing.
They form q = fp32(amax * fp32(1 / D)), D = fp32(dstTypeMax): q is within 2.5 ulp of S, so
when q's exponent field is in [1, 253] and its mantissa field in [4, 2^23 - 5] the byte is
q's exponent field plus one. Otherwise (rare) q is next to a power of two 2^k and S <= 2^k
exactly when amax - D 2^k <= D 2^(k - 24), a difference one FMA gives exactly (the two
terms are within a factor two: Sterbenz); the byte is then k + 127, else k + 128. This CPU
test restates that rule with numpy float32 arithmetic (the exact difference taken in
float64) and checks it against the oracle's bytes, which come from numpy's correctly
rounded float32 division: on random maxima down to subnormal ones, on maxima a few ulps around D * 2^k (where the
byte turns), and on maxima whose quotient falls next to an fp32 midpoint. It also checks
that the rare branch is rare on maxima of ordinary size."""

import numpy as np
import pytest

import oracle


def _method_byte(amax, D):
    """(common-path mask, byte) of the kernels' rule; exact differences taken in float64."""
    a = np.asarray(amax, dtype=np.float32)
    D32 = np.float32(D)
    inv32 = np.float32(1.0 / np.float64(D32))
    q = (a * inv32).astype(np.float32)
    qb = q.view(np.uint32).astype(np.int64)
    Eq, Mq = (qb >> 23) & 0xFF, qb & 0x7FFFFF
    common = (Eq >= 1) & (Eq <= 253) & (Mq >= 4) & (Mq <= 0x7FFFFA)
    k = np.where(Eq == 0, -126, np.where(Mq <= 3, Eq - 127, Eq - 126))
    # S next to 2^-126: 0 (subnormal S), 1 (S = 2^-126) or 2, from terms scaled by 2^64 (only
    # used there: for large amax the scaled term overflows to inf and is not read)
    with np.errstate(over="ignore"):
        a64 = (a.astype(np.float64) * 2.0 ** 64).astype(np.float32)
    r0 = (a64.astype(np.float64) - np.float64(D32) * 2.0 ** -62).astype(np.float32)
    t0 = np.float32(np.float64(D32) * 2.0 ** -86)
    bottom = np.where(r0 > t0, 2, np.where(r0 >= -t0, 1, 0))
    kk = np.maximum(k, -125)
    r = (a.astype(np.float64) - np.float64(D32) * np.ldexp(1.0, kk)).astype(np.float32)
    t = (np.float64(D32) * np.ldexp(1.0, kk - 24)).astype(np.float32)
    near = np.where(r <= t, kk + 127, kk + 128)
    return common, np.where(common, Eq + 1, np.where(k <= -126, bottom, near))


def _cases(D, rng):
    rand = np.abs((rng.standard_normal(200000) * np.exp2(rng.integers(-149, 120, 200000))).astype(np.float32))
    base = (np.float32(D) * np.exp2(np.arange(-149, 124)).astype(np.float32)).astype(np.float32)
    near = [base]
    up, dn = base, base
    for _ in range(8):
        up = np.nextafter(up, np.float32(np.inf))
        dn = np.nextafter(dn, np.float32(0))
        near += [up, dn]
    # quotients next to an fp32 midpoint: amax = fp32(D * (m + half ulp)) for random m
    m = (1.0 + rng.random(50000)) * np.exp2(rng.integers(-30, 30, 50000))
    m32 = m.astype(np.float32).astype(np.float64)
    ulp = np.spacing(m32.astype(np.float32)).astype(np.float64)
    mid = (np.float64(np.float32(D)) * (m32 + ulp / 2)).astype(np.float32)
    a = np.concatenate([rand] + near + [mid, np.nextafter(mid, np.float32(np.inf)),
                                        np.nextafter(mid, np.float32(0))])
    return a[np.isfinite(a) & (a > 0)]


@pytest.mark.parametrize("D", [6.5, 8.0, 9.5, 10.0, 11.0, 12.0, 10.3, 7.25, 11.9])
def test_rule_gives_the_bytes_of_the_correctly_rounded_quotient(D):
    rng = np.random.default_rng(int(D * 100))
    a = _cases(D, rng)
    byte, _ = oracle.mx_scale_exponent(a, D)
    common, b = _method_byte(a, D)
    np.testing.assert_array_equal(b, byte.astype(np.int64))
    assert common.any() and (~common).any()
    ordinary = np.abs(rng.standard_normal(200000).astype(np.float32) * np.float32(3.0))
    c, _ = _method_byte(ordinary[ordinary > 0], D)
    assert c.mean() > 0.99999
