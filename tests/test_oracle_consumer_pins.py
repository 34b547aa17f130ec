"""Pins of the consumer-side oracle (unpacking, dequantization, FP4 x FP4 contraction).

Page: "aclnnFlatQuantV2 complete guide: from two-level matmul to FP4 E2M1 quantization
fusion" (http://www.zwxr.cn/news/277566), "per-token mode" (quantScale is emitted for
later dequantization) and "per-group mode" cases 1-3 (the encodings that the
dequantization inverts). Each test says which slip it catches: a swapped nibble, an
exponent offset off by one, a group index taken per row instead of per flattened token,
a transposed operand. None of these tests touches a GPU.
"""

from fractions import Fraction

import numpy as np
import pytest

from oracle import consumer as cs
from oracle import flatquant as fq

CASES = [0.0, 6.0, 7.0, 10.0]


def _rng(seed=99):
    return np.random.default_rng(seed)


def test_unpack_inverts_pack_for_every_byte():
    """All 256 bytes: unpack then pack gives the byte back; 0x21 is element 0 = 1 (bits 0-3)
    and element 1 = 2 (bits 4-7), the LSB-first order of the packing."""
    b = np.arange(256, dtype=np.uint8).reshape(1, 256)
    n = cs.unpack_nibbles(b, 512)
    assert np.array_equal(fq.pack_nibbles(n), b)
    assert list(cs.unpack_nibbles(np.array([[0x21]], np.uint8), 2)[0]) == [1, 2]


def test_code_values_hand():
    """INT4 two's complement and the E2M1 table, written out."""
    assert list(cs.int4_value(np.arange(16))) == [0, 1, 2, 3, 4, 5, 6, 7, -8, -7, -6, -5, -4, -3, -2, -1]
    want = [0, 0.5, 1, 1.5, 2, 3, 4, 6, 0, -0.5, -1, -1.5, -2, -3, -4, -6]
    assert list(cs.e2m1_value(np.arange(16, dtype=np.uint8))) == want


def test_per_token_dequant_host_example():
    """The page's host example (x = 1, P1 = P2 = ones(16, 16)): x'' = 256, every code 7 and
    quantScale = fp32(256 / 7), so every dequantized element is 7 * fp32(256 / 7), within
    one fp32 ulp of 256; the INT32 bytes dequantize the same."""
    x = np.ones((2, 16, 16))
    P = np.ones((16, 16))
    for fmt in ("int4", "int32"):
        out, qs, _ = fq.flat_quant_per_token(x, P, P, 1.0, fmt)
        xh = cs.dequantize_per_token(out, qs, 16, 16)
        assert np.all(xh == 7.0 * float(np.float32(256.0 / 7.0)))
        assert np.all(np.abs(xh - 256.0) <= 256.0 * 2.0 ** -23)


def test_per_token_dequant_error_bound():
    """Identity rotation, clipRatio 1: |x_hat - x| <= quantScale / 2 (plus the float32
    rounding of x / quantScale), and the token's largest element comes back to within that
    bound of itself. A code taken from the wrong nibble breaks the bound."""
    rng = _rng(3)
    K, M, N = 5, 8, 12
    x = rng.standard_normal((K, M, N)) * rng.lognormal(0, 1, (K, 1, 1))
    out, qs, _ = fq.flat_quant_per_token(x, np.eye(M), np.eye(N), 1.0)
    xh = cs.dequantize_per_token(out, qs, M, N)
    bound = qs.astype(np.float64)[:, None, None] * (0.5 + 1e-5)
    assert np.all(np.abs(xh - x) <= bound)


def _on_grid_tokens(rng, K, M, N):
    """Tokens whose every 32-group holds E2M1 grid values times 2^e_g with one element at
    +-6 * 2^e_g: every dstTypeMax rule then picks byte e_g + 127 and encodes the group
    exactly. e_g varies per group, so a group index or an exponent offset taken wrong
    shows up in the values."""
    L = M * N
    G = -(-L // 32)
    e = rng.integers(-20, 20, size=(K, G))
    mags = fq.E2M1_GRID[rng.integers(0, 8, size=(K, G * 32))]
    signs = np.where(rng.random((K, G * 32)) < 0.5, -1.0, 1.0)
    v = (mags * signs).reshape(K, G, 32)
    v[:, :, 5] = np.where(rng.random((K, G)) < 0.5, -6.0, 6.0)
    x = (v * np.ldexp(1.0, e)[:, :, None]).reshape(K, G * 32)[:, :L]
    return x.reshape(K, M, N), e


@pytest.mark.parametrize("D", CASES)
def test_mx_dequant_exact_on_grid(D):
    """Quantize (identity rotation) then dequantize returns grid-valued tokens exactly, for
    every dstTypeMax rule; M * N = 144 gives groups that straddle rows and a padded last
    group."""
    rng = _rng(11)
    K, M, N = 3, 3, 48
    x, e = _on_grid_tokens(rng, K, M, N)
    out, scales, info = fq.flat_quant_mx(x, np.eye(M), np.eye(N), D)
    assert np.array_equal(info["group_bytes"].astype(np.int64), e + 127)
    xh = cs.dequantize_mx(out, scales, M, N)
    assert np.array_equal(xh, x)


@pytest.mark.parametrize("D", CASES)
def test_mx_dequant_error_bound(D):
    """Random tokens (identity rotation): every element comes back within one grid step of
    its group's scale 2^(byte - 127), or within the saturation margin above 6 that its rule
    allows (case 1: values below 8; cases 2 and 3: values up to dstTypeMax). An exponent
    offset off by one doubles or halves the large elements and breaks the bound."""
    rng = _rng(5)
    K, M, N = 4, 4, 40
    x = rng.standard_normal((K, M, N)) * rng.lognormal(0, 2, (K, 1, 1))
    out, scales, info = fq.flat_quant_mx(x, np.eye(M), np.eye(N), D)
    xh = cs.dequantize_mx(out, scales, M, N).reshape(K, -1)
    L = M * N
    step = np.ldexp(1.0, np.repeat(info["group_bytes"].astype(np.int64), 32, axis=1)[:, :L] - 127)
    top = 8.0 if D == 0.0 else D
    margin = max(1.0, top - 6.0) * (1 + 1e-6)
    assert np.all(np.abs(xh - x.reshape(K, -1)) <= margin * step)
    # the largest element of each token never dequantizes to 0
    big = np.abs(x.reshape(K, -1)) == np.abs(x.reshape(K, -1)).max(axis=1, keepdims=True)
    assert np.all(np.abs(xh[big]) > 0)


def _random_mx_operand(rng, R, L):
    codes = rng.integers(0, 16, size=(R, L), dtype=np.uint8)
    G = -(-L // 32)
    gb = rng.integers(120, 135, size=(R, G)).astype(np.uint8)
    return fq.pack_nibbles(codes), fq.mx_scale_layout(gb), codes, gb


def test_mx_matmul_matches_exact_rational_loops():
    """C[t, o] = sum_i A_hat[t, i] W_hat[o, i], summed exactly in rationals by plain loops
    (the values are dyadic, so the fp64 result must equal it exactly). L = 96 spans three
    groups, so a scale taken from the wrong group or a transposed operand fails."""
    rng = _rng(21)
    T, O, L = 3, 2, 96
    a, a_s, ac, ag = _random_mx_operand(rng, T, L)
    w, w_s, wc, wg = _random_mx_operand(rng, O, L)
    got = cs.mx_matmul(a, a_s, w, w_s, L)
    table = [Fraction(v).limit_denominator() for v in [0, 0.5, 1, 1.5, 2, 3, 4, 6]]

    def val(code, byte):
        mag = table[int(code) & 7]
        s = -mag if int(code) & 8 else mag
        return s * (Fraction(2) ** (int(byte) - 127))

    for t in range(T):
        for o in range(O):
            acc = Fraction(0)
            for i in range(L):
                acc += val(ac[t, i], ag[t, i // 32]) * val(wc[o, i], wg[o, i // 32])
            assert Fraction(got[t, o]) == acc


def test_mx_matmul_one_hot_weights_select_columns():
    """A weight row that is E2M1 1.0 (code 0x2, byte 127) at column j and 0 elsewhere makes
    output column o equal to dequantized activation column j."""
    rng = _rng(8)
    M, N = 4, 24
    L = M * N
    x = rng.standard_normal((6, M, N))
    a, a_s, _ = fq.flat_quant_mx(x, np.eye(M), np.eye(N), 0.0)
    cols = [0, 31, 32, 95]
    wc = np.zeros((len(cols), L), dtype=np.uint8)
    for o, j in enumerate(cols):
        wc[o, j] = 0x2
    wg = np.full((len(cols), -(-L // 32)), 127, dtype=np.uint8)
    C = cs.mx_matmul(a, a_s, fq.pack_nibbles(wc), fq.mx_scale_layout(wg), L)
    A_hat = cs.dequantize_mx(a, a_s, M, N).reshape(6, L)
    assert np.array_equal(C, A_hat[:, cols])


def test_mx_matmul_scale_shift():
    """Raising every weight byte by 3 multiplies the product by 2^3 exactly; raising one
    group's activation bytes moves only that group's share."""
    rng = _rng(13)
    T, O, L = 4, 3, 64
    a, a_s, ac, ag = _random_mx_operand(rng, T, L)
    w, w_s, wc, wg = _random_mx_operand(rng, O, L)
    C = cs.mx_matmul(a, a_s, w, w_s, L)
    C3 = cs.mx_matmul(a, a_s, w, fq.mx_scale_layout(wg + 3), L)
    assert np.array_equal(C3, 8.0 * C)
    ag2 = ag.copy()
    ag2[:, 1] += 1
    C1 = cs.mx_matmul(a, fq.mx_scale_layout(ag2), w, w_s, L)
    ac_g1 = ac.copy()
    ac_g1[:, :32] = 0  # group 0 zeroed: what is left is group 1's share
    a_only_g1 = cs.mx_matmul(fq.pack_nibbles(ac_g1), a_s, w, w_s, L)
    assert np.array_equal(C1 - C, a_only_g1)


def test_planted_mistakes_are_caught(monkeypatch):
    """Each slip below, planted in the oracle on the CPU, makes one of the pins above fail."""
    rng = _rng(17)
    # an E8M0 offset of 126 instead of 127 fails the exact on-grid round trip
    x, _ = _on_grid_tokens(rng, 2, 3, 48)
    out, scales, _ = fq.flat_quant_mx(x, np.eye(3), np.eye(48), 0.0)
    real_ldexp = cs.np.ldexp

    class _OffByOne:
        def __getattr__(self, name):
            return getattr(np, name)

        @staticmethod
        def ldexp(a, b):
            return real_ldexp(a, np.asarray(b) + 1)
    monkeypatch.setattr(cs, "np", _OffByOne())
    assert not np.array_equal(cs.dequantize_mx(out, scales, 3, 48), x)
    monkeypatch.setattr(cs, "np", np)

    # swapped nibbles fail the LSB-first unpack pin
    def swapped(packed, L):
        n = cs.unpack_nibbles(packed, L)
        return n.reshape(n.shape[:-1] + (-1, 2))[..., ::-1].reshape(n.shape)
    assert list(swapped(np.array([[0x21]], np.uint8), 2)[0]) != [1, 2]

    # one byte per row of N instead of per 32 flattened elements fails the round trip
    gb = cs.group_bytes_from_layout(scales, 144).astype(np.int64)
    codes = cs.unpack_nibbles(out.reshape(2, -1), 144)
    per_row = np.repeat(gb[:, :3], 48, axis=1)
    wrong = (cs.e2m1_value(codes) * np.ldexp(1.0, per_row - 127)).reshape(2, 3, 48)
    assert not np.array_equal(wrong, x)
