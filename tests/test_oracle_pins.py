"""Pins of the CPU oracle against values fixed by the page and by mathematics.

The page is "aclnnFlatQuantV2 complete guide: from two-level matmul to FP4 E2M1
quantization fusion" (http://www.zwxr.cn/news/277566). Each test names what it pins
and why a plausible slip in the oracle (a dropped term, a swapped operand, a wrong
exponent offset, a wrong rounding mode) would fail it. None of these tests touches a GPU.
"""

import os

import numpy as np
import pytest
import torch

import oracle
from oracle import flatquant as fq

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed=1234):
    return np.random.default_rng(seed)


def _haar(n, rng):
    q, r = np.linalg.qr(rng.standard_normal((n, n)))
    return q * np.sign(np.diag(r))[None, :]


# --------------------------------------------------------------------------------------
# rotation ("How it works": x' = x . kroneckerP2, x'' = kroneckerP1 . x')
# --------------------------------------------------------------------------------------

def test_rotation_matches_kronecker_brute_force():
    """vec_row(P1 X P2) = (P1 kron P2^T) vec_row(X): an explicit 16x16 operator on 4x4
    tokens pins the multiply order and both transposes."""
    rng = _rng()
    x = rng.standard_normal((2, 4, 4))
    P1 = rng.standard_normal((4, 4))
    P2 = rng.standard_normal((4, 4))
    big = np.kron(P1, P2.T)
    want = np.stack([(big @ x[k].reshape(-1)).reshape(4, 4) for k in range(2)])
    got = oracle.rotate(x, P1, P2)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_rotation_matches_scalar_loops():
    """x''[m,n] = sum_i sum_j P1[m,i] x[i,j] P2[j,n], written as plain loops (M != N)."""
    rng = _rng(7)
    K, M, N = 2, 3, 5
    x = rng.standard_normal((K, M, N))
    P1 = rng.standard_normal((M, M))
    P2 = rng.standard_normal((N, N))
    want = np.zeros((K, M, N))
    for k in range(K):
        for m in range(M):
            for n in range(N):
                s = 0.0
                for i in range(M):
                    for j in range(N):
                        s += P1[m, i] * x[k, i, j] * P2[j, n]
                want[k, m, n] = s
    np.testing.assert_allclose(oracle.rotate(x, P1, P2), want, rtol=0, atol=1e-12)


def test_rotation_orthogonal_preserves_frobenius_norm():
    """Orthogonal P1, P2 preserve each token's Frobenius norm."""
    rng = _rng(3)
    x = rng.standard_normal((5, 16, 24))
    x2 = oracle.rotate(x, _haar(16, rng), _haar(24, rng))
    np.testing.assert_allclose(np.linalg.norm(x2.reshape(5, -1), axis=1),
                               np.linalg.norm(x.reshape(5, -1), axis=1), rtol=1e-12)


def test_rotation_identity_and_skip():
    rng = _rng(4)
    x = rng.standard_normal((3, 6, 8))
    assert np.array_equal(oracle.rotate(x, np.eye(6), np.eye(8)), x)
    P1 = rng.standard_normal((6, 6))
    # kroneckerP2 = [0, 0] skips the right multiply (parameter table, per-group only)
    np.testing.assert_allclose(oracle.rotate(x, P1, np.zeros((0, 0))), P1 @ x, atol=1e-13)
    np.testing.assert_allclose(oracle.rotate(x, P1, None), P1 @ x, atol=1e-13)


# --------------------------------------------------------------------------------------
# per-token mode
# --------------------------------------------------------------------------------------

def _read_golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


def test_host_example_closed_form():
    """The page's complete host example (all-ones inputs, INT32 out)."""
    g = dict(ln.split() for ln in _read_golden_lines("host_example.txt"))
    K, M, N = int(g["K"]), int(g["M"]), int(g["N"])
    x = np.ones((K, M, N))
    P = np.ones((M, M))
    out, qs, info = oracle.flat_quant_per_token(x, P, np.ones((N, N)), 1.0, "int32")
    assert np.all(info["x2"] == float(g["x2"]))
    assert out.shape == (K, M, N // 8) and out.dtype == np.dtype("<i4")
    assert np.all(out == int(g["word"]))
    assert np.all(qs.view(np.uint32) == int(g["quantScale_bits"], 16))


def test_per_token_hand_worked():
    for ln in _read_golden_lines("hand_worked_groups.txt"):
        f = [s.strip() for s in ln.split("|")]
        if f[0] != "pt":
            continue
        clip = float(f[1])
        vals = np.array([float(s) for s in f[2].split()])
        want_codes = [int(s) for s in f[4].split()]
        tok = np.zeros((1, 4, 8))
        tok.reshape(-1)[: len(vals)] = vals
        codes, qs, _ = oracle.per_token_quantize(tok, clip)
        assert qs[0] == np.float32(float(f[3])), ln
        assert list(codes.reshape(-1)[: len(vals)]) == want_codes, ln
        assert np.all(codes.reshape(-1)[len(vals):] == 0)


def test_per_token_identity_matches_torch_quantize_per_tensor():
    """With P1 = P2 = I the per-token path is plain symmetric absmax quantization;
    torch.quantize_per_tensor (round half to even) gives the codes of every token."""
    rng = _rng(11)
    K, M, N = 6, 8, 16
    x = rng.standard_normal((K, M, N)).astype(np.float32).astype(np.float64)
    for clip in (1.0, 0.9, 0.55):
        codes, qs, _ = oracle.per_token_quantize(oracle.rotate(x, np.eye(M), np.eye(N)), clip)
        for k in range(K):
            q = torch.quantize_per_tensor(torch.from_numpy(x[k].astype(np.float32)),
                                          float(qs[k]), 0, torch.qint8)
            want = np.clip(q.int_repr().numpy().astype(np.int64), -8, 7)
            assert np.array_equal(codes[k].astype(np.int64), want)
        # quantScale * 7 / clipRatio recovers the token's absmax (closed form)
        amax = np.abs(x).reshape(K, -1).max(axis=1)
        np.testing.assert_allclose(qs.astype(np.float64) * 7.0 / clip, amax, rtol=2e-7)


def test_per_token_rounding_error_bound_and_range():
    """Unclamped codes are the nearest integers to x''/quantScale; with clipRatio 1 the
    largest element lands on +-7 and -8 never appears."""
    rng = _rng(12)
    x2 = rng.standard_normal((20, 8, 8)) * rng.lognormal(size=(20, 1, 1))
    codes, qs, v = oracle.per_token_quantize(x2, 1.0)
    assert codes.min() >= -7 and codes.max() <= 7
    assert np.all(np.abs(codes.reshape(20, -1)).max(axis=1) == 7)
    assert np.all(np.abs(v - codes) <= 0.5)


def test_per_token_zero_token():
    codes, qs, _ = oracle.per_token_quantize(np.zeros((2, 4, 4)), 0.7)
    assert np.all(qs == 0) and np.all(codes == 0)


def test_per_token_power_of_two_scale_invariance():
    """Scaling a token by 2^j scales quantScale by 2^j and leaves every code unchanged."""
    rng = _rng(13)
    x2 = rng.standard_normal((4, 8, 8))
    c0, q0, _ = oracle.per_token_quantize(x2, 0.8)
    for j in (-5, 3, 17):
        c1, q1, _ = oracle.per_token_quantize(x2 * 2.0 ** j, 0.8)
        assert np.array_equal(c0, c1)
        assert np.array_equal(q1, (q0.astype(np.float64) * 2.0 ** j).astype(np.float32))


# --------------------------------------------------------------------------------------
# packing (parameter table: INT4 two per byte, INT32 = eight INT4 along the last axis)
# --------------------------------------------------------------------------------------

def test_pack_nibbles_order():
    assert list(oracle.pack_nibbles(np.array([1, 2]))) == [0x21]
    assert list(oracle.pack_nibbles(np.array([-1, 7, -8, 0]))) == [0x7F, 0x08]
    words = oracle.pack_nibbles(np.arange(8)[None, :]).view("<i4")
    assert words[0, 0] == 0x76543210


# --------------------------------------------------------------------------------------
# E2M1 cast and per-group mode
# --------------------------------------------------------------------------------------

def _e2m1_by_scaling(v):
    """Independent E2M1 cast: scale each value into its binade's integer grid and round
    half to even there (binade spacing 0.5 below 2, 1 in [2,4), 2 in [4,8)), saturate."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    step = np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0))
    q = np.minimum(np.rint(a / step) * step, 6.0)
    idx = np.searchsorted(oracle.E2M1_GRID, q)
    return (idx | (((v < 0) & (idx > 0)) << 3)).astype(np.uint8)


def test_e2m1_grid_and_ties():
    grid = oracle.E2M1_GRID
    assert list(oracle.e2m1_encode(grid)) == list(range(8))
    assert list(oracle.e2m1_encode(-grid[1:])) == [8 + c for c in range(1, 8)]
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    assert list(oracle.e2m1_decode(oracle.e2m1_encode(mids))) == [0, 1, 1, 2, 2, 4, 4]
    assert list(oracle.e2m1_encode([6.5, 100.0, -7.0])) == [7, 7, 15]
    assert list(oracle.e2m1_encode([0.0, -0.0, -0.1, 0.1, -0.25])) == [0, 0, 0, 0, 0]


def test_e2m1_matches_independent_scaled_rounding():
    rng = _rng(21)
    v = np.concatenate([rng.uniform(-8, 8, 20000), rng.standard_normal(2000) * 0.3,
                        np.arange(-70, 71) / 10.0, np.arange(-32, 33) / 4.0])
    assert np.array_equal(oracle.e2m1_encode(v), _e2m1_by_scaling(v))


def _mx_group(vals):
    g = np.zeros((1, 1, 32))
    g.reshape(-1)[: len(vals)] = vals
    return g


def test_mx_hand_worked_groups():
    n = 0
    for ln in _read_golden_lines("hand_worked_groups.txt"):
        f = [s.strip() for s in ln.split("|")]
        if f[0] != "mx":
            continue
        D = float(f[1])
        vals = [float(s) for s in f[2].split()]
        codes, gbytes, _, _ = oracle.mx_quantize(_mx_group(vals), D)
        assert int(gbytes[0, 0]) == int(f[3]), ln
        assert [int(c) for c in codes[0, : len(vals)]] == [int(s, 16) for s in f[4].split()], ln
        assert np.all(codes[0, len(vals):] == 0)
        n += 1
    assert n >= 10


def _amax_f32(rng, n):
    return (rng.lognormal(0, 4, n) * rng.choice([1, 1, 1, 0], n)).astype(np.float32)


def test_mx_case1_exponent_is_floor_log2_minus_2():
    """Case 1: 2^(e+2) <= amax < 2^(e+3), found by brute force over e."""
    rng = _rng(31)
    a = _amax_f32(rng, 3000)
    byte, R = oracle.mx_scale_exponent(a, 0.0)
    for ai, bi, ri in zip(a.astype(np.float64), byte, R):
        e = int(bi) - 127
        assert ri == 2.0 ** -e
        if ai == 0:
            assert bi == 0
            continue
        want = next(t for t in range(-140, 140) if 2.0 ** (t + 2) <= ai < 2.0 ** (t + 3))
        assert e == max(want, -127)


@pytest.mark.parametrize("D", [6.0, 7.0])
def test_mx_case2_is_smallest_exponent_within_dst_max(D):
    """Case 2: for dstTypeMax in (4, 8), the mantissa check picks the smallest e with
    amax / 2^e <= dstTypeMax (brute force over e)."""
    rng = _rng(32)
    a = _amax_f32(rng, 3000)
    # values on and next to the thresholds 1.5*2^E / 1.75*2^E
    edge = np.array([1.5, 1.75], dtype=np.float32)
    a = np.concatenate([a, edge, np.nextafter(edge, np.float32(3)), edge * 8, edge / 4])
    byte, R = oracle.mx_scale_exponent(a, D)
    for ai, bi in zip(a.astype(np.float64), byte):
        if ai == 0:
            assert bi == 0
            continue
        want = next(t for t in range(-140, 140) if ai / 2.0 ** t <= D)
        assert int(bi) - 127 == want


@pytest.mark.parametrize("D", [8.0, 10.0, 12.0, 9.5])
def test_mx_case3_is_smallest_power_covering_fp32_scale(D):
    """Case 3: byte E is the smallest E with fp32(amax/D) <= 2^(E-127) (normal S)."""
    rng = _rng(33)
    a = _amax_f32(rng, 3000)
    byte, R = oracle.mx_scale_exponent(a, D)
    S = (a / np.float32(D)).astype(np.float32).astype(np.float64)
    for si, bi, ri in zip(S, byte, R):
        if si == 0:
            assert bi == 0
            continue
        want = next(E for E in range(1, 255) if si <= 2.0 ** (E - 127))
        assert int(bi) == want
        assert ri == 2.0 ** (127 - int(bi))


def test_mx_identity_reconstruction_bound():
    """With P1 = P2 = I, unsaturated elements reconstruct to within half an E2M1 step
    times the group scale, and the group's maximum never exceeds dstTypeMax*scale
    for cases 2 and 3 (no overflow by construction)."""
    rng = _rng(34)
    K, M, N = 4, 8, 64
    x = (rng.standard_normal((K, M, N)) * rng.lognormal(0, 2, (K, 1, 1))).astype(np.float32)
    for D in (0.0, 6.0, 7.0, 10.0):
        out, scales, info = oracle.flat_quant_mx(x, np.eye(M), np.eye(N), D)
        codes = info["codes"].reshape(K, -1, 32)
        e = info["group_bytes"].astype(np.int64) - 127
        recon = oracle.e2m1_decode(codes) * (2.0 ** e)[..., None]
        xg = x.reshape(K, -1, 32).astype(np.float64)
        v = xg / (2.0 ** e)[..., None]
        step = np.where(np.abs(v) < 2, 0.5, np.where(np.abs(v) < 4, 1.0, 2.0))
        unsat = np.abs(v) <= 6.0
        assert np.all(np.abs(recon - xg)[unsat] <= (0.5 * step * (2.0 ** e)[..., None])[unsat])
        if D:
            assert np.all(np.abs(v).max(axis=-1) <= D)


def test_mx_power_of_two_shift_invariance():
    """Scaling x by 2^j shifts every E8M0 byte by j and leaves every code unchanged."""
    rng = _rng(35)
    x2 = rng.standard_normal((3, 4, 48)) * 3
    for D in (0.0, 6.0, 7.0, 10.0):
        c0, b0, _, _ = oracle.mx_quantize(x2, D)
        for j in (-9, 4):
            c1, b1, _, _ = oracle.mx_quantize(x2 * 2.0 ** j, D)
            assert np.array_equal(c0, c1)
            assert np.array_equal(b1.astype(int), b0.astype(int) + j)


def test_mx_groups_straddle_rows_and_pad():
    """Groups run over the flattened [K, M*N] axis, across row ends (N = 112 gives 3.5
    groups per row), and a short last group is zero padded; the scale tensor is
    [K, ceilDiv(M*N, 64), 2] with the spare slot of an odd group count holding 0x7F (2^0)."""
    rng = _rng(36)
    x2 = rng.standard_normal((2, 3, 14))  # M*N = 42: one full group + a group of 10
    codes, gbytes, v, amax = oracle.mx_quantize(x2, 0.0)
    flat = x2.reshape(2, -1).astype(np.float32)
    assert np.array_equal(amax[:, 0], np.abs(flat[:, :32]).max(axis=1))
    assert np.array_equal(amax[:, 1], np.abs(flat[:, 32:]).max(axis=1))
    sc = oracle.mx_scale_layout(gbytes)
    assert sc.shape == (2, 1, 2)
    x3 = rng.standard_normal((2, 1, 96))  # three groups -> ceilDiv(96, 64) = 2 -> pad slot
    _, gb3, _, _ = oracle.mx_quantize(x3, 0.0)
    sc3 = oracle.mx_scale_layout(gb3)
    assert sc3.shape == (2, 2, 2) and np.all(sc3[:, 1, 1] == 0x7F)
    assert np.array_equal(sc3.reshape(2, -1)[:, :3], gb3)


def test_flat_quant_mx_output_layout():
    rng = _rng(37)
    K, M, N = 3, 4, 16
    x = rng.standard_normal((K, M, N))
    out, scales, info = oracle.flat_quant_mx(x, _haar(M, rng), _haar(N, rng), 0.0)
    assert out.shape == (K, M * N // 2) and out.dtype == np.uint8
    assert scales.shape == (K, 1, 2)
    lo = out & 0xF
    hi = out >> 4
    assert np.array_equal(lo, info["codes"][:, 0::2]) and np.array_equal(hi, info["codes"][:, 1::2])


# --------------------------------------------------------------------------------------
# planted mistakes: each pin above must catch at least one of these, on the CPU
# --------------------------------------------------------------------------------------

def test_planted_mistakes_are_caught(monkeypatch):
    rng = _rng(41)
    x = rng.standard_normal((2, 4, 4))
    P1, P2 = rng.standard_normal((4, 4)), rng.standard_normal((4, 4))
    big = np.kron(P1, P2.T)
    want = np.stack([(big @ x[k].reshape(-1)).reshape(4, 4) for k in range(2)])
    # a transposed right operand
    assert not np.allclose(np.matmul(P1, np.matmul(x, P2.T)), want)
    # the two matmuls applied in the wrong places
    assert not np.allclose(np.matmul(P2, np.matmul(x, P1)), want)

    # a case-1 exponent offset of 3 instead of 2 fails the hand-worked group
    real = fq._floor_log2
    monkeypatch.setattr(fq, "_floor_log2", lambda a: real(a) - 1)
    _, gbytes, _, _ = oracle.mx_quantize(_mx_group([0.3, -1.1, 5.0, 2.6]), 0.0)
    assert int(gbytes[0, 0]) != 127
    monkeypatch.setattr(fq, "_floor_log2", real)

    # ties away from zero instead of to even fails the E2M1 tie pin
    def away(v):
        v = np.asarray(v, dtype=np.float64)
        d = np.abs(np.abs(v)[..., None] - fq.E2M1_GRID)
        idx = (d.shape[-1] - 1) - np.argmin(d[..., ::-1], axis=-1)
        return (idx | ((v < 0) << 3)).astype(np.uint8)
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    assert list(fq.e2m1_decode(away(mids))) != [0, 1, 1, 2, 2, 4, 4]

    # dropping clipRatio fails the clip-0.9 hand-worked token
    tok = np.zeros((1, 2, 4))
    tok.reshape(-1)[:3] = [3.5, 1.25, -3.5]
    codes_no_clip, _, _ = oracle.per_token_quantize(tok, 1.0)
    assert list(codes_no_clip.reshape(-1)[:3]) != [7, 3, -8]


# --------------------------------------------------------------------------------------
# intermediate rounding (x' kept in the input type between the two products)
# --------------------------------------------------------------------------------------

def test_rounded_intermediate_tie_and_exact_sum():
    """Hand cases pin the reading x' = round16(exact x . P2). Tie: x' = 1 + 2^-8 is halfway
    between the bf16 neighbours 1 and 1 + 2^-7, so it rounds to the even one, 1 (fp16 holds
    it exactly). Exactness: 2^24 + 1 - 2^24 is 1 (a float32 running sum in index order would
    give 0). Just above the tie: 1 + 2^-8 + 2^-60 rounds up to 1 + 2^-7, although its float64
    sum is the tie itself (this takes the oracle's exact-rational branch). A rounding step
    dropped, a float32 or float64 sum used as if exact, or a wrong tie rule fails one."""
    P1 = np.ones((1, 1))
    x = np.array([[[1.0, 2.0 ** -8]]])
    P2 = np.array([[1.0, 0.0], [1.0, 0.0]])
    assert oracle.rotate_rounded(x, P1, P2, "bf16")[0, 0, 0] == 1.0
    assert oracle.rotate_rounded(x, P1, P2, "fp16")[0, 0, 0] == 1.0 + 2.0 ** -8
    assert oracle.rotate(x, P1, P2)[0, 0, 0] == 1.0 + 2.0 ** -8
    x = np.array([[[2.0 ** 24, 1.0, -(2.0 ** 24)]]])
    P2 = np.ones((3, 3))
    assert np.all(oracle.rotate_rounded(x, P1, P2, "bf16") == 1.0)
    x = np.array([[[1.0, 2.0 ** -8, 2.0 ** -60]]])
    P2 = np.zeros((3, 3))
    P2[:, 0] = 1.0
    assert oracle.rotate_rounded(x, P1, P2, "bf16")[0, 0, 0] == 1.0 + 2.0 ** -7
    assert oracle.rotate_rounded(x, P1, P2, "fp16")[0, 0, 0] == 1.0 + 2.0 ** -8
    x = np.array([[[-1.0, -(2.0 ** -8), -(2.0 ** -60)]]])
    assert oracle.rotate_rounded(x, P1, P2, "bf16")[0, 0, 0] == -(1.0 + 2.0 ** -7)


def _int_round_half_even(num, shift):
    """num / 2^shift (shift >= 0) rounded to an integer, ties to even, in integers."""
    if shift == 0:
        return num
    q, r = divmod(num, 1 << shift)
    half = 1 << (shift - 1)
    if r > half or (r == half and q % 2 == 1):
        q += 1
    return q


def test_rounded_intermediate_on_integer_grid_matches_integer_arithmetic():
    """x on the grid k / 8 and P2 on the grid j / 16 (|k|, |j| <= 15): every x' element is an
    integer multiple of 2^-7, computed here with Python integers. Rounded to 8 significant
    bits (bf16) or 11 (fp16) with an integer ties-to-even rule, it must equal the oracle's x'
    (read back through P1 = I). Ties occur on this grid, so a wrong tie rule, a truncation or
    a transposed P2 fails."""
    rng = _rng(79)
    K, M, N = 3, 8, 24
    xi = rng.integers(-15, 16, size=(K, M, N))
    pi = rng.integers(-15, 16, size=(N, N))
    x = xi / 8.0
    P2 = pi / 16.0
    ties = 0
    for dtype, p in (("bf16", 8), ("fp16", 11)):
        got = oracle.rotate_rounded(x, np.eye(M), P2, dtype)
        for k in range(K):
            for m in range(M):
                for n in range(N):
                    s = int(sum(int(xi[k, m, j]) * int(pi[j, n]) for j in range(N)))  # x' * 2^7
                    a = abs(s)
                    if a == 0:
                        want = 0.0
                    else:
                        shift = max(a.bit_length() - p, 0)
                        r = _int_round_half_even(a, shift)
                        want = float(r) * 2.0 ** (shift - 7)
                        if shift > 0 and a % (1 << shift) == 1 << (shift - 1):
                            ties += 1
                    want = -want if s < 0 else want
                    assert got[k, m, n] == want, (dtype, k, m, n, s)
    assert ties > 0


def test_round_f64_to_16bit_ties_subnormals_overflow():
    """Direct float64 -> 16-bit rounding: agrees with torch's casts on float32 values (ties
    and subnormals included); a value just above a tie, which a float32 step would turn into
    the tie, rounds up; fp16 overflows to inf at 65520 and keeps 65504 below it; half the
    smallest fp16 subnormal rounds to 0 (even), three quarters of it to 2^-24."""
    rng = _rng(80)
    v = np.concatenate([
        (rng.standard_normal(20000) * np.exp(rng.uniform(-30, 30, 20000))).astype(np.float32),
        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 2.0 ** -130, 0.0], dtype=np.float32)])
    want_bf = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(fq.round_f64_to_16bit(v.astype(np.float64), "bf16"), want_bf)
    small = v[np.abs(v) < 60000]
    want_h = torch.from_numpy(small).to(torch.float16).to(torch.float64).numpy()
    assert np.array_equal(fq.round_f64_to_16bit(small.astype(np.float64), "fp16"), want_h)
    assert fq.round_f64_to_16bit(np.array([1 + 2 ** -8 + 2 ** -40]), "bf16")[0] == 1 + 2 ** -7
    h = fq.round_f64_to_16bit(np.array([65519.99, 65520.0, 2.0 ** -25, 0.75 * 2.0 ** -24]), "fp16")
    assert h[0] == 65504.0 and np.isinf(h[1]) and h[2] == 0.0 and h[3] == 2.0 ** -24


def test_round_to_16bit_matches_torch_casts():
    """The oracle's bf16 rounding (on the float32 bit pattern) and fp16 rounding agree with
    torch's float32 -> bfloat16 / float16 casts, ties and subnormals included."""
    rng = _rng(77)
    v = np.concatenate([
        (rng.standard_normal(20000) * np.exp(rng.uniform(-30, 30, 20000))).astype(np.float32),
        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 2.0 ** -130, 0.0, -0.0],
                 dtype=np.float32)])
    want_bf = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(oracle.round_to_16bit(v, "bf16"), want_bf)
    small = v[np.abs(v) < 60000]
    want_h = torch.from_numpy(small).to(torch.float16).to(torch.float64).numpy()
    assert np.array_equal(oracle.round_to_16bit(small, "fp16"), want_h)


def test_rounded_intermediate_identity_and_skip_reduce_to_exact_path():
    """With P2 = I every x' sum has one nonzero term, so x' = x exactly and the rounded path
    equals the exact one; skipping P2 (per-group mode) does too."""
    rng = _rng(78)
    x = torch.from_numpy(rng.standard_normal((3, 8, 16))).to(torch.bfloat16).double().numpy()
    P1 = rng.standard_normal((8, 8))
    assert np.array_equal(oracle.rotate_rounded(x, P1, np.eye(16)), oracle.rotate(x, P1, np.eye(16)))
    assert np.array_equal(oracle.rotate_rounded(x, P1, None), oracle.rotate(x, P1, None))
