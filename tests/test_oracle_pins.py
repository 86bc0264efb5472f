"""Pins for the CPU oracle, independent of the oracle itself.

Each test checks the oracle against something the pages or mathematics fix:
the hand-worked example, the packing layout example, exhaustive round trips,
closed forms (Gaussian zero fraction, identity weights, constant rows),
library routines (math.fsum, torch's bf16 cast, numpy's integer matmul),
exact rational arithmetic (fractions.Fraction) and invariants of the method.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from conftest import load_golden, parse_float, rn32_of_fraction

FLOOR = np.float32(1e-5)


def bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


# --------------------------------------------------------------------------
# Worked examples
# --------------------------------------------------------------------------
def test_hand_example_every_stage(O):
    g = load_golden("hand_example_4x8.txt")
    W = np.array([[parse_float(v) for v in g["W_row%d" % i]] for i in range(4)], np.float32)
    t_exp = np.array([[int(v) for v in g["t_row%d" % i]] for i in range(4)], np.int8)
    P_exp = np.array([[int(v, 16) for v in g["P_hex"]]], np.uint8)
    x = np.array([[parse_float(v) for v in g["x_row%d" % i]] for i in range(4)], np.float32)
    s_exp = np.array([parse_float(v) for v in g["s_x"]], np.float32)
    q_exp = np.array([[int(v) for v in g["q_row%d" % i]] for i in range(4)], np.int8)
    acc_exp = np.array([[int(v) for v in g["acc_row%d" % i]] for i in range(4)], np.int32)
    y_exp = np.array([[rn32_of_fraction(Fraction(v)) for v in g["y_row%d" % i]]
                      for i in range(4)], np.float32)

    beta = O.weight_scale(W)
    assert beta == parse_float(g["beta"][0])
    t = O.ternarize(W, beta)
    np.testing.assert_array_equal(t, t_exp)
    P = O.pack(t)
    np.testing.assert_array_equal(P, P_exp)
    np.testing.assert_array_equal(O.unpack(P), t_exp)

    xb = bf16(x)  # every x value is exact in bf16
    np.testing.assert_array_equal(O.bf16_to_f32(xb), x)
    q, s, rs = O.quantize_input(xb)
    np.testing.assert_array_equal(s, s_exp)
    np.testing.assert_array_equal(q, q_exp)
    np.testing.assert_array_equal(rs, q_exp.astype(np.int32).sum(1))

    acc = O.ternary_matmul(q, t)
    np.testing.assert_array_equal(acc, acc_exp)
    y = O.rescale(acc, s, beta)
    np.testing.assert_array_equal(y.view(np.uint32), y_exp.view(np.uint32))

    out = O.forward(xb, P, beta)
    np.testing.assert_array_equal(out["y"].view(np.uint32), y_exp.view(np.uint32))
    np.testing.assert_array_equal(out["acc"], acc_exp)
    np.testing.assert_array_equal(out["q"], q_exp)
    # the zero row gives +0, not -0
    assert not np.signbit(out["y"][1]).any()


def test_pack_layout_example(O):
    g = load_golden("pack_layout_n8.txt")
    t = np.array([int(v) for v in g["t"]], np.int8).reshape(8, 1)
    P = O.pack(t)
    np.testing.assert_array_equal(P.ravel(), [int(v, 16) for v in g["P_hex"]])
    assert list(P.ravel()) != [int(v, 16) for v in g["P_hex_interleaved_alternative"]]
    np.testing.assert_array_equal(O.unpack(P), t)


# --------------------------------------------------------------------------
# Round trips
# --------------------------------------------------------------------------
def test_every_valid_byte_round_trips(O):
    """The 3^4 = 81 bytes whose four bit pairs are all in {0,1,2}."""
    valid = [b for b in range(256) if all(((b >> (2 * i)) & 3) != 3 for i in range(4))]
    assert len(valid) == 81
    P = np.array(valid, np.uint8).reshape(1, -1)  # N=4, K=81
    t = O.unpack(P)
    for k, b in enumerate(valid):
        for i in range(4):
            assert t[i, k] == ((b >> (2 * i)) & 3) - 1
    np.testing.assert_array_equal(O.pack(t), P)


def test_unused_code_decodes_to_plus_two(O):
    """Bit pair 11 is never written; unpack maps it arithmetically to +2."""
    P = np.array([[0xFF, 0x03, 0xC0]], np.uint8)
    t = O.unpack(P)
    np.testing.assert_array_equal(t[:, 0], [2, 2, 2, 2])
    np.testing.assert_array_equal(t[:, 1], [2, -1, -1, -1])
    np.testing.assert_array_equal(t[:, 2], [-1, -1, -1, 2])
    with pytest.raises(ValueError):
        O.pack(t)


@pytest.mark.parametrize("N,K", [(4, 1), (8, 16), (64, 48), (132, 33)])
def test_random_ternary_round_trip(O, N, K):
    rng = np.random.default_rng(N * 1000 + K)
    t = rng.integers(-1, 2, (N, K)).astype(np.int8)
    P = O.pack(t)
    assert P.shape == (N // 4, K)
    np.testing.assert_array_equal(O.unpack(P), t)
    # bit pair i of packed row r is row i*N/4 + r
    R = N // 4
    for i in range(4):
        np.testing.assert_array_equal(((P >> (2 * i)) & 3).astype(np.int8) - 1, t[i * R:(i + 1) * R])


def test_pack_rejects_bad_shape_and_values(O):
    with pytest.raises(ValueError):
        O.pack(np.zeros((6, 4), np.int8))
    with pytest.raises(ValueError):
        O.pack(np.full((4, 4), 2, np.int8))


# --------------------------------------------------------------------------
# Building blocks against library routines / exact arithmetic
# --------------------------------------------------------------------------
def test_exact_sum_matches_fsum(O):
    rng = np.random.default_rng(7)
    for trial in range(40):
        n = int(rng.integers(1, 3000))
        mant = rng.standard_normal(n)
        expo = rng.integers(-60, 60, n) if trial % 2 else rng.integers(-1070, 1000, n)
        v = np.ldexp(mant, expo)
        assert O.exact_sum(v) == math.fsum(v.tolist())
    # heavy cancellation and subnormals
    cases = [[1e308, 1e308, -1e308, -1e308, 1.0], [1e100, 1.0, -1e100, 1e-100],
             [5e-324, 5e-324, -1e-323, 2.5e-323], [0.1] * 10, [2.0 ** 53, 1.0, 1.0],
             [2.0 ** 53, 1.0], [-0.0, 0.0], [1.0, 2.0 ** -60, -1.0]]
    for c in cases:
        # exact rational sum, rounded once (float(Fraction) rounds correctly)
        assert O.exact_sum(np.array(c)) == float(sum(Fraction(v) for v in c))


def test_bf16_cast_matches_torch(O):
    rng = np.random.default_rng(3)
    bits = rng.integers(0, 2 ** 32, 200000, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    f = np.concatenate([f, np.array([0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 3.4e38,
                                     -3.4e38, 1e-45, 2 ** -133], np.float32)])
    np.testing.assert_array_equal(O.f32_to_bf16(f), bf16(f))
    xb = bf16(rng.standard_normal(1000))
    np.testing.assert_array_equal(O.bf16_to_f32(xb),
                                  torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16)
                                  .float().numpy())


def _beta_exact(W):
    s = sum(Fraction(float(abs(v))) for v in W.ravel())
    mean = float(s) / float(W.size)  # float(Fraction) rounds correctly to binary64
    b = np.float32(mean)
    return max(b, FLOOR)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_weight_scale_is_rounded_exact_mean(O, seed):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((12, 40)) * np.exp(rng.uniform(-20, 5, (12, 40)))).astype(np.float32)
    assert O.weight_scale(W) == _beta_exact(W)


def test_weight_scale_floor(O):
    assert O.weight_scale(np.zeros((8, 16), np.float32)) == FLOOR
    tiny = np.full((4, 4), 1e-7, np.float32)
    assert O.weight_scale(tiny) == FLOOR


def test_ternary_matmul_vs_numpy(O):
    rng = np.random.default_rng(11)
    for (M, K, N) in [(1, 16, 4), (3, 48, 20), (7, 130, 12)]:
        q = rng.integers(-127, 128, (M, K)).astype(np.int8)
        t = rng.integers(-1, 2, (N, K)).astype(np.int8)
        ref = np.matmul(q.astype(np.int64), t.astype(np.int64).T)
        np.testing.assert_array_equal(O.ternary_matmul(q, t), ref)


# --------------------------------------------------------------------------
# Closed forms and special cases
# --------------------------------------------------------------------------
def test_gaussian_zero_fraction(O):
    """For W ~ N(0, s^2), t = 0 iff |W| < beta/2 with beta = E|W| = s*sqrt(2/pi),
    so P(t=0) = erf(1/(2 sqrt(pi))) = 0.3101 and P(t=+1) = P(t=-1)."""
    rng = np.random.default_rng(2560)
    W = (rng.standard_normal((2560, 2560)) * 0.02).astype(np.float32)
    t = O.ternarize(W, O.weight_scale(W))
    n = t.size
    p0 = math.erf(1.0 / (2.0 * math.sqrt(math.pi)))
    sigma = math.sqrt(p0 * (1 - p0) / n)
    frac0 = float((t == 0).mean())
    assert abs(frac0 - p0) < 5 * sigma + 1e-4  # +1e-4: beta is the sample, not population, mean
    pp = float((t == 1).mean())
    pm = float((t == -1).mean())
    assert abs(pp - pm) < 5 * math.sqrt(0.5 * 0.5 / n) * 2
    assert set(np.unique(t)) <= {-1, 0, 1}


def test_all_zero_weights(O):
    W = np.zeros((8, 32), np.float32)
    beta = O.weight_scale(W)
    assert beta == FLOOR
    t = O.ternarize(W, beta)
    assert not t.any()
    x = bf16(np.random.default_rng(0).standard_normal((3, 32)))
    out = O.forward(x, O.pack(t), beta)
    assert not out["y"].any()


def test_constant_rows_quantise_to_full_scale(O):
    for c in (0.37, -5.0, 1e-3, -2.0 ** -10, 300.0):
        xb = bf16(np.full((1, 64), c, np.float32))
        q, s, rs = O.quantize_input(xb)
        assert (q == (127 if c > 0 else -127)).all()
        assert rs[0] == 64 * (127 if c > 0 else -127)


def test_identity_weights(O):
    """W = I (N = K = 256): beta = 1/256 exactly, t = I, so acc = q and
    y = RN32(q * 2^-8 / s_x)."""
    K = 256
    W = np.eye(K, dtype=np.float32)
    beta = O.weight_scale(W)
    assert beta == np.float32(1.0 / 256.0)
    t = O.ternarize(W, beta)
    np.testing.assert_array_equal(t, np.eye(K, dtype=np.int8))
    x = bf16(np.random.default_rng(5).standard_normal((4, K)))
    out = O.forward(x, O.pack(t), beta)
    np.testing.assert_array_equal(out["acc"], out["q"].astype(np.int32))
    for m in range(4):
        for n in range(0, K, 17):
            exp = rn32_of_fraction(Fraction(int(out["q"][m, n]), 256) / Fraction(float(out["s_x"][m])))
            assert out["y"][m, n] == exp


def test_power_of_two_scaling_leaves_codes(O):
    rng = np.random.default_rng(9)
    x = rng.standard_normal((5, 96)).astype(np.float32)
    q0, s0, _ = O.quantize_input(bf16(x))
    for k in (-6, -1, 3, 8):
        q1, s1, _ = O.quantize_input(bf16(x * np.float32(2.0 ** k)))
        np.testing.assert_array_equal(q1, q0)
        np.testing.assert_array_equal(s1, s0 * np.float32(2.0 ** -k))


def test_act_quant_invariants(O):
    rng = np.random.default_rng(12)
    h = (rng.standard_normal((64, 200)) * np.exp(rng.uniform(-14, 6, (64, 1)))).astype(np.float32)
    h[3] = 0.0
    h[7] = 3e-6  # below the floor
    q, s, rs = O.act_quant(h)
    mx = np.abs(h).max(1)
    big = mx >= FLOOR
    assert (np.abs(q.astype(np.int32)).max(1)[big] == 127).all()
    assert (np.abs(q.astype(np.int32)).max(1)[~big] < 127).all()
    assert (q[3] == 0).all() and s[3] == np.float32(12700000.0)
    assert q.min() >= -127  # -128 is never reached: |h*s| <= 127 (1 + 2^-23)
    np.testing.assert_array_equal(rs, q.astype(np.int32).sum(1))
    # s_x is the correctly rounded 127 / max(m, 1e-5)
    for m in range(0, 64, 5):
        assert s[m] == rn32_of_fraction(Fraction(127) / Fraction(float(max(mx[m], FLOOR))))
    # dequantisation error is at most half a step on unclamped rows
    deq = q.astype(np.float64) / s[:, None].astype(np.float64)
    err = np.abs(deq - h.astype(np.float64))
    assert (err[big] <= (0.5 / s[big, None].astype(np.float64)) * (1 + 1e-6)).all()


TIE_VALUES = [127.0, 0.5, 1.5, 2.5, 3.5, -0.5, -1.5, -2.5, 126.5, -126.5, 4.5, -3.5]
TIE_CODES = [127, 0, 2, 2, 4, 0, -2, -2, 126, -126, 4, -4]  # halves go to the even neighbour


def test_act_quant_rounds_ties_to_even(O):
    """With max|h| = 127 the scale is exactly 1, so h = k + 1/2 lands on a tie:
    the codes are the even neighbours (round half to even, as torch.round)."""
    h = np.zeros((2, 16), np.float32)
    h[0, :len(TIE_VALUES)] = TIE_VALUES
    h[1, :len(TIE_VALUES)] = [-v for v in TIE_VALUES]
    q, s, rs = O.act_quant(h)
    assert s[0] == s[1] == np.float32(1.0)
    np.testing.assert_array_equal(q[0, :len(TIE_CODES)], TIE_CODES)
    np.testing.assert_array_equal(q[1, :len(TIE_CODES)], [-c for c in TIE_CODES])
    np.testing.assert_array_equal(rs, [sum(TIE_CODES), -sum(TIE_CODES)])


# --------------------------------------------------------------------------
# RMSNorm
# --------------------------------------------------------------------------
def _r_exact(xrow_f32, K, eps):
    ss = sum(Fraction(float(v)) ** 2 for v in xrow_f32)
    ssd = float(ss)                 # RN64 of the exact sum
    rd = 1.0 / math.sqrt(ssd / K + float(np.float32(eps)))   # IEEE binary64 ops
    return np.float32(rd)


def test_rmsnorm_factor_exact(O):
    rng = np.random.default_rng(21)
    x = rng.standard_normal((6, 64)) * np.exp(rng.uniform(-30, 10, (6, 64)))
    xb = bf16(x.astype(np.float32))
    h, r = O.rmsnorm(xb, None, 1e-5)
    xf = O.bf16_to_f32(xb)
    for m in range(6):
        assert r[m] == _r_exact(xf[m], 64, 1e-5)
        np.testing.assert_array_equal(h[m], (xf[m] * r[m]).astype(np.float32))


@pytest.mark.parametrize("K", [16, 256, 2560])
def test_rmsnorm_factor_on_rounding_boundaries(O, K):
    """Rows whose exact sum of squares sits where RN64 of it decides between two
    binary32 factors: the oracle gives the factor of the exact sum, and a plain
    binary64 running sum of the same squares misses at least one of them."""
    from rms_boundary import exact_sum_squares, factor_from_sum, straddle_rows
    rows = straddle_rows(8, K, 1e-5, seed=K + 7)
    _, r = O.rmsnorm(rows, None, 1e-5)
    exact = np.array([factor_from_sum(float(exact_sum_squares(b)), K, 1e-5) for b in rows])
    np.testing.assert_array_equal(r, exact)
    xf = O.bf16_to_f32(rows).astype(np.float64)
    running = np.array([factor_from_sum(float(np.cumsum(v * v)[-1]), K, 1e-5) for v in xf])
    assert (running != exact).any()


def test_rmsnorm_matches_textbook_formula(O):
    rng = np.random.default_rng(22)
    K = 2560
    x = rng.standard_normal((4, K)).astype(np.float32)
    g = rng.uniform(0.5, 1.5, K).astype(np.float32)
    xb, gb = bf16(x), bf16(g)
    h, _ = O.rmsnorm(xb, gb, 1e-5)
    xf = O.bf16_to_f32(xb).astype(np.float64)
    gf = O.bf16_to_f32(gb).astype(np.float64)
    ref = xf / np.sqrt((xf ** 2).mean(1, keepdims=True) + 1e-5) * gf
    np.testing.assert_allclose(h, ref, rtol=4 * 2.0 ** -24, atol=0)


def test_rmsnorm_applies_the_gain_after_the_factor(O):
    """h = RN32(RN32(x r) g), not RN32(x RN32(r g)): r is recomputed here from
    the exact sum of squares (math.fsum of exact binary64 squares, then
    binary64 IEEE divide, add, sqrt, reciprocal, one rounding to binary32), and
    the row holds elements where the two orders round differently."""
    import math
    rng = np.random.default_rng(23)
    K = 2560
    xb = bf16(rng.standard_normal((3, K)))
    gb = bf16(rng.uniform(0.5, 1.5, K))
    h, r_o = O.rmsnorm(xb, gb, 1e-5)
    xf, gf = O.bf16_to_f32(xb), O.bf16_to_f32(gb)
    eps = float(np.float32(1e-5))
    for m in range(3):
        ss = math.fsum(float(v) * float(v) for v in xf[m])  # each square exact in binary64
        r = np.float32(1.0 / math.sqrt(ss / K + eps))
        assert r == r_o[m]
        after = ((xf[m] * r).astype(np.float32) * gf).astype(np.float32)
        before = (xf[m] * np.float32(r * gf.astype(np.float32))).astype(np.float32)
        assert (after != before).sum() > 10  # the row separates the two orders
        assert (h[m].view(np.uint32) == after.view(np.uint32)).all()


def test_rescale_is_two_correctly_rounded_steps(O):
    """y = RN32(RN32(acc * beta) / s_x), each step the correctly rounded value
    of the exact rational (multiply first, then divide); the other order
    differs on most of these samples."""
    rng = np.random.default_rng(5)
    M, N = 8, 64
    acc = rng.integers(-877824, 877825, (M, N)).astype(np.int32)  # |acc| <= 127 * 6912
    acc[0, :4] = [0, 1, -1, 877824]
    s = (np.float32(127) / rng.uniform(0.5, 40, M).astype(np.float32)).astype(np.float32)
    beta = np.float32(0.0173)
    y = O.rescale(acc, s, float(beta))
    swapped = 0
    for m in range(M):
        for n in range(N):
            p = rn32_of_fraction(Fraction(int(acc[m, n])) * Fraction(float(beta)))
            assert y[m, n] == rn32_of_fraction(Fraction(float(p)) / Fraction(float(s[m])))
            d = rn32_of_fraction(Fraction(int(acc[m, n])) / Fraction(float(s[m])))
            swapped += rn32_of_fraction(Fraction(float(d)) * Fraction(float(beta))) != y[m, n]
    assert swapped > 0


# --------------------------------------------------------------------------
# Forward vs brute force
# --------------------------------------------------------------------------
@pytest.mark.parametrize("M,K,N,norm", [(3, 48, 20, False), (5, 256, 64, True), (2, 96, 8, True)])
def test_forward_vs_float64_brute_force(O, M, K, N, norm):
    rng = np.random.default_rng(M * K + N)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    x = bf16(rng.standard_normal((M, K)))
    gain = bf16(rng.uniform(0.5, 1.5, K)) if norm else None
    P, beta = O.pack_master(W)
    out = O.forward(x, P, beta, gain=gain, norm=norm)
    t = O.unpack(P).astype(np.int64)
    # integer accumulator: numpy's matmul of the dequantised operands' integers
    np.testing.assert_array_equal(out["acc"], out["q"].astype(np.int64) @ t.T)
    # y against the fp64 value of sum_k (q/s_x) (t*beta): at most ~2 binary32 ulps away
    ref = (out["q"].astype(np.float64) / out["s_x"][:, None].astype(np.float64)) @ \
        (t.astype(np.float64) * float(beta)).T
    np.testing.assert_allclose(out["y"], ref, rtol=2 * 2.0 ** -23, atol=1e-30)
    # and the dequantised weight is a ternary multiple of beta
    Wq = t * float(beta)
    assert np.all(np.isin(np.unique(Wq / beta), [-1.0, 0.0, 1.0]))


def test_forward_equals_its_steps(O):
    rng = np.random.default_rng(31)
    M, K, N = 4, 128, 32
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    x = bf16(rng.standard_normal((M, K)))
    gain = bf16(rng.uniform(0.5, 1.5, K))
    P, beta = O.pack_master(W)
    out = O.forward(x, P, beta, gain=gain, norm=True)
    h, _ = O.rmsnorm(x, gain, 1e-5)
    q, s, _ = O.act_quant(h)
    acc = O.ternary_matmul(q, O.unpack(P))
    y = O.rescale(acc, s, beta)
    np.testing.assert_array_equal(out["y"], y)


# --------------------------------------------------------------------------
# FFN block glue
# --------------------------------------------------------------------------
# Single-rounding bound of the FFN glue: two binary32 roundings (relative
# error <= 2^-24 each) and one bf16 rounding (8-bit significand: <= 2^-8) of
# the exact value give at most 2^-8 + 2^-23 + (smaller terms)
# < 2^-8 (1 + 2^-14) relative error.  An intermediate rounded to bf16 would
# double the bf16 term; test_relu2_mul_keeps_the_square_in_binary32 tells the
# two readings apart bit for bit.
GLUE_RTOL = 2.0 ** -8 * (1 + 2.0 ** -14)


def test_relu2_mul_vs_float64(O):
    rng = np.random.default_rng(41)
    a = bf16(rng.standard_normal(5000) * 3)
    b = bf16(rng.standard_normal(5000) * 3)
    z = O.bf16_to_f32(O.relu2_mul(a, b)).astype(np.float64)
    af = O.bf16_to_f32(a).astype(np.float64)
    bf = O.bf16_to_f32(b).astype(np.float64)
    ref = np.maximum(af, 0) ** 2 * bf
    np.testing.assert_allclose(z, ref, rtol=GLUE_RTOL, atol=0)
    assert (z[af <= 0] == 0).all()


def _torch_bf16_bits(v):
    """bf16 bits of binary32 values by torch's round-to-nearest-even cast."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(np.asarray(v, np.float32)))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_relu2_mul_keeps_the_square_in_binary32(O):
    """Pairs where rounding relu(a)^2 to bf16 before the multiply changes the
    result: the oracle gives the binary32-intermediate value, not the other."""
    rng = np.random.default_rng(43)
    a = bf16(np.abs(rng.standard_normal(20000)) * 3 + 0.01)
    b = bf16(rng.standard_normal(20000) * 3)
    af, bf = O.bf16_to_f32(a), O.bf16_to_f32(b)
    sq = (af * af).astype(np.float32)                       # RN32(a^2), a > 0
    keep = _torch_bf16_bits((sq * bf).astype(np.float32))   # bf16(RN32(RN32(a^2) b))
    sq_b = O.bf16_to_f32(_torch_bf16_bits(sq))
    early = _torch_bf16_bits((sq_b * bf).astype(np.float32))  # bf16(RN32(bf16(a^2) b))
    differ = np.flatnonzero(keep != early)
    assert differ.size > 100  # the two readings are distinguishable on these inputs
    z = O.relu2_mul(a[differ], b[differ])
    assert (z == keep[differ]).all()
    assert not (z == early[differ]).any()


def test_residual_add_vs_float64(O):
    rng = np.random.default_rng(42)
    x = bf16(rng.standard_normal(5000))
    d = bf16(rng.standard_normal(5000) * 0.1)
    out = O.bf16_to_f32(O.residual_add(x, d)).astype(np.float64)
    ref = O.bf16_to_f32(x).astype(np.float64) + O.bf16_to_f32(d).astype(np.float64)
    np.testing.assert_allclose(out, ref, rtol=GLUE_RTOL, atol=0)


def _packed(O, W):
    return O.pack_master(W.astype(np.float32))


def test_ffn_block_zero_down_is_identity(O):
    rng = np.random.default_rng(51)
    M, H, I = 3, 64, 128
    x = bf16(rng.standard_normal((M, H)))
    g1, g2 = bf16(rng.uniform(.5, 1.5, H)), bf16(rng.uniform(.5, 1.5, I))
    Pg, bg = _packed(O, rng.standard_normal((I, H)) * .02)
    Pu, bu = _packed(O, rng.standard_normal((I, H)) * .02)
    Pd, bd = _packed(O, np.zeros((H, I)))
    np.testing.assert_array_equal(O.ffn_block(x, g1, g2, 1e-5, Pg, bg, Pu, bu, Pd, bd), x)


def test_ffn_block_gate_is_the_relu_operand(O):
    """Gate outputs all negative (positive inputs, all -1 gate weights): relu
    zeroes z, so the block is the identity.  Swapping gate and up, dropping the
    relu, or dropping the residual would all change the output."""
    rng = np.random.default_rng(52)
    M, H, I = 2, 64, 128
    x = bf16(np.abs(rng.standard_normal((M, H))) + 0.1)
    g1, g2 = bf16(rng.uniform(.5, 1.5, H)), bf16(rng.uniform(.5, 1.5, I))
    Pg, bg = _packed(O, -np.abs(rng.standard_normal((I, H))) - 0.5)
    Pu, bu = _packed(O, np.abs(rng.standard_normal((I, H))) + 0.5)
    Pd, bd = _packed(O, rng.standard_normal((H, I)) * .02)
    out = O.ffn_block(x, g1, g2, 1e-5, Pg, bg, Pu, bu, Pd, bd)
    np.testing.assert_array_equal(out, x)
    # swapped roles: up (positive) as the relu operand gives a non-trivial update
    out_sw = O.ffn_block(x, g1, g2, 1e-5, Pu, bu, Pg, bg, Pd, bd)
    assert (out_sw != x).any()


def test_ffn_block_equals_its_steps(O):
    rng = np.random.default_rng(53)
    M, H, I = 4, 64, 96
    x = bf16(rng.standard_normal((M, H)))
    g1, g2 = bf16(rng.uniform(.5, 1.5, H)), bf16(rng.uniform(.5, 1.5, I))
    Pg, bg = _packed(O, rng.standard_normal((I, H)) * .02)
    Pu, bu = _packed(O, rng.standard_normal((I, H)) * .02)
    Pd, bd = _packed(O, rng.standard_normal((H, I)) * .02)
    out = O.ffn_block(x, g1, g2, 1e-5, Pg, bg, Pu, bu, Pd, bd)
    a = O.f32_to_bf16(O.forward(x, Pg, bg, gain=g1, norm=True)["y"])
    b = O.f32_to_bf16(O.forward(x, Pu, bu, gain=g1, norm=True)["y"])
    z = O.relu2_mul(a, b)
    d = O.f32_to_bf16(O.forward(z, Pd, bd, gain=g2, norm=True)["y"])
    np.testing.assert_array_equal(out, O.residual_add(x, d))


def test_openmp_build_gives_identical_results(O):
    """The oracle's OpenMP build (matmul rows on all host cores, used for the
    CPU baseline) returns the plain build's results bit for bit."""
    rng = np.random.default_rng(77)
    W = (rng.standard_normal((256, 512)) * 0.02).astype(np.float32)
    P, beta = O.pack_master(W)
    x = bf16(rng.standard_normal((5, 512)))
    g = bf16(rng.uniform(0.5, 1.5, 512))
    ref = O.forward(x, P, beta, gain=g, eps=1e-5, norm=True)
    try:
        O.set_parallel(True)
        par = O.forward(x, P, beta, gain=g, eps=1e-5, norm=True)
    finally:
        O.set_parallel(False)
    assert (par["acc"] == ref["acc"]).all()
    assert (par["y"].view(np.uint32) == ref["y"].view(np.uint32)).all()


# --------------------------------------------------------------------------
# Online QAT: forward with on-the-fly ternarisation, straight-through backward
# --------------------------------------------------------------------------
def test_online_forward_reproduces_the_hand_example(O):
    """The online forward starts from the fp32 masters: on the hand-worked
    example it must land on the hand-derived beta, ternary weights and y."""
    g = load_golden("hand_example_4x8.txt")
    W = np.array([[parse_float(v) for v in g["W_row%d" % i]] for i in range(4)], np.float32)
    t_exp = np.array([[int(v) for v in g["t_row%d" % i]] for i in range(4)], np.int8)
    x = np.array([[parse_float(v) for v in g["x_row%d" % i]] for i in range(4)], np.float32)
    y_exp = np.array([[rn32_of_fraction(Fraction(v)) for v in g["y_row%d" % i]]
                      for i in range(4)], np.float32)
    out = O.online_forward(bf16(x), W)
    assert out["beta"] == parse_float(g["beta"][0])
    np.testing.assert_array_equal(out["t"], t_exp)
    np.testing.assert_array_equal(out["y"].view(np.uint32), y_exp.view(np.uint32))


def test_online_forward_is_the_forward_of_the_packed_masters(O):
    rng = np.random.default_rng(90)
    W = (rng.standard_normal((64, 96)) * 0.02).astype(np.float32)
    x = bf16(rng.standard_normal((3, 96)))
    gain = bf16(rng.uniform(0.5, 1.5, 96))
    P, beta = O.pack_master(W)
    for norm in (False, True):
        on = O.online_forward(x, W, gain=gain, eps=1e-5, norm=norm)
        ref = O.forward(x, P, beta, gain=gain, eps=1e-5, norm=norm)
        assert on["beta"] == beta
        assert (on["y"].view(np.uint32) == ref["y"].view(np.uint32)).all()


def _dequantised(O, q, s_x, t, beta):
    """W_q = RN32(t / RN32(1/beta)), x_q = RN32(q / s_x), by numpy binary32."""
    s_w = np.float32(1.0) / np.float32(beta)
    W_q = (t.astype(np.float32) / s_w).astype(np.float32)
    x_q = (q.astype(np.float32) / s_x[:, None].astype(np.float32)).astype(np.float32)
    return W_q, x_q


def test_ste_backward_one_hot_gradients(O):
    """A one-hot output gradient selects one row of each dequantised operand:
    gx[m0] = W_q[n0] and gw[n0] = x_q[m0] exactly, zeros elsewhere."""
    rng = np.random.default_rng(91)
    M, K, N = 3, 40, 8
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    beta = O.weight_scale(W)
    t = O.ternarize(W, beta)
    q, s, _ = O.quantize_input(bf16(rng.standard_normal((M, K)) * 3))
    W_q, x_q = _dequantised(O, q, s, t, beta)
    for m0, n0 in ((0, 0), (2, 5), (1, 7)):
        gy = np.zeros((M, N), np.float32)
        gy[m0, n0] = 1.0
        gx, gw = O.ste_backward(gy, q, s, t, beta)
        exp_gx = np.zeros((M, K))
        exp_gx[m0] = W_q[n0]
        exp_gw = np.zeros((N, K))
        exp_gw[n0] = x_q[m0]
        np.testing.assert_array_equal(gx, exp_gx)
        np.testing.assert_array_equal(gw, exp_gw)
    # the dequantised weight magnitude is RN32(1 / RN32(1 / beta)): beta give or take an ulp
    mag = np.abs(W_q[W_q != 0])
    assert np.all(mag == mag[0]) and abs(float(mag[0]) - beta) <= float(np.spacing(np.float32(beta)))


def test_ste_backward_against_exact_rationals(O):
    """Tiny shapes: the binary64 sums against exact rational sums of the same
    binary32 products, within the rounding bound of n binary64 additions."""
    rng = np.random.default_rng(92)
    M, K, N = 4, 6, 8
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    beta = O.weight_scale(W)
    t = O.ternarize(W, beta)
    q, s, _ = O.quantize_input(bf16(rng.standard_normal((M, K))))
    gy = rng.standard_normal((M, N)).astype(np.float32)
    gx, gw = O.ste_backward(gy, q, s, t, beta)
    W_q, x_q = _dequantised(O, q, s, t, beta)
    u = 2.0 ** -53
    for m in range(M):
        for k in range(K):
            terms = [Fraction(float(gy[m, n])) * Fraction(float(W_q[n, k])) for n in range(N)]
            exact = sum(terms, Fraction(0))
            bound = N * u * float(sum(abs(v) for v in terms))
            assert abs(Fraction(gx[m, k]) - exact) <= Fraction(bound) + Fraction(1, 10 ** 300)
    for n in range(N):
        for k in range(K):
            terms = [Fraction(float(gy[m, n])) * Fraction(float(x_q[m, k])) for m in range(M)]
            exact = sum(terms, Fraction(0))
            bound = M * u * float(sum(abs(v) for v in terms))
            assert abs(Fraction(gw[n, k]) - exact) <= Fraction(bound) + Fraction(1, 10 ** 300)
