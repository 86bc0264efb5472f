"""Token rows whose RMSNorm factor sits on a binary32 rounding boundary.

The factor r = RN32(1 / sqrt(RN64(SS/K) + eps)) is computed from the exact sum
of squares SS.  A fast implementation may start from an approximate SS and
accept it only when its error interval cannot change r; these rows put the
exact SS within ~2^-66 relative of the point where r changes from one binary32
value to the next, so any such interval straddles it and the implementation
has to fall back to the exact sum; a plain binary64 sum lands on the wrong
side about half the time.

Construction (exact rational arithmetic, no library rounding on the way):
random bf16 values fill all but six positions; r0 is the factor of that bulk.
Near SS* = K (1 / r_mid^2 - eps), r_mid the midpoint between r0 and the next
binary32 value below it, bisection over binary64 values finds the neighbours
d1 < d2 at which the factor steps from r0 down; the target is their midpoint,
where RN64(SS) itself decides.  It exceeds the bulk's sum by a relative ~2^-24;
five bf16 values whose squares greedily fill the gap from below (each step
removes ~7 bits of it) and a sixth rounded down or up put SS just below or just
above the target, so any error in the sum of squares can flip r.
"""
import math
from fractions import Fraction

import numpy as np

_SLOTS = 6


def bf16_value(bits):
    return float(np.array([int(bits) << 16], np.uint32).view(np.float32)[0])


def _bf16_sqrt(R, up):
    """Smallest (up) or largest (down) positive bf16 d with d*d >= R (<= R)."""
    f = math.sqrt(float(R))
    b = int(np.array([f], np.float32).view(np.uint32)[0]) >> 16
    while Fraction(bf16_value(b + 1)) ** 2 <= R:
        b += 1
    while b > 0 and Fraction(bf16_value(b)) ** 2 > R:
        b -= 1
    if up and Fraction(bf16_value(b)) ** 2 < R:
        b += 1
    return b


def factor_from_sum(ss, K, eps):
    """r from a binary64 sum of squares, each step an IEEE binary64 operation."""
    ms = ss / K
    var = ms + float(np.float32(eps))
    return np.float32(1.0 / math.sqrt(var))


def _first_double_below_factor(guess, r0, K, eps):
    """Smallest binary64 d near guess whose factor is below r0 (the factor is
    non-increasing in d), by bisection over the bit patterns."""
    lo = int(np.array([guess * (1 - 2.0 ** -40)]).view(np.int64)[0])
    hi = int(np.array([guess * (1 + 2.0 ** -40)]).view(np.int64)[0])
    val = lambda i: float(np.array([i], np.int64).view(np.float64)[0])
    if factor_from_sum(val(lo), K, eps) < r0 or factor_from_sum(val(hi), K, eps) >= r0:
        return None
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if factor_from_sum(val(mid), K, eps) < r0:
            hi = mid
        else:
            lo = mid
    return val(hi)


def exact_sum_squares(bits):
    return sum(Fraction(bf16_value(b)) ** 2 for b in bits)


def straddles(bits, K, eps):
    """True when a relative (K + 64) 2^-52 interval around RN64(SS) maps to two
    different binary32 factors."""
    ss = float(exact_sum_squares(bits))
    d = (K + 64) * 2.0 ** -52
    return factor_from_sum(ss * (1 - d), K, eps) != factor_from_sum(ss * (1 + d), K, eps)


def straddle_rows(n, K, eps, seed):
    """n rows of K bf16 bit patterns (uint16), alternately just below and just
    above the boundary, each checked to straddle it."""
    rng = np.random.default_rng(seed)
    eps32 = Fraction(float(np.float32(eps)))
    out = []
    attempts = 0
    while len(out) < n:
        attempts += 1
        assert attempts < 8 * n + 16, "could not place rows on a rounding boundary"
        vals = (rng.standard_normal(K) * rng.uniform(0.05, 4.0)).astype(np.float32)
        bits = (vals.view(np.uint32) >> 16).astype(np.uint16)  # truncation: any bf16 will do
        slots = rng.choice(K, _SLOTS, replace=False)
        bits[slots] = 0
        ss_bulk = exact_sum_squares(bits)
        r0 = factor_from_sum(float(ss_bulk), K, eps)
        r_next = np.nextafter(r0, np.float32(0))
        r_mid = (Fraction(float(r0)) + Fraction(float(r_next))) / 2
        d2 = _first_double_below_factor(float(K * (1 / (r_mid * r_mid) - eps32)), r0, K, eps)
        if d2 is None:
            continue
        d1 = float(np.nextafter(d2, 0.0))
        target = (Fraction(d1) + Fraction(d2)) / 2  # RN64 of SS picks d1 (r0) below, d2 above
        R = target - ss_bulk
        if R <= 0:
            continue
        up = len(out) % 2 == 1
        for i, pos in enumerate(slots):
            last = i == _SLOTS - 1
            b = _bf16_sqrt(R, up and last)
            if b == 0:
                break
            R -= Fraction(bf16_value(b)) ** 2
            bits[pos] = b | (0x8000 if rng.random() < 0.5 else 0)
        if straddles(bits, K, eps):
            out.append(bits)
    return np.stack(out)
