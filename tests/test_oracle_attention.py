"""Pins of the attention-block oracle (RoPE, GQA decode attention) against
what fixes it other than itself: a hand-worked example, closed forms,
invariants of a rotation and of a softmax average, and a brute force written
with scalar Python loops.  CPU only."""
import math
import os

import numpy as np
import pytest

import oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))


def test_rope_hand_example():
    rows = []
    with open(os.path.join(HERE, "golden", "rope_hand_d4.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([float(v) for v in line.split()])
    for r in rows:
        pos, x, want = int(r[0]), np.array(r[1:5]), np.array(r[5:9])
        got = O.rope(x[None, :], [pos], 1, 4, 10000.0)[0]
        assert np.allclose(got, want, rtol=0, atol=1e-15), (r, got)


def test_rope_inv_freq_closed_form():
    f = O.rope_inv_freq(128, 10000.0)
    assert f.shape == (64,)
    assert f[0] == 1.0
    assert abs(f[32] - 0.01) < 1e-17          # 10000^(-64/128)
    assert abs(f[63] - 10000.0 ** (-126 / 128)) < 1e-20
    assert np.all(np.diff(f) < 0)


def test_rope_position_zero_is_identity():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((3, 5 * 128))
    assert np.array_equal(O.rope(x, [0, 0, 0], 5, 128, 500000.0), x)


def test_rope_preserves_each_pair_norm():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((4, 2 * 64))
    y = O.rope(x, [1, 17, 511, 2047], 2, 64, 10000.0)
    xr, yr = x.reshape(4, 2, 64), y.reshape(4, 2, 64)
    nx = xr[..., :32] ** 2 + xr[..., 32:] ** 2
    ny = yr[..., :32] ** 2 + yr[..., 32:] ** 2
    assert np.allclose(nx, ny, rtol=1e-12, atol=0)


def test_rope_dot_products_depend_on_relative_position_only():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 128))
    k = rng.standard_normal((1, 128))
    d0 = float((O.rope(q, [40], 1, 128, 10000.0) @ O.rope(k, [25], 1, 128, 10000.0).T)[0, 0])
    d1 = float((O.rope(q, [1040], 1, 128, 10000.0) @ O.rope(k, [1025], 1, 128, 10000.0).T)[0, 0])
    assert abs(d0 - d1) < 1e-9 * (1 + abs(d0))
    d2 = float((O.rope(q, [41], 1, 128, 10000.0) @ O.rope(k, [25], 1, 128, 10000.0).T)[0, 0])
    assert abs(d0 - d2) > 1e-6  # and it does depend on it


def test_rope_rotates_first_half_into_second():
    # a sign or pairing mistake (interleaved pairs, swapped sin sign) fails here
    x = np.zeros((1, 8))
    x[0, 1] = 1.0  # pair 1 = (x1, x5)
    y = O.rope(x, [3], 1, 8, 10000.0)[0]
    a = 3 * 10000.0 ** (-2 / 8)
    want = np.zeros(8)
    want[1], want[5] = math.cos(a), math.sin(a)
    assert np.allclose(y, want, rtol=0, atol=1e-15)


def _brute_attn(q, K, V, L, H, Hkv, d, scale):
    out = []
    group = H // Hkv
    for h in range(H):
        g = h // group
        s = [sum(q[h * d + i] * K[j][g][i] for i in range(d)) * scale for j in range(L)]
        m = max(s)
        e = [math.exp(v - m) for v in s]
        tot = sum(e)
        out.extend(sum(e[j] * V[j][g][i] for j in range(L)) / tot for i in range(d))
    return np.array(out)


@pytest.mark.parametrize("L,H,Hkv,d", [(1, 4, 2, 4), (5, 4, 1, 8), (9, 6, 3, 4), (13, 8, 2, 16)])
def test_attn_brute_force(L, H, Hkv, d):
    rng = np.random.default_rng(L * 100 + H)
    q = rng.standard_normal(H * d)
    K = rng.standard_normal((L + 3, Hkv, d))
    V = rng.standard_normal((L + 3, Hkv, d))
    scale = 1.0 / math.sqrt(d)
    got = O.attn_decode(q, K, V, L, H, Hkv, d, scale)
    want = _brute_attn(q, K.tolist(), V.tolist(), L, H, Hkv, d, scale)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def test_attn_single_position_returns_its_value():
    rng = np.random.default_rng(5)
    K = rng.standard_normal((1, 5, 128))
    V = rng.standard_normal((1, 5, 128))
    out = O.attn_decode(rng.standard_normal(20 * 128), K, V, 1, 20, 5, 128, 128 ** -0.5).reshape(20, 128)
    for h in range(20):
        assert np.array_equal(out[h], V[0, h // 4])


def test_attn_zero_query_is_the_mean_of_values():
    rng = np.random.default_rng(6)
    K = rng.standard_normal((37, 5, 128))
    V = rng.standard_normal((37, 5, 128))
    out = O.attn_decode(np.zeros(20 * 128), K, V, 37, 20, 5, 128, 128 ** -0.5).reshape(20, 128)
    for h in range(20):
        assert np.allclose(out[h], V[:, h // 4].mean(axis=0), rtol=1e-12, atol=1e-14)


def test_attn_gqa_group_of_each_query_head():
    # values constant per kv head: head h must return the constant of h // 4
    # (a query head paired by h % 5 instead would not)
    L, H, Hkv, d = 11, 20, 5, 128
    rng = np.random.default_rng(7)
    K = rng.standard_normal((L, Hkv, d))
    V = np.zeros((L, Hkv, d))
    for g in range(Hkv):
        V[:, g, :] = g + 1.0
    out = O.attn_decode(rng.standard_normal(H * d), K, V, L, H, Hkv, d, d ** -0.5).reshape(H, d)
    for h in range(H):
        assert np.allclose(out[h], h // 4 + 1.0, rtol=1e-13)


def test_attn_peaked_scores_select_one_value():
    L, d = 16, 64
    K = np.zeros((L, 1, d))
    for j in range(L):
        K[j, 0, j] = 1.0
    V = np.arange(L * d, dtype=np.float64).reshape(L, 1, d)
    q = np.zeros(d)
    q[9] = 1.0
    out = O.attn_decode(q, K, V, L, 1, 1, d, 1000.0)  # exp(-1000) vanishes
    assert np.array_equal(out, V[9, 0])


def test_attn_reads_no_position_past_L_and_ignores_their_order():
    rng = np.random.default_rng(8)
    L = 23
    K = rng.standard_normal((L + 5, 5, 128))
    V = rng.standard_normal((L + 5, 5, 128))
    K[L:], V[L:] = np.nan, np.nan
    q = rng.standard_normal(20 * 128)
    a = O.attn_decode(q, K, V, L, 20, 5, 128, 0.1)
    assert np.all(np.isfinite(a))
    perm = rng.permutation(L)
    b = O.attn_decode(q, K[perm], V[perm], L, 20, 5, 128, 0.1)
    assert np.allclose(a, b, rtol=1e-12, atol=1e-14)
