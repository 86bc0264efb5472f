"""The attention block around the projections (bitlinear_rope,
bitlinear_attn_decode) against the float64 oracle through the C ABI, at the
2B4T head shapes and the cache lengths up to the model's 2048 positions.

Tolerances (binary32 and binary64 arithmetic against float64, one bf16
rounding at the output):
  RoPE      |gpu - exact| <= 2^-8 |exact| + 2^-133: the kernel works in
            binary64 and rounds once to bf16 (half an ulp of an 8-bit
            significand is at most 2^-8 of the value; 2^-133 covers bf16
            subnormals);
  attention |gpu - exact| <= 2^-8 |exact| + (2^-17 + L 2^-22) max|v|: the
            bf16 rounding plus binary32 error in the scores (a 128-term dot
            product), in exp2f and in the L-term sums of weights and values.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import ternary_weight_bitlinear_b200 as B
from ternary_weight_bitlinear_b200 import workloads as WL
from gpu_util import bf16_dev, bf16_host, f32_of_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device_status_clean():
    yield
    assert B.bitlinear_device_status() == 0


def _rope_case(M, heads, d, theta, seed, guard, in_place=False):
    x = WL.activations(M, heads * d, seed=seed)
    pos = WL.rope_positions(M, seed=seed + 1)
    xd = guard.copy(bf16_dev(x).reshape(M, heads * d))
    pd = guard.copy(torch.from_numpy(pos).cuda())
    out = xd if in_place else guard.empty((M, heads * d), torch.bfloat16)
    B.bitlinear_rope(xd, pd, heads, theta, out=out)
    torch.cuda.synchronize()
    got = f32_of_bf16(bf16_host(out)).astype(np.float64)
    want = O.rope(f32_of_bf16(x).reshape(M, heads * d), pos, heads, d, theta)
    err = np.abs(got - want)
    bound = 2.0 ** -8 * np.abs(want) + 2.0 ** -133
    assert np.all(err <= bound), "max excess %g at %s" % (
        float((err - bound).max()), np.unravel_index(int(np.argmax(err - bound)), err.shape))
    return out


@pytest.mark.parametrize("M", [1, 4, 17])
@pytest.mark.parametrize("heads", [WL.Q_HEADS, WL.KV_HEADS])
@pytest.mark.parametrize("theta", [10000.0, 500000.0])
def test_rope_matches_oracle(M, heads, theta, guard):
    _rope_case(M, heads, WL.HEAD_DIM, theta, seed=M * 7 + heads, guard=guard)


def test_rope_in_place_and_other_head_width(guard):
    a = _rope_case(9, 8, 64, 10000.0, seed=3, guard=guard, in_place=True)
    assert a.shape == (9, 512)


def test_rope_position_zero_is_bit_identity(guard):
    x = WL.activations(3, WL.Q_HEADS * WL.HEAD_DIM, seed=11)
    xd = bf16_dev(x).reshape(3, -1)
    pd = torch.zeros(3, dtype=torch.int32, device="cuda")
    y = B.bitlinear_rope(xd, pd, WL.Q_HEADS, 500000.0, out=guard.empty(xd.shape, torch.bfloat16))
    assert np.array_equal(bf16_host(y), bf16_host(xd))


def _attn_case(L, H, Hkv, d, seed, guard, q_std=1.0):
    q, k, v = WL.attention_decode_inputs(L, seed, H, Hkv, d, q_std=q_std)
    scale = 1.0 / math.sqrt(d)
    # caches padded past L with NaN: nothing past L may be read
    kpad = np.concatenate([k, np.full((3, Hkv, d), 0x7FC0, np.uint16)])
    vpad = np.concatenate([v, np.full((3, Hkv, d), 0x7FC0, np.uint16)])
    kd, vd = guard.copy(bf16_dev(kpad)), guard.copy(bf16_dev(vpad))
    qd = guard.copy(bf16_dev(q))
    ws = guard.workspace(B.bitlinear_attn_decode_workspace_size(L, H, Hkv, d))
    out = guard.empty(H * d, torch.bfloat16)
    B.bitlinear_attn_decode(qd, kd, vd, L, H, Hkv, scale, out=out, workspace=ws)
    torch.cuda.synchronize()
    got = f32_of_bf16(bf16_host(out)).astype(np.float64)
    vf = f32_of_bf16(v)
    want = O.attn_decode(f32_of_bf16(q), f32_of_bf16(k), vf, L, H, Hkv, d, scale)
    err = np.abs(got - want)
    bound = 2.0 ** -8 * np.abs(want) + (2.0 ** -17 + L * 2.0 ** -22) * float(np.abs(vf).max())
    assert np.all(np.isfinite(got))
    assert np.all(err <= bound), "L=%d: max excess %g at %d" % (L, float((err - bound).max()),
                                                                 int(np.argmax(err - bound)))
    return got, v


@pytest.mark.parametrize("L", [1, 2, 31, 32, 33, 100, 1000, 2048])
def test_attn_decode_2b4t_heads(L, guard):
    got, v = _attn_case(L, WL.Q_HEADS, WL.KV_HEADS, WL.HEAD_DIM, seed=L, guard=guard)
    if L == 1:  # one position: every head of a group returns its value row exactly
        vv = f32_of_bf16(v).reshape(WL.KV_HEADS, WL.HEAD_DIM)
        for h in range(WL.Q_HEADS):
            assert np.array_equal(got.reshape(WL.Q_HEADS, -1)[h], vv[h // 4])


@pytest.mark.parametrize("H,Hkv,d", [(8, 8, 64), (16, 2, 128), (4, 2, 64), (8, 1, 128)])
def test_attn_decode_other_groupings(H, Hkv, d, guard):
    _attn_case(257, H, Hkv, d, seed=H * 10 + Hkv, guard=guard)


def test_attn_decode_peaked_scores(guard):
    # large queries: softmax close to one-hot, the max subtraction matters
    _attn_case(640, WL.Q_HEADS, WL.KV_HEADS, WL.HEAD_DIM, seed=77, guard=guard, q_std=8.0)


def test_attention_half_of_a_decoder_layer_stagewise(guard):
    """One decode token through the attention half of a 2B4T decoder layer on
    the GPU (input RMSNorm + q, k, v BitLinear, RoPE, attention over a cache
    that ends with the token's own key and value, attn_sub_norm + o BitLinear),
    each stage checked against the oracle on that stage's GPU inputs: bit for
    bit for the BitLinear stages, within the tolerances above for RoPE and
    attention."""
    from gpu_util import assert_bf16_output
    H, Hkv, d, L = WL.Q_HEADS, WL.KV_HEADS, WL.HEAD_DIM, 300
    x = WL.activations(1, WL.HIDDEN, seed=5)
    g_in, g_sub = WL.gain(WL.HIDDEN, 1010), WL.gain(WL.HIDDEN, 1012)
    xd = bf16_dev(x).reshape(1, -1)
    dev, ora = {}, {}
    for p in WL.PROJECTIONS[:4]:
        W = WL.master_weights(p.N, p.K, WL.master_seed(0, p.name))
        P, b = B.bitlinear_pack(torch.from_numpy(W).cuda())
        dev[p.name] = (P, float(b.item()))
        ora[p.name] = O.pack_master(W)
    # q, k, v projections with the input norm
    y = {}
    for n in ("q", "k", "v"):
        y[n] = B.bitlinear_forward(xd, dev[n][0], dev[n][1], gain=bf16_dev(g_in), eps=WL.RMS_EPS,
                                   out=guard.empty((1, 2560 if n == "q" else 640), torch.bfloat16))
        ref = O.f32_to_bf16(O.forward(x, ora[n][0], ora[n][1], gain=g_in, eps=WL.RMS_EPS, norm=True)["y"])
        assert_bf16_output(bf16_host(y[n]), ref, n)
    # RoPE of q and k at the token's position (the cache's last)
    pos = torch.full((1,), L - 1, dtype=torch.int32, device="cuda")
    qr = B.bitlinear_rope(y["q"], pos, H, 500000.0, out=guard.empty((1, H * d), torch.bfloat16))
    kr = B.bitlinear_rope(y["k"], pos, Hkv, 500000.0, out=guard.empty((1, Hkv * d), torch.bfloat16))
    torch.cuda.synchronize()
    for got, src, heads in ((qr, y["q"], H), (kr, y["k"], Hkv)):
        want = O.rope(f32_of_bf16(bf16_host(src)), [L - 1], heads, d, 500000.0)
        g = f32_of_bf16(bf16_host(got)).astype(np.float64)
        assert np.all(np.abs(g - want) <= 2.0 ** -8 * np.abs(want) + 2.0 ** -133)
    # the cache: L - 1 earlier positions, then this token's rotated key and its value
    _, k0, v0 = WL.attention_decode_inputs(L - 1, seed=21)
    kc = guard.empty((L, Hkv, d), torch.bfloat16)
    vc = guard.empty((L, Hkv, d), torch.bfloat16)
    kc[:L - 1] = bf16_dev(k0)
    vc[:L - 1] = bf16_dev(v0)
    kc[L - 1] = kr.reshape(Hkv, d)
    vc[L - 1] = y["v"].reshape(Hkv, d)
    ws = guard.workspace(B.bitlinear_attn_decode_workspace_size(L, H, Hkv, d))
    att = B.bitlinear_attn_decode(qr.reshape(-1), kc, vc, L, H, Hkv, d ** -0.5,
                                  out=guard.empty(H * d, torch.bfloat16), workspace=ws)
    torch.cuda.synchronize()
    vf = f32_of_bf16(bf16_host(vc))
    want = O.attn_decode(f32_of_bf16(bf16_host(qr)), f32_of_bf16(bf16_host(kc)), vf, L, H, Hkv, d, d ** -0.5)
    got = f32_of_bf16(bf16_host(att)).astype(np.float64)
    assert np.all(np.abs(got - want) <= 2.0 ** -8 * np.abs(want)
                  + (2.0 ** -17 + L * 2.0 ** -22) * float(np.abs(vf).max()))
    # attn_sub_norm + o projection on the attention output
    a_bits = bf16_host(att).reshape(1, -1)
    o = B.bitlinear_forward(att.reshape(1, -1), dev["o"][0], dev["o"][1], gain=bf16_dev(g_sub),
                            eps=WL.RMS_EPS, out=guard.empty((1, 2560), torch.bfloat16))
    ref = O.f32_to_bf16(O.forward(a_bits, ora["o"][0], ora["o"][1], gain=g_sub, eps=WL.RMS_EPS,
                                  norm=True)["y"])
    assert_bf16_output(bf16_host(o), ref, "o after attn_sub_norm")
