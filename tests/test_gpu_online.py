"""Quantisation-aware training on the GPU against the oracle: the online
forward (weight scale and ternary weights derived from fp32 masters on every
call, then the inference forward) bit for bit, and the straight-through
backward within the rounding bound of binary32 sums.

Backward tolerance (derived from the arithmetic): the GPU adds n products
(n = N for grad_x, M for grad_w) in binary32 with fused multiply-adds in an
unspecified order; recursive summation errs by at most (n - 1) 2^-24 of the
sum of |terms|, and the oracle's binary64 sums by far less, so every output
must agree with the oracle within (n + 1) 2^-24 * sum|terms| (+ the smallest
normal binary32 for sums that vanish).
"""
import numpy as np
import pytest
import torch

import oracle as O
import ternary_weight_bitlinear_b200 as B
from ternary_weight_bitlinear_b200 import workloads as WL
from gpu_util import assert_bf16_output, assert_exact, assert_f32_output, bf16_dev, bf16_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device_status_clean():
    yield
    assert B.bitlinear_device_status() == 0


def online(x, W, gain, out_dtype, guard):
    M, K = x.shape
    N = W.shape[0]
    ws = guard.workspace(B.bitlinear_forward_online_workspace_size(M, K, N))
    return B.bitlinear_forward_online(bf16_dev(x), torch.from_numpy(W).cuda(),
                                      gain=None if gain is None else bf16_dev(gain), eps=WL.RMS_EPS,
                                      out=guard.empty((M, N), out_dtype), workspace=ws)


@pytest.mark.parametrize("M,K,N,norm,out", [
    (1, 2560, 2560, True, "bf16"), (3, 272, 36, False, "f32"), (5, 2560, 640, True, "bf16"),
    (16, 6912, 2560, True, "bf16"), (64, 400, 180, False, "f32"), (65, 2560, 640, True, "bf16"),
])
def test_online_forward_matches_oracle(M, K, N, norm, out, guard):
    x = WL.activations(M, K, seed=5000 + M, outlier_frac=0.001, row_std=(0.1, 10.0))
    W = WL.master_weights(N, K, seed=5100 + N)
    g = WL.gain(K, seed=5200) if norm else None
    dt = torch.float32 if out == "f32" else torch.bfloat16
    y, saved = online(x, W, g, dt, guard)
    ref = O.online_forward(x, W, gain=g, eps=WL.RMS_EPS, norm=norm)
    assert np.float32(saved["beta"].item()) == np.float32(ref["beta"])
    assert_exact(saved["P"].cpu().numpy(), O.pack(ref["t"]), "packed weights of the call")
    q_o, s_o, rs_o = O.quantize_input(x, g, WL.RMS_EPS, norm=norm)
    assert_exact(saved["q"].cpu().numpy(), q_o, "codes")
    assert_exact(saved["s_x"].cpu().numpy().view(np.uint32), s_o.view(np.uint32), "s_x")
    if out == "f32":
        assert_f32_output(y.cpu().numpy(), ref["y"], "online M=%d" % M)
    else:
        assert_bf16_output(bf16_host(y), O.f32_to_bf16(ref["y"]), "online M=%d" % M)


@pytest.mark.parametrize("name", WL.CONFIG4_PROJECTIONS)
def test_online_forward_config4_sampled_rows(name, guard):
    """M = 4096 at the prefill shapes: every row on the GPU, the oracle's online
    forward on a sample of rows (rows are independent; the weights it derives
    are the whole matrix's)."""
    c = WL.config4_projection(name)
    p = WL.PROJECTIONS[WL.PROJ_INDEX[name]]
    W = WL.master_weights(p.N, p.K, WL.master_seed(0, name))
    y, saved = online(c["x"], W, c["gain"], torch.bfloat16, guard)
    rows = np.unique(np.concatenate([[0, 4095], np.random.default_rng(5300).integers(0, 4096, 14)]))
    ref = O.online_forward(c["x"][rows], W, gain=c["gain"], eps=WL.RMS_EPS, norm=True)
    assert np.float32(saved["beta"].item()) == np.float32(ref["beta"])
    assert_exact(saved["P"].cpu().numpy(), O.pack(ref["t"]), "packed weights of the call")
    assert_bf16_output(bf16_host(y)[rows], O.f32_to_bf16(ref["y"]), "online config 4 %s" % name)


def _dequantised(q, s_x, t, beta):
    s_w = np.float32(1.0) / np.float32(beta)
    W_q = (t.astype(np.float32) / s_w).astype(np.float32)
    x_q = (q.astype(np.float32) / s_x[:, None].astype(np.float32)).astype(np.float32)
    return W_q, x_q


def _check_grad(got, ref, abs_terms, n, what):
    bound = (n + 1) * 2.0 ** -24 * abs_terms + 2.0 ** -126
    err = np.abs(got.astype(np.float64) - ref)
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert (err <= bound).all(), "%s: error %g > bound %g at %s" % (
        what, err[worst], bound[worst], worst)


@pytest.mark.parametrize("M,K,N", [(5, 272, 36), (64, 2560, 640), (130, 400, 2560)])
def test_backward_ste_matches_oracle(M, K, N, guard):
    x = WL.activations(M, K, seed=5400 + M, row_std=(0.1, 10.0))
    W = WL.master_weights(N, K, seed=5500 + N)
    y, saved = online(x, W, None, torch.float32, guard)
    gy = np.random.default_rng(5600 + M).standard_normal((M, N)).astype(np.float32)
    gx, gw = B.bitlinear_backward_ste(torch.from_numpy(gy).cuda(), saved, K)
    ref = O.online_forward(x, W)
    q_o, s_o, _ = O.quantize_input(x)
    gx_o, gw_o = O.ste_backward(gy, q_o, s_o, ref["t"], ref["beta"])
    W_q, x_q = _dequantised(q_o, s_o, ref["t"], ref["beta"])
    agy = np.abs(gy).astype(np.float64)
    _check_grad(gx.cpu().numpy(), gx_o, agy @ np.abs(W_q).astype(np.float64), N, "grad_x")
    _check_grad(gw.cpu().numpy(), gw_o, agy.T @ np.abs(x_q).astype(np.float64), M, "grad_w")


def test_backward_ste_config4_sampled(guard):
    """M = 4096 at the gate shape: all gradients on the GPU; the oracle
    recomputes sampled rows of grad_x (sampled tokens) and of grad_w (sampled
    output rows)."""
    name = "gate"
    c = WL.config4_projection(name)
    p = WL.PROJECTIONS[WL.PROJ_INDEX[name]]
    W = WL.master_weights(p.N, p.K, WL.master_seed(0, name))
    y, saved = online(c["x"], W, c["gain"], torch.bfloat16, guard)
    M, K, N = 4096, p.K, p.N
    gy = (np.random.default_rng(5700).standard_normal((M, N)) * 1e-3).astype(np.float32)
    gx, gw = B.bitlinear_backward_ste(torch.from_numpy(gy).cuda(), saved, K)
    gx, gw = gx.cpu().numpy(), gw.cpu().numpy()
    beta = float(np.float32(saved["beta"].item()))
    t = O.unpack(saved["P"].cpu().numpy())
    assert_exact(saved["P"].cpu().numpy(), O.pack(O.ternarize(W, O.weight_scale(W))), "packed")
    q, s = saved["q"].cpu().numpy(), saved["s_x"].cpu().numpy()
    rng = np.random.default_rng(5701)
    ms = np.unique(np.concatenate([[0, M - 1], rng.integers(0, M, 6)]))
    ns = np.unique(np.concatenate([[0, N - 1], rng.integers(0, N, 6)]))
    gx_o, _ = O.ste_backward(gy[ms], q[ms], s[ms], t, beta)
    W_q, _ = _dequantised(q[ms], s[ms], t, beta)
    _check_grad(gx[ms], gx_o, np.abs(gy[ms]).astype(np.float64) @ np.abs(W_q).astype(np.float64),
                N, "grad_x rows")
    _, gw_o = O.ste_backward(np.ascontiguousarray(gy[:, ns]), q, s, t[ns], beta)
    _, x_q = _dequantised(q, s, t[ns], beta)
    _check_grad(gw[ns], gw_o, np.abs(gy[:, ns]).astype(np.float64).T @ np.abs(x_q).astype(np.float64),
                M, "grad_w rows")
