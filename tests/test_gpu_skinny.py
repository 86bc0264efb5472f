"""5..64 tokens: the weight-streaming tensor-core kernel vs the oracle.

Covers both CTA schedules: equal shares with row tiles split across CTAs
(entry points with a workspace: bitlinear_forward, bitlinear_forward_batch) and
shares cut at row-tile boundaries (no workspace: bitlinear_forward_quantized*,
bitlinear_accumulate).  Accumulators bit-exact; outputs bit-exact and within
the stated tolerances.
"""
import numpy as np
import pytest
import torch

import oracle as O
import ternary_weight_bitlinear_b200 as B
from ternary_weight_bitlinear_b200 import workloads as WL
from gpu_util import assert_bf16_output, assert_exact, assert_f32_output, bf16_dev, bf16_host
from test_gpu_parity import _batch_case, _check_batch, both_pack, run_batch, run_quantized_batch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device_status_clean():
    yield
    assert B.bitlinear_device_status() == 0


@pytest.mark.parametrize("M,K,N", [
    (5, 272, 36),        # R = 9: one ragged row tile, K not a multiple of 128
    (8, 16384, 128),     # one row tile of 128 items: every CTA holds a piece of it
    (16, 400, 4 * 45),   # R = 45: two tiles, the second ragged
    (33, 2560, 640),     # npad 48
    (64, 6912, 2560),    # npad 64, the down projection's shape
])
def test_skinny_accumulate_is_exact(M, K, N, guard):
    x = WL.activations(M, K, seed=3100 + M + K, row_std=(0.1, 10.0))
    P_d, beta, P_o, beta_o = both_pack(WL.master_weights(N, K, seed=3200 + N))
    q, s, rs = B.bitlinear_act_quant(bf16_dev(x))
    q_o, s_o, rs_o = O.quantize_input(x)
    assert_exact(q.cpu().numpy(), q_o, "codes")
    acc = B.bitlinear_accumulate(q, rs, P_d, out=guard.empty((M, N), torch.int32))
    assert_exact(acc.cpu().numpy(), O.ternary_matmul(q_o, O.unpack(P_o)), "int32 accumulators")


@pytest.mark.parametrize("M,K,N,norm,out", [
    (5, 272, 36, False, "f32"),
    (8, 16384, 128, True, "bf16"),   # one tile split over every CTA: 127 partial sums
    (16, 400, 4 * 45, True, "f32"),
    (48, 2560, 6912, True, "bf16"),
    (64, 6912, 2560, False, "f32"),
])
def test_skinny_forward_split_tiles(M, K, N, norm, out, guard):
    x = WL.activations(M, K, seed=3300 + M, outlier_frac=0.001, row_std=(0.1, 10.0))
    g = WL.gain(K, seed=3400 + K) if norm else None
    P_d, beta, P_o, beta_o = both_pack(WL.master_weights(N, K, seed=3500 + N))
    dt = torch.float32 if out == "f32" else torch.bfloat16
    # a workspace of exactly the reported size, filled with garbage first
    ws = guard.empty((B.bitlinear_forward_workspace_size(M, K, N),), torch.uint8, fill=0x5A)
    ref = O.forward(x, P_o, beta_o, gain=g, eps=WL.RMS_EPS, norm=norm)["y"]
    for call in range(2):  # the second call reuses the workspace its predecessor left
        y = B.bitlinear_forward(bf16_dev(x), P_d, beta, gain=None if g is None else bf16_dev(g),
                                eps=WL.RMS_EPS, out=guard.empty((M, N), dt), workspace=ws)
        what = "skinny forward M=%d K=%d N=%d call %d" % (M, K, N, call)
        if out == "f32":
            assert_f32_output(y.cpu().numpy(), ref, what)
        else:
            assert_bf16_output(bf16_host(y), O.f32_to_bf16(ref), what)


@pytest.mark.parametrize("M", [5, 8, 17, 32, 64])
def test_skinny_batch_seven_projections(M, guard):
    """Config 3's shapes: the seven 2B4T projections as one batch (split schedule),
    then the same codes through the quantized batch (tile-cut schedule)."""
    specs = [(p.K, p.N, True, torch.bfloat16, p.name == "down") for p in WL.PROJECTIONS]
    items, refs = _batch_case(specs, M, seed=3600 + M, guard=guard)
    run_batch(items, M, guard)
    _check_batch(items, refs, "skinny batch M=%d" % M)
    qitems = []
    for it in items:
        q, s, rs = B.bitlinear_act_quant(it["x"], it["gain"], WL.RMS_EPS)
        y2 = guard.empty(it["y"].shape, it["y"].dtype)
        d = dict(q=q, s_x=s, rowsum=rs, P=it["P"], beta=it["beta"], y=y2)
        if "residual" in it:
            d["residual"] = it["residual"]
        qitems.append(d)
    B.bitlinear_forward_quantized_batch(B.make_quantized_batch(qitems), M)  # no workspace
    for i, (it, d) in enumerate(zip(items, qitems)):
        assert torch.equal(it["y"].view(torch.int16), d["y"].view(torch.int16)), \
            "quantized batch differs from forward batch, problem %d" % i


def test_skinny_batch_more_problems_than_one_launch(guard):
    """70 problems (two launches of the kernel) with M = 12."""
    specs = [(16 * (1 + i % 9), 4 * (1 + i % 11), i % 2 == 0,
              torch.float32 if i % 5 == 0 else torch.bfloat16, i % 3 == 0 and i % 5 != 0)
             for i in range(70)]
    items, refs = _batch_case(specs, 12, seed=3700, guard=guard)
    run_batch(items, 12, guard)
    _check_batch(items, refs, "70-problem skinny batch")


def test_skinny_quantized_single_matches_forward(guard):
    M, K, N = 24, 2560, 2560
    x = WL.activations(M, K, seed=3800, outlier_frac=0.001)
    P_d, beta, P_o, beta_o = both_pack(WL.master_weights(N, K, seed=3801))
    q, s, rs = B.bitlinear_act_quant(bf16_dev(x))
    y1 = B.bitlinear_forward_quantized(q, s, rs, P_d, beta, out=guard.empty((M, N), torch.bfloat16))
    ref = O.forward(x, P_o, beta_o, norm=False)["y"]
    assert_bf16_output(bf16_host(y1), O.f32_to_bf16(ref), "skinny quantized single")
