"""The FFN block's gate/up pair in one pass (bitlinear_pack_gate_up,
bitlinear_forward_gate_up) against the oracle.

The oracle has no fused function: the expected packed bytes are the oracle's
pack of the two separately ternarised matrices stacked as [gate; up], and the
expected output is the oracle's relu2_mul of the two projections' bf16
outputs, each computed by the oracle's forward with its own weight scale.
Every shape runs through the decode kernel (M <= 4), the 5..64-token kernel
(with and without its split workspace) or the tensor-core GEMM; outputs sit in
guarded buffers.
"""
import numpy as np
import pytest
import torch

import oracle as O
import ternary_weight_bitlinear_b200 as B
from ternary_weight_bitlinear_b200 import workloads as WL
from gpu_util import assert_bf16_output, assert_exact, bf16_dev, bf16_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device_status_clean():
    yield
    assert B.bitlinear_device_status() == 0


def pack_pair(Wg, Wu, guard=None):
    """(P2, beta_g, beta_u) on the device, checked bit for bit against the
    oracle's pack of [ternarise(Wg); ternarise(Wu)], plus the oracle's
    separate packings (Pg, bg, Pu, bu)."""
    I, K = Wg.shape
    P2 = guard.empty((I // 2, K), torch.uint8) if guard else None
    P2, beta = B.bitlinear_pack_gate_up(torch.from_numpy(Wg).cuda(), torch.from_numpy(Wu).cuda(),
                                        P2=P2)
    bg, bu = (float(v) for v in beta.cpu().numpy())
    bg_o, bu_o = O.weight_scale(Wg), O.weight_scale(Wu)
    assert np.float32(bg) == np.float32(bg_o) and np.float32(bu) == np.float32(bu_o)
    tg, tu = O.ternarize(Wg, bg_o), O.ternarize(Wu, bu_o)
    assert_exact(P2.cpu().numpy(), O.pack(np.concatenate([tg, tu])), "packed gate/up pair")
    # packing the stacked ternary matrices gives the same bytes
    t_cat = torch.from_numpy(np.concatenate([tg, tu])).cuda()
    assert_exact(B.bitlinear_pack_ternary(t_cat).cpu().numpy(), P2.cpu().numpy(), "pack_ternary")
    return P2, bg, bu, (O.pack(tg), bg_o, O.pack(tu), bu_o)


def oracle_gate_up(x, gain, norm, ora):
    Pg, bg, Pu, bu = ora
    g = O.f32_to_bf16(O.forward(x, Pg, bg, gain=gain, eps=WL.RMS_EPS, norm=norm)["y"])
    u = O.f32_to_bf16(O.forward(x, Pu, bu, gain=gain, eps=WL.RMS_EPS, norm=norm)["y"])
    return O.relu2_mul(g, u)


@pytest.mark.parametrize("I,K", [(8, 16), (12, 48), (72, 272), (6912, 2560)])
def test_pack_gate_up_matches_oracle(I, K, guard):
    pack_pair(WL.master_weights(I, K, seed=I + K), WL.master_weights(I, K, seed=I + K + 1), guard)


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 16, 33, 64, 65, 130])
@pytest.mark.parametrize("I,K,norm", [(6912, 2560, True), (72, 272, False)])
def test_forward_gate_up_matches_oracle(M, I, K, norm, guard):
    Wg = WL.master_weights(I, K, seed=4000 + I)
    Wu = WL.master_weights(I, K, seed=4001 + I)
    P2, bg, bu, ora = pack_pair(Wg, Wu)
    x = WL.activations(M, K, seed=4100 + M, outlier_frac=0.001, row_std=(0.1, 10.0))
    g = WL.gain(K, seed=4200) if norm else None
    q, s, rs = B.bitlinear_act_quant(bf16_dev(x), None if g is None else bf16_dev(g), WL.RMS_EPS)
    ref = oracle_gate_up(x, g, norm, ora)
    ws = guard.workspace(B.bitlinear_quantized_batch_workspace_size(M))
    for w in (ws, None):  # equal CTA shares (split tiles), then shares cut at row tiles
        z = B.bitlinear_forward_gate_up(q, s, rs, P2, bg, bu, out=guard.empty((M, I), torch.bfloat16),
                                        workspace=w)
        assert_bf16_output(bf16_host(z), ref, "gate/up M=%d I=%d K=%d ws=%s" % (M, I, K, w is not None))


def test_gate_up_prefill_sampled_rows(guard):
    """M = 4096 tokens at the FFN shape through the tensor-core GEMM; the
    oracle recomputes a sample of rows (rows are independent)."""
    M, I, K = 4096, WL.INTERMEDIATE, WL.HIDDEN
    P2, bg, bu, ora = pack_pair(WL.master_weights(I, K, seed=4300), WL.master_weights(I, K, seed=4301))
    c = WL.config4_projection("gate", M)
    q, s, rs = B.bitlinear_act_quant(bf16_dev(c["x"]), bf16_dev(c["gain"]), WL.RMS_EPS)
    z = bf16_host(B.bitlinear_forward_gate_up(q, s, rs, P2, bg, bu,
                                              out=guard.empty((M, I), torch.bfloat16)))
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 4095],
                                     np.random.default_rng(4302).integers(0, M, 27)]))
    ref = oracle_gate_up(c["x"][rows], c["gain"], True, ora)
    assert_bf16_output(z[rows], ref, "gate/up prefill")


def test_config5_chain_with_fused_gate_up(guard):
    """Config 5 (30 FFN blocks in order, M = 16) with the fused gate/up pass:
    bit for bit the oracle's FFN block after every layer."""
    M = 16
    x = WL.config5_input(M)
    x_d = guard.copy(bf16_dev(x))
    x_o = x.copy()
    H, I = WL.HIDDEN, WL.INTERMEDIATE
    ws = guard.workspace(B.bitlinear_quantized_batch_workspace_size(M))
    z = guard.empty((M, I), torch.bfloat16)
    for layer in range(WL.LAYERS):
        L = WL.config5_layer(layer)
        P2, bg, bu, (Pg_o, bg_o, Pu_o, bu_o) = pack_pair(L["W_gate"], L["W_up"])
        Pd, bd = B.bitlinear_pack(torch.from_numpy(L["W_down"]).cuda())
        bd = float(bd.item())
        Pd_o, bd_o = O.pack_master(L["W_down"])
        q, s, rs = B.bitlinear_act_quant(x_d, bf16_dev(L["g_in"]), WL.RMS_EPS)
        B.bitlinear_forward_gate_up(q, s, rs, P2, bg, bu, out=z, workspace=ws)
        q2, s2, rs2 = B.bitlinear_act_quant(z, bf16_dev(L["g_sub"]), WL.RMS_EPS)
        B.bitlinear_forward_quantized(q2, s2, rs2, Pd, bd, residual=x_d, out=x_d)
        x_o = O.ffn_block(x_o, L["g_in"], L["g_sub"], WL.RMS_EPS, Pg_o, bg_o, Pu_o, bu_o, Pd_o, bd_o)
        assert_bf16_output(bf16_host(x_d), x_o, "fused config 5 after layer %d" % layer)
