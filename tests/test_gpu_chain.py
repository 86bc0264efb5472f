"""One token through dependent decoder steps in one persistent launch
(bitlinear_decode_chain_*) against the oracle and against the same steps run
launch by launch.

Per layer (BitNet-2B4T shapes, attention omitted): step A quantises the layer
input (RMSNorm) and runs q, k, v and o, o's output added to the residual
stream into a second buffer; step B the FFN input norm and the fused gate|up
relu^2 pass; step C the sub-norm and down, added back into the first buffer.
The oracle composes its forward, relu2_mul and residual_add in that order.
"""
import numpy as np
import pytest
import torch

import oracle as O
import ternary_weight_bitlinear_b200 as B
from ternary_weight_bitlinear_b200 import workloads as WL
from gpu_util import assert_bf16_output, bf16_dev, bf16_host

pytestmark = pytest.mark.gpu
H, I = WL.HIDDEN, WL.INTERMEDIATE


@pytest.fixture(scope="module", autouse=True)
def _device_status_clean():
    yield
    assert B.bitlinear_device_status() == 0


def layer_weights(l):
    """Device and oracle weights of layer l (seeded masters), and its gains."""
    W = {n: WL.master_weights(p.N, p.K, WL.master_seed(l, n))
         for n, p in zip([q.name for q in WL.PROJECTIONS], WL.PROJECTIONS)}
    dev, ora = {}, {}
    for n in ("q", "k", "v", "o", "down"):
        P, b = B.bitlinear_pack(torch.from_numpy(W[n]).cuda())
        dev[n] = (P, float(b.item()))
        ora[n] = O.pack_master(W[n])
        assert np.float32(dev[n][1]) == np.float32(ora[n][1])
    P2, b2 = B.bitlinear_pack_gate_up(torch.from_numpy(W["gate"]).cuda(),
                                      torch.from_numpy(W["up"]).cuda())
    dev["pair"] = (P2, [float(v) for v in b2.cpu()])
    ora["gate"], ora["up"] = O.pack_master(W["gate"]), O.pack_master(W["up"])
    gains = dict(a=WL.gain(H, 1000 * (l + 1) + 12), f=WL.gain(H, 1000 * (l + 1) + 10),
                 s=WL.gain(I, 1000 * (l + 1) + 11))
    return dev, ora, gains


class Chain:
    """Device buffers and the chain of 3 steps per layer."""

    def __init__(self, layers, x0):
        self.layers = [layer_weights(l) for l in range(layers)]
        self.xa = bf16_dev(x0).reshape(-1).clone()
        self.xb = torch.empty_like(self.xa)
        self.z = torch.empty(I, dtype=torch.bfloat16, device="cuda")
        self.qkv = {n: torch.empty(p.N, dtype=torch.bfloat16, device="cuda")
                    for n, p in zip(("q", "k", "v"), WL.PROJECTIONS[:3])}
        self.gains = [{k: bf16_dev(v) for k, v in g.items()} for _, _, g in self.layers]
        steps = []
        for (dev, _, _), g in zip(self.layers, self.gains):
            steps.append(dict(x=self.xa, gain=g["a"], eps=WL.RMS_EPS, problems=[
                dict(P=dev[n][0], beta=dev[n][1], y=self.qkv[n]) for n in ("q", "k", "v")] + [
                dict(P=dev["o"][0], beta=dev["o"][1], y=self.xb, residual=self.xa)]))
            steps.append(dict(x=self.xb, gain=g["f"], eps=WL.RMS_EPS, problems=[
                dict(P=dev["pair"][0], beta=dev["pair"][1][0], beta_up=dev["pair"][1][1],
                     y=self.z, kind="gate_up")]))
            steps.append(dict(x=self.z, gain=g["s"], eps=WL.RMS_EPS, problems=[
                dict(P=dev["down"][0], beta=dev["down"][1], y=self.xa, residual=self.xb)]))
        self.arr = B.make_chain(steps)
        self.ws = B.bitlinear_decode_chain_prepare(self.arr)

    def run(self):
        B.bitlinear_decode_chain_run(self.ws, len(self.arr))

    def run_launch_by_launch(self):
        """The same steps through the separate entry points."""
        for (dev, _, _), g in zip(self.layers, self.gains):
            xa, xb = self.xa.view(1, H), self.xb.view(1, H)
            q, s, rs = B.bitlinear_act_quant(xa, g["a"], WL.RMS_EPS)
            for n in ("q", "k", "v"):
                B.bitlinear_forward_quantized(q, s, rs, dev[n][0], dev[n][1], out=self.qkv[n].view(1, -1))
            xb.copy_(xa)
            B.bitlinear_forward_quantized(q, s, rs, dev["o"][0], dev["o"][1], residual=xb, out=xb)
            q, s, rs = B.bitlinear_act_quant(xb, g["f"], WL.RMS_EPS)
            P2, (bg, bu) = dev["pair"]
            B.bitlinear_forward_gate_up(q, s, rs, P2, bg, bu, out=self.z.view(1, I))
            q, s, rs = B.bitlinear_act_quant(self.z.view(1, I), g["s"], WL.RMS_EPS)
            xa.copy_(xb)
            B.bitlinear_forward_quantized(q, s, rs, dev["down"][0], dev["down"][1], residual=xa, out=xa)


def oracle_chain(layers, x0):
    """(final residual stream, last layer's q, k, v outputs, last z) by the oracle."""
    xa = x0.copy()
    for _, ora, g in layers:
        f = lambda x, n, gain: O.f32_to_bf16(O.forward(x, ora[n][0], ora[n][1], gain=gain,
                                                       eps=WL.RMS_EPS, norm=True)["y"])
        qkv = {n: f(xa, n, g["a"]) for n in ("q", "k", "v")}
        xb = O.residual_add(xa, f(xa, "o", g["a"]))
        z = O.relu2_mul(f(xb, "gate", g["f"]), f(xb, "up", g["f"]))
        xa = O.residual_add(xb, f(z, "down", g["s"]))
    return xa, qkv, z, xb


@pytest.mark.parametrize("layers", [1, 3])
def test_decode_chain_matches_oracle(layers):
    x0 = WL.activations(1, H, seed=7)
    ch = Chain(layers, x0)
    ch.run()
    torch.cuda.synchronize()
    xa, qkv, z, xb = oracle_chain(ch.layers, x0)
    assert_bf16_output(bf16_host(ch.xa).reshape(1, H), xa, "residual stream after %d layers" % layers)
    assert_bf16_output(bf16_host(ch.xb).reshape(1, H), xb, "stream after the last o")
    assert_bf16_output(bf16_host(ch.z).reshape(1, I), z, "last z")
    for n in ("q", "k", "v"):
        assert_bf16_output(bf16_host(ch.qkv[n]).reshape(1, -1), qkv[n], "last %s" % n)


def test_decode_chain_30_layers_equals_launch_by_launch_and_oracle():
    x0 = WL.activations(1, H, seed=8)
    ch = Chain(WL.LAYERS, x0)
    for rep in range(2):  # the second run finds the first one's counter and buffers
        ch.xa.copy_(bf16_dev(x0).reshape(-1))
        ch.run()
    torch.cuda.synchronize()
    got = bf16_host(ch.xa).copy()
    ch.xa.copy_(bf16_dev(x0).reshape(-1))
    ch.run_launch_by_launch()
    torch.cuda.synchronize()
    assert np.array_equal(got, bf16_host(ch.xa)), "persistent chain differs from the launches"
    xa, _, _, _ = oracle_chain(ch.layers, x0)
    assert_bf16_output(got.reshape(1, H), xa, "residual stream after 30 layers")


@pytest.mark.parametrize("K", [2560, 6912])
def test_chain_quantiser_on_rms_boundary_rows(K):
    """Input rows whose RMSNorm factor is decided by the rounding of the exact
    sum of squares (the chain's quantiser must take its exact-sum path), one
    step each, fp32 outputs, against the oracle's forward."""
    from rms_boundary import straddle_rows
    rows = straddle_rows(4, K, WL.RMS_EPS, seed=K + 11)
    N = 256
    W = WL.master_weights(N, K, seed=K + 12)
    P, b = B.bitlinear_pack(torch.from_numpy(W).cuda())
    P_o, b_o = O.pack_master(W)
    gain = WL.gain(K, seed=K + 13)
    g_d = bf16_dev(gain)
    xs = [bf16_dev(rows[i]).reshape(-1) for i in range(len(rows))]
    ys = [torch.empty(N, dtype=torch.float32, device="cuda") for _ in xs]
    steps = [dict(x=x, gain=g_d, eps=WL.RMS_EPS,
                  problems=[dict(P=P, beta=float(b.item()), y=y, kind="f32")])
             for x, y in zip(xs, ys)]
    arr = B.make_chain(steps)
    ws = B.bitlinear_decode_chain_prepare(arr)
    B.bitlinear_decode_chain_run(ws, len(arr))
    torch.cuda.synchronize()
    from gpu_util import assert_f32_output
    for i, y in enumerate(ys):
        ref = O.forward(rows[i:i + 1], P_o, b_o, gain=gain, eps=WL.RMS_EPS, norm=True)["y"]
        assert_f32_output(y.cpu().numpy().reshape(1, N), ref, "boundary row %d K=%d" % (i, K))
