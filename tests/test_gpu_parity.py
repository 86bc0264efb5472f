"""GPU vs oracle parity, through the C ABI, on the seeded workloads.

Bit-exact: packed bytes, beta, int8 codes, s_x, row sums, int32 accumulators.
Outputs: bit-exact and within the stated tolerances (fp32 1e-6, bf16 8e-3 rel).
Every input comes from the seeded generators; each side prepares its own
weights from the same fp32 masters.
"""
import numpy as np
import pytest
import torch

import oracle as O
import ternary_weight_bitlinear_b200 as B
from ternary_weight_bitlinear_b200 import workloads as WL
from gpu_util import (assert_bf16_output, assert_exact, assert_f32_output, bf16_dev, bf16_host)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device_status_clean():
    yield
    assert B.bitlinear_device_status() == 0


def both_pack(W):
    """(P_gpu, beta_gpu_float, P_oracle, beta_oracle) after checking they agree."""
    P_d, beta_d = B.bitlinear_pack(torch.from_numpy(W).cuda())
    P_o, beta_o = O.pack_master(W)
    beta_g = float(beta_d.item())
    assert np.float32(beta_g) == np.float32(beta_o), (beta_g, beta_o)
    assert_exact(P_d.cpu().numpy(), P_o, "packed bytes")
    return P_d, beta_g, P_o, beta_o


def run_forward(cfg, P_d, beta, P_o, beta_o, what, guard):
    """Forward through the C ABI into a guarded output and an exactly sized
    guarded workspace, checked against the oracle."""
    x = cfg["x"]
    gain = cfg.get("gain") if cfg["norm"] else None
    out_dtype = torch.float32 if cfg["out"] == "f32" else torch.bfloat16
    M, K = x.shape
    N = 4 * P_d.shape[0]
    y = B.bitlinear_forward(bf16_dev(x), P_d, beta, gain=None if gain is None else bf16_dev(gain),
                            eps=WL.RMS_EPS, out=guard.empty((M, N), out_dtype),
                            workspace=guard.workspace(B.bitlinear_forward_workspace_size(M, K, N)))
    ref = O.forward(x, P_o, beta_o, gain=gain, eps=WL.RMS_EPS, norm=cfg["norm"])
    if out_dtype == torch.float32:
        assert_f32_output(y.cpu().numpy(), ref["y"], what)
    else:
        assert_bf16_output(bf16_host(y), O.f32_to_bf16(ref["y"]), what)
    return y, ref


# ---------------------------------------------------------------------------
# weight preparation
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("N,K", [(4, 16), (12, 48), (128, 256), (132, 80), (640, 2560),
                                 (2560, 6912), (6912, 2560)])
def test_pack_matches_oracle(N, K):
    both_pack(WL.master_weights(N, K, seed=N * 7 + K))


def test_pack_special_weights():
    both_pack(np.zeros((8, 32), np.float32))                       # beta floors at 1e-5
    both_pack(np.eye(256, dtype=np.float32))                       # t = I
    W = WL.master_weights(64, 64, seed=3)
    W[::3] *= 1e-20                                               # tiny magnitudes mixed in
    both_pack(W)
    both_pack(np.full((16, 32), 0.5, np.float32) * np.sign(WL.master_weights(16, 32, 4)))


@pytest.mark.parametrize("N,K", [(4, 16), (36, 64), (640, 2560)])
def test_pack_ternary_and_unpack(N, K):
    rng = np.random.default_rng(N + K)
    t = rng.integers(-1, 2, (N, K)).astype(np.int8)
    P_d = B.bitlinear_pack_ternary(torch.from_numpy(t).cuda())
    assert_exact(P_d.cpu().numpy(), O.pack(t), "pack_ternary")
    assert_exact(B.bitlinear_unpack(P_d).cpu().numpy(), t, "unpack")
    # the never-written bit pair 11 decodes to +2 on both sides
    P_bad = rng.integers(0, 256, (N // 4, K)).astype(np.uint8)
    assert_exact(B.bitlinear_unpack(torch.from_numpy(P_bad).cuda()).cpu().numpy(),
                 O.unpack(P_bad), "unpack of arbitrary bytes")


# ---------------------------------------------------------------------------
# activation quantisation
# ---------------------------------------------------------------------------
def special_rows(x):
    """Overwrite a few rows with the method's degenerate cases."""
    M, K = x.shape
    f = WL.to_bf16_bits
    if M > 1:
        x[1] = 0                                                    # all zero: 1e-5 floor
    if M > 2:
        x[2] = f(np.full(K, 3e-7, np.float32))                      # below the floor
    if M > 3:
        x[3] = f(np.full(K, -2.5, np.float32))                      # constant row
    if M > 4:
        r = np.zeros(K, np.float32)
        r[K // 2] = 1000.0
        x[4] = f(r)                                                 # single spike
    return x


def guarded_quant(guard, M, K):
    """Guarded code, scale and row-sum buffers for an [M,K] quantisation."""
    return dict(q=guard.empty((M, K), torch.int8), s_x=guard.empty(M, torch.float32),
                rowsum=guard.empty(M, torch.int32))


@pytest.mark.parametrize("norm", [False, True])
@pytest.mark.parametrize("M,K", [(1, 16), (3, 256), (4, 2560), (7, 6912), (64, 2560), (257, 272),
                                 # 1024+ rows: the register-resident kernels (two warps per
                                 # row up to K = 2560, four up to 7168) and, past that, the
                                 # shared-memory warp kernel
                                 (1024, 2560), (1031, 6912), (1100, 272), (1024, 2576),
                                 (1025, 7168), (1024, 8192), (1030, 8208)])
def test_act_quant_matches_oracle(M, K, norm, guard):
    x = special_rows(WL.activations(M, K, seed=M * 131 + K, outlier_frac=0.001))
    gain = WL.gain(K, seed=K) if norm else None
    q, s, rs = B.bitlinear_act_quant(bf16_dev(x), None if gain is None else bf16_dev(gain),
                                     WL.RMS_EPS, **guarded_quant(guard, M, K))
    q_o, s_o, rs_o = O.quantize_input(x, gain, WL.RMS_EPS, norm=norm)
    assert_exact(s.cpu().numpy().view(np.uint32), s_o.view(np.uint32), "s_x")
    assert_exact(q.cpu().numpy(), q_o, "codes")
    assert_exact(rs.cpu().numpy(), rs_o, "row sums")


@pytest.mark.parametrize("M,K", [(3, 256), (1024, 2560), (1030, 6912), (1024, 8208)])
def test_act_quant_tie_rows(M, K, guard):
    """Rows with max|x| = 127 (scale exactly 1) and half-integer entries: every
    quantiser kernel rounds the ties to the even neighbour, as the oracle."""
    ties = [127.0, 0.5, 1.5, 2.5, 3.5, -0.5, -1.5, -2.5, 126.5, -126.5, 4.5, -3.5]
    codes = [127, 0, 2, 2, 4, 0, -2, -2, 126, -126, 4, -4]
    x = WL.activations(M, K, seed=M + 3 * K)
    at = np.linspace(0, M - 1, min(M, 6)).astype(int)
    row = np.zeros(K, np.float32)
    row[:len(ties)] = ties
    for i, m in enumerate(at):
        x[m] = WL.to_bf16_bits(row if i % 2 == 0 else -row)
    q, s, rs = B.bitlinear_act_quant(bf16_dev(x), **guarded_quant(guard, M, K))
    q_o, s_o, rs_o = O.quantize_input(x)
    qh = q.cpu().numpy()
    for i, m in enumerate(at):
        sign = 1 if i % 2 == 0 else -1
        assert list(qh[m, :len(codes)]) == [sign * c for c in codes]
    assert_exact(s.cpu().numpy().view(np.uint32), s_o.view(np.uint32), "s_x")
    assert_exact(qh, q_o, "codes")
    assert_exact(rs.cpu().numpy(), rs_o, "row sums")


@pytest.mark.parametrize("M,K", [(8, 2560),      # one CTA per row
                                 (1024, 2560),   # many rows: two warps per row
                                 (1031, 6912),   # four warps per row
                                 (1024, 8208),   # past 7168: the shared-memory warp kernel
                                 (1, 16)])
def test_act_quant_rms_boundary_rows(M, K, guard):
    """Rows whose RMSNorm factor is decided by the rounding of the exact sum of
    squares (the fast interval test must fall back to the exact sum) at
    several places of the batch."""
    from rms_boundary import straddle_rows
    x = WL.activations(M, K, seed=M * 7 + K)
    n = min(M, 8)
    at = np.linspace(0, M - 1, n).astype(int)
    x[at] = straddle_rows(n, K, WL.RMS_EPS, seed=K + M)
    gain = WL.gain(K, seed=K + 1)
    q, s, rs = B.bitlinear_act_quant(bf16_dev(x), bf16_dev(gain), WL.RMS_EPS,
                                     **guarded_quant(guard, M, K))
    q_o, s_o, rs_o = O.quantize_input(x, gain, WL.RMS_EPS, norm=True)
    assert_exact(s.cpu().numpy().view(np.uint32), s_o.view(np.uint32), "s_x")
    assert_exact(q.cpu().numpy(), q_o, "codes")
    assert_exact(rs.cpu().numpy(), rs_o, "row sums")


# ---------------------------------------------------------------------------
# exact int32 accumulators
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("M,K,N", [(1, 16, 4), (2, 64, 12), (3, 256, 128), (4, 2560, 640),
                                   (5, 272, 36), (9, 6912, 2560), (1, 65536, 8), (2, 65536, 8)])
def test_accumulate_is_exact(M, K, N, guard):
    x = special_rows(WL.activations(M, K, seed=M + K + N, row_std=(0.1, 10.0)))
    W = WL.master_weights(N, K, seed=K + N)
    P_d, beta, P_o, beta_o = both_pack(W)
    q, s, rs = B.bitlinear_act_quant(bf16_dev(x))
    q_o, s_o, rs_o = O.quantize_input(x)
    assert_exact(q.cpu().numpy(), q_o, "codes")
    acc = B.bitlinear_accumulate(q, rs, P_d, out=guard.empty((M, N), torch.int32))
    acc_o = O.ternary_matmul(q_o, O.unpack(P_o))
    assert_exact(acc.cpu().numpy(), acc_o, "int32 accumulators")


# ---------------------------------------------------------------------------
# the five workloads
# ---------------------------------------------------------------------------
def test_config1_single_bitlinear_fp32(guard):
    c = WL.config1()
    P_d, beta, P_o, beta_o = both_pack(c["W"])
    y, ref = run_forward(c, P_d, beta, P_o, beta_o, "config 1", guard)
    assert not y[1].any()                      # the all-zero token gives +0 outputs
    assert not torch.signbit(y[1]).any()


@pytest.mark.parametrize("layer", [0, 29])
def test_config2_decode_all_projections(layer, guard):
    for p in WL.PROJECTIONS:
        c = WL.config2_projection(layer, p.name)
        W = WL.master_weights(p.N, p.K, WL.master_seed(layer, p.name))
        P_d, beta, P_o, beta_o = both_pack(W)
        run_forward(c, P_d, beta, P_o, beta_o, "config 2 %s" % p.name, guard)


@pytest.mark.parametrize("M", [8, 32, 64])
def test_config3_batched_decode(M, guard):
    for p in WL.PROJECTIONS:
        c = WL.config3_projection(0, p.name, M)
        W = WL.master_weights(p.N, p.K, WL.master_seed(0, p.name))
        P_d, beta, P_o, beta_o = both_pack(W)
        run_forward(c, P_d, beta, P_o, beta_o, "config 3 %s M=%d" % (p.name, M), guard)


def test_config4_prefill_sampled_rows(guard):
    """M=4096: the GPU computes every row; the oracle recomputes a sample of
    rows (rows are independent) and the full int8 codes of one projection."""
    rng = np.random.default_rng(4096)
    for name in WL.CONFIG4_PROJECTIONS:
        c = WL.config4_projection(name)
        p = WL.PROJECTIONS[WL.PROJ_INDEX[name]]
        W = WL.master_weights(p.N, p.K, WL.master_seed(0, name))
        P_d, beta, P_o, beta_o = both_pack(W)
        x_d, g_d = bf16_dev(c["x"]), bf16_dev(c["gain"])
        M = c["x"].shape[0]
        y = bf16_host(B.bitlinear_forward(
            x_d, P_d, beta, gain=g_d, eps=WL.RMS_EPS, out=guard.empty((M, p.N), torch.bfloat16),
            workspace=guard.workspace(B.bitlinear_forward_workspace_size(M, p.K, p.N))))
        rows = np.unique(np.concatenate([[0, 1, 4095], rng.integers(0, 4096, 29)]))
        ref = O.forward(c["x"][rows], P_o, beta_o, gain=c["gain"], eps=WL.RMS_EPS, norm=True)
        assert_bf16_output(y[rows], O.f32_to_bf16(ref["y"]), "config 4 %s" % name)
        if name == "down":
            q, s, _ = B.bitlinear_act_quant(x_d, g_d, WL.RMS_EPS)
            q_o, s_o, _ = O.quantize_input(c["x"], c["gain"], WL.RMS_EPS, norm=True)
            assert_exact(q.cpu().numpy(), q_o, "config 4 codes")
            assert_exact(s.cpu().numpy().view(np.uint32), s_o.view(np.uint32), "config 4 s_x")


def gpu_ffn_block(x_d, g_in, g_sub, Pg, bg, Pu, bu, Pd, bd, guard):
    """One FFN block through the C ABI, every intermediate in a guarded
    buffer; updates x_d in place."""
    M, H = x_d.shape
    I = 4 * Pg.shape[0]
    q, s, rs = B.bitlinear_act_quant(x_d, g_in, WL.RMS_EPS, **guarded_quant(guard, M, H))
    a = B.bitlinear_forward_quantized(q, s, rs, Pg, bg, out=guard.empty((M, I), torch.bfloat16))
    b = B.bitlinear_forward_quantized(q, s, rs, Pu, bu, out=guard.empty((M, I), torch.bfloat16))
    z = B.bitlinear_relu2_mul(a, b, out=guard.empty((M, I), torch.bfloat16))
    q2, s2, rs2 = B.bitlinear_act_quant(z, g_sub, WL.RMS_EPS, **guarded_quant(guard, M, I))
    B.bitlinear_forward_quantized(q2, s2, rs2, Pd, bd, residual=x_d, out=x_d)
    return x_d


def test_config5_ffn_chain_30_layers(guard):
    M = 16
    x = WL.config5_input(M)
    x_d = guard.copy(bf16_dev(x))
    x_o = x.copy()
    for layer in range(WL.LAYERS):
        L = WL.config5_layer(layer)
        Pg, bg, Pg_o, bg_o = both_pack(L["W_gate"])
        Pu, bu, Pu_o, bu_o = both_pack(L["W_up"])
        Pd, bd, Pd_o, bd_o = both_pack(L["W_down"])
        gpu_ffn_block(x_d, bf16_dev(L["g_in"]), bf16_dev(L["g_sub"]), Pg, bg, Pu, bu, Pd, bd,
                      guard)
        x_o = O.ffn_block(x_o, L["g_in"], L["g_sub"], WL.RMS_EPS, Pg_o, bg_o, Pu_o, bu_o, Pd_o,
                          bd_o)
        assert_bf16_output(bf16_host(x_d), x_o, "config 5 after layer %d" % layer)


# ---------------------------------------------------------------------------
# glue and edge cases
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("n", [8, 13, 6912 * 16, 1000003])
def test_relu2_mul_matches_oracle(n, guard):
    rng = np.random.default_rng(n)
    a = WL.to_bf16_bits((rng.standard_normal(n) * 3).astype(np.float32))
    b = WL.to_bf16_bits((rng.standard_normal(n) * 3).astype(np.float32))
    z = B.bitlinear_relu2_mul(bf16_dev(a), bf16_dev(b), out=guard.empty(n, torch.bfloat16))
    assert_exact(bf16_host(z), O.relu2_mul(a, b), "relu2_mul")


def test_residual_epilogue_matches_oracle(guard):
    M, K, N = 6, 256, 64
    x = WL.activations(M, K, seed=77)
    res = WL.activations(M, N, seed=78)
    W = WL.master_weights(N, K, seed=79)
    P_d, beta, P_o, beta_o = both_pack(W)
    q, s, rs = B.bitlinear_act_quant(bf16_dev(x))
    r_d = guard.copy(bf16_dev(res))
    B.bitlinear_forward_quantized(q, s, rs, P_d, beta, residual=r_d, out=r_d)
    y_o = O.forward(x, P_o, beta_o)["y"]
    assert_exact(bf16_host(r_d), O.residual_add(res, O.f32_to_bf16(y_o)), "residual epilogue")


def test_empty_batch_is_a_no_op():
    P = torch.zeros(8, 64, dtype=torch.uint8, device="cuda")
    x = torch.zeros(0, 64, dtype=torch.bfloat16, device="cuda")
    y = B.bitlinear_forward(x, P, 1.0)
    assert y.shape == (0, 32)


@pytest.mark.parametrize("M,K,N", [(1, 16, 4), (2, 32, 8), (3, 4096 + 16, 12), (4, 16384, 20),
                                   (5, 64, 4), (1, 65536, 16), (3, 65536, 8)])
def test_ragged_and_extreme_shapes(M, K, N, guard):
    x = WL.activations(M, K, seed=M * K + N, outlier_frac=0.01)
    g = WL.gain(K, seed=N)
    W = WL.master_weights(N, K, seed=K - N)
    P_d, beta, P_o, beta_o = both_pack(W)
    for norm in (False, True):
        c = dict(x=x, gain=g, norm=norm, out="f32")
        run_forward(c, P_d, beta, P_o, beta_o, "M=%d K=%d N=%d norm=%s" % (M, K, N, norm),
                    guard)


# ---------------------------------------------------------------------------
# batched forwards (independent problems in one call)
# ---------------------------------------------------------------------------
def _batch_case(specs, M, seed, guard):
    """specs: list of (K, N, norm, out dtype, residual) -> (items, oracle outputs);
    outputs in guarded buffers."""
    items, refs = [], []
    for i, (K, N, norm, dt, res) in enumerate(specs):
        x = WL.activations(M, K, seed=seed + i, outlier_frac=0.001)
        g = WL.gain(K, seed=seed + 100 + i) if norm else None
        P_d, beta, P_o, beta_o = both_pack(WL.master_weights(N, K, seed=seed + 200 + i))
        y_o = O.forward(x, P_o, beta_o, gain=g, eps=WL.RMS_EPS, norm=norm)["y"]
        it = dict(x=bf16_dev(x), P=P_d, beta=beta, y=guard.empty((M, N), dt))
        if norm:
            it["gain"] = bf16_dev(g)
        if res:
            r = WL.activations(M, N, seed=seed + 300 + i)
            it["residual"] = bf16_dev(r)
            refs.append(("bf16", O.residual_add(r, O.f32_to_bf16(y_o))))
        elif dt == torch.float32:
            refs.append(("f32", y_o))
        else:
            refs.append(("bf16", O.f32_to_bf16(y_o)))
        items.append(it)
    return items, refs


def run_batch(items, M, guard):
    """bitlinear_forward_batch with an exactly sized guarded workspace."""
    arr = B.make_batch(items)
    B.bitlinear_forward_batch(arr, M, WL.RMS_EPS,
                              workspace=guard.workspace(B.bitlinear_forward_batch_workspace_size(arr, M)))


def run_quantized_batch(items, M, guard):
    """bitlinear_forward_quantized_batch with an exactly sized guarded workspace."""
    B.bitlinear_forward_quantized_batch(
        B.make_quantized_batch(items), M,
        workspace=guard.workspace(B.bitlinear_quantized_batch_workspace_size(M)))


def _check_batch(items, refs, what):
    for i, (it, (kind, ref)) in enumerate(zip(items, refs)):
        if kind == "f32":
            assert_f32_output(it["y"].cpu().numpy(), ref, "%s problem %d" % (what, i))
        else:
            assert_bf16_output(bf16_host(it["y"]), ref, "%s problem %d" % (what, i))


@pytest.mark.parametrize("layer", [0, 17])
def test_batch_config2_layer(layer, guard):
    """A decode layer's seven projections (independent inputs) as one batch."""
    items, refs = [], []
    for p in WL.PROJECTIONS:
        c = WL.config2_projection(layer, p.name)
        P_d, beta, P_o, beta_o = both_pack(WL.master_weights(p.N, p.K, WL.master_seed(layer, p.name)))
        refs.append(("bf16", O.f32_to_bf16(O.forward(c["x"], P_o, beta_o, gain=c["gain"],
                                                     eps=WL.RMS_EPS, norm=True)["y"])))
        items.append(dict(x=bf16_dev(c["x"]), gain=bf16_dev(c["gain"]), P=P_d, beta=beta,
                          y=guard.empty((1, p.N), torch.bfloat16)))
    run_batch(items, 1, guard)
    _check_batch(items, refs, "config 2 layer %d batch" % layer)


def test_batch_whole_token_as_timed(guard):
    """The timed decode step: all 210 projections of one token (30 layers) in one
    batched call.  The GPU computes all of them; the oracle recomputes three
    layers' seven outputs each (those layers with their seeded master weights,
    the others with seeded weights drawn on the device)."""
    items, check = [], {}
    gen = torch.Generator(device="cuda")
    gen.manual_seed(210)
    for layer in range(WL.LAYERS):
        for p in WL.PROJECTIONS:
            c = WL.config2_projection(layer, p.name)
            if layer in (0, 14, 29):
                W = WL.master_weights(p.N, p.K, WL.master_seed(layer, p.name))
                W_d = torch.from_numpy(W).cuda()
            else:
                W = None
                W_d = torch.randn(p.N, p.K, device="cuda", generator=gen) * WL.MASTER_STD
            P_d, beta_d = B.bitlinear_pack(W_d)
            del W_d
            items.append(dict(x=bf16_dev(c["x"]), gain=bf16_dev(c["gain"]), P=P_d,
                              beta=float(beta_d.item()),
                              y=guard.empty((1, p.N), torch.bfloat16)))
            if W is not None:
                check[len(items) - 1] = (c, W)
    assert len(items) == 210
    run_batch(items, 1, guard)
    for i, (c, W) in check.items():
        P_o, beta_o = O.pack_master(W)
        assert np.float32(items[i]["beta"]) == np.float32(beta_o)
        assert_exact(items[i]["P"].cpu().numpy(), P_o, "packed bytes %d" % i)
        ref = O.f32_to_bf16(O.forward(c["x"], P_o, beta_o, gain=c["gain"], eps=WL.RMS_EPS,
                                      norm=True)["y"])
        assert_bf16_output(bf16_host(items[i]["y"]), ref, "token batch problem %d" % i)


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5])
def test_batch_mixed_problems(M, guard):
    specs = [(256, 128, True, torch.bfloat16, False), (2560, 640, False, torch.float32, False),
             (6912, 2560, True, torch.bfloat16, True), (16, 4, False, torch.bfloat16, False),
             (4096 + 16, 12, True, torch.float32, False)]
    items, refs = _batch_case(specs, M, seed=5000 + M, guard=guard)
    run_batch(items, M, guard)
    _check_batch(items, refs, "mixed batch M=%d" % M)


def test_batch_many_problems(guard):
    specs = [(16 * (1 + i % 7), 4 * (1 + i % 5), i % 2 == 0, torch.bfloat16, i % 3 == 0)
             for i in range(40)]
    items, refs = _batch_case(specs, 2, seed=7000, guard=guard)
    run_batch(items, 2, guard)
    _check_batch(items, refs, "40-problem batch")


def test_quantized_batch_shared_input_qkv_and_gate_up(guard):
    """q|k|v share one quantised input, gate|up another: one launch each."""
    for M in (1, 3, 6):
        x = WL.activations(M, 2560, seed=8000 + M, outlier_frac=0.001)
        g = WL.gain(2560, seed=8100)
        q, s, rs = B.bitlinear_act_quant(bf16_dev(x), bf16_dev(g), WL.RMS_EPS)
        for names in (("q", "k", "v"), ("gate", "up")):
            items, refs = [], []
            for name in names:
                p = WL.PROJECTIONS[WL.PROJ_INDEX[name]]
                P_d, beta, P_o, beta_o = both_pack(WL.master_weights(p.N, p.K,
                                                                     WL.master_seed(3, name)))
                refs.append(O.f32_to_bf16(O.forward(x, P_o, beta_o, gain=g, eps=WL.RMS_EPS,
                                                    norm=True)["y"]))
                items.append(dict(q=q, s_x=s, rowsum=rs, P=P_d, beta=beta,
                                  y=guard.empty((M, p.N), torch.bfloat16)))
            run_quantized_batch(items, M, guard)
            for it, ref, name in zip(items, refs, names):
                assert_bf16_output(bf16_host(it["y"]), ref, "shared-input %s M=%d" % (name, M))


def test_batch_of_many_tiny_problems_and_one_large(guard):
    """100 one-row problems land in the first CTA's byte range (more problems
    than a CTA stages), next to a large one: both code paths in one launch."""
    specs = [(16, 4, i % 2 == 0, torch.bfloat16, False) for i in range(100)]
    specs.append((2560, 2560, True, torch.float32, False))
    items, refs = _batch_case(specs, 1, seed=9000, guard=guard)
    run_batch(items, 1, guard)
    _check_batch(items, refs, "100 tiny + 1 large")


# ---------------------------------------------------------------------------
# tensor-core GEMM path (M > 4): ragged tiles, store paths, persistent loop
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("M,K,N,out,residual", [
    (5, 16, 4, "f32", False),          # everything smaller than one tile
    (129, 272, 36, "f32", False),      # token tile + 1, K not a multiple of 128, R=9
    (300, 4112, 12, "bf16", True),     # R=3: scalar store path with residual
    (257, 128, 256, "bf16", False),    # exactly one K stage, one weight tile
    (1000, 2560, 6912, "bf16", True),  # 216 tiles > 148 CTAs: both accumulators reused
    (130, 6912, 2560, "i32", False),   # exact int32 accumulators, 54 K stages
    # last wave split in N: 160 tiles on 148 CTAs leave 12 tiles for 24 halves
    (256, 128, 20304, "bf16", False),  # R=5076: last tile 20 rows, its second half empty
    (256, 144, 20384, "f32", False),   # R=5096: second half of the last tile 8 rows
    (200, 256, 20480, "i32", False),   # R=5120: every half full, int32 accumulators
])
def test_gemm_path_shapes(M, K, N, out, residual, guard):
    x = special_rows(WL.activations(M, K, seed=M * 7 + K, row_std=(0.1, 10.0)))
    W = WL.master_weights(N, K, seed=N * 3 + K)
    P_d, beta, P_o, beta_o = both_pack(W)
    q, s, rs = B.bitlinear_act_quant(bf16_dev(x))
    q_o, s_o, rs_o = O.quantize_input(x)
    assert_exact(q.cpu().numpy(), q_o, "codes")
    if out == "i32":
        acc = B.bitlinear_accumulate(q, rs, P_d, out=guard.empty((M, N), torch.int32))
        assert_exact(acc.cpu().numpy(), O.ternary_matmul(q_o, O.unpack(P_o)), "int32 accumulators")
        return
    y_o = O.forward(x, P_o, beta_o)["y"]
    if out == "f32":
        y = B.bitlinear_forward_quantized(q, s, rs, P_d, beta,
                                          out=guard.empty((M, N), torch.float32))
        assert_f32_output(y.cpu().numpy(), y_o, "gemm f32")
    else:
        r = WL.activations(M, N, seed=M + N) if residual else None
        y = guard.copy(bf16_dev(r)) if residual else guard.empty((M, N), torch.bfloat16)
        B.bitlinear_forward_quantized(q, s, rs, P_d, beta, residual=y if residual else None, out=y)
        ref = O.residual_add(r, O.f32_to_bf16(y_o)) if residual else O.f32_to_bf16(y_o)
        assert_bf16_output(bf16_host(y), ref, "gemm bf16")
