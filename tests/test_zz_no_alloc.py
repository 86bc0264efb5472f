"""bitlinear_forward_noalloc: the BitLinear forward for callers that cannot
allocate device memory (latency-critical loops that must not trigger
cudaMalloc's implicit device synchronisation, plugins inside an engine that
owns every allocation).  It keeps its intermediate int8 codes in a fixed device
array inside the library instead of a caller workspace.

Checked through the C ABI against the oracle (bit for bit, and within the
stated tolerances) and against bitlinear_forward, on two calls in a row (the
second call finds the first one's leftovers in the shared array), with every
output in a guarded buffer.  The shapes cover the decode kernel (M <= 4), the
5..64-token kernel with and without room for its split-tile tail in the fixed
array, and the tensor-core GEMM.  This file is named so that pytest collects
it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import ternary_weight_bitlinear_b200 as B
from ternary_weight_bitlinear_b200 import workloads as WL
from gpu_util import assert_bf16_output, assert_f32_output, bf16_dev, bf16_host

SCRATCH_BYTES = 2 << 20  # BL_NOALLOC_SCRATCH_BYTES


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def noalloc_forward(x, gain, P, beta, out):
    M, K = x.shape
    N = out.shape[1]
    code = B.BL_OUT_BF16 if out.dtype == torch.bfloat16 else B.BL_OUT_F32
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return B.lib().bitlinear_forward_noalloc(_p(x), _p(gain), WL.RMS_EPS, _p(P), float(beta),
                                             M, K, N, _p(out), code, stream)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # 4096 x 2560 codes need ~10 MB of scratch: refused on the host, nothing launched
    st = B.lib().bitlinear_forward_noalloc(ctypes.c_void_p(0x10000), None, 1e-5,
                                           ctypes.c_void_p(0x10000), 1.0, 4096, 2560, 640,
                                           ctypes.c_void_p(0x10000), 0, None)
    assert st == 5  # BL_ERR_WORKSPACE
    msg = B.lib().bitlinear_last_error().decode()
    assert str(SCRATCH_BYTES) in msg and "needs" in msg


CASES = [  # (M, K, N, norm, out dtype)
    (1, 2560, 2560, True, torch.bfloat16),    # decode kernel
    (4, 6912, 2560, False, torch.float32),    # decode kernel, four tokens
    (9, 6912, 2560, False, torch.float32),    # 5..64 tokens, split-tile tail fits
    (16, 2560, 640, True, torch.bfloat16),    # 5..64 tokens, split-tile tail fits
    (32, 2560, 6912, True, torch.bfloat16),   # 5..64 tokens, tail does not fit: tile-cut shares
    (64, 6912, 2560, True, torch.bfloat16),   # the same at 64 tokens
    (96, 2560, 640, False, torch.float32),    # tensor-core GEMM
]


@pytest.mark.gpu
def test_noalloc_matches_oracle_and_forward_on_two_calls(guard):
    prepared = []
    for i, (M, K, N, norm, dt) in enumerate(CASES):
        x = WL.activations(M, K, seed=900 + i, outlier_frac=0.001, row_std=(0.1, 10.0))
        g = WL.gain(K, seed=910 + i) if norm else None
        W = WL.master_weights(N, K, seed=920 + i)
        P, beta = B.bitlinear_pack(torch.from_numpy(W).cuda())
        P_o, beta_o = O.pack_master(W)
        assert np.float32(beta.item()) == np.float32(beta_o)
        ref = O.forward(x, P_o, beta_o, gain=g, eps=WL.RMS_EPS, norm=norm)["y"]
        prepared.append((x, g, P, float(beta.item()), dt, ref))
    for call in range(2):  # two rounds of calls sharing the library's one scratch array
        for (M, K, N, norm, dt), (x, g, P, beta, _, ref) in zip(CASES, prepared):
            xd, gd = bf16_dev(x), None if g is None else bf16_dev(g)
            y = guard.empty((M, N), dt)
            assert noalloc_forward(xd, gd, P, beta, y) == 0
            y_fw = B.bitlinear_forward(xd, P, beta, gain=gd, eps=WL.RMS_EPS, out_dtype=dt)
            torch.cuda.synchronize()
            what = "noalloc call %d M=%d K=%d N=%d" % (call, M, K, N)
            if dt == torch.bfloat16:
                assert_bf16_output(bf16_host(y), O.f32_to_bf16(ref), what)
                assert_bf16_output(bf16_host(y), bf16_host(y_fw), what + " vs bitlinear_forward")
            else:
                assert_f32_output(y.cpu().numpy(), ref, what)
                assert_f32_output(y.cpu().numpy(), y_fw.cpu().numpy(), what + " vs bitlinear_forward")
    assert B.bitlinear_device_status() == 0
