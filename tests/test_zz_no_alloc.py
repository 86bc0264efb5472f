"""bitlinear_forward_noalloc: the BitLinear forward for callers that cannot
allocate device memory (code inside a CUDA-graph capture, latency-critical
loops that must not trigger cudaMalloc's device synchronisation, plugins in an
engine that owns every allocation).  It keeps its intermediate int8 codes in a
fixed device array inside the library instead of a caller workspace.

Checked through the C ABI against bitlinear_forward, on two calls in a row
(the second call finds the first one's leftovers in the shared array), with
the same bit-exact / tolerance bar as the other parity tests.  This file is
named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

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
    assert B.bitlinear_forward_workspace_size(4096, 2560, 640) > SCRATCH_BYTES


@pytest.mark.gpu
def test_noalloc_matches_forward_on_two_calls():
    cases = [  # (M, K, N, norm, out dtype): both need scratch (M > 4)
        (16, 2560, 640, True, torch.bfloat16),
        (9, 6912, 2560, False, torch.float32),
    ]
    prepared = []
    for i, (M, K, N, norm, dt) in enumerate(cases):
        assert 0 < B.bitlinear_forward_workspace_size(M, K, N) <= SCRATCH_BYTES
        x = bf16_dev(WL.activations(M, K, seed=900 + i, outlier_frac=0.001))
        g = bf16_dev(WL.gain(K, seed=910 + i)) if norm else None
        P, beta = B.bitlinear_pack(torch.from_numpy(WL.master_weights(N, K, seed=920 + i)).cuda())
        prepared.append((x, g, P, float(beta.item()), torch.empty((M, N), dtype=dt, device="cuda")))
    # two calls in a row, sharing the library's one scratch array
    got = []
    for x, g, P, beta, y in prepared:
        assert noalloc_forward(x, g, P, beta, y) == 0
        got.append(y)
    ref = [B.bitlinear_forward(x, P, beta, gain=g, eps=WL.RMS_EPS, out_dtype=y.dtype)
           for x, g, P, beta, y in prepared]
    torch.cuda.synchronize()
    assert B.bitlinear_device_status() == 0
    for (M, K, N, norm, dt), y, r in zip(cases, got, ref):
        what = "noalloc M=%d K=%d N=%d" % (M, K, N)
        if dt == torch.bfloat16:
            assert_bf16_output(bf16_host(y), bf16_host(r), what)
        else:
            assert_f32_output(y.cpu().numpy(), r.cpu().numpy(), what)
