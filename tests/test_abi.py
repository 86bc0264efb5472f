"""The C ABI without a GPU: the library loads, exports every entry point the
header declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest
import torch

from conftest import ROOT

B = pytest.importorskip("ternary_weight_bitlinear_b200")

HEADER = os.path.join(ROOT, "include", "bitlinear.h")
NULL = None
P16 = ctypes.c_void_p(0x10000)  # 16-byte aligned, never dereferenced by host checks
P17 = ctypes.c_void_p(0x10001)


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bitlinear_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    return B.lib()


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 13
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(B.bitlinear.SIGNATURES)


def test_abi_version_and_status_strings(L):
    assert L.bitlinear_abi_version() == 1
    for code in range(9):
        assert B.status_string(code)
    assert "unknown" in B.status_string(99)


def test_workspace_sizes(L):
    assert B.bitlinear_forward_workspace_size(1, 2560, 6912) >= 2560 + 8
    assert B.bitlinear_forward_workspace_size(4, 6912, 2560) >= 4 * 6912 + 32
    assert B.bitlinear_forward_workspace_size(0, 2560, 2560) == 0
    big = B.bitlinear_forward_workspace_size(4096, 2560, 6912)
    assert big >= 4096 * 2560 + 2 * 4096 * 4
    assert B.bitlinear_pack_workspace_size(2560, 2560) > 0
    with pytest.raises(B.BitLinearError):
        B.bitlinear_forward_workspace_size(1, 2561, 16)


def test_skinny_workspace_sizes(L):
    """5..64 tokens add one split area (a counter and two blocks of 128 x npad
    int32 per CTA)."""
    Q = B.bitlinear_quantized_batch_workspace_size
    assert Q(0) == Q(1) == Q(4) == Q(65) == Q(4096) == 0
    s5, s16, s17, s64 = Q(5), Q(16), Q(17), Q(64)
    assert 0 < s5 == s16 < s17 < s64           # npad 16, 16, 32, 64
    assert s64 - s16 == 3 * (s17 - s16)        # linear in npad
    assert s64 >= 148 * 2 * 64 * 128 * 4      # room for every CTA of a B200
    own = 8 * 2560 + 2 * 256                  # codes + s_x + row sums (256-byte slices)
    assert B.bitlinear_forward_workspace_size(8, 2560, 640) == own + Q(8)
    assert B.bitlinear_forward_workspace_size(4, 2560, 640) == 4 * 2560 + 2 * 256
    sz = ctypes.c_size_t()
    arr = _batch(7, K=2560, N=640)
    assert L.bitlinear_forward_batch_workspace_size(arr, 7, 8, ctypes.byref(sz)) == 0
    assert sz.value == 7 * own + Q(8)          # one split area for the whole batch
    assert L.bitlinear_quantized_batch_workspace_size(8, None) == 1
    assert L.bitlinear_quantized_batch_workspace_size(-1, ctypes.byref(sz)) == 2


def _fwd(L, x=P16, gain=NULL, P=P16, M=1, K=256, N=128, y=P16, dt=0, ws=P16, wsb=1 << 30):
    return L.bitlinear_forward(x, gain, 1e-5, P, 1.0, M, K, N, y, dt, ws, wsb, NULL)


def test_forward_argument_checks(L):
    assert _fwd(L, K=250) == 2          # K % 16
    assert _fwd(L, K=0) == 2
    assert _fwd(L, N=130) == 2          # N % 4
    assert _fwd(L, M=-1) == 2
    assert _fwd(L, K=65536 + 16) == 2   # > BL_MAX_K
    assert _fwd(L, dt=7) == 4           # unknown dtype
    assert _fwd(L, M=0, x=NULL, P=NULL, y=NULL) == 0   # empty: no-op
    assert _fwd(L, x=NULL) == 1
    assert _fwd(L, y=NULL) == 1
    assert _fwd(L, x=P17) == 3
    assert _fwd(L, gain=P17) == 3
    assert _fwd(L, M=64, K=2560, ws=NULL) == 5   # needs a workspace
    assert _fwd(L, M=64, K=2560, ws=P16, wsb=16) == 5
    assert _fwd(L, ws=P17) == 3


def test_other_entry_points_check_arguments(L):
    assert L.bitlinear_pack(NULL, 8, 16, P16, P16, P16, 1 << 20, NULL) == 1
    assert L.bitlinear_pack(P16, 6, 16, P16, P16, P16, 1 << 20, NULL) == 2
    assert L.bitlinear_pack(P16, 8, 16, P16, P16, P16, 8, NULL) == 5
    assert L.bitlinear_pack_ternary(P16, 8, 24, P16, NULL) == 2
    assert L.bitlinear_unpack(P17, 8, 16, P16, NULL) == 3
    assert L.bitlinear_act_quant(NULL, NULL, 1e-5, 2, 64, P16, P16, P16, NULL) == 1
    assert L.bitlinear_act_quant(P16, NULL, 1e-5, 0, 64, NULL, NULL, NULL, NULL) == 0
    assert L.bitlinear_forward_quantized(P16, P16, P16, P16, 1.0, 2, 64, 8, P16, 1, P16, NULL) == 4
    assert L.bitlinear_forward_quantized(P16, P16, NULL, P16, 1.0, 2, 64, 8, P16, 0, NULL, NULL) == 1
    assert L.bitlinear_accumulate(P16, P16, P16, 2, 64, 10, P16, NULL) == 2
    assert L.bitlinear_relu2_mul(P16, P16, -1, P16, NULL) == 2
    assert L.bitlinear_relu2_mul(NULL, NULL, 0, NULL, NULL) == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_no_device_is_reported_not_faked(L):
    # valid arguments, but no CUDA device: the library refuses, it never falls back
    assert _fwd(L) == 8
    assert L.bitlinear_act_quant(P16, NULL, 1e-5, 2, 64, P16, P16, P16, NULL) == 8
    assert L.bitlinear_device_status(NULL) == 8


def _batch(n, K=256, N=128, x=P16, dt=0, residual=None):
    arr = (B.bitlinear.Problem * n)()
    for i in range(n):
        arr[i] = B.bitlinear.Problem(x.value, None, P16.value, P16.value,
                                     residual.value if residual else None, K, N, 1.0, dt)
    return arr


def test_batch_argument_checks(L):
    sz = ctypes.c_size_t()
    arr = _batch(7)
    assert L.bitlinear_forward_batch_workspace_size(arr, 7, 1, ctypes.byref(sz)) == 0
    assert sz.value == 7 * B.bitlinear_forward_workspace_size(1, 256, 128)
    assert L.bitlinear_forward_batch_workspace_size(arr, 0, 1, ctypes.byref(sz)) == 2
    big = _batch(257)
    assert L.bitlinear_forward_batch_workspace_size(big, 257, 1, ctypes.byref(sz)) == 2
    assert L.bitlinear_forward_batch(_batch(3, K=250), 3, 1, 1e-5, P16, 1 << 30, NULL) == 2
    assert L.bitlinear_forward_batch(_batch(3, dt=9), 3, 1, 1e-5, P16, 1 << 30, NULL) == 4
    assert L.bitlinear_forward_batch(_batch(3, dt=1, residual=P16), 3, 1, 1e-5, P16, 1 << 30,
                                     NULL) == 4
    assert L.bitlinear_forward_batch(_batch(3, x=P17), 3, 1, 1e-5, P16, 1 << 30, NULL) == 3
    assert L.bitlinear_forward_batch(arr, 7, 1, 1e-5, NULL, 0, NULL) == 5
    assert L.bitlinear_forward_batch(arr, 7, 0, 1e-5, NULL, 0, NULL) == 0  # M = 0: no-op


def _qbatch(n, K=256, N=128, q=P16, rowsum=P16, dt=0, residual=None):
    arr = (B.bitlinear.QuantizedProblem * n)()
    for i in range(n):
        arr[i] = B.bitlinear.QuantizedProblem(q.value if q else None, P16.value,
                                              rowsum.value if rowsum else None, P16.value,
                                              P16.value, residual.value if residual else None,
                                              K, N, 1.0, dt)
    return arr


def test_quantized_batch_argument_checks(L):
    Q = L.bitlinear_forward_quantized_batch
    assert Q(NULL, 1, 8, NULL, 0, NULL) == 1
    assert Q(_qbatch(1), 0, 8, NULL, 0, NULL) == 2                # count 0
    assert Q(_qbatch(257), 257, 8, NULL, 0, NULL) == 2            # > BL_MAX_BATCH
    assert Q(_qbatch(2), 2, -1, NULL, 0, NULL) == 2               # M < 0
    assert Q(_qbatch(2, K=250), 2, 8, NULL, 0, NULL) == 2         # K % 16
    assert Q(_qbatch(2, N=130), 2, 8, NULL, 0, NULL) == 2         # N % 4
    assert Q(_qbatch(2, dt=5), 2, 8, NULL, 0, NULL) == 4          # unknown dtype
    assert Q(_qbatch(2, dt=1, residual=P16), 2, 8, NULL, 0, NULL) == 4  # residual wants bf16
    assert Q(_qbatch(2, q=None), 2, 8, NULL, 0, NULL) == 1
    assert Q(_qbatch(2, rowsum=None), 2, 8, NULL, 0, NULL) == 1
    assert Q(_qbatch(2, q=P17), 2, 8, NULL, 0, NULL) == 3
    assert Q(_qbatch(2, q=None), 2, 0, NULL, 0, NULL) == 0        # M = 0: no-op, pointers unread


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_selftest_and_quantized_batch_need_a_device(L):
    assert L.bitlinear_selftest_wait_timeout(1000000, NULL) == 8
    assert L.bitlinear_forward_quantized_batch(_qbatch(2), 2, 8, NULL, 0, NULL) == 8


def test_binding_rejects_cpu_tensors():
    x = torch.zeros(1, 256, dtype=torch.bfloat16)
    P = torch.zeros(32, 256, dtype=torch.uint8)
    with pytest.raises(TypeError):
        B.bitlinear_forward(x, P, 1.0)


def test_gate_up_argument_checks(L):
    sz = ctypes.c_size_t()
    assert L.bitlinear_pack_gate_up_workspace_size(6912, 2560, ctypes.byref(sz)) == 0
    assert sz.value > 0
    assert L.bitlinear_pack_gate_up_workspace_size(7, 2560, ctypes.byref(sz)) == 2   # I odd
    assert L.bitlinear_pack_gate_up_workspace_size(8, 24, ctypes.byref(sz)) == 2     # K % 16
    ws = ctypes.c_size_t(1 << 20)
    assert L.bitlinear_pack_gate_up(NULL, P16, 8, 32, P16, P16, P16, ws, NULL) == 1
    assert L.bitlinear_pack_gate_up(P16, P16, 8, 32, P16, P16, P16, 0, NULL) == 5
    assert L.bitlinear_pack_gate_up(P17, P16, 8, 32, P16, P16, P16, ws, NULL) == 3

    def fgu(q=P16, s=P16, rs=P16, P=P16, M=2, K=32, I=8, z=P16, w=NULL, wb=0):
        return L.bitlinear_forward_gate_up(q, s, rs, P, 1.0, 1.0, M, K, I, z, w, wb, NULL)

    assert fgu(I=7) == 2
    assert fgu(K=24) == 2
    assert fgu(M=0) == 0                     # empty: nothing to do
    assert fgu(z=NULL) == 1
    assert fgu(P=P17) == 3
    assert fgu(w=P17, wb=64) == 3


def test_binding_exports_gate_up():
    for n in ("bitlinear_pack_gate_up", "bitlinear_forward_gate_up",
              "bitlinear_pack_gate_up_workspace_size"):
        assert callable(getattr(B, n))



def test_online_and_backward_argument_checks(L):
    sz = ctypes.c_size_t()
    assert L.bitlinear_forward_online_workspace_size(8, 256, 128, ctypes.byref(sz)) == 0
    small = sz.value
    assert small > 0
    assert L.bitlinear_forward_online_workspace_size(1, 256, 128, ctypes.byref(sz)) == 0
    assert sz.value < small                      # no split area below five tokens
    assert L.bitlinear_forward_online_workspace_size(1, 250, 128, ctypes.byref(sz)) == 2

    def fon(x=P16, W=P16, M=2, K=32, N=8, y=P16, P=P16, beta=P16, q=P16, s=P16, rs=P16, ws=P16,
            wsb=1 << 30):
        return L.bitlinear_forward_online(x, NULL, 1e-5, W, M, K, N, y, 0, P, beta, q, s, rs, ws,
                                          wsb, NULL)

    assert fon(K=24) == 2
    assert fon(W=NULL) == 1
    assert fon(beta=NULL) == 1
    assert fon(ws=NULL) == 5
    assert fon(wsb=16) == 5
    assert fon(W=P17) == 3
    assert L.bitlinear_forward_online(P16, NULL, 1e-5, P16, 2, 32, 8, P16, 7, P16, P16, P16, P16,
                                      P16, P16, 1 << 30, NULL) == 4          # bad dtype

    def bwd(gy=P16, q=P16, s=P16, P=P16, beta=P16, M=2, K=32, N=8, gx=P16, gw=P16):
        return L.bitlinear_backward_ste(gy, q, s, P, beta, M, K, N, gx, gw, NULL)

    assert bwd(M=0) == 0
    assert bwd(N=6) == 2
    assert bwd(gx=NULL, gw=NULL) == 1
    assert bwd(P=NULL) == 1                      # grad_x needs the packed weights
    assert bwd(q=NULL, gx=NULL) == 1             # grad_w needs the codes


def test_decode_chain_argument_checks(L):
    sz = ctypes.c_size_t()
    assert L.bitlinear_decode_chain_workspace_size(0, ctypes.byref(sz)) == 2
    assert L.bitlinear_decode_chain_workspace_size(90, ctypes.byref(sz)) == 0
    assert sz.value > 90 * 64
    steps = (B.bitlinear.ChainStep * 2)()
    for st in steps:
        st.x, st.eps, st.K, st.count = 0x10000, 1e-5, 256, 1
        st.p[0] = B.bitlinear.ChainProblem(0x10000, 0x10000, None, 128, 1.0, 0.0, 0)
    ws = ctypes.c_void_p(0x10000)
    big = 1 << 20
    assert L.bitlinear_decode_chain_prepare(steps, 2, None, big) == 5
    assert L.bitlinear_decode_chain_prepare(None, 2, ws, big) == 1
    steps[1].K = 8208                             # beyond the chain's row limit
    assert L.bitlinear_decode_chain_prepare(steps, 2, ws, big) == 2
    steps[1].K = 256
    steps[1].count = 5
    assert L.bitlinear_decode_chain_prepare(steps, 2, ws, big) == 2
    steps[1].count = 1
    steps[1].p[0].kind = 7
    assert L.bitlinear_decode_chain_prepare(steps, 2, ws, big) == 4
    steps[1].p[0].kind = 2                        # a gate/up pair needs an even N, no residual
    steps[1].p[0].N = 7
    assert L.bitlinear_decode_chain_prepare(steps, 2, ws, big) == 2
    steps[1].p[0].N = 128
    steps[1].p[0].P = 0x10001
    assert L.bitlinear_decode_chain_prepare(steps, 2, ws, big) == 3
    assert L.bitlinear_decode_chain_run(ws, 16, 2, None) == 5


def test_rope_and_attention_argument_checks(L):
    # RoPE: shape and theta are checked first, then pointers
    assert L.bitlinear_rope(P16, P16, -1, 20, 128, 10000.0, P16, NULL) == 2
    assert L.bitlinear_rope(P16, P16, 1, 20, 127, 10000.0, P16, NULL) == 2   # odd head_dim
    assert L.bitlinear_rope(P16, P16, 1, 20, 2048, 10000.0, P16, NULL) == 2  # > 1024
    assert L.bitlinear_rope(P16, P16, 1, 20, 128, 0.0, P16, NULL) == 2
    assert L.bitlinear_rope(P16, P16, 1, 20, 128, float("inf"), P16, NULL) == 2
    assert L.bitlinear_rope(NULL, NULL, 0, 20, 128, 10000.0, NULL, NULL) == 0  # M == 0
    assert L.bitlinear_rope(NULL, P16, 1, 20, 128, 10000.0, P16, NULL) == 1
    # attention: shapes before pointers and device
    sz = ctypes.c_size_t()
    assert L.bitlinear_attn_decode_workspace_size(0, 20, 5, 128, ctypes.byref(sz)) == 2
    assert L.bitlinear_attn_decode_workspace_size(16, 20, 6, 128, ctypes.byref(sz)) == 2  # 20 % 6
    assert L.bitlinear_attn_decode_workspace_size(16, 48, 3, 128, ctypes.byref(sz)) == 2  # group 16
    assert L.bitlinear_attn_decode_workspace_size(16, 20, 5, 96, ctypes.byref(sz)) == 2
    assert L.bitlinear_attn_decode_workspace_size(16, 20, 5, 128, None) == 1
    a = [P16, P16, P16]
    assert L.bitlinear_attn_decode(*a, 0, 20, 5, 128, 0.088, P16, P16, 1 << 20, NULL) == 2
    assert L.bitlinear_attn_decode(*a, 16, 20, 5, 128, float("nan"), P16, P16, 1 << 20, NULL) == 2
    assert L.bitlinear_attn_decode(P16, NULL, P16, 16, 20, 5, 128, 0.088, P16, P16, 1 << 20, NULL) == 1
    assert L.bitlinear_attn_decode(P16, P17, P16, 16, 20, 5, 128, 0.088, P16, P16, 1 << 20, NULL) == 3


def test_binding_exports_attention_block():
    for name in ("bitlinear_rope", "bitlinear_attn_decode", "bitlinear_attn_decode_workspace_size"):
        assert callable(getattr(B, name))
