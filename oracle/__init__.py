"""CPU oracle of the BitNet b1.58 BitLinear forward (W1.58A8).

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package; the product path
(``ternary_weight_bitlinear_b200``) never does and shares no code with it.

Each function is a thin numpy <-> ctypes shim over ``bitlinear_oracle.c``,
whose comments cite the page and section every step follows.  bf16 tensors are
passed as ``numpy.uint16`` arrays holding the bf16 bit patterns.

Function          Definition followed
----------------  ----------------------------------------------------------
weight_scale      absmean of |W| clamped at 1e-5 (the per-tensor weight scale)
ternarize         clamp(round(W * RN32(1/beta)), -1, 1): multiply by the scale
pack / unpack     2-bit codes t+1, four rows per byte, bit pair i = quarter i
rmsnorm           exact-sum RMSNorm, gain after the rms factor
act_quant         per-token absmax int8: s = 127/max(max|h|,1e-5), round, clamp
ternary_matmul    exact int32 sum_k q[m,k] t[n,k]
rescale           RN32(RN32(acc * beta) / s_x)
forward           norm -> unpack -> quant -> matmul -> rescale
relu2_mul         bf16(relu(a)^2 * b)
residual_add      bf16(x + d)
ffn_block         one FFN block of the 30-layer chain
online_forward    weight scale + ternarise on this call, then forward (online QAT)
ste_backward      linear backward on the dequantised operands (straight-through)
rope, attn_decode the attention block's RoPE and GQA decode attention, float64
                  numpy (``oracle/attention.py``)
"""
import ctypes
import os

import numpy as np

from . import build as _build
from .attention import attn_decode, rope, rope_inv_freq  # noqa: F401

_LIB = None
_PARALLEL = False


def set_parallel(on):
    """Use the OpenMP build (matmul rows on all host cores, identical results)
    for the calls that follow; the plain single-core build otherwise."""
    global _LIB, _PARALLEL
    if bool(on) != _PARALLEL:
        _PARALLEL = bool(on)
        _LIB = None


def lib():
    """Load (building first if needed) liboracle.so, or liboracle_omp.so after
    set_parallel(True)."""
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(_build.LIB_OMP if _PARALLEL else path)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        f32 = ctypes.c_float
        L.ref_exact_sum_f64.argtypes = [P, i64]
        L.ref_exact_sum_f64.restype = ctypes.c_double
        L.ref_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.ref_bf16_to_f32.restype = f32
        L.ref_f32_to_bf16.argtypes = [f32]
        L.ref_f32_to_bf16.restype = ctypes.c_uint16
        L.ref_weight_scale.argtypes = [P, i64, i64]
        L.ref_weight_scale.restype = f32
        L.ref_ternarize.argtypes = [P, i64, f32, P]
        L.ref_ternarize.restype = None
        L.ref_pack.argtypes = [P, i64, i64, P]
        L.ref_pack.restype = ctypes.c_int
        L.ref_unpack.argtypes = [P, i64, i64, P]
        L.ref_unpack.restype = None
        L.ref_bf16_to_f32_buf.argtypes = [P, i64, P]
        L.ref_bf16_to_f32_buf.restype = None
        L.ref_f32_to_bf16_buf.argtypes = [P, i64, P]
        L.ref_f32_to_bf16_buf.restype = None
        L.ref_rmsnorm.argtypes = [P, P, f32, i64, i64, P, P]
        L.ref_rmsnorm.restype = None
        L.ref_act_quant.argtypes = [P, i64, i64, P, P, P]
        L.ref_act_quant.restype = None
        L.ref_ternary_matmul.argtypes = [P, P, i64, i64, i64, P]
        L.ref_ternary_matmul.restype = None
        L.ref_rescale.argtypes = [P, P, f32, i64, i64, P]
        L.ref_rescale.restype = None
        L.ref_forward.argtypes = [P, P, ctypes.c_int, f32, P, f32, i64, i64, i64, P, P, P, P]
        L.ref_forward.restype = ctypes.c_int
        L.ref_relu2_mul.argtypes = [P, P, i64, P]
        L.ref_relu2_mul.restype = None
        L.ref_residual_add.argtypes = [P, P, i64, P]
        L.ref_residual_add.restype = None
        L.ref_ffn_block.argtypes = [P, P, P, f32, P, f32, P, f32, P, f32, i64, i64, i64, P]
        L.ref_ffn_block.restype = ctypes.c_int
        L.ref_online_forward.argtypes = [P, P, ctypes.c_int, f32, P, i64, i64, i64, P, P, P]
        L.ref_online_forward.restype = ctypes.c_int
        L.ref_ste_backward.argtypes = [P, P, P, P, f32, i64, i64, i64, P, P]
        L.ref_ste_backward.restype = None
        _LIB = L
    return _LIB


def _c(a, dtype):
    """Contiguous array of the exact dtype (no silent conversion of values)."""
    a = np.asarray(a)
    if a.dtype != np.dtype(dtype):
        raise TypeError("expected %s, got %s" % (np.dtype(dtype), a.dtype))
    return np.ascontiguousarray(a)


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


# --- scalar helpers -------------------------------------------------------
def exact_sum(v):
    v = _c(v, np.float64).ravel()
    return float(lib().ref_exact_sum_f64(_p(v), v.size))


def f32_to_bf16(y):
    y = _c(y, np.float32)
    out = np.empty(y.shape, np.uint16)
    lib().ref_f32_to_bf16_buf(_p(y), y.size, _p(out))
    return out


def bf16_to_f32(x):
    x = _c(x, np.uint16)
    out = np.empty(x.shape, np.float32)
    lib().ref_bf16_to_f32_buf(_p(x), x.size, _p(out))
    return out


# --- weight side ----------------------------------------------------------
def weight_scale(W):
    W = _c(W, np.float32)
    N, K = W.shape
    return float(np.float32(lib().ref_weight_scale(_p(W), N, K)))


def ternarize(W, beta):
    W = _c(W, np.float32)
    t = np.empty(W.shape, np.int8)
    lib().ref_ternarize(_p(W), W.size, ctypes.c_float(beta), _p(t))
    return t


def pack(t):
    t = _c(t, np.int8)
    N, K = t.shape
    P = np.empty((N // 4, K), np.uint8)
    if lib().ref_pack(_p(t), N, K, _p(P)) != 0:
        raise ValueError("pack: N must be a multiple of 4 and values in {-1,0,1}")
    return P


def unpack(P, N=None):
    P = _c(P, np.uint8)
    R, K = P.shape
    N = 4 * R if N is None else N
    t = np.empty((N, K), np.int8)
    lib().ref_unpack(_p(P), N, K, _p(t))
    return t


def pack_master(W):
    """Master fp32 weights -> (packed codes, beta): absmean scale, ternarise, pack."""
    beta = weight_scale(W)
    return pack(ternarize(W, beta)), beta


# --- activation side ------------------------------------------------------
def rmsnorm(x, gain, eps):
    x = _c(x, np.uint16)
    M, K = x.shape
    g = None if gain is None else _c(gain, np.uint16)
    h = np.empty((M, K), np.float32)
    r = np.empty(M, np.float32)
    lib().ref_rmsnorm(_p(x), _p(g), ctypes.c_float(eps), M, K, _p(h), _p(r))
    return h, r


def act_quant(h):
    h = _c(h, np.float32)
    M, K = h.shape
    q = np.empty((M, K), np.int8)
    s = np.empty(M, np.float32)
    rs = np.empty(M, np.int32)
    lib().ref_act_quant(_p(h), M, K, _p(q), _p(s), _p(rs))
    return q, s, rs


def quantize_input(x, gain=None, eps=1e-5, norm=False):
    """bf16 x -> (q, s_x, rowsum), through the RMSNorm first when ``norm``."""
    h = rmsnorm(x, gain, eps)[0] if norm else bf16_to_f32(x)
    return act_quant(h)


# --- matmul / rescale / forward ------------------------------------------
def ternary_matmul(q, t):
    q = _c(q, np.int8)
    t = _c(t, np.int8)
    M, K = q.shape
    N = t.shape[0]
    acc = np.empty((M, N), np.int32)
    lib().ref_ternary_matmul(_p(q), _p(t), M, K, N, _p(acc))
    return acc


def rescale(acc, s_x, beta):
    acc = _c(acc, np.int32)
    s_x = _c(s_x, np.float32)
    M, N = acc.shape
    y = np.empty((M, N), np.float32)
    lib().ref_rescale(_p(acc), _p(s_x), ctypes.c_float(beta), M, N, _p(y))
    return y


def forward(x, P, beta, N=None, gain=None, eps=1e-5, norm=False):
    """Full BitLinear forward.  Returns dict(y=fp32 [M,N], q, s_x, acc)."""
    x = _c(x, np.uint16)
    P = _c(P, np.uint8)
    M, K = x.shape
    N = 4 * P.shape[0] if N is None else N
    g = None if gain is None else _c(gain, np.uint16)
    y = np.empty((M, N), np.float32)
    q = np.empty((M, K), np.int8)
    s = np.empty(M, np.float32)
    acc = np.empty((M, N), np.int32)
    rc = lib().ref_forward(_p(x), _p(g), 1 if norm else 0, ctypes.c_float(eps), _p(P),
                           ctypes.c_float(beta), M, K, N, _p(y), _p(q), _p(s), _p(acc))
    if rc != 0:
        raise ValueError("forward: bad shape")
    return dict(y=y, q=q, s_x=s, acc=acc)


# --- FFN glue -------------------------------------------------------------
def relu2_mul(a, b):
    a = _c(a, np.uint16)
    b = _c(b, np.uint16)
    z = np.empty(a.shape, np.uint16)
    lib().ref_relu2_mul(_p(a), _p(b), a.size, _p(z))
    return z


def residual_add(x, d):
    x = _c(x, np.uint16)
    d = _c(d, np.uint16)
    out = np.empty(x.shape, np.uint16)
    lib().ref_residual_add(_p(x), _p(d), x.size, _p(out))
    return out


def ffn_block(x, g_in, g_sub, eps, Pg, bg, Pu, bu, Pd, bd):
    x = _c(x, np.uint16)
    M, H = x.shape
    I = 4 * Pg.shape[0]
    out = np.empty_like(x)
    rc = lib().ref_ffn_block(_p(x), _p(_c(g_in, np.uint16)), _p(_c(g_sub, np.uint16)),
                             ctypes.c_float(eps), _p(_c(Pg, np.uint8)), ctypes.c_float(bg),
                             _p(_c(Pu, np.uint8)), ctypes.c_float(bu), _p(_c(Pd, np.uint8)),
                             ctypes.c_float(bd), M, H, I, _p(out))
    if rc != 0:
        raise ValueError("ffn_block: bad shape")
    return out


# --- online QAT -------------------------------------------------------------
def online_forward(x, W, gain=None, eps=1e-5, norm=False):
    """Forward with the weights quantised on this call from fp32 masters W
    [N,K].  Returns dict(y=fp32 [M,N], beta, t=int8 [N,K])."""
    x = _c(x, np.uint16)
    W = _c(W, np.float32)
    M, K = x.shape
    N = W.shape[0]
    g = None if gain is None else _c(gain, np.uint16)
    y = np.empty((M, N), np.float32)
    beta = ctypes.c_float()
    t = np.empty((N, K), np.int8)
    rc = lib().ref_online_forward(_p(x), _p(g), 1 if norm else 0, ctypes.c_float(eps), _p(W), M,
                                  K, N, _p(y), ctypes.byref(beta), _p(t))
    if rc != 0:
        raise ValueError("online_forward: bad shape")
    return dict(y=y, beta=float(np.float32(beta.value)), t=t)


def ste_backward(gy, q, s_x, t, beta):
    """Gradients (gx [M,K], gw [N,K], float64) of the layer under the
    straight-through estimator, from the output gradient gy [M,N] (fp32), the
    forward's codes q [M,K] and scales s_x [M], and the ternary weights t
    [N,K] with their absmean beta."""
    gy = _c(gy, np.float32)
    q = _c(q, np.int8)
    s_x = _c(s_x, np.float32)
    t = _c(t, np.int8)
    M, N = gy.shape
    K = q.shape[1]
    gx = np.empty((M, K), np.float64)
    gw = np.empty((N, K), np.float64)
    lib().ref_ste_backward(_p(gy), _p(q), _p(s_x), _p(t), ctypes.c_float(beta), M, K, N, _p(gx),
                           _p(gw))
    return gx, gw

