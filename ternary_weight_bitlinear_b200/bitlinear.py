"""Python binding of libbitlinear.so (ctypes): argument marshalling only.

Every function has the name of the C entry point it calls and takes CUDA
torch tensors; all arithmetic runs in the library's kernels.  There is no
fallback: if ``libbitlinear.so`` is missing or no sm_100 device is current,
calls raise.
"""
import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbitlinear.so")

BL_OUT_BF16 = 0
BL_OUT_F32 = 1
BL_MAX_K = 65536

STATUS = {0: "BL_OK", 1: "BL_ERR_NULL", 2: "BL_ERR_SHAPE", 3: "BL_ERR_ALIGN", 4: "BL_ERR_DTYPE",
          5: "BL_ERR_WORKSPACE", 6: "BL_ERR_CUDA", 7: "BL_ERR_TIMEOUT", 8: "BL_ERR_DEVICE"}

# C signatures: name -> (argtypes, restype)
_P, _I64, _F32, _SZ, _INT = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t, \
    ctypes.c_int
SIGNATURES = {
    "bitlinear_abi_version": ([], _INT),
    "bitlinear_status_string": ([_INT], ctypes.c_char_p),
    "bitlinear_last_error": ([], ctypes.c_char_p),
    "bitlinear_pack_workspace_size": ([_I64, _I64, ctypes.POINTER(_SZ)], _INT),
    "bitlinear_pack": ([_P, _I64, _I64, _P, _P, _P, _SZ, _P], _INT),
    "bitlinear_pack_ternary": ([_P, _I64, _I64, _P, _P], _INT),
    "bitlinear_unpack": ([_P, _I64, _I64, _P, _P], _INT),
    "bitlinear_act_quant": ([_P, _P, _F32, _I64, _I64, _P, _P, _P, _P], _INT),
    "bitlinear_forward_workspace_size": ([_I64, _I64, _I64, ctypes.POINTER(_SZ)], _INT),
    "bitlinear_forward": ([_P, _P, _F32, _P, _F32, _I64, _I64, _I64, _P, _INT, _P, _SZ, _P], _INT),
    "bitlinear_forward_quantized": ([_P, _P, _P, _P, _F32, _I64, _I64, _I64, _P, _INT, _P, _P],
                                    _INT),
    "bitlinear_accumulate": ([_P, _P, _P, _I64, _I64, _I64, _P, _P], _INT),
    "bitlinear_relu2_mul": ([_P, _P, _I64, _P, _P], _INT),
    "bitlinear_rope": ([_P, _P, _I64, _I64, _I64, _F32, _P, _P], _INT),
    "bitlinear_attn_decode_workspace_size": ([_I64, _I64, _I64, _I64, ctypes.POINTER(_SZ)], _INT),
    "bitlinear_attn_decode": ([_P, _P, _P, _I64, _I64, _I64, _I64, _F32, _P, _P, _SZ, _P], _INT),
    "bitlinear_pack_gate_up_workspace_size": ([_I64, _I64, ctypes.POINTER(_SZ)], _INT),
    "bitlinear_pack_gate_up": ([_P, _P, _I64, _I64, _P, _P, _P, _SZ, _P], _INT),
    "bitlinear_forward_gate_up": ([_P, _P, _P, _P, _F32, _F32, _I64, _I64, _I64, _P, _P, _SZ, _P],
                                  _INT),
    "bitlinear_forward_online_workspace_size": ([_I64, _I64, _I64, ctypes.POINTER(_SZ)], _INT),
    "bitlinear_forward_online": ([_P, _P, _F32, _P, _I64, _I64, _I64, _P, _INT, _P, _P, _P, _P, _P,
                                  _P, _SZ, _P], _INT),
    "bitlinear_backward_ste": ([_P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _P], _INT),
    "bitlinear_decode_chain_workspace_size": ([_INT, ctypes.POINTER(_SZ)], _INT),
    "bitlinear_decode_chain_prepare": ([_P, _INT, _P, _SZ], _INT),
    "bitlinear_decode_chain_run": ([_P, _SZ, _INT, _P], _INT),
    "bitlinear_forward_noalloc": ([_P, _P, _F32, _P, _F32, _I64, _I64, _I64, _P, _INT, _P], _INT),
    "bitlinear_device_status": ([_P], _INT),
    "bitlinear_selftest_wait_timeout": ([_I64, _P], _INT),
    "bitlinear_forward_batch_workspace_size": ([_P, _INT, _I64, ctypes.POINTER(_SZ)], _INT),
    "bitlinear_forward_batch": ([_P, _INT, _I64, _F32, _P, _SZ, _P], _INT),
    "bitlinear_quantized_batch_workspace_size": ([_I64, ctypes.POINTER(_SZ)], _INT),
    "bitlinear_forward_quantized_batch": ([_P, _INT, _I64, _P, _SZ, _P], _INT),
}


class Problem(ctypes.Structure):
    """bl_problem: one independent BitLinear forward of a batch."""
    _fields_ = [("x", _P), ("gain", _P), ("P", _P), ("y", _P), ("residual", _P),
                ("K", _I64), ("N", _I64), ("beta", _F32), ("y_dtype", _INT)]


class QuantizedProblem(ctypes.Structure):
    """bl_quantized_problem: one matmul on already-quantised activations."""
    _fields_ = [("q", _P), ("s_x", _P), ("rowsum", _P), ("P", _P), ("y", _P), ("residual", _P),
                ("K", _I64), ("N", _I64), ("beta", _F32), ("y_dtype", _INT)]


BL_CHAIN_BF16, BL_CHAIN_F32, BL_CHAIN_GATE_UP = 0, 1, 2
BL_CHAIN_MAX_PROBLEMS = 4


class ChainProblem(ctypes.Structure):
    """bl_chain_problem: one projection of a chain step (M = 1)."""
    _fields_ = [("P", _P), ("y", _P), ("residual", _P), ("N", _I64), ("beta", _F32),
                ("beta_up", _F32), ("kind", _INT)]


class ChainStep(ctypes.Structure):
    """bl_chain_step: up to four projections of one input row."""
    _fields_ = [("x", _P), ("gain", _P), ("eps", _F32), ("K", _I64), ("count", _INT),
                ("p", ChainProblem * BL_CHAIN_MAX_PROBLEMS)]


class BitLinearError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        detail = lib().bitlinear_last_error().decode() if status == 6 else ""
        super().__init__("%s failed: %s (%s)%s" % (fn, STATUS.get(status, status),
                                                    status_string(status),
                                                    " -- " + detail if detail else ""))


_lib = None


def lib():
    """The loaded libbitlinear.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libbitlinear.so is not built; run "
                              "`python -m ternary_weight_bitlinear_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def status_string(status):
    return lib().bitlinear_status_string(status).decode()


def _check(fn, status):
    if status != 0:
        raise BitLinearError(fn, status)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, dtype, name, ndim=None):
    if not (isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == dtype and t.is_contiguous()):
        raise TypeError("%s must be a contiguous CUDA %s tensor" % (name, dtype))
    if ndim is not None and t.dim() != ndim:
        raise TypeError("%s must have %d dimensions" % (name, ndim))
    return t


# --- sizes --------------------------------------------------------------------
def bitlinear_pack_workspace_size(N, K):
    n = ctypes.c_size_t()
    _check("bitlinear_pack_workspace_size", lib().bitlinear_pack_workspace_size(N, K, ctypes.byref(n)))
    return n.value


def bitlinear_forward_workspace_size(M, K, N):
    n = ctypes.c_size_t()
    _check("bitlinear_forward_workspace_size",
           lib().bitlinear_forward_workspace_size(M, K, N, ctypes.byref(n)))
    return n.value


def _workspace(nbytes, device):
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)


# --- weights --------------------------------------------------------------------
def bitlinear_pack(W, P=None, beta=None, workspace=None, stream=None):
    """fp32 master W[N,K] -> (P uint8 [N/4,K], beta fp32 [1] on the device)."""
    _need(W, torch.float32, "W", 2)
    N, K = W.shape
    P = torch.empty((N // 4, K), dtype=torch.uint8, device=W.device) if P is None else P
    beta = torch.empty(1, dtype=torch.float32, device=W.device) if beta is None else beta
    ws = _workspace(bitlinear_pack_workspace_size(N, K), W.device) if workspace is None else workspace
    _check("bitlinear_pack", lib().bitlinear_pack(_ptr(W), N, K, _ptr(P), _ptr(beta), _ptr(ws),
                                                  ws.numel(), _stream(stream)))
    return P, beta


def bitlinear_pack_ternary(t, P=None, stream=None):
    _need(t, torch.int8, "t", 2)
    N, K = t.shape
    P = torch.empty((N // 4, K), dtype=torch.uint8, device=t.device) if P is None else P
    _check("bitlinear_pack_ternary", lib().bitlinear_pack_ternary(_ptr(t), N, K, _ptr(P),
                                                                  _stream(stream)))
    return P


def bitlinear_unpack(P, N=None, t=None, stream=None):
    _need(P, torch.uint8, "P", 2)
    R, K = P.shape
    N = 4 * R if N is None else N
    t = torch.empty((N, K), dtype=torch.int8, device=P.device) if t is None else t
    _check("bitlinear_unpack", lib().bitlinear_unpack(_ptr(P), N, K, _ptr(t), _stream(stream)))
    return t


# --- activations ------------------------------------------------------------------
def bitlinear_act_quant(x, gain=None, eps=1e-5, q=None, s_x=None, rowsum=None, stream=None):
    """bf16 x[M,K] (+ optional RMSNorm gain) -> (q int8 [M,K], s_x fp32 [M], rowsum int32 [M])."""
    _need(x, torch.bfloat16, "x", 2)
    if gain is not None:
        _need(gain, torch.bfloat16, "gain", 1)
    M, K = x.shape
    dev = x.device
    q = torch.empty((M, K), dtype=torch.int8, device=dev) if q is None else q
    s_x = torch.empty(M, dtype=torch.float32, device=dev) if s_x is None else s_x
    rowsum = torch.empty(M, dtype=torch.int32, device=dev) if rowsum is None else rowsum
    _check("bitlinear_act_quant", lib().bitlinear_act_quant(
        _ptr(x), _ptr(gain), eps, M, K, _ptr(q), _ptr(s_x), _ptr(rowsum), _stream(stream)))
    return q, s_x, rowsum


# --- forward ----------------------------------------------------------------------
def _out_code(dtype):
    if dtype == torch.bfloat16:
        return BL_OUT_BF16
    if dtype == torch.float32:
        return BL_OUT_F32
    raise TypeError("output dtype must be torch.bfloat16 or torch.float32")


def bitlinear_forward(x, P, beta, gain=None, eps=1e-5, out_dtype=torch.bfloat16, out=None,
                      workspace=None, N=None, stream=None):
    """Full BitLinear forward: bf16 x[M,K] -> y[M,N] (bf16 or fp32).  ``beta`` is a host float."""
    _need(x, torch.bfloat16, "x", 2)
    _need(P, torch.uint8, "P", 2)
    if gain is not None:
        _need(gain, torch.bfloat16, "gain", 1)
    M, K = x.shape
    N = 4 * P.shape[0] if N is None else N
    y = torch.empty((M, N), dtype=out_dtype, device=x.device) if out is None else out
    if workspace is None:
        need = bitlinear_forward_workspace_size(M, K, N)
        workspace = _workspace(need, x.device) if need else None
    _check("bitlinear_forward", lib().bitlinear_forward(
        _ptr(x), _ptr(gain), eps, _ptr(P), float(beta), M, K, N, _ptr(y), _out_code(y.dtype),
        _ptr(workspace), 0 if workspace is None else workspace.numel(), _stream(stream)))
    return y


def make_batch(items):
    """Build a bl_problem array from dicts with keys x, P, beta, y and optional
    gain, residual (all CUDA tensors except the float beta)."""
    arr = (Problem * len(items))()
    for i, it in enumerate(items):
        x, P, y = it["x"], it["P"], it["y"]
        _need(x, torch.bfloat16, "x", 2)
        _need(P, torch.uint8, "P", 2)
        arr[i] = Problem(x.data_ptr(), _addr(it.get("gain")), P.data_ptr(), y.data_ptr(),
                         _addr(it.get("residual")), x.shape[1], y.shape[1], float(it["beta"]),
                         _out_code(y.dtype))
    return arr


def _addr(t):
    return None if t is None else t.data_ptr()


def bitlinear_forward_batch_workspace_size(batch, M):
    n = ctypes.c_size_t()
    _check("bitlinear_forward_batch_workspace_size", lib().bitlinear_forward_batch_workspace_size(
        ctypes.cast(batch, _P), len(batch), M, ctypes.byref(n)))
    return n.value


def bitlinear_forward_batch(batch, M, eps=1e-5, workspace=None, stream=None):
    """Run a bl_problem array (see make_batch) of independent forwards with M tokens each."""
    if workspace is None:
        workspace = _workspace(bitlinear_forward_batch_workspace_size(batch, M), "cuda")
    _check("bitlinear_forward_batch", lib().bitlinear_forward_batch(
        ctypes.cast(batch, _P), len(batch), M, eps, _ptr(workspace), workspace.numel(),
        _stream(stream)))


def make_quantized_batch(items):
    """Build a bl_quantized_problem array from dicts with keys q, s_x, rowsum, P,
    beta, y and optional residual."""
    arr = (QuantizedProblem * len(items))()
    for i, it in enumerate(items):
        q, P, y = it["q"], it["P"], it["y"]
        _need(q, torch.int8, "q", 2)
        _need(P, torch.uint8, "P", 2)
        arr[i] = QuantizedProblem(q.data_ptr(), it["s_x"].data_ptr(), it["rowsum"].data_ptr(),
                                  P.data_ptr(), y.data_ptr(), _addr(it.get("residual")),
                                  q.shape[1], y.shape[1], float(it["beta"]), _out_code(y.dtype))
    return arr


def bitlinear_quantized_batch_workspace_size(M):
    n = ctypes.c_size_t()
    _check("bitlinear_quantized_batch_workspace_size",
           lib().bitlinear_quantized_batch_workspace_size(M, ctypes.byref(n)))
    return n.value


def bitlinear_forward_quantized_batch(batch, M, workspace=None, stream=None):
    """``workspace``: None, or a uint8 CUDA tensor of at least
    bitlinear_quantized_batch_workspace_size(M) bytes (equal CTA shares for
    5 <= M <= 64)."""
    _check("bitlinear_forward_quantized_batch", lib().bitlinear_forward_quantized_batch(
        ctypes.cast(batch, _P), len(batch), M, _ptr(workspace),
        0 if workspace is None else workspace.numel(), _stream(stream)))


def bitlinear_forward_quantized(q, s_x, rowsum, P, beta, out_dtype=torch.bfloat16, residual=None,
                                out=None, N=None, stream=None):
    _need(q, torch.int8, "q", 2)
    _need(P, torch.uint8, "P", 2)
    M, K = q.shape
    N = 4 * P.shape[0] if N is None else N
    y = torch.empty((M, N), dtype=out_dtype, device=q.device) if out is None else out
    _check("bitlinear_forward_quantized", lib().bitlinear_forward_quantized(
        _ptr(q), _ptr(s_x), _ptr(rowsum), _ptr(P), float(beta), M, K, N, _ptr(y),
        _out_code(y.dtype), _ptr(residual), _stream(stream)))
    return y


def bitlinear_accumulate(q, rowsum, P, N=None, out=None, stream=None):
    _need(q, torch.int8, "q", 2)
    _need(P, torch.uint8, "P", 2)
    M, K = q.shape
    N = 4 * P.shape[0] if N is None else N
    acc = torch.empty((M, N), dtype=torch.int32, device=q.device) if out is None else out
    _check("bitlinear_accumulate", lib().bitlinear_accumulate(
        _ptr(q), _ptr(rowsum), _ptr(P), M, K, N, _ptr(acc), _stream(stream)))
    return acc


def bitlinear_relu2_mul(a, b, out=None, stream=None):
    _need(a, torch.bfloat16, "a")
    _need(b, torch.bfloat16, "b")
    z = torch.empty_like(a) if out is None else out
    _check("bitlinear_relu2_mul", lib().bitlinear_relu2_mul(_ptr(a), _ptr(b), a.numel(), _ptr(z),
                                                            _stream(stream)))
    return z


def bitlinear_rope(x, pos, heads, theta, out=None, stream=None):
    """RoPE of bf16 x [M, heads * head_dim] at int32 positions pos [M] (out may be x)."""
    _need(x, torch.bfloat16, "x", 2)
    _need(pos, torch.int32, "pos", 1)
    M, W = x.shape
    if W % heads:
        raise TypeError("x's width must be heads * head_dim")
    y = torch.empty_like(x) if out is None else out
    _check("bitlinear_rope", lib().bitlinear_rope(_ptr(x), _ptr(pos), M, heads, W // heads, float(theta),
                                                  _ptr(y), _stream(stream)))
    return y


def bitlinear_attn_decode_workspace_size(L, q_heads, kv_heads, head_dim):
    n = ctypes.c_size_t()
    _check("bitlinear_attn_decode_workspace_size",
           lib().bitlinear_attn_decode_workspace_size(L, q_heads, kv_heads, head_dim, ctypes.byref(n)))
    return n.value


def bitlinear_attn_decode(q, k_cache, v_cache, L, q_heads, kv_heads, scale, out=None, workspace=None,
                          stream=None):
    """One decode token's GQA attention: q bf16 [q_heads * d], caches bf16
    [>= L, kv_heads, d] -> bf16 [q_heads * d]."""
    _need(q, torch.bfloat16, "q")
    _need(k_cache, torch.bfloat16, "k_cache")
    _need(v_cache, torch.bfloat16, "v_cache")
    d = q.numel() // q_heads
    y = torch.empty(q_heads * d, dtype=torch.bfloat16, device=q.device) if out is None else out
    nbytes = bitlinear_attn_decode_workspace_size(L, q_heads, kv_heads, d)
    ws = _workspace(nbytes, q.device) if workspace is None else workspace
    _check("bitlinear_attn_decode",
           lib().bitlinear_attn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), L, q_heads, kv_heads, d,
                                       float(scale), _ptr(y), _ptr(ws), ws.numel() * ws.element_size(),
                                       _stream(stream)))
    return y


def bitlinear_pack_gate_up_workspace_size(I, K):
    n = ctypes.c_size_t()
    _check("bitlinear_pack_gate_up_workspace_size",
           lib().bitlinear_pack_gate_up_workspace_size(I, K, ctypes.byref(n)))
    return n.value


def bitlinear_pack_gate_up(W_gate, W_up, P2=None, beta=None, workspace=None, stream=None):
    """fp32 masters W_gate, W_up [I,K] -> (P2 uint8 [I/2,K], beta fp32 [2] = {gate, up})."""
    _need(W_gate, torch.float32, "W_gate", 2)
    _need(W_up, torch.float32, "W_up", 2)
    I, K = W_gate.shape
    if W_up.shape != W_gate.shape:
        raise TypeError("W_gate and W_up must have the same shape")
    P2 = torch.empty((I // 2, K), dtype=torch.uint8, device=W_gate.device) if P2 is None else P2
    beta = torch.empty(2, dtype=torch.float32, device=W_gate.device) if beta is None else beta
    ws = _workspace(bitlinear_pack_gate_up_workspace_size(I, K), W_gate.device) \
        if workspace is None else workspace
    _check("bitlinear_pack_gate_up", lib().bitlinear_pack_gate_up(
        _ptr(W_gate), _ptr(W_up), I, K, _ptr(P2), _ptr(beta), _ptr(ws), ws.numel(), _stream(stream)))
    return P2, beta


def bitlinear_forward_gate_up(q, s_x, rowsum, P2, beta_gate, beta_up, out=None, workspace=None,
                              stream=None):
    """z = relu(gate)^2 * up (bf16 [M, I]) from quantised activations and a packed pair."""
    _need(q, torch.int8, "q", 2)
    _need(P2, torch.uint8, "P2", 2)
    M, K = q.shape
    I = 2 * P2.shape[0]
    z = torch.empty((M, I), dtype=torch.bfloat16, device=q.device) if out is None else out
    _check("bitlinear_forward_gate_up", lib().bitlinear_forward_gate_up(
        _ptr(q), _ptr(s_x), _ptr(rowsum), _ptr(P2), float(beta_gate), float(beta_up), M, K, I,
        _ptr(z), _ptr(workspace), 0 if workspace is None else workspace.numel(), _stream(stream)))
    return z


def bitlinear_forward_online_workspace_size(M, K, N):
    n = ctypes.c_size_t()
    _check("bitlinear_forward_online_workspace_size",
           lib().bitlinear_forward_online_workspace_size(M, K, N, ctypes.byref(n)))
    return n.value


def bitlinear_forward_online(x, W, gain=None, eps=1e-5, out_dtype=torch.bfloat16, out=None,
                             workspace=None, stream=None):
    """Training forward from fp32 masters W [N,K]: returns (y, saved) where
    saved = dict(P, beta (device fp32 [1]), q, s_x, rowsum) feeds the backward."""
    _need(x, torch.bfloat16, "x", 2)
    _need(W, torch.float32, "W", 2)
    if gain is not None:
        _need(gain, torch.bfloat16, "gain", 1)
    M, K = x.shape
    N = W.shape[0]
    dev = x.device
    y = torch.empty((M, N), dtype=out_dtype, device=dev) if out is None else out
    saved = dict(P=torch.empty((N // 4, K), dtype=torch.uint8, device=dev),
                 beta=torch.empty(1, dtype=torch.float32, device=dev),
                 q=torch.empty((M, K), dtype=torch.int8, device=dev),
                 s_x=torch.empty(M, dtype=torch.float32, device=dev),
                 rowsum=torch.empty(M, dtype=torch.int32, device=dev))
    ws = _workspace(bitlinear_forward_online_workspace_size(M, K, N), dev) \
        if workspace is None else workspace
    _check("bitlinear_forward_online", lib().bitlinear_forward_online(
        _ptr(x), _ptr(gain), eps, _ptr(W), M, K, N, _ptr(y), _out_code(y.dtype), _ptr(saved["P"]),
        _ptr(saved["beta"]), _ptr(saved["q"]), _ptr(saved["s_x"]), _ptr(saved["rowsum"]),
        _ptr(ws), ws.numel(), _stream(stream)))
    return y, saved


def bitlinear_backward_ste(grad_y, saved, K, grad_x=True, grad_w=True, stream=None):
    """Straight-through backward: (grad_x fp32 [M,K] or None, grad_w fp32 [N,K] or None)."""
    _need(grad_y, torch.float32, "grad_y", 2)
    M, N = grad_y.shape
    dev = grad_y.device
    gx = torch.empty((M, K), dtype=torch.float32, device=dev) if grad_x else None
    gw = torch.empty((N, K), dtype=torch.float32, device=dev) if grad_w else None
    _check("bitlinear_backward_ste", lib().bitlinear_backward_ste(
        _ptr(grad_y), _ptr(saved["q"]), _ptr(saved["s_x"]), _ptr(saved["P"]), _ptr(saved["beta"]),
        M, K, N, _ptr(gx), _ptr(gw), _stream(stream)))
    return gx, gw


def make_chain(steps):
    """bl_chain_step array from dicts: x (bf16 [1,K] or [K]), optional gain,
    eps, problems = [dict(P, y, beta, optional residual, beta_up, kind)]
    (kind: "bf16", "f32" or "gate_up"; N is taken from y)."""
    kinds = {"bf16": BL_CHAIN_BF16, "f32": BL_CHAIN_F32, "gate_up": BL_CHAIN_GATE_UP}
    arr = (ChainStep * len(steps))()
    for i, st in enumerate(steps):
        x = st["x"]
        _need(x, torch.bfloat16, "x")
        arr[i].x = x.data_ptr()
        arr[i].gain = _addr(st.get("gain"))
        arr[i].eps = float(st.get("eps", 1e-5))
        arr[i].K = x.numel()
        probs = st["problems"]
        arr[i].count = len(probs)
        for j, pr in enumerate(probs):
            _need(pr["P"], torch.uint8, "P", 2)
            arr[i].p[j] = ChainProblem(pr["P"].data_ptr(), pr["y"].data_ptr(),
                                       _addr(pr.get("residual")), pr["y"].numel(),
                                       float(pr["beta"]), float(pr.get("beta_up", 0.0)),
                                       kinds[pr.get("kind", "bf16")])
    return arr


def bitlinear_decode_chain_workspace_size(nsteps):
    n = ctypes.c_size_t()
    _check("bitlinear_decode_chain_workspace_size",
           lib().bitlinear_decode_chain_workspace_size(nsteps, ctypes.byref(n)))
    return n.value


def bitlinear_decode_chain_prepare(chain, workspace=None):
    """Copy a make_chain() array into a (new or given) device workspace; returns it."""
    ws = _workspace(bitlinear_decode_chain_workspace_size(len(chain)), "cuda") \
        if workspace is None else workspace
    _check("bitlinear_decode_chain_prepare", lib().bitlinear_decode_chain_prepare(
        ctypes.cast(chain, _P), len(chain), _ptr(ws), ws.numel()))
    return ws


def bitlinear_decode_chain_run(workspace, nsteps, stream=None):
    _check("bitlinear_decode_chain_run", lib().bitlinear_decode_chain_run(
        _ptr(workspace), workspace.numel(), nsteps, _stream(stream)))


def bitlinear_selftest_wait_timeout(limit_ns, stream=None):
    """Launch the bounded-wait self-test (see include/bitlinear.h)."""
    _check("bitlinear_selftest_wait_timeout",
           lib().bitlinear_selftest_wait_timeout(int(limit_ns), _stream(stream)))


def bitlinear_device_status(stream=None):
    """Synchronise and return (and clear) the library's device status code."""
    return lib().bitlinear_device_status(_stream(stream))
