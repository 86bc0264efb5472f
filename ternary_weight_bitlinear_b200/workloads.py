"""Seeded synthetic inputs at BitNet b1.58 2B4T shapes.

This module only draws random numbers and casts them to the input dtypes; it
holds none of the BitLinear arithmetic, so both the CUDA path and the CPU
oracle can take their inputs from it.

Shapes come from the "BitNet" transformers model doc (BitNetConfig defaults:
hidden_size 2560, intermediate_size 6912, 30 hidden layers, 20 query heads and
5 key/value heads of width 128, rms_norm_eps 1e-5).  Each decoder layer holds
seven BitLinear projections:

    q 2560->2560, k 2560->640, v 2560->640, o 2560->2560,
    gate 2560->6912, up 2560->6912, down 6912->2560

Seeds (numpy ``default_rng``):
    master weights of layer l, projection p (index into PROJECTIONS): 1000*(l+1)+p
    input-norm gain of layer l: 1000*(l+1)+10,  sub-norm gain: 1000*(l+1)+11
    activations for layer l, projection p: 1000*(l+1)+20+p   (stream "x")
    per-row standard deviations: the activation seed + 500      (stream "std")

bf16 arrays are returned as ``numpy.uint16`` bit patterns (rounded to nearest
even by torch's cast from the fp32 draw).
"""
from collections import namedtuple

import numpy as np
import torch

HIDDEN = 2560
INTERMEDIATE = 6912
LAYERS = 30
RMS_EPS = 1e-5
MASTER_STD = 0.02

Projection = namedtuple("Projection", "name K N")
PROJECTIONS = (
    Projection("q", HIDDEN, HIDDEN),
    Projection("k", HIDDEN, 640),
    Projection("v", HIDDEN, 640),
    Projection("o", HIDDEN, HIDDEN),
    Projection("gate", HIDDEN, INTERMEDIATE),
    Projection("up", HIDDEN, INTERMEDIATE),
    Projection("down", INTERMEDIATE, HIDDEN),
)
PROJ_INDEX = {p.name: i for i, p in enumerate(PROJECTIONS)}


def to_bf16_bits(a):
    """fp32 numpy array -> bf16 bit patterns (uint16), via torch's RN cast."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def master_seed(layer, proj):
    p = PROJ_INDEX[proj] if isinstance(proj, str) else proj
    return 1000 * (layer + 1) + p


def x_seed(layer, proj):
    p = PROJ_INDEX[proj] if isinstance(proj, str) else proj
    return 1000 * (layer + 1) + 20 + p


def master_weights(N, K, seed, std=MASTER_STD):
    """Gaussian master weights W[N,K] ~ N(0, std^2), fp32."""
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((N, K), dtype=np.float32) * np.float32(std)).astype(np.float32)


def gain(K, seed):
    """RMSNorm gain ~ U(0.5, 1.5), bf16 bits [K]."""
    rng = np.random.default_rng(seed)
    return to_bf16_bits(rng.uniform(0.5, 1.5, K).astype(np.float32))


def activations(M, K, seed, outlier_frac=0.0, outlier_scale=20.0, row_std=None,
                zero_rows=()):
    """x[M,K] ~ N(0,1) as bf16 bits.

    outlier_frac: fraction of elements (chosen by a uniform mask) multiplied by
        ``outlier_scale``;
    row_std: (lo, hi) -> each row is scaled by a std drawn from U(lo, hi) on a
        separate stream;
    zero_rows: rows forced to exactly zero.
    """
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K), dtype=np.float32)
    if outlier_frac > 0.0:
        mask = rng.random((M, K)) < outlier_frac
        x[mask] *= np.float32(outlier_scale)
    if row_std is not None:
        srng = np.random.default_rng(seed + 500)
        std = srng.uniform(row_std[0], row_std[1], M).astype(np.float32)
        x *= std[:, None]
    for r in zero_rows:
        x[r, :] = 0.0
    return to_bf16_bits(x)


# --- the five workloads ----------------------------------------------------
# 1: single BitLinear, M=4 K=256 N=128, row 1 all zeros, no norm, fp32 out.
def config1():
    x = activations(4, 256, seed=0, zero_rows=(1,))
    W = master_weights(128, 256, seed=1000)
    return dict(x=x, W=W, M=4, K=256, N=128, norm=False, out="f32")


# 2: decode GEMV, M=1, 0.1% outliers x20, fused RMSNorm with U(0.5,1.5) gain.
def config2_projection(layer, proj, M=1):
    p = PROJECTIONS[PROJ_INDEX[proj]]
    return dict(x=activations(M, p.K, x_seed(layer, proj), outlier_frac=0.001),
                gain=gain(p.K, 1000 * (layer + 1) + 10),
                M=M, K=p.K, N=p.N, norm=True, out="bf16", name=proj, layer=layer)


# 3: batched decode, M in {8,32,64}, per-row std ~ U(0.1,10), no norm.
def config3_projection(layer, proj, M):
    p = PROJECTIONS[PROJ_INDEX[proj]]
    return dict(x=activations(M, p.K, x_seed(layer, proj), row_std=(0.1, 10.0)),
                M=M, K=p.K, N=p.N, norm=False, out="bf16", name=proj, layer=layer)


# 4: prefill GEMM, M=4096, fused RMSNorm, on gate/up/down/q/o.
CONFIG4_PROJECTIONS = ("gate", "up", "down", "q", "o")


def config4_projection(proj, M=4096, layer=0):
    p = PROJECTIONS[PROJ_INDEX[proj]]
    return dict(x=activations(M, p.K, x_seed(layer, proj)),
                gain=gain(p.K, 1000 * (layer + 1) + 10),
                M=M, K=p.K, N=p.N, norm=True, out="bf16", name=proj, layer=layer)


# 5: 30-layer FFN chain at M=16 (attention omitted).
def config5_input(M=16, H=HIDDEN):
    return activations(M, H, seed=0)


def config5_layer(layer, H=HIDDEN, I=INTERMEDIATE):
    return dict(W_gate=master_weights(I, H, master_seed(layer, "gate")),
                W_up=master_weights(I, H, master_seed(layer, "up")),
                W_down=master_weights(H, I, master_seed(layer, "down")),
                g_in=gain(H, 1000 * (layer + 1) + 10),
                g_sub=gain(I, 1000 * (layer + 1) + 11))


# ---------------------------------------------------------------------------
# attention block of the decoder layer (20 query heads, 5 key/value heads of 128)
# ---------------------------------------------------------------------------
Q_HEADS = 20
KV_HEADS = 5
HEAD_DIM = 128
MAX_POSITIONS = 2048


def attention_decode_inputs(L, seed, q_heads=Q_HEADS, kv_heads=KV_HEADS, head_dim=HEAD_DIM,
                            q_std=1.0):
    """One decode token over an L-position cache: q [q_heads * head_dim] ~
    N(0, q_std^2), k_cache and v_cache [L, kv_heads, head_dim] ~ N(0, 1), all
    bf16 bits (seed, seed + 1, seed + 2)."""
    q = np.random.default_rng(seed).standard_normal(q_heads * head_dim).astype(np.float32)
    k = np.random.default_rng(seed + 1).standard_normal((L, kv_heads, head_dim)).astype(np.float32)
    v = np.random.default_rng(seed + 2).standard_normal((L, kv_heads, head_dim)).astype(np.float32)
    return to_bf16_bits(q * np.float32(q_std)), to_bf16_bits(k), to_bf16_bits(v)


def rope_positions(M, seed, max_pos=MAX_POSITIONS):
    """M token positions in [0, max_pos), the first 0 and the last max_pos - 1."""
    p = np.random.default_rng(seed).integers(0, max_pos, M).astype(np.int32)
    p[0] = 0
    if M > 1:
        p[-1] = max_pos - 1
    return p
