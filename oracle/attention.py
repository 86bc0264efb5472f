"""CPU oracle of the rest of the BitNet b1.58 decoder layer's attention block:
rotary position embeddings and grouped-query decode attention, in float64.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: the tests, the smoke
check and the benchmark's CPU leg may call it; the product path never does.

What the pages fix: the "BitNet" model doc, model details, says the decoder
uses rotary position embeddings (RoPE) and its BitNetConfig gives 20 attention
heads over hidden size 2560 (head dimension 128), 5 key/value heads (grouped
query attention: each key/value head serves a group of query heads) and at
most 2048 positions; the layer order is q, k, v -> RoPE + attention ->
attn_sub_norm -> o.  The pages give no formula for either operation, so both
are the textbook definitions (the readings are listed with the design):

* RoPE, in the rotate-half form: for head dimension d and i < d/2 the pair
  (x[i], x[i + d/2]) of every head is rotated by the angle pos * theta^(-2i/d):
      y[i]       = x[i] cos(a) - x[i + d/2] sin(a)
      y[i + d/2] = x[i + d/2] cos(a) + x[i] sin(a)
  theta is a parameter (the pages name rope_theta without a value).
* Decode attention for one query token over the L cached positions (the
  current token's key and value included): query head h reads key/value head
  h // (H / H_kv); scores s_j = (q_h . k_j) * scale, p = softmax(s),
  out_h = sum_j p_j v_j.

Function        Definition followed
--------------  -------------------------------------------------------------
rope_inv_freq   theta^(-2i/d), i < d/2
rope            the rotation above, per token position
attn_decode     softmax(q k^T * scale) v per query head, kv head h // group
"""
import numpy as np


def rope_inv_freq(head_dim, theta):
    """Angular frequency of pair i: theta^(-2i/d), float64."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    return np.power(float(theta), -2.0 * i / head_dim)


def rope(x, pos, heads, head_dim, theta):
    """x: [M, heads * head_dim] (any float dtype; bf16 inputs as their float
    values), pos: [M] integer positions -> float64 [M, heads * head_dim]."""
    pos = np.asarray(pos, dtype=np.int64).reshape(-1)
    M = pos.shape[0]
    x = np.asarray(x, dtype=np.float64).reshape(M, heads, head_dim)
    ang = pos.astype(np.float64)[:, None] * rope_inv_freq(head_dim, theta)[None, :]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    h = head_dim // 2
    x1, x2 = x[..., :h], x[..., h:]
    y = np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)
    return y.reshape(M, heads * head_dim)


def attn_decode(q, k_cache, v_cache, L, q_heads, kv_heads, head_dim, scale):
    """q: [q_heads * head_dim]; k_cache, v_cache: [>= L, kv_heads, head_dim]
    (positions past L are not read) -> float64 [q_heads * head_dim]."""
    if q_heads % kv_heads:
        raise ValueError("query heads must be a multiple of key/value heads")
    q = np.asarray(q, dtype=np.float64).reshape(q_heads, head_dim)
    K = np.asarray(k_cache, dtype=np.float64).reshape(-1, kv_heads, head_dim)[:L]
    V = np.asarray(v_cache, dtype=np.float64).reshape(-1, kv_heads, head_dim)[:L]
    group = q_heads // kv_heads
    out = np.empty((q_heads, head_dim), dtype=np.float64)
    for h in range(q_heads):
        g = h // group
        s = (K[:, g, :] @ q[h]) * float(scale)
        p = np.exp(s - s.max())
        out[h] = (p @ V[:, g, :]) / p.sum()
    return out.reshape(-1)
