"""FP64 oracle of the whole Flint attention layer around the attention core:
the QKV projections in front of it and o_proj behind it.

TEST INFRASTRUCTURE ONLY: the test suite is the only caller; the product
never imports it.

FlintAttention.forward ("flint.layers" API page) maps hidden states
[T, hidden] to [T, hidden]: q_proj, k_proj and v_proj (no bias: FlintConfig
attention_bias = False, and HF discussion #26 notes that this makes fused
QKV kernels trivial), the per-head q_norm/k_norm and RoPE, the sink-aware
attention, then o_proj.  The checkpoint's sizes ("flint" model page, "Model
Architecture"): hidden 2048, 32 query heads and 4 key/value heads of 128.

Weights use the PyTorch Linear layout [out_features, in_features]:

    q = h W_q^T  [T, 4096] -> [T, 32, 128]   (head-major: column h*128 + c)
    k = h W_k^T  [T, 512]  -> [T, 4, 128]
    v = h W_v^T  [T, 512]  -> [T, 4, 128]
    a = attention(q, k, v)  [T, 32, 128] -> [T, 4096] (column h*128 + c)
    y = a W_o^T  [T, hidden]

The attention core is the C oracle (``oracle.attn_fwd``), fed the projections
in FP64 (no intermediate rounding: the exact composition).
"""
from __future__ import annotations

import numpy as np

from . import D, HKV, HQ, _f64, attn_fwd


def project_qkv(hidden, w_q, w_k, w_v):
    """The three projections: returns q [T,32,128], k and v [T,4,128]."""
    h = _f64(hidden)
    T = h.shape[0]
    q = (h @ _f64(w_q).T).reshape(T, HQ, D)
    k = (h @ _f64(w_k).T).reshape(T, HKV, D)
    v = (h @ _f64(w_v).T).reshape(T, HKV, D)
    return q, k, v


def attn_layer(hidden, w_q, w_k, w_v, w_o, q_norm_w, k_norm_w, sinks, *, pos_ids=None,
               cu_seqlens=None, pad_mask=None, window=0, use_rope=False, rope_theta=10000.0,
               eps=1e-6):
    """The layer's output [T, hidden] and the attention core's lse [T, 32]."""
    q, k, v = project_qkv(hidden, w_q, w_k, w_v)
    T = q.shape[0]
    a, lse = attn_fwd(q, k, v, q_norm_w, k_norm_w, sinks, pos_ids=pos_ids, cu_seqlens=cu_seqlens,
                      pad_mask=pad_mask, window=window, use_rope=use_rope, rope_theta=rope_theta,
                      eps=eps)
    y = a.reshape(T, HQ * D) @ _f64(w_o).T
    return y, lse
