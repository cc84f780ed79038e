"""FP64 oracle of one decode step of the Flint sink-aware GQA attention
against a key/value cache.

TEST INFRASTRUCTURE ONLY: the test suite and the decode leg of the
benchmark's CPU baseline are the only callers; the product never imports it.

One new token per sequence b sits at position p = cache_len[b].  Following
FlintAttention.forward on the NeMo AutoModel "flint.layers" API page (per-head
RMSNorm in weight form, then NeoX RoPE on sliding layers, learned sink as an
extra zero-value softmax column in natural-logit units: HF discussion #26 on
RecursiveSI/flint):

    q~ = RoPE(RMSNorm(q, w_q), p),  k~ = RoPE(RMSNorm(k, w_k), p)
    keys j in [lo, p]: lo = max(0, p - W + 1) on a sliding layer of window W
    (the window counts the current token), lo = 0 on a full layer
    K_j, V_j = the cached key and value of position j for j < p; k~, v for j = p
    s_j = q~ . K_j / sqrt(128)
    Z = e^{sink_h} + sum_j e^{s_j},  out = sum_j e^{s_j} V_j / Z,  lse = ln Z

The cache stores position j in slot j mod cap, which makes a cache of
capacity >= W a ring for sliding layers (the "flint" model page's hybrid KV
cache, where per-layer window sizes must be honoured).  Cached keys are taken
as given: they are the normalised, rotated keys of earlier steps, in whatever
precision the cache holds.  Query head h reads KV head h // 8.

The norm and rotation of single rows reuse the C oracle's routines
(``oracle.rmsnorm``, ``oracle.rope``); the attention over the window is
written out here in float64 with log-sum-exp stabilisation.
"""
from __future__ import annotations

import numpy as np

from . import D, HKV, HQ, _f64, rmsnorm, rope

GROUP = HQ // HKV


def normalise(x, w, pos: int, use_rope: bool, theta: float, eps: float) -> np.ndarray:
    """RMSNorm (weight form) then, if use_rope, NeoX RoPE at pos: one row."""
    y = rmsnorm(x, w, eps)
    return rope(y, pos, theta) if use_rope else y


def decode_step(q, k, v, k_cache, v_cache, cache_len, q_norm_w, k_norm_w, sinks, *,
                window: int, use_rope: bool, rope_theta: float = 10000.0, eps: float = 1e-6):
    """One decode step for B sequences.

    q [B,32,128], k and v [B,4,128]: the new token's projections (BF16 bit
    patterns or floats); k_cache, v_cache [B,4,cap,128] (BF16 bit patterns or
    floats; head-major: slot j of KV head g is k_cache[b, g, j]); cache_len [B].  Returns out [B,32,128], lse [32,B] and the new
    token's normalised, rotated keys k~ [B,4,128], all float64.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    kc, vc = _f64(k_cache), _f64(v_cache)
    sinks = np.asarray(sinks, np.float64).reshape(HQ)
    B, cap = kc.shape[0], kc.shape[2]
    q = q.reshape(B, HQ, D)
    k = k.reshape(B, HKV, D)
    v = v.reshape(B, HKV, D)
    out = np.zeros((B, HQ, D))
    lse = np.zeros((HQ, B))
    k_new = np.zeros((B, HKV, D))
    scale = 1.0 / np.sqrt(D)
    for b in range(B):
        p = int(cache_len[b])
        lo = max(0, p - window + 1) if window > 0 else 0
        if p - lo + 1 > cap:
            raise ValueError("the window does not fit the cache capacity")
        pos = np.arange(lo, p)                       # cached positions in the window
        slots = pos % cap
        for g in range(HKV):
            k_new[b, g] = normalise(k[b, g], k_norm_w, p, use_rope, rope_theta, eps)
            keys = np.concatenate([kc[b, g, slots], k_new[b, g][None]], axis=0)
            vals = np.concatenate([vc[b, g, slots], v[b, g][None]], axis=0)
            for h in range(GROUP * g, GROUP * (g + 1)):
                qt = normalise(q[b, h], q_norm_w, p, use_rope, rope_theta, eps)
                s = keys @ qt * scale
                sink = sinks[h]
                if sink == np.inf:
                    out[b, h] = 0.0
                    lse[h, b] = np.inf
                    continue
                m = max(s.max(), sink)
                e = np.exp(s - m)
                z = e.sum() + (np.exp(sink - m) if sink > -np.inf else 0.0)
                out[b, h] = (e @ vals) / z
                lse[h, b] = m + np.log(z)
    return out, lse, k_new
