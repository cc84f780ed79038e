"""FP64 oracle of the gradient of the Flint sink-aware GQA attention forward.

TEST INFRASTRUCTURE ONLY: the test suite and the backward leg of the
benchmark's CPU baseline are the only callers; the product never imports it.

The pages make every head's sink a trainable parameter held in FP32 and note
that the sink's adjoint needs care in context-parallel training ("flint"
model page on NeMo AutoModel, "Parallelism and backends"; FA4 rejects learned
sinks in backward, same section).  They give no formula, so this module takes
the plain reading: the exact derivative of the forward (FlintAttention.forward
on the "flint.layers" API page; the sink as a zero-value softmax column, HF
discussion #26 on RecursiveSI/flint) for a scalar loss that depends on `out`
only (lse is an auxiliary output and receives no gradient).

For one document, query head h (KV head g = h // 8), rows i, keys j:

    n = x r w,  r = (mean(x^2) + eps)^(-1/2)           RMSNorm, weight form
    x~ = R(p) n                                        NeoX RoPE (sliding layers)
    s_ij = q~_i . k~_j / sqrt(128) on allowed pairs     causal, same document,
                                                       i - j < W on sliding layers
    lse_i = ln(e^{sink_h} + sum_j e^{s_ij})
    P_ij = e^{s_ij - lse_i},  P_sink,i = e^{sink_h - lse_i}
    out_i = sum_j P_ij v_j

Given dO = dLoss/d out, the adjoint of each step in reverse order:

    D_i    = dO_i . out_i
    dv_j   = sum_{h in g} sum_i P_ij dO_i
    dS_ij  = P_ij (dO_i . v_j - D_i)
    dsink  = -sum_i P_sink,i D_i        (the sink column carries a zero value)
    dq~_i  = sum_j dS_ij k~_j / sqrt(128),   dk~_j = sum_{h in g} sum_i dS_ij q~_i / sqrt(128)
    dn     = R(p)^T dx~                  (rotation by -p)
    dw    += dn * x r                    (summed over every row that uses w)
    dx     = r (w * dn) - x r^3 (sum_c w_c dn_c x_c) / 128

Padded tokens have out = 0 whatever the inputs, so every gradient through
them is zero.  A head with sink = +inf has out = 0 (all gradients 0); with
sink = -inf the sink column vanishes (dsink = 0).
"""
from __future__ import annotations

import numpy as np

from . import D, HKV, HQ, _f64, doc_ids

GROUP = HQ // HKV


def _inv_freq(theta: float) -> np.ndarray:
    return theta ** (-2.0 * np.arange(D // 2) / D)


def _norm(x, w, eps):
    """Rows of x [..., 128]: returns n and the per-row r."""
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return x * r * w, r


def _rope(x, pos, theta, sign=1.0):
    """NeoX half-split rotation of rows x [n, H, 128] by sign * pos[n]."""
    ang = sign * pos[:, None].astype(np.float64) * _inv_freq(theta)[None, :]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    lo, hi = x[..., :D // 2], x[..., D // 2:]
    return np.concatenate([lo * c - hi * s, hi * c + lo * s], axis=-1)


def _segments(doc):
    """(start, end) of each run of equal non-negative segment ids."""
    out, T, i = [], len(doc), 0
    while i < T:
        if doc[i] < 0:
            i += 1
            continue
        j = i
        while j < T and doc[j] == doc[i]:
            j += 1
        out.append((i, j))
        i = j
    return out


def attn_bwd(q, k, v, q_norm_w, k_norm_w, sinks, dout, *, pos_ids=None, cu_seqlens=None,
             pad_mask=None, window=0, use_rope=False, rope_theta=10000.0, eps=1e-6, out_given=None):
    """Gradients of sum(dout * out) for the forward with these arguments.

    q [T,32,128], k and v [T,4,128] (BF16 bit patterns or floats), weights
    [128], sinks [32], dout [T,32,128] (or [T,4096]); pos_ids None means the
    index of each token within its document.  Returns a dict of
    float64 arrays: dq [T,32,128], dk, dv [T,4,128], dq_norm_w, dk_norm_w
    [128], dsinks [32], and the forward's out [T,32,128] and lse [T,32].

    out_given: a forward output [T,32,128] to take D_i = dO_i . out_i from
    instead of the exact one (the same formula evaluated at a stored forward
    output, as a backward that receives `out` does); None: the exact output.
    """
    qx, kx, vx = _f64(q), _f64(k), _f64(v)
    T = qx.shape[0]
    qx = qx.reshape(T, HQ, D)
    kx = kx.reshape(T, HKV, D)
    vx = vx.reshape(T, HKV, D)
    do = _f64(dout).reshape(T, HQ, D)
    og = None if out_given is None else _f64(out_given).reshape(T, HQ, D)
    wq = _f64(q_norm_w).reshape(D)
    wk = _f64(k_norm_w).reshape(D)
    sk = np.asarray(sinks, np.float64).reshape(HQ)
    doc = doc_ids(T, cu_seqlens, pad_mask)
    if pos_ids is None:                 # default: index of the token within its document
        pos = np.zeros(T, np.int64)
        for a, b in _segments(doc):
            pos[a:b] = np.arange(b - a)
    else:
        pos = np.asarray(pos_ids, np.int64).reshape(T)
    scale = 1.0 / np.sqrt(D)

    # forward quantities
    nq, rq = _norm(qx, wq, eps)
    nk, rk = _norm(kx, wk, eps)
    qt = _rope(nq, pos, rope_theta) if use_rope else nq
    kt = _rope(nk, pos, rope_theta) if use_rope else nk

    out = np.zeros((T, HQ, D))
    lse = np.zeros((T, HQ))
    dqt = np.zeros((T, HQ, D))
    dkt = np.zeros((T, HKV, D))
    dv = np.zeros((T, HKV, D))
    dsinks = np.zeros(HQ)
    lse[doc < 0] = sk[None, :]

    for a, b in _segments(doc):
        L = b - a
        i = np.arange(L)[:, None]
        j = np.arange(L)[None, :]
        allowed = j <= i
        if window > 0:
            allowed &= (i - j) < window
        for g in range(HKV):
            K, V = kt[a:b, g], vx[a:b, g]
            for h in range(GROUP * g, GROUP * (g + 1)):
                sink = sk[h]
                if sink == np.inf:
                    lse[a:b, h] = np.inf
                    continue
                S = np.where(allowed, qt[a:b, h] @ K.T * scale, -np.inf)
                m = np.maximum(S.max(axis=1), sink)
                Z = np.exp(S - m[:, None]).sum(axis=1) + np.exp(sink - m)
                ls = m + np.log(Z)
                P = np.exp(S - ls[:, None])
                Psink = np.exp(sink - ls)
                O = P @ V
                out[a:b, h] = O
                lse[a:b, h] = ls
                dO = do[a:b, h]
                Dr = np.sum(dO * (O if og is None else og[a:b, h]), axis=1)
                dv[a:b, g] += P.T @ dO
                dS = P * (dO @ V.T - Dr[:, None])
                dsinks[h] += -np.sum(Psink * Dr)
                dqt[a:b, h] = dS @ K * scale
                dkt[a:b, g] += dS.T @ qt[a:b, h] * scale

    # back through RoPE: the transpose of a rotation is the rotation by -p
    dnq = _rope(dqt, pos, rope_theta, -1.0) if use_rope else dqt
    dnk = _rope(dkt, pos, rope_theta, -1.0) if use_rope else dkt

    # back through RMSNorm
    def norm_bwd(x, r, w, dn):
        dw = np.sum(dn * x * r, axis=(0, 1))
        t = np.sum(w * dn * x, axis=-1, keepdims=True)
        dx = r * w * dn - x * r ** 3 * t / D
        return dx, dw

    dq, dwq = norm_bwd(qx, rq, wq, dnq)
    dk, dwk = norm_bwd(kx, rk, wk, dnk)
    return dict(dq=dq, dk=dk, dv=dv, dq_norm_w=dwq, dk_norm_w=dwk, dsinks=dsinks,
                out=out, lse=lse)


def attn_bwd_workload(w, dout, out_given=None):
    """The oracle on a ``workloads.Workload`` with upstream gradient dout."""
    return attn_bwd(w.q, w.k, w.v, w.q_norm_w, w.k_norm_w, w.sinks, dout, pos_ids=w.pos_ids,
                    cu_seqlens=w.cu_seqlens, pad_mask=w.pad_mask, window=w.window,
                    use_rope=w.use_rope, rope_theta=w.rope_theta, eps=w.eps, out_given=out_given)
