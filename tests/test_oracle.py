"""Pins for the FP64 oracle: checks against facts the pages and mathematics fix,
never against the oracle's own formulas retyped.

Independent routes used here:
  * torch.nn.functional.rms_norm for the per-head norm;
  * complex multiplication (numpy) for the NeoX rotation;
  * torch scaled_dot_product_attention (float64, CPU) with an explicit
    boolean/additive mask, the sink entered as an extra zero-value key column
    whose additive bias is the sink logit;
  * closed forms (4-token hand case, uniform logits, window counts);
  * numpy's float16 conversion and an integer bit trick for the roundings.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f64(bits):
    return W.bf16_to_f64(bits)


def reference_sdpa(w, rows=None):
    """Independent FP64 evaluation through torch SDPA.

    The sink enters as one extra key whose key vector and value vector are
    zero and whose additive bias equals the sink logit, so its score is the
    unscaled sink and it adds nothing to the numerator."""
    T = w.T
    q = torch.tensor(f64(w.q))
    k = torch.tensor(f64(w.k))
    v = torch.tensor(f64(w.v))
    qn = F.rms_norm(q, (128,), weight=torch.tensor(w.q_norm_w, dtype=torch.float64), eps=w.eps)
    kn = F.rms_norm(k, (128,), weight=torch.tensor(w.k_norm_w, dtype=torch.float64), eps=w.eps)
    doc = oracle.doc_ids(T, w.cu_seqlens, w.pad_mask)
    if w.use_rope:
        pos = w.pos_ids.astype(np.float64)
        inv = np.exp(-np.log(w.rope_theta) * np.arange(64) / 64.0)
        rot = np.exp(1j * pos[:, None] * inv[None, :])          # [T,64]

        def rotate(x):
            xn = x.numpy()
            z = (xn[..., :64] + 1j * xn[..., 64:]) * rot[:, None, :]
            return torch.tensor(np.concatenate([z.real, z.imag], axis=-1))
        qn, kn = rotate(qn), rotate(kn)
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    allow = (j <= i) & (doc[:, None] == doc[None, :]) & (doc[None, :] >= 0) & (doc[:, None] >= 0)
    if w.window > 0:
        allow &= (i - j) <= (w.window - 1)
    bias = np.where(allow, 0.0, -np.inf)
    sinks = np.asarray(w.sinks, np.float64)
    full_bias = np.concatenate([np.broadcast_to(bias, (32, T, T)),
                                np.broadcast_to(sinks[:, None, None], (32, T, 1))], axis=2)
    kr = kn.repeat_interleave(8, dim=1)           # query head h reads KV head h // 8
    vr = v.repeat_interleave(8, dim=1)
    zero = torch.zeros(1, 32, 128, dtype=torch.float64)
    kh = torch.cat([kr, zero], 0).permute(1, 0, 2)[None]
    vh = torch.cat([vr, zero], 0).permute(1, 0, 2)[None]
    qh = qn.permute(1, 0, 2)[None]
    bias_t = torch.tensor(full_bias)[None]
    out = F.scaled_dot_product_attention(qh, kh, vh, attn_mask=bias_t)   # [1,32,T,128]
    scores = (qh @ kh.transpose(-1, -2)) / math.sqrt(128.0) + bias_t
    lse = torch.logsumexp(scores, dim=-1)                                 # [1,32,T]
    out = out[0].permute(1, 0, 2).numpy()
    lse = lse[0].permute(1, 0).numpy()
    if rows is not None:
        out, lse = out[rows], lse[rows]
    return out, lse


def run(w, **kw):
    return oracle.attn_fwd_workload(w, rows=kw.pop("rows", None), **kw)


# ---------------------------------------------------------------- library pins

@pytest.mark.parametrize("window,use_rope", [(0, False), (0, True), (7, True), (513, True)])
def test_matches_sdpa_with_sink_column(window, use_rope):
    w = W.make_small(45, seed=11, window=window, use_rope=use_rope)
    out, lse = run(w)
    ro, rl = reference_sdpa(w)
    np.testing.assert_allclose(out, ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=0, atol=1e-12)


def test_sink_minus_inf_is_textbook_causal_softmax():
    w = W.make_small(40, seed=12, window=0, use_rope=True, sinks=-np.inf)
    out, lse = run(w)
    # textbook causal softmax attention, no extra column at all
    T = w.T
    q = torch.tensor(f64(w.q)); k = torch.tensor(f64(w.k)); v = torch.tensor(f64(w.v))
    qn = F.rms_norm(q, (128,), weight=torch.tensor(w.q_norm_w, dtype=torch.float64), eps=w.eps)
    kn = F.rms_norm(k, (128,), weight=torch.tensor(w.k_norm_w, dtype=torch.float64), eps=w.eps)
    pos = w.pos_ids.astype(np.float64)
    inv = np.exp(-np.log(w.rope_theta) * np.arange(64) / 64.0)
    rot = np.exp(1j * pos[:, None] * inv[None, :])

    def rotate(x):
        xn = x.numpy()
        z = (xn[..., :64] + 1j * xn[..., 64:]) * rot[:, None, :]
        return torch.tensor(np.concatenate([z.real, z.imag], axis=-1))
    qh = rotate(qn).permute(1, 0, 2)[None]
    kh = rotate(kn).repeat_interleave(8, dim=1).permute(1, 0, 2)[None]
    vh = v.repeat_interleave(8, dim=1).permute(1, 0, 2)[None]
    ref = F.scaled_dot_product_attention(qh, kh, vh, is_causal=True)[0].permute(1, 0, 2).numpy()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    assert np.all(np.isfinite(lse))


def test_gqa_head_mapping_is_contiguous_groups():
    """Query head h must read KV head h // 8: perturbing KV head 2 may change
    only query heads 16..23."""
    w = W.make_small(20, seed=13)
    out0, _ = run(w)
    k2 = w.k.copy()
    k2[:, 2, :] = W.bf16_bits(np.random.default_rng(1).standard_normal((20, 128)).astype(np.float32))
    w.k = k2
    out1, _ = run(w)
    changed = np.abs(out1 - out0).max(axis=(0, 2)) > 0
    assert list(np.nonzero(changed)[0]) == list(range(16, 24))


def test_rmsnorm_matches_torch():
    rng = np.random.default_rng(3)
    for scale in (1e-3, 1.0, 1e4):
        x = rng.standard_normal(128) * scale
        wv = 1 + 0.1 * rng.standard_normal(128)
        y = oracle.rmsnorm(x, wv, 1e-6)
        ref = F.rms_norm(torch.tensor(x)[None], (128,), weight=torch.tensor(wv), eps=1e-6)[0].numpy()
        np.testing.assert_allclose(y, ref, rtol=1e-14, atol=1e-300)


def test_rmsnorm_unit_rms():
    rng = np.random.default_rng(4)
    x = rng.standard_normal(128) * 3.0
    y = oracle.rmsnorm(x, np.ones(128), 0.0)
    assert abs(math.sqrt(np.mean(y * y)) - 1.0) < 1e-14


def test_rope_identity_at_zero_and_pair_norms():
    rng = np.random.default_rng(5)
    x = rng.standard_normal(128)
    np.testing.assert_array_equal(oracle.rope(x, 0), x)
    for p in (1, 77, 262143):
        y = oracle.rope(x, p)
        np.testing.assert_allclose(y[:64] ** 2 + y[64:] ** 2, x[:64] ** 2 + x[64:] ** 2,
                                   rtol=1e-13)


def test_rope_matches_complex_rotation():
    rng = np.random.default_rng(6)
    x = rng.standard_normal(128)
    for p in (3, 4097, 262143):
        y = oracle.rope(x, p, 10000.0)
        inv = 10000.0 ** (-np.arange(64) / 64.0)
        z = (x[:64] + 1j * x[64:]) * np.exp(1j * p * inv)
        np.testing.assert_allclose(y, np.concatenate([z.real, z.imag]), rtol=0, atol=1e-9)
    # channel 0 has inverse frequency 1: a quarter turn at pos = pi/2 is not
    # integral, so check the first channel's angle directly at pos = 1
    e0 = np.zeros(128); e0[0] = 1.0
    y = oracle.rope(e0, 1)
    assert abs(y[0] - math.cos(1.0)) < 1e-15 and abs(y[64] - math.sin(1.0)) < 1e-15


def test_relative_position_property():
    """Shifting every position by a constant leaves attention unchanged."""
    w = W.make_small(30, seed=7, window=9, use_rope=True)
    out0, lse0 = run(w)
    w.pos_ids = w.pos_ids + 1000
    out1, lse1 = run(w)
    np.testing.assert_allclose(out1, out0, rtol=0, atol=1e-9)
    np.testing.assert_allclose(lse1, lse0, rtol=0, atol=1e-9)


# ---------------------------------------------------------------- sink pins

def test_large_sink_takes_all_mass():
    w = W.make_small(16, seed=8, sinks=1e4)
    out, lse = run(w)
    assert np.all(out == 0.0)
    assert np.all(lse == 1e4)


def test_probability_mass_sums_to_one():
    """With every value row equal to ones, out = sum_j p_ij, so
    out + exp(sink - lse) = 1 (the sink takes the remaining mass)."""
    w = W.make_small(50, seed=9, window=13, use_rope=True)
    w.v = np.full_like(w.v, 0x3F80)          # BF16 1.0
    out, lse = run(w)
    tot = out[:, :, 0] + np.exp(w.sinks[None, :].astype(np.float64) - lse)
    np.testing.assert_allclose(tot, 1.0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(out, out[:, :, :1].repeat(128, axis=2), rtol=0, atol=1e-15)


def test_sink_is_unscaled_natural_logit():
    """With q = 0 every logit is 0, so Z = e^sink + n and lse = ln(e^sink + n)
    exactly; a sink scaled by 1/sqrt(128) or taken in log2 units would fail."""
    w = W.make_small(5, seed=10, sinks=2.5)
    w.q = np.zeros_like(w.q)
    _, lse = run(w)
    n = np.arange(1, 6)[:, None]
    np.testing.assert_allclose(lse, np.log(np.exp(2.5) + n) * np.ones((1, 32)), rtol=0, atol=1e-14)


# ---------------------------------------------------------------- mask pins

def test_window_counts_current_token():
    """Flint model page, "Model Architecture": the window holds the current
    token and the 512 before it.  With q = 0 all logits are 0 and
    exp(lse) - exp(sink) is the number of visible keys."""
    facts = json.load(open(os.path.join(GOLDEN, "flint_attention_facts.json")))
    Wn = facts["sliding_window"]["value"]
    assert Wn == 513 == W.WINDOW
    w = W.make_small(600, seed=14, window=Wn, use_rope=True, sinks=0.0)
    w.q = np.zeros_like(w.q)
    rows = np.array([0, 1, 511, 512, 513, 514, 599])
    _, lse = run(w, rows=rows)
    n = np.exp(lse[:, 0]) - 1.0
    np.testing.assert_allclose(n, np.minimum(rows + 1, 513), rtol=1e-12)


def test_window_ge_T_equals_full():
    w = W.make_small(70, seed=15, window=0, use_rope=True)
    out0, lse0 = run(w)
    w.window = 70
    out1, lse1 = run(w)
    w.window = 1000
    out2, lse2 = run(w)
    np.testing.assert_array_equal(out0, out1)
    np.testing.assert_array_equal(out0, out2)
    np.testing.assert_array_equal(lse0, lse2)


def test_window_one_is_self_only():
    """Window 1: each query sees itself only: out = v_i * e^s_ii / (e^sink + e^s_ii)."""
    w = W.make_small(12, seed=16, window=1)
    out, lse = run(w)
    v = f64(w.v)
    for h in (0, 9, 31):
        p = 1.0 - np.exp(w.sinks[h] - lse[:, h])
        np.testing.assert_allclose(out[:, h, :], v[:, h // 8, :] * p[:, None], rtol=1e-12, atol=1e-14)


def test_packed_documents_equal_separate_runs():
    lens = [5, 17, 1, 30]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    w = W.make_small(T, seed=17, window=9, use_rope=True, cu_seqlens=cu)
    out, lse = run(w)
    for d in range(len(lens)):
        a, b = int(cu[d]), int(cu[d + 1])
        sub = W.Workload("doc", w.q[a:b], w.k[a:b], w.v[a:b], w.q_norm_w, w.k_norm_w,
                         w.sinks, pos_ids=w.pos_ids[a:b], cu_seqlens=None, pad_mask=None,
                         window=9, use_rope=True)
        o2, l2 = run(sub)
        np.testing.assert_allclose(out[a:b], o2, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[a:b], l2, rtol=0, atol=1e-13)
    # default positions equal document-local indices
    w.pos_ids = None
    o3, l3 = run(w)
    np.testing.assert_array_equal(o3, out)


def test_thd_tail_and_padmask_rows_are_padding():
    B, S = 3, 20
    lens = [20, 13, 0]
    mask = np.zeros((B, S), np.uint8)
    for b, L in enumerate(lens):
        mask[b, :L] = 1
    w = W.make_small(B * S, seed=18, window=0, use_rope=True, pad_mask=mask)
    out, lse = run(w)
    doc = oracle.doc_ids(B * S, pad_mask=mask)
    pad = doc < 0
    assert np.all(out[pad] == 0.0)
    np.testing.assert_array_equal(lse[pad], np.broadcast_to(w.sinks, (pad.sum(), 32)))
    # valid rows equal a THD packing of the same valid tokens
    keep = np.nonzero(~pad)[0]
    cu = np.concatenate([[0], np.cumsum([L for L in lens])]).astype(np.int32)
    thd = W.Workload("thd", w.q[keep], w.k[keep], w.v[keep], w.q_norm_w, w.k_norm_w, w.sinks,
                     pos_ids=w.pos_ids[keep], cu_seqlens=cu, pad_mask=None, window=0,
                     use_rope=True)
    o2, l2 = run(thd)
    np.testing.assert_allclose(out[keep], o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse[keep], l2, rtol=0, atol=1e-13)
    # THD tokens beyond cu[-1] are padding too
    cu2 = np.array([0, 7, 11], np.int32)
    w2 = W.make_small(16, seed=19, cu_seqlens=cu2)
    o4, l4 = run(w2)
    assert np.all(o4[11:] == 0.0)
    np.testing.assert_array_equal(l4[11:], np.broadcast_to(w2.sinks, (5, 32)))


# ---------------------------------------------------------------- closed form

def test_hand_computed_four_tokens():
    """T=4, one document, weights 1, q and k one-hot in channel 0, v_j = e_j.
    After the norm the only nonzero channel is a = 1/sqrt(1/128 + eps); NeoX
    RoPE with inverse frequency 1 on channel 0 turns it by p_i, so
    s_ij = a^2 cos(p_i - p_j) / sqrt(128) and out[i, j] = e^s_ij / Z_i."""
    T = 4
    q = np.zeros((T, 32, 128), np.float64); q[:, :, 0] = 1.0
    k = np.zeros((T, 4, 128), np.float64); k[:, :, 0] = 1.0
    v = np.zeros((T, 4, 128), np.float64)
    for j in range(T):
        v[j, :, j] = 1.0
    pos = np.array([0, 1, 2, 3], np.int32)
    sinks = np.linspace(-1.0, 1.0, 32)
    out, lse = oracle.attn_fwd(q, k, v, np.ones(128), np.ones(128), sinks, pos_ids=pos,
                               window=0, use_rope=True)
    a2 = 1.0 / (1.0 / 128 + 1e-6)
    for i in range(T):
        for h in range(32):
            s = [a2 * math.cos(i - j) / math.sqrt(128.0) for j in range(i + 1)]
            Z = math.exp(sinks[h]) + sum(math.exp(x) for x in s)
            assert abs(lse[i, h] - math.log(Z)) < 1e-12
            for j in range(T):
                exp_v = math.exp(s[j]) / Z if j <= i else 0.0
                assert abs(out[i, h, j] - exp_v) < 1e-12
    # window 2 drops key i-2
    out2, lse2 = oracle.attn_fwd(q, k, v, np.ones(128), np.ones(128), sinks, pos_ids=pos,
                                 window=2, use_rope=True)
    assert out2[3, 0, 1] == 0.0 and out2[3, 0, 2] > 0.0


def test_default_positions_within_segment():
    w = W.make_small(24, seed=20, window=0, use_rope=True)
    out0, _ = run(w)
    w.pos_ids = None
    out1, _ = run(w)
    np.testing.assert_array_equal(out0, out1)


# ---------------------------------------------------------------- roundings

def test_round_bf16_matches_bit_rounding():
    rng = np.random.default_rng(21)
    x = (rng.standard_normal(2000) * np.exp(rng.uniform(-20, 20, 2000))).astype(np.float32)
    bits = W.bf16_bits(x)
    ref = W.bf16_to_f64(bits)
    got = np.array([oracle.round_bf16(float(t)) for t in x])
    np.testing.assert_array_equal(got, ref)


def test_round_fp16_matches_numpy():
    rng = np.random.default_rng(22)
    x = rng.standard_normal(2000) * np.exp(rng.uniform(-12, 10, 2000))
    ref = x.astype(np.float16).astype(np.float64)
    got = np.array([oracle.round_fp16(float(t)) for t in x])
    np.testing.assert_array_equal(got, ref)


def test_golden_facts_file_is_cited():
    facts = json.load(open(os.path.join(GOLDEN, "flint_attention_facts.json")))
    for key, item in facts.items():
        assert "source" in item and item["source"], key
    assert facts["num_attention_heads"]["value"] == W.HQ
    assert facts["num_key_value_heads"]["value"] == W.HKV
    assert facts["head_dim"]["value"] == W.D
    assert facts["rms_norm_eps"]["value"] == W.EPS
