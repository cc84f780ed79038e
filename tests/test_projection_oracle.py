"""Pins of the attention-layer oracle (oracle/projection.py): projections in
front of the attention core and o_proj behind it.  CPU only.

Each pin is something the layer must satisfy whatever the attention core
does: closed forms for one and two tokens, the scale invariance of the
per-head RMSNorm, linearity in the value and output weights, and the
symmetries of the head layout (query heads within a KV group, KV groups with
their query heads).
"""
import numpy as np
import pytest

from oracle import projection as OP

HID = 64                      # a small hidden size; the oracle is generic in it


def _weights(seed, scale=0.2):
    rng = np.random.default_rng(seed)
    return dict(w_q=rng.standard_normal((4096, HID)) * scale,
                w_k=rng.standard_normal((512, HID)) * scale,
                w_v=rng.standard_normal((512, HID)) * scale,
                w_o=rng.standard_normal((HID, 4096)) * scale / 8,
                q_norm_w=1 + 0.1 * rng.standard_normal(128),
                k_norm_w=1 + 0.1 * rng.standard_normal(128),
                sinks=rng.standard_normal(32))


def _hidden(T, seed):
    return np.random.default_rng(seed).standard_normal((T, HID))


def _layer(h, p, **kw):
    return OP.attn_layer(h, p["w_q"], p["w_k"], p["w_v"], p["w_o"], p["q_norm_w"], p["k_norm_w"],
                         p["sinks"], **kw)[0]


def test_single_token_without_sink_is_value_then_output_projection():
    """One token, sink = -inf: every head's attention output is its KV head's
    value, so y = sum_h W_o[:, 128h:128h+128] W_v[128g(h):128g(h)+128] h."""
    p = _weights(1)
    p["sinks"] = np.full(32, -np.inf)
    h = _hidden(1, 2)
    y = _layer(h, p, use_rope=True, pos_ids=np.array([5], np.int32))
    want = np.zeros(HID)
    for hq in range(32):
        g = hq // 8
        v_g = p["w_v"][128 * g:128 * g + 128] @ h[0]
        want += p["w_o"][:, 128 * hq:128 * hq + 128] @ v_g
    np.testing.assert_allclose(y[0], want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("rope", [False, True])
def test_two_tokens_closed_form(rope):
    """Two tokens, full causal, sink = -inf: row 1 mixes the two values with
    the logistic weight of the logit difference.  The logits are built here
    from plain numpy norms of the projected rows and, with RoPE, a rotation
    of channel i against i + 64 by angle p * 10000^(-i/64) (positions 3, 11)."""
    p = _weights(3)
    p["sinks"] = np.full(32, -np.inf)
    h = _hidden(2, 4)
    pos = np.array([3, 11], np.int32)
    y = _layer(h, p, use_rope=rope, pos_ids=pos if rope else None)

    def norm(x, w, t):
        n = x / np.sqrt(np.mean(x * x) + 1e-6) * w
        if not rope:
            return n
        ang = pos[t] * 10000.0 ** (-np.arange(64) / 64.0)
        c, s_ = np.cos(ang), np.sin(ang)
        return np.concatenate([n[:64] * c - n[64:] * s_, n[64:] * c + n[:64] * s_])
    want = np.zeros(HID)
    for hq in range(32):
        g = hq // 8
        qn = norm(p["w_q"][128 * hq:128 * hq + 128] @ h[1], p["q_norm_w"], 1)
        k0 = norm(p["w_k"][128 * g:128 * g + 128] @ h[0], p["k_norm_w"], 0)
        k1 = norm(p["w_k"][128 * g:128 * g + 128] @ h[1], p["k_norm_w"], 1)
        d = (qn @ k1 - qn @ k0) / np.sqrt(128)
        w1 = 1.0 / (1.0 + np.exp(-d))
        v0 = p["w_v"][128 * g:128 * g + 128] @ h[0]
        v1 = p["w_v"][128 * g:128 * g + 128] @ h[1]
        want += p["w_o"][:, 128 * hq:128 * hq + 128] @ (w1 * v1 + (1 - w1) * v0)
    np.testing.assert_allclose(y[1], want, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("name", ["w_q", "w_k"])
def test_norm_makes_the_layer_invariant_to_query_and_key_weight_scale(name):
    """With eps = 0 the per-head RMSNorm removes any positive scale of the
    projected queries or keys."""
    p = _weights(5)
    h = _hidden(12, 6)
    kw = dict(window=5, use_rope=True, pos_ids=np.arange(12, dtype=np.int32), eps=0.0)
    y = _layer(h, p, **kw)
    p2 = dict(p)
    p2[name] = p[name] * 7.25
    np.testing.assert_allclose(_layer(h, p2, **kw), y, rtol=1e-10, atol=1e-12)


def test_linear_in_value_and_output_weights():
    p = _weights(7)
    h = _hidden(10, 8)
    y = _layer(h, p, window=0)
    p2 = dict(p, w_v=p["w_v"] * -2.5)
    np.testing.assert_allclose(_layer(h, p2, window=0), -2.5 * y, rtol=1e-11, atol=1e-12)
    extra = np.random.default_rng(9).standard_normal(p["w_o"].shape) * 0.01
    p3 = dict(p, w_o=p["w_o"] + extra)
    p4 = dict(p, w_o=extra)
    np.testing.assert_allclose(_layer(h, p3, window=0), y + _layer(h, p4, window=0), rtol=1e-11,
                               atol=1e-12)


def _blocks(w, perm, axis):
    """Reorder 128-wide blocks of w along `axis` by perm."""
    parts = np.split(w, len(perm), axis=axis)
    return np.concatenate([parts[i] for i in perm], axis=axis)


def test_query_heads_within_a_group_are_interchangeable():
    """Permuting the query heads of each KV group (their W_q rows, sinks and
    W_o columns together) leaves the layer unchanged."""
    p = _weights(11)
    h = _hidden(9, 12)
    y = _layer(h, p, window=4, use_rope=True, pos_ids=np.arange(9, dtype=np.int32))
    rng = np.random.default_rng(13)
    perm = np.concatenate([8 * g + rng.permutation(8) for g in range(4)])
    p2 = dict(p, w_q=_blocks(p["w_q"], perm, 0), w_o=_blocks(p["w_o"], perm, 1),
              sinks=p["sinks"][perm])
    np.testing.assert_allclose(_layer(h, p2, window=4, use_rope=True, pos_ids=np.arange(9, dtype=np.int32)),
                               y, rtol=1e-11, atol=1e-12)


def test_kv_groups_move_with_their_query_heads():
    """Permuting the KV heads (W_k, W_v rows) together with their groups of 8
    query heads leaves the layer unchanged; moving the KV heads alone does
    not."""
    p = _weights(17)
    h = _hidden(8, 18)
    y = _layer(h, p, window=0)
    kv_perm = [2, 0, 3, 1]
    q_perm = np.concatenate([np.arange(8 * g, 8 * g + 8) for g in kv_perm])
    p2 = dict(p, w_k=_blocks(p["w_k"], kv_perm, 0), w_v=_blocks(p["w_v"], kv_perm, 0),
              w_q=_blocks(p["w_q"], q_perm, 0), w_o=_blocks(p["w_o"], q_perm, 1), sinks=p["sinks"][q_perm])
    np.testing.assert_allclose(_layer(h, p2, window=0), y, rtol=1e-11, atol=1e-12)
    p3 = dict(p, w_k=_blocks(p["w_k"], kv_perm, 0), w_v=_blocks(p["w_v"], kv_perm, 0))
    assert np.max(np.abs(_layer(h, p3, window=0) - y)) > 1e-3
