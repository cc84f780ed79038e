"""Pins of the decode-step oracle (oracle/decode.py) against the independent
prefill oracle and closed forms.  CPU only."""
import numpy as np
import pytest

import oracle
import workloads as W
from oracle import decode as OD


def _cache_from_prefill(w, L, window, use_rope, cap, fill=0.0):
    """Cache of capacity cap holding the exact normalised, rotated keys and the
    values of positions lo..L-1 at slots j mod cap; other slots hold `fill`."""
    kc = np.full((1, 4, cap, 128), fill)
    vc = np.full((1, 4, cap, 128), fill)
    kf, vf = oracle._f64(w.k), oracle._f64(w.v)
    lo = max(0, L - window + 1) if window > 0 else 0
    for j in range(lo, L):
        for g in range(4):
            kc[0, g, j % cap] = OD.normalise(kf[j, g], w.k_norm_w, j, use_rope, 1e4, 1e-6)
        vc[0, :, j % cap] = vf[j]
    return kc, vc


@pytest.mark.parametrize("L,window,rope,cap", [(0, 0, False, 4), (37, 0, False, 40), (37, 0, True, 64),
                                               (60, 17, True, 17), (60, 17, True, 23), (16, 17, True, 17),
                                               (700, 513, True, 513)])
def test_decode_equals_last_row_of_prefill(L, window, rope, cap):
    """Decoding token L against the cache of tokens < L is row L of the
    prefill over tokens 0..L (same positions, window, sink)."""
    w = W.make_small(L + 1, seed=30 + L, window=window, use_rope=rope)
    ref_o, ref_l = oracle.attn_fwd(w.q, w.k, w.v, w.q_norm_w, w.k_norm_w, w.sinks,
                                   pos_ids=w.pos_ids, window=window, use_rope=rope, rows=[L])
    kc, vc = _cache_from_prefill(w, L, window, rope, cap, fill=1e6)   # slots outside the window are poison
    out, lse, k_new = OD.decode_step(w.q[L:L + 1], w.k[L:L + 1], w.v[L:L + 1], kc, vc, [L],
                                     w.q_norm_w, w.k_norm_w, w.sinks, window=window, use_rope=rope)
    np.testing.assert_allclose(out[0], ref_o[0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[:, 0], ref_l[0], rtol=0, atol=1e-12)
    kf = oracle._f64(w.k)
    for g in range(4):
        np.testing.assert_allclose(k_new[0, g], OD.normalise(kf[L, g], w.k_norm_w, L, rope, 1e4, 1e-6),
                                   rtol=0, atol=0)


def test_single_key_closed_form():
    """Empty cache and sink = -inf: the only key is the token itself, so
    out = v and lse = q~ . k~ / sqrt(128)."""
    w = W.make_small(1, seed=40, window=0, use_rope=True, sinks=-np.inf)
    kc = np.zeros((1, 4, 2, 128))
    out, lse, k_new = OD.decode_step(w.q, w.k, w.v, kc, kc, [0], w.q_norm_w, w.k_norm_w, w.sinks,
                                     window=513, use_rope=True)
    q, v = oracle._f64(w.q), oracle._f64(w.v)
    for h in range(32):
        g = h // 8
        np.testing.assert_array_equal(out[0, h], v[0, g])
        qt = OD.normalise(q[0, h], w.q_norm_w, 0, True, 1e4, 1e-6)
        assert abs(lse[h, 0] - qt @ k_new[0, g] / np.sqrt(128)) < 1e-12


def test_infinite_sinks():
    w = W.make_small(1, seed=41, window=0, use_rope=False, sinks=np.inf)
    kc = np.zeros((1, 4, 1, 128))
    out, lse, _ = OD.decode_step(w.q, w.k, w.v, kc, kc, [0], w.q_norm_w, w.k_norm_w, w.sinks,
                                 window=0, use_rope=False)
    assert np.all(out == 0) and np.all(lse == np.inf)


def test_batch_is_independent_sequences():
    """A batch of sequences with different lengths equals one call per sequence."""
    d = W.make_decode(3, cap=40, seed=42, window=33, use_rope=True, max_len=120)
    out, lse, k_new = OD.decode_step(d.q, d.k, d.v, d.k_cache, d.v_cache, d.cache_len, d.q_norm_w,
                                     d.k_norm_w, d.sinks, window=33, use_rope=True)
    for b in range(3):
        o1, l1, k1 = OD.decode_step(d.q[b:b + 1], d.k[b:b + 1], d.v[b:b + 1], d.k_cache[b:b + 1],
                                    d.v_cache[b:b + 1], d.cache_len[b:b + 1], d.q_norm_w, d.k_norm_w,
                                    d.sinks, window=33, use_rope=True)
        np.testing.assert_array_equal(out[b], o1[0])
        np.testing.assert_array_equal(lse[:, b], l1[:, 0])
        np.testing.assert_array_equal(k_new[b], k1[0])


def test_window_larger_than_cache_is_rejected():
    d = W.make_decode(1, cap=8, seed=43, window=33, use_rope=False, max_len=100, min_len=50)
    with pytest.raises(ValueError):
        OD.decode_step(d.q, d.k, d.v, d.k_cache, d.v_cache, d.cache_len, d.q_norm_w, d.k_norm_w,
                       d.sinks, window=33, use_rope=False)
