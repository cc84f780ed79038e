"""GPU parity of the decode step (flint_attn_decode through the C ABI) with the
FP64 decode oracle on the same seeded inputs.

Tolerances are those of the attention forward (output max abs 2e-2, relative
L2 5e-3, LSE 1e-3); the decode path computes in FP32 from exact BF16 inputs,
so its error is essentially the BF16 rounding of the output.  The new token's
key is written to the cache rounded to BF16 from an FP32 value; it may differ
from the oracle's FP64 value by the BF16 rounding plus the FP32 error of the
rotation (about 1e-6 absolute at positions up to 2^18)."""
import numpy as np
import pytest

import workloads as W
from oracle import decode as OD

pytestmark = pytest.mark.gpu

TOL = dict(max_abs=2e-2, rel_l2=5e-3, lse=1e-3)


def to_dev(d):
    import torch
    dev = torch.device("cuda:0")

    def bf(x):
        return torch.from_numpy(np.ascontiguousarray(x)).view(torch.bfloat16).to(dev)
    return dict(q=bf(d.q), k=bf(d.k), v=bf(d.v), k_cache=bf(d.k_cache), v_cache=bf(d.v_cache),
                cache_len=torch.from_numpy(d.cache_len).to(dev),
                q_norm_w=torch.from_numpy(d.q_norm_w).to(dev), k_norm_w=torch.from_numpy(d.k_norm_w).to(dev),
                sinks=torch.from_numpy(np.ascontiguousarray(d.sinks, np.float32)).to(dev))


def run(d, t):
    import torch
    import full_gqa_learned_b200 as fa
    out, lse = fa.attn_decode(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["sinks"],
                              t["k_cache"], t["v_cache"], t["cache_len"], window=d.window,
                              use_rope=d.use_rope, rope_theta=d.rope_theta, eps=d.eps)
    st = fa.device_status(fa.attn_decode.last_workspace)
    torch.cuda.synchronize()
    return st, out.float().cpu().numpy().reshape(d.B, 32, 128).astype(np.float64), lse.cpu().numpy()


def compare(d, got_o, got_l, ref_o, ref_l):
    err = np.abs(got_o - ref_o)
    fin = np.isfinite(ref_l)
    assert np.array_equal(np.isfinite(got_l), fin)
    assert np.all(got_l[~fin] == ref_l[~fin])
    lse_err = float(np.abs(got_l[fin] - ref_l[fin]).max()) if fin.any() else 0.0
    rel = float(np.linalg.norm(got_o - ref_o) / max(np.linalg.norm(ref_o), 1e-300))
    msg = "%s: max_abs %.3e rel_l2 %.3e lse %.3e" % (d.name, err.max(), rel, lse_err)
    print(msg)
    assert err.max() <= TOL["max_abs"], msg
    assert rel <= TOL["rel_l2"] or np.linalg.norm(ref_o) == 0, msg
    assert lse_err <= TOL["lse"], msg


def check_appended(d, t, k_new_ref):
    """The new token's key and value sit in slot cache_len mod cap."""
    kc = t["k_cache"].view(__import__("torch").int16).cpu().numpy().view(np.uint16)
    vc = t["v_cache"].view(__import__("torch").int16).cpu().numpy().view(np.uint16)
    for b in range(d.B):
        slot = int(d.cache_len[b]) % d.cap
        np.testing.assert_array_equal(vc[b, :, slot], d.v[b])
        got = W.bf16_to_f64(kc[b, :, slot])
        # BF16 rounding (half a unit, 2^-9 relative) of an FP32 value whose
        # rotation carries ~1e-6 absolute error at positions up to 2^18
        err = np.abs(got - k_new_ref[b])
        assert np.all(err <= 2.0 ** -8 * np.abs(k_new_ref[b]) + 1e-5), float(err.max())


@pytest.mark.parametrize("B,cap,window,rope,max_len", [(5, 513, 513, True, 3000), (4, 700, 0, False, 700),
                                                       (3, 300, 0, True, 300), (6, 40, 33, True, 200),
                                                       (2, 1, 1, True, 50), (3, 1000, 513, True, 5000),
                                                       (2, 2600, 0, True, 2600)])
def test_decode_matches_oracle(B, cap, window, rope, max_len):
    d = W.make_decode(B, cap, seed=50 + B + cap, window=window, use_rope=rope, max_len=max_len)
    ref_o, ref_l, k_new = OD.decode_step(d.q, d.k, d.v, d.k_cache, d.v_cache, d.cache_len, d.q_norm_w,
                                         d.k_norm_w, d.sinks, window=window, use_rope=rope)
    t = to_dev(d)
    st, o, l = run(d, t)
    assert st == 0
    compare(d, o, l, ref_o, ref_l)
    check_appended(d, t, k_new)


def test_empty_cache_and_extreme_sinks():
    for sink in (-np.inf, np.inf, 20.0, -20.0):
        d = W.make_decode(3, 16, seed=60, window=0, use_rope=True, max_len=1, sinks=sink)
        assert np.all(d.cache_len == 0)
        ref_o, ref_l, _ = OD.decode_step(d.q, d.k, d.v, d.k_cache, d.v_cache, d.cache_len, d.q_norm_w,
                                         d.k_norm_w, d.sinks, window=0, use_rope=True)
        st, o, l = run(d, to_dev(d))
        assert st == 0
        compare(d, o, l, ref_o, ref_l)
        if sink == np.inf:
            assert np.all(o == 0) and np.all(l == np.inf)


def test_consecutive_steps_stream_through_the_ring():
    """Three steps in a row on a ring of exactly the window: each step must
    see the keys the previous steps appended (read back from the device)."""
    import torch
    d = W.make_decode(4, 17, seed=61, window=17, use_rope=True, max_len=90, min_len=20)
    t = to_dev(d)
    for step in range(3):
        kc = t["k_cache"].view(torch.int16).cpu().numpy().view(np.uint16).copy()
        vc = t["v_cache"].view(torch.int16).cpu().numpy().view(np.uint16).copy()
        ref_o, ref_l, k_new = OD.decode_step(d.q, d.k, d.v, kc, vc, d.cache_len, d.q_norm_w, d.k_norm_w,
                                             d.sinks, window=17, use_rope=True)
        st, o, l = run(d, t)
        assert st == 0
        compare(d, o, l, ref_o, ref_l)
        check_appended(d, t, k_new)
        # next token of every sequence: new projections, one position later
        rng = np.random.default_rng(100 + step)
        d.q = W.bf16_bits(rng.standard_normal(d.q.shape).astype(np.float32))
        d.k = W.bf16_bits(rng.standard_normal(d.k.shape).astype(np.float32))
        d.v = W.bf16_bits(rng.standard_normal(d.v.shape).astype(np.float32))
        d.cache_len = d.cache_len + 1
        n = to_dev(d)
        for key in ("q", "k", "v", "cache_len"):
            t[key] = n[key]


def test_window_that_does_not_fit_the_cache_reports_invalid():
    import full_gqa_learned_b200 as fa
    d = W.make_decode(2, 8, seed=62, window=33, use_rope=False, max_len=60, min_len=40)
    st, _, _ = run(d, to_dev(d))
    assert st == 1


@pytest.mark.parametrize("name", sorted(W.DECODE_CONFIGS))
def test_named_decode_workloads(name):
    d = W.make_decode_named(name)
    ref_o, ref_l, k_new = OD.decode_step(d.q, d.k, d.v, d.k_cache, d.v_cache, d.cache_len, d.q_norm_w,
                                         d.k_norm_w, d.sinks, window=d.window, use_rope=d.use_rope)
    t = to_dev(d)
    st, o, l = run(d, t)
    assert st == 0
    compare(d, o, l, ref_o, ref_l)
    check_appended(d, t, k_new)


@pytest.mark.parametrize("scale", [1.0, 3.0])
def test_both_decode_paths(scale):
    """Norm weights scaled by 3 put the logit bound (16.45 max|w_q| max|w_k|)
    far above 48: the step then runs the CUDA-core split kernel instead of the
    tensor-core tile kernel; both must match the oracle.  A ring larger than
    the window holds stale positions outside it."""
    d = W.make_decode(4, 600, seed=63, window=513, use_rope=True, max_len=4000)
    d.q_norm_w = (np.asarray(d.q_norm_w, np.float32) * scale).astype(np.float32)
    d.k_norm_w = (np.asarray(d.k_norm_w, np.float32) * scale).astype(np.float32)
    bound = 16.45 * np.abs(d.q_norm_w).max() * np.abs(d.k_norm_w).max()
    assert (bound <= 48) == (scale == 1.0)
    ref_o, ref_l, k_new = OD.decode_step(d.q, d.k, d.v, d.k_cache, d.v_cache, d.cache_len, d.q_norm_w,
                                         d.k_norm_w, d.sinks, window=513, use_rope=True)
    t = to_dev(d)
    st, o, l = run(d, t)
    assert st == 0
    compare(d, o, l, ref_o, ref_l)
    check_appended(d, t, k_new)
