"""Parity of the CUDA backward (flint_attn_bwd) with the FP64 backward oracle.

The GPU path is the one a training step runs: the library's forward produces
out and lse, and the backward takes them with a BF16 upstream gradient.  The
oracle computes the exact gradient from the same inputs (its own forward).

The backward takes the forward's out and computes D_i = dO_i . out_i from it
(include/flint_attn.h, flint_attn_bwd), so the reference is the gradient
formula evaluated at the same stored output (the oracle's out_given); the
forward's own error is covered by the forward's parity tests.  Against that
reference, from the arithmetic:
* each probability is exp(s - lse) with the forward's FP32 lse, whose error
  is at most the forward's LSE bound (1e-3) and in practice the FP16-operand
  floor (~5e-4); that scales a row's probabilities by at most 1e-3;
* the products run on the tensor cores with q~, k~ and dS in FP16 and P in
  BF16 (an FP64 emulation of those roundings: dv 1.7e-3, dq and dk 7e-4
  relative L2), accumulating in FP32.
So dq, dk, dv: relative L2 <= 5e-3 and max |err| <= 1e-2 max |ref|.
dsinks_h = -sum_i exp(sink_h - lse_i) D_i sums signed terms, so its bound is
relative to the sum of absolute terms A_h = sum_i exp(sink_h - lse_i)
sum_c |dO_ic out_ic|: |err| <= 1e-2 A_h.  The norm weights' gradients sum
T x heads signed row terms: relative L2 <= 1e-2.

End to end, against the exact gradient (exact out in D), the forward's BF16
output adds its rounding to D; where a row's D nearly cancels dO . v (a row
dominated by one key) that error is amplified, so the bound there is 1e-2.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from oracle import backward as OB
from test_parity import to_device

pytestmark = pytest.mark.gpu


def _torch():
    import torch
    return torch


def _run(w, dO_bits):
    """Library forward then backward on the GPU; returns the gradients (numpy)."""
    torch = _torch()
    import full_gqa_learned_b200 as fa
    dev = torch.device("cuda:0")
    t = to_device(w)
    q, k, v = t["q"], t["k"], t["v"]
    wq, wk, sk = t["q_norm_w"], t["k_norm_w"], t["sinks"]
    kw = dict(pos_ids=t["pos_ids"], cu_seqlens=t["cu_seqlens"], pad_mask=t["pad_mask"],
              window=w.window, use_rope=w.use_rope, rope_theta=w.rope_theta, eps=w.eps)
    out, lse = fa.attn_fwd(q, k, v, wq, wk, sk, **kw)
    assert fa.device_status(fa.attn_fwd.last_workspace) == 0
    dO = torch.from_numpy(np.ascontiguousarray(dO_bits)).view(torch.bfloat16).to(dev).reshape(w.T, 4096)
    g = fa.attn_bwd(q, k, v, wq, wk, sk, out, lse, dO, **kw)
    assert fa.device_status(fa.attn_bwd.last_workspace) == 0
    torch.cuda.synchronize()
    got = {n: x.cpu().numpy().astype(np.float64) for n, x in g.items()}
    got["fwd_out"] = out.float().cpu().numpy().astype(np.float64).reshape(w.T, 32, 128)
    return got, (q, k, v, wq, wk, sk, out, lse, dO, kw)


def _dout_bits(T, seed):
    return W.bf16_bits(np.random.default_rng(seed).standard_normal((T, 32, 128)).astype(np.float32))


def _compare(w, dO_bits, got):
    exact = OB.attn_bwd_workload(w, oracle._f64(dO_bits))
    for key in ("dq", "dk", "dv"):
        e = got[key] - exact[key]
        assert np.linalg.norm(e) <= 1e-2 * np.linalg.norm(exact[key]) + 1e-30, \
            ("end to end", key, np.linalg.norm(e) / np.linalg.norm(exact[key]))
    ref = OB.attn_bwd_workload(w, oracle._f64(dO_bits), out_given=got["fwd_out"])
    for key in ("dq", "dk", "dv"):
        e = got[key] - ref[key]
        scale = np.abs(ref[key]).max()
        assert np.linalg.norm(e) <= 5e-3 * np.linalg.norm(ref[key]) + 1e-30, (key, np.linalg.norm(e) / np.linalg.norm(ref[key]))
        assert np.abs(e).max() <= 1e-2 * scale + 1e-30, (key, np.abs(e).max(), scale)
    for key in ("dq_norm_w", "dk_norm_w"):
        e = got[key] - ref[key]
        assert np.linalg.norm(e) <= 1e-2 * np.linalg.norm(ref[key]) + 1e-30, (key, np.linalg.norm(e), np.linalg.norm(ref[key]))
    dO = oracle._f64(dO_bits).reshape(w.T, 32, 128)
    sk = np.asarray(w.sinks, np.float64)
    with np.errstate(invalid="ignore", over="ignore"):
        share = np.where(np.isfinite(sk)[None, :], np.exp(sk[None, :] - ref["lse"]), 0.0)
    A = np.sum(share * np.sum(np.abs(dO * ref["out"]), axis=2), axis=0)
    e = np.abs(got["dsinks"] - ref["dsinks"])
    assert np.all(e <= 1e-2 * A + 1e-6), (e, A)
    # padded tokens: exactly zero rows
    doc = oracle.doc_ids(w.T, w.cu_seqlens, w.pad_mask)
    for key in ("dq", "dk", "dv"):
        assert np.all(got[key][doc < 0] == 0.0), key
    return ref


CASES = {
    "full_t300": lambda: W.make_small(300, seed=81, window=0, use_rope=False),
    "sliding_thd_pad_t700": lambda: W.make_small(700, seed=82, window=513, use_rope=True,
                                                 cu_seqlens=[0, 250, 600]),
    "padmask_2x160": lambda: W.make_small(320, seed=83, window=513, use_rope=True,
                                          pad_mask=np.concatenate([np.ones((1, 160), np.uint8),
                                                                   (np.arange(160) < 97).astype(np.uint8)[None]])),
    "window_1": lambda: W.make_small(40, seed=84, window=1, use_rope=True),
    "window_7_docs": lambda: W.make_small(90, seed=85, window=7, use_rope=True, cu_seqlens=[0, 1, 30, 31, 77]),
    "single_token": lambda: W.make_small(1, seed=86, window=513, use_rope=True),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_backward_matches_oracle(name):
    w = CASES[name]()
    dO = _dout_bits(w.T, 90)
    got, _ = _run(w, dO)
    _compare(w, dO, got)


def test_infinite_and_extreme_sinks():
    """Heads with sink = +inf (out = 0: no gradient), -inf (no sink column)
    and large finite sinks."""
    w = W.make_small(64, seed=87, window=0, use_rope=False)
    s = np.asarray(w.sinks, np.float32).copy()
    s[0], s[9], s[17], s[30] = np.inf, -np.inf, 20.0, -20.0
    w.sinks = s
    dO = _dout_bits(64, 91)
    got, _ = _run(w, dO)
    _compare(w, dO, got)
    assert np.all(got["dq"][:, 0] == 0.0) and got["dsinks"][0] == 0.0 and got["dsinks"][9] == 0.0


@pytest.mark.parametrize("T,window", [(700, 513), (2000, 0)])
def test_repeated_calls_are_bitwise_identical(T, window):
    """T = 700 gives every warp several work items, so one CTA meets the same
    head more than once: the per-CTA sums must still be in a fixed order.  On
    both sequences the dk/dv kernel cuts each key tile's queries into pieces
    that different CTAs run (10 pieces of 13 query tiles on the causal
    T = 2000): their sum must be taken in piece order."""
    torch = _torch()
    import full_gqa_learned_b200 as fa
    w = W.make_small(T, seed=88, window=window, use_rope=window > 0)
    got, (q, k, v, wq, wk, sk, out, lse, dO, kw) = _run(w, _dout_bits(T, 92))
    g2 = fa.attn_bwd(q, k, v, wq, wk, sk, out, lse, dO, **kw)
    torch.cuda.synchronize()
    for n, x in g2.items():
        assert np.array_equal(x.cpu().numpy().astype(np.float64), got[n]), n


def test_ill_formed_boundaries_set_the_device_status():
    """A decreasing cu_seqlens and a non-trailing mask are reported through
    the workspace status (every access stays inside the buffers: each token's
    document bounds are checked against [0, T] before use)."""
    torch = _torch()
    import full_gqa_learned_b200 as fa
    dev = torch.device("cuda:0")
    T = 64
    z = lambda *sh, dt=torch.bfloat16: torch.zeros(sh, dtype=dt, device=dev)
    q, k, v = z(T, 32, 128), z(T, 4, 128), z(T, 4, 128)
    wq, wk = torch.ones(128, device=dev), torch.ones(128, device=dev)
    sk = torch.zeros(32, device=dev)
    out, lse, dO = z(T, 4096), z(32, T, dt=torch.float32), z(T, 4096)
    cu = torch.tensor([0, 50, 30, 64], dtype=torch.int32, device=dev)
    fa.attn_bwd(q, k, v, wq, wk, sk, out, lse, dO, cu_seqlens=cu, window=0, use_rope=False)
    assert fa.device_status(fa.attn_bwd.last_workspace) == 1
    m = torch.tensor([[1] * 30 + [0] * 2, [1, 0, 1] + [0] * 29], dtype=torch.uint8, device=dev)
    fa.attn_bwd(q, k, v, wq, wk, sk, out, lse, dO, pad_mask=m, window=0, use_rope=False)
    assert fa.device_status(fa.attn_bwd.last_workspace) == 2


def test_empty_input_zeroes_the_small_gradients():
    torch = _torch()
    import full_gqa_learned_b200 as fa
    dev = torch.device("cuda:0")
    e = lambda *sh, dt=torch.bfloat16: torch.empty(sh, dtype=dt, device=dev)
    grads = {"dq": e(0, 32, 128, dt=torch.float32), "dk": e(0, 4, 128, dt=torch.float32),
             "dv": e(0, 4, 128, dt=torch.float32), "dq_norm_w": torch.full((128,), 7.0, device=dev),
             "dk_norm_w": torch.full((128,), 7.0, device=dev), "dsinks": torch.full((32,), 7.0, device=dev)}
    fa.attn_bwd(e(0, 32, 128), e(0, 4, 128), e(0, 4, 128), torch.ones(128, device=dev),
                torch.ones(128, device=dev), torch.zeros(32, device=dev), e(0, 4096),
                e(32, 0, dt=torch.float32), e(0, 4096), grads=grads)
    torch.cuda.synchronize()
    for n in ("dq_norm_w", "dk_norm_w", "dsinks"):
        assert torch.all(grads[n] == 0).item(), n
