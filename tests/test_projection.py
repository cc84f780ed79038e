"""GPU parity of the projection GEMMs and of the whole attention layer
(flint_qkv_proj, flint_o_proj, flint_attn_layer_fwd) against FP64 references.

The layer is FlintAttention.forward on the NeMo AutoModel "flint.layers" API
page: bias-free q/k/v projections (FlintConfig attention_bias = False), the
sink-aware attention, then o_proj.  Its FP64 oracle is oracle/projection.py.

Bounds:
* A projection output is an FP32 tensor-core sum rounded once to BF16: at most
  half a BF16 ulp from the exact product (2^-8 relative at the bottom of a
  binade), plus the FP32 accumulation error, bounded here by 2^-16 times the
  sum of |x_i w_i|.
* The layer's attention runs on its own BF16 q and v and on keys taken from
  the projection's FP32 accumulator (the fused key prologue): it is compared
  with the attention oracle on exactly those inputs (the GPU's BF16 q and v,
  the exact FP64 k), under the attention's stated bounds.
* y is o_proj of the GPU's BF16 attention output: same bound as a projection.
  Against the exact FP64 composition (no intermediate rounding) the BF16
  roundings of q, v and the attention output leave a relative L2 error of a
  few 1e-3; the bound there is 1e-2.
"""
import numpy as np
import pytest

import oracle
from oracle import projection as OP
import workloads as W

pytestmark = pytest.mark.gpu

TOL = dict(max_abs=2e-2, rel_l2=5e-3, lse=1e-3)


def _dev():
    import torch
    return torch.device("cuda:0")


def _bf(x):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x)).view(torch.bfloat16).to(_dev())


def _bits(t):
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _check_gemm(got_bits, a_bits, b_bits):
    """got [M, N] BF16 against A B^T in FP64."""
    a, b = W.bf16_to_f64(a_bits), W.bf16_to_f64(b_bits)
    ref = a @ b.T
    absum = np.abs(a) @ np.abs(b).T
    got = W.bf16_to_f64(got_bits).reshape(ref.shape)
    err = np.abs(got - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -16 * absum + 1e-30
    worst = float((err / bound).max())
    assert worst <= 1.0, "worst error / bound = %.3f" % worst
    return ref


@pytest.mark.parametrize("T,hidden", [(1, 2048), (100, 2048), (300, 2048), (1000, 64), (129, 192)])
def test_qkv_proj_matches_fp64_product(T, hidden):
    import full_gqa_learned_b200 as fa
    lw = W.make_layer(T, seed=300 + T, hidden=hidden)
    q, k, v = fa.qkv_proj(_bf(lw.x), _bf(lw.w_qkv))
    got = np.concatenate([_bits(q).reshape(T, 4096), _bits(k).reshape(T, 512),
                          _bits(v).reshape(T, 512)], axis=1)
    _check_gemm(got, lw.x, lw.w_qkv)


@pytest.mark.parametrize("T,hidden", [(1, 2048), (300, 2048), (257, 64)])
def test_o_proj_matches_fp64_product(T, hidden):
    import full_gqa_learned_b200 as fa
    lw = W.make_layer(T, seed=400 + T, hidden=hidden)
    a = W.bf16_bits(np.random.default_rng(T).standard_normal((T, 4096)).astype(np.float32))
    y = fa.o_proj(_bf(a), _bf(lw.w_o))
    _check_gemm(_bits(y), a, lw.w_o)


def _layer_case(name):
    if name == "sliding_thd":
        cu = np.array([0, 120, 121, 380, 600], np.int32)
        return W.make_layer(640, seed=51, window=129, use_rope=True, cu_seqlens=cu, name=name)
    if name == "full_pad":
        mask = np.zeros((3, 200), np.uint8)
        for b, L in enumerate([200, 57, 0]):
            mask[b, :L] = 1
        return W.make_layer(600, seed=52, window=0, use_rope=True, pad_mask=mask, name=name)
    return W.make_layer(500, seed=53, window=0, use_rope=False, name=name)


@pytest.mark.parametrize("name", ["sliding_thd", "full_pad", "full"])
def test_layer_matches_the_oracle(name):
    import torch
    import full_gqa_learned_b200 as fa
    lw = _layer_case(name)
    w = lw.attn
    dev = _dev()
    kw = dict(window=w.window, use_rope=w.use_rope, rope_theta=w.rope_theta, eps=w.eps)
    for key in ("pos_ids", "cu_seqlens", "pad_mask"):
        if getattr(w, key) is not None:
            kw[key] = torch.from_numpy(getattr(w, key)).to(dev)
    qn, kn = torch.from_numpy(w.q_norm_w).to(dev), torch.from_numpy(w.k_norm_w).to(dev)
    sk = torch.from_numpy(np.asarray(w.sinks, np.float32)).to(dev)
    r = fa.attn_layer_fwd(_bf(lw.x), _bf(lw.w_qkv), _bf(lw.w_o), qn, kn, sk, **kw)
    assert fa.device_status(fa.attn_layer_fwd.last_workspace) == 0
    torch.cuda.synchronize()
    T = lw.T
    # projections
    got_qkv = np.concatenate([_bits(r["q"]).reshape(T, 4096), _bits(r["k"]).reshape(T, 512),
                              _bits(r["v"]).reshape(T, 512)], axis=1)
    exact = _check_gemm(got_qkv, lw.x, lw.w_qkv)
    # attention on the GPU's BF16 q and v and the exact keys
    q_g = W.bf16_to_f64(_bits(r["q"]))
    v_g = W.bf16_to_f64(_bits(r["v"]))
    k_x = exact[:, 4096:4608].reshape(T, 4, 128)
    ref_a, ref_l = oracle.attn_fwd(q_g, k_x, v_g, w.q_norm_w, w.k_norm_w, w.sinks, pos_ids=w.pos_ids,
                                   cu_seqlens=w.cu_seqlens, pad_mask=w.pad_mask, window=w.window,
                                   use_rope=w.use_rope, rope_theta=w.rope_theta, eps=w.eps)
    got_a = W.bf16_to_f64(_bits(r["attn_out"])).reshape(T, 32, 128)
    got_l = r["lse"].cpu().numpy().T.astype(np.float64)
    err = np.abs(got_a - ref_a).max()
    rel = np.linalg.norm(got_a - ref_a) / np.linalg.norm(ref_a)
    fin = np.isfinite(ref_l)
    lerr = np.abs(got_l[fin] - ref_l[fin]).max()
    print("%s attention: max_abs %.3e rel_l2 %.3e lse %.3e" % (name, err, rel, lerr))
    # derived edge bound for LSE as in test_parity (rows of one or few keys)
    assert err <= TOL["max_abs"] and rel <= TOL["rel_l2"] and lerr <= 2e-3
    doc = oracle.doc_ids(T, w.cu_seqlens, w.pad_mask)
    pad = np.nonzero(doc < 0)[0]
    assert np.all(_bits(r["attn_out"])[pad] == 0)
    # o_proj of the GPU's attention output
    _check_gemm(_bits(r["y"]), _bits(r["attn_out"]), lw.w_o)
    # the whole layer against the exact FP64 composition
    y_ref, l_ref = OP.attn_layer(W.bf16_to_f64(lw.x), W.bf16_to_f64(lw.w_qkv[:4096]),
                                 W.bf16_to_f64(lw.w_qkv[4096:4608]), W.bf16_to_f64(lw.w_qkv[4608:]),
                                 W.bf16_to_f64(lw.w_o), w.q_norm_w, w.k_norm_w, w.sinks,
                                 pos_ids=w.pos_ids, cu_seqlens=w.cu_seqlens, pad_mask=w.pad_mask,
                                 window=w.window, use_rope=w.use_rope, rope_theta=w.rope_theta,
                                 eps=w.eps)
    y = W.bf16_to_f64(_bits(r["y"])).reshape(y_ref.shape)
    rel_y = np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref)
    print("%s layer: rel_l2 %.3e" % (name, rel_y))
    assert rel_y <= 1e-2


def test_layer_empty_input_is_a_noop():
    import torch
    import full_gqa_learned_b200 as fa
    dev = _dev()
    x = torch.zeros((0, 2048), dtype=torch.bfloat16, device=dev)
    wq = torch.zeros((5120, 2048), dtype=torch.bfloat16, device=dev)
    wo = torch.zeros((2048, 4096), dtype=torch.bfloat16, device=dev)
    w1 = torch.ones(128, dtype=torch.float32, device=dev)
    s = torch.zeros(32, dtype=torch.float32, device=dev)
    r = fa.attn_layer_fwd(x, wq, wo, w1, w1, s, window=0, use_rope=False)
    assert r["y"].shape == (0, 2048)
