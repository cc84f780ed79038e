"""Host-side wiring of the differentiable entry (flint_attention): with the
two library calls replaced by CPU stand-ins built on the oracle, autograd must
hand back exactly the oracle's gradients for the upstream gradient it sees
(argument order, reshapes, dtype casts, configuration pass-through).  CPU
only; tests/test_zzz_autograd.py runs the same entry on the GPU."""
import numpy as np
import pytest
import torch

import full_gqa_learned_b200 as fa
import oracle
import workloads as W
from oracle import backward as OB


def _np(t):
    return None if t is None else t.detach().cpu().numpy()


def _cfg_np(cfg):
    return dict(pos_ids=_np(cfg["pos_ids"]), cu_seqlens=_np(cfg["cu_seqlens"]),
                pad_mask=_np(cfg["pad_mask"]), window=cfg["window"], use_rope=cfg["use_rope"],
                rope_theta=cfg["rope_theta"], eps=cfg["eps"])


def fake_fwd(q, k, v, q_norm_w, k_norm_w, sinks, **cfg):
    c = _cfg_np(cfg)
    out, lse = oracle.attn_fwd(q.float().numpy().astype(np.float64), k.float().numpy().astype(np.float64),
                               v.float().numpy().astype(np.float64), _np(q_norm_w), _np(k_norm_w),
                               _np(sinks), **c)
    T = q.shape[0]
    return (torch.from_numpy(out.reshape(T, 4096)).to(torch.bfloat16),
            torch.from_numpy(lse.T.copy()).to(torch.float32))


def fake_bwd(q, k, v, q_norm_w, k_norm_w, sinks, out, lse, dout, **cfg):
    assert dout.dtype == torch.bfloat16 and dout.is_contiguous() and tuple(dout.shape) == (q.shape[0], 4096)
    g = OB.attn_bwd(q.float().numpy().astype(np.float64), k.float().numpy().astype(np.float64),
                    v.float().numpy().astype(np.float64), _np(q_norm_w), _np(k_norm_w), _np(sinks),
                    dout.float().numpy().astype(np.float64), **_cfg_np(cfg))
    return {n: torch.from_numpy(np.ascontiguousarray(g[n])).to(torch.float32)
            for n in ("dq", "dk", "dv", "dq_norm_w", "dk_norm_w", "dsinks")}


@pytest.mark.parametrize("kind", ["sliding_thd", "full"])
def test_autograd_returns_the_oracle_gradients(kind, monkeypatch):
    monkeypatch.setattr(fa, "attn_fwd", fake_fwd)
    monkeypatch.setattr(fa, "attn_bwd", fake_bwd)
    if kind == "sliding_thd":
        w = W.make_small(24, seed=61, window=5, use_rope=True, cu_seqlens=[0, 10, 21])
    else:
        w = W.make_small(16, seed=62, window=0, use_rope=False)
    T = w.T
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).clone().requires_grad_(True)
    q, k, v = bf(w.q), bf(w.k), bf(w.v)
    wq = torch.from_numpy(w.q_norm_w.copy()).requires_grad_(True)
    wk = torch.from_numpy(w.k_norm_w.copy()).requires_grad_(True)
    sk = torch.from_numpy(np.asarray(w.sinks, np.float32).copy()).requires_grad_(True)
    kw = dict(window=w.window, use_rope=w.use_rope)
    if w.pos_ids is not None:
        kw["pos_ids"] = torch.from_numpy(w.pos_ids)
    if w.cu_seqlens is not None:
        kw["cu_seqlens"] = torch.from_numpy(w.cu_seqlens)
    out, lse = fa.flint_attention(q, k, v, wq, wk, sk, **kw)
    assert out.shape == (T, 4096) and lse.shape == (32, T) and not lse.requires_grad
    G = torch.from_numpy(np.random.default_rng(63).standard_normal((T, 4096)).astype(np.float32))
    (out.float() * G).sum().backward()
    dO = G.to(torch.bfloat16).float().numpy().astype(np.float64)       # what reaches out (bf16)
    ref = OB.attn_bwd(w.q, w.k, w.v, w.q_norm_w, w.k_norm_w, w.sinks, dO, pos_ids=w.pos_ids,
                      cu_seqlens=w.cu_seqlens, window=w.window, use_rope=w.use_rope)
    for t, n, dt in ((q, "dq", torch.bfloat16), (k, "dk", torch.bfloat16), (v, "dv", torch.bfloat16)):
        assert t.grad.dtype == dt
        want = torch.from_numpy(ref[n].astype(np.float32)).to(dt).float()
        assert torch.equal(t.grad.float(), want), n
    for t, n in ((wq, "dq_norm_w"), (wk, "dk_norm_w"), (sk, "dsinks")):
        assert t.grad.dtype == torch.float32
        assert torch.equal(t.grad, torch.from_numpy(ref[n].astype(np.float32))), n
