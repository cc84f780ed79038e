"""The differentiable entry (flint_attention) on the GPU: autograd's
gradients are bit for bit those of a direct flint_attn_bwd call on the same
forward result and upstream gradient (the backward is deterministic), and
the entry's output is the forward's.  Parity of those gradients with the
oracle is tests/test_backward.py."""
import numpy as np
import pytest

import workloads as W
from test_parity import to_device

pytestmark = pytest.mark.gpu


def test_autograd_gradients_equal_the_direct_backward():
    import torch
    import full_gqa_learned_b200 as fa
    w = W.make_small(300, seed=64, window=513, use_rope=True, cu_seqlens=[0, 120, 290])
    t = to_device(w)
    kw = dict(pos_ids=t["pos_ids"], cu_seqlens=t["cu_seqlens"], pad_mask=t["pad_mask"], window=w.window,
              use_rope=w.use_rope, rope_theta=w.rope_theta, eps=w.eps)
    names = ("q", "k", "v", "q_norm_w", "k_norm_w", "sinks")
    leaves = {n: t[n].clone().requires_grad_(True) for n in names}
    out, lse = fa.flint_attention(*(leaves[n] for n in names), **kw)
    assert not lse.requires_grad
    G = torch.from_numpy(np.random.default_rng(65).standard_normal((w.T, 4096)).astype(np.float32)).to(out.device)
    (out.float() * G).sum().backward()
    g = fa.attn_bwd(*(t[n] for n in names), out.detach(), lse, G.to(torch.bfloat16).contiguous(), **kw)
    assert fa.device_status(fa.attn_bwd.last_workspace) == 0
    torch.cuda.synchronize()
    for n, key in (("q", "dq"), ("k", "dk"), ("v", "dv")):
        assert torch.equal(leaves[n].grad, g[key].to(torch.bfloat16)), n
    for n, key in (("q_norm_w", "dq_norm_w"), ("k_norm_w", "dk_norm_w"), ("sinks", "dsinks")):
        assert torch.equal(leaves[n].grad, g[key]), n
    # the entry passes its configuration to the forward unchanged (a wrong
    # window, mask or RoPE flag would change the output wholesale)
    out2, lse2 = fa.attn_fwd(*(t[n] for n in names), **kw)
    torch.cuda.synchronize()
    scale = out2.float().abs().max().item()
    assert (out.detach().float() - out2.float()).abs().max().item() <= 1e-2 * scale
    assert (lse - lse2).abs().max().item() <= 1e-3
