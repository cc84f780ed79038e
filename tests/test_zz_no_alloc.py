"""flint_attn_fwd_static, the entry point for callers that cannot allocate
device memory when they run the layer (its scratch is a fixed device array
inside the library), must give the same results as flint_attn_fwd.

The test calls it through the C ABI twice in a row on different problems, so
the second call runs on scratch the first one left behind, and compares each
output with flint_attn_fwd's within the parity tolerances.  This file is
collected last on purpose."""
import numpy as np
import pytest

import workloads as W

pytestmark = pytest.mark.gpu

TOL = dict(max_abs=2e-2, rel_l2=5e-3, lse=1e-3)


def _device(w):
    import torch
    dev = torch.device("cuda:0")

    def bf(x):
        return torch.from_numpy(np.ascontiguousarray(x)).view(torch.bfloat16).to(dev)
    t = dict(q=bf(w.q), k=bf(w.k), v=bf(w.v), q_norm_w=torch.from_numpy(w.q_norm_w).to(dev),
             k_norm_w=torch.from_numpy(w.k_norm_w).to(dev),
             sinks=torch.from_numpy(np.asarray(w.sinks, np.float32)).to(dev))
    kw = dict(window=w.window, use_rope=w.use_rope, rope_theta=w.rope_theta, eps=w.eps)
    if w.pos_ids is not None:
        kw["pos_ids"] = torch.from_numpy(w.pos_ids).to(dev)
    if w.cu_seqlens is not None:
        kw["cu_seqlens"] = torch.from_numpy(w.cu_seqlens).to(dev)
    if w.pad_mask is not None:
        kw["pad_mask"] = torch.from_numpy(w.pad_mask).to(dev)
    return t, kw


def _compare(out_a, lse_a, out_b, lse_b):
    a = out_a.float().cpu().numpy().astype(np.float64)
    b = out_b.float().cpu().numpy().astype(np.float64)
    assert np.abs(a - b).max() <= TOL["max_abs"]
    assert np.linalg.norm(a - b) <= TOL["rel_l2"] * max(np.linalg.norm(b), 1e-30)
    la, lb = lse_a.cpu().numpy(), lse_b.cpu().numpy()
    fin = np.isfinite(lb)
    assert np.array_equal(np.isfinite(la), fin)
    assert np.abs(la[fin] - lb[fin]).max() <= TOL["lse"]


def test_static_entry_matches_workspace_entry_twice():
    import torch
    import full_gqa_learned_b200 as fa
    cases = [W.make_small(3000, seed=31, window=513, use_rope=True),
             W.make_small(2000, seed=32, window=0, use_rope=False,
                          cu_seqlens=np.array([0, 700, 701, 1600, 1990], np.int32))]
    for w in cases:
        t, kw = _device(w)
        ref_out, ref_lse = fa.attn_fwd(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"],
                                       t["sinks"], **kw)
        out = torch.empty_like(ref_out)
        lse = torch.empty_like(ref_lse)
        fa.attn_fwd_static(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["sinks"],
                           out, lse, **kw)
        torch.cuda.synchronize()
        _compare(out, lse, ref_out, ref_lse)


def test_static_entry_rejects_problems_beyond_its_scratch():
    import torch
    import full_gqa_learned_b200 as fa
    T = 20000                          # needs ~20 MiB of scratch > 16 MiB
    assert fa.workspace_bytes(T, 1) > fa.STATIC_SCRATCH_BYTES
    dev = torch.device("cuda:0")
    q = torch.zeros((T, 32, 128), dtype=torch.bfloat16, device=dev)
    kv = torch.zeros((T, 4, 128), dtype=torch.bfloat16, device=dev)
    w = torch.ones(128, dtype=torch.float32, device=dev)
    s = torch.zeros(32, dtype=torch.float32, device=dev)
    out = torch.empty((T, 4096), dtype=torch.bfloat16, device=dev)
    with pytest.raises(fa.FlintError) as e:
        fa.attn_fwd_static(q, kv, kv, w, w, s, out, None, window=0, use_rope=False)
    assert e.value.status == 5
