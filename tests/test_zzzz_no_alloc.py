"""flint_attn_fwd_static, the entry point for callers that cannot allocate
device memory when they run the layer (its scratch is a fixed device array
inside the library), must give the same results as flint_attn_fwd.

Both entries run the same kernels on the same inputs; only the scratch's
address differs, and no result depends on it, so the outputs and LSE must be
bit-identical.  The calls come one after another on different problems and
mask kinds (single sequence, packed documents, a trailing-padding mask), so
each runs on scratch the previous one left behind.  One case is also checked
against the FP64 oracle, and the status word in the static scratch is read
back after an ill-formed call and after a good one.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test."""
import numpy as np
import pytest

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

TOL = dict(max_abs=2e-2, rel_l2=5e-3, lse=1e-3)      # stated parity bounds


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


def _run_both(w):
    import torch
    import full_gqa_learned_b200 as fa
    t, kw = _device(w)
    ref_out, ref_lse = fa.attn_fwd(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"],
                                   t["sinks"], **kw)
    assert fa.device_status(fa.attn_fwd.last_workspace) == 0
    # poison the outputs: every element the call must write is overwritten
    out = torch.full_like(ref_out, float("nan"))
    lse = torch.full_like(ref_lse, float("nan"))
    fa.attn_fwd_static(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["sinks"],
                       out, lse, **kw)
    assert fa.static_status() == 0
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))
    assert torch.equal(lse.view(torch.int32), ref_lse.view(torch.int32))
    return out, lse


def test_static_entry_bitwise_equal_to_workspace_entry():
    cu = np.array([0, 700, 701, 1600, 1990], np.int32)
    mask = np.zeros((3, 700), np.uint8)
    for b, L in enumerate([700, 0, 333]):
        mask[b, :L] = 1
    cases = [W.make_small(3000, seed=31, window=513, use_rope=True),
             W.make_small(2000, seed=32, window=0, use_rope=False, cu_seqlens=cu),
             W.make_small(2100, seed=33, window=129, use_rope=True, pad_mask=mask),
             W.make_small(40, seed=34, window=0, use_rope=True)]
    for i, w in enumerate(cases):
        out, lse = _run_both(w)
        if i == 0:
            # the first case against the FP64 oracle as well
            rows = np.arange(w.T)
            ref_o, ref_l = oracle.attn_fwd_workload(w, rows=rows)
            got = out.float().cpu().numpy().reshape(w.T, 32, 128).astype(np.float64)
            got_l = lse.cpu().numpy().T.astype(np.float64)
            err = np.abs(got - ref_o)
            rel = np.linalg.norm(got - ref_o) / np.linalg.norm(ref_o)
            lerr = np.abs(got_l - ref_l).max()
            assert err.max() <= TOL["max_abs"] and rel <= TOL["rel_l2"] and lerr <= TOL["lse"], \
                (err.max(), rel, lerr)
        if w.pad_mask is not None:
            # padded rows +0.0 exactly, their LSE the sink
            import torch
            pad = np.nonzero(w.pad_mask.reshape(-1) == 0)[0]
            o = out.view(torch.int16).cpu().numpy()
            assert np.all(o[pad] == 0)
            np.testing.assert_array_equal(lse.cpu().numpy()[:, pad], np.broadcast_to(
                np.asarray(w.sinks, np.float32)[:, None], (32, pad.size)))


def test_static_status_reports_device_errors():
    import torch
    import full_gqa_learned_b200 as fa
    w = W.make_small(64, seed=35)
    t, _ = _device(w)
    out = torch.empty((64, 4096), dtype=torch.bfloat16, device="cuda:0")
    bad = torch.tensor([0, 40, 20, 64], dtype=torch.int32, device="cuda:0")
    fa.attn_fwd_static(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["sinks"], out,
                       None, cu_seqlens=bad, window=0, use_rope=False)
    assert fa.static_status() == 1                       # FLINT_ERR_INVALID_ARG
    good = torch.tensor([0, 20, 64], dtype=torch.int32, device="cuda:0")
    fa.attn_fwd_static(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["sinks"], out,
                       None, cu_seqlens=good, window=0, use_rope=False)
    assert fa.static_status() == 0


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
