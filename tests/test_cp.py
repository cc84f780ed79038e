"""Head-split context parallelism (full_gqa_learned_b200/cp.py).

CPU: world sizes 2 and 4 on gloo.  The per-slice attention is a stand-in
built on the FP64 oracle (each head depends only on its own KV head, so the
slice is computed by placing it in full-size inputs and reading its heads
back); every rank's shard of the output and LSE must equal the oracle run on
the whole sequence, bit for bit.  This checks the data movement: the
all-to-all of head slices, the sink slices and the return to sequence shards.

GPU: flint_attn_fwd_heads on each head slice equals the corresponding heads of
flint_attn_fwd bit for bit (the work units of a slice are those of the full
call).
"""
import os

import numpy as np
import pytest

import workloads as W

HQ, HKV, D = 32, 4, 128


def _oracle_slice(q_h, k_h, v_h, q_norm_w, k_norm_w, sinks_h, **kw):
    """Stand-in per-slice attention on the oracle (test infrastructure only)."""
    import torch
    import oracle
    T, nh = q_h.shape[0], q_h.shape[1]
    g = k_h.shape[1]
    q = np.zeros((T, HQ, D))
    k = np.zeros((T, HKV, D))
    v = np.zeros((T, HKV, D))
    q[:, :nh] = q_h.numpy()
    k[:, :g] = k_h.numpy()
    v[:, :g] = v_h.numpy()
    s = np.zeros(HQ)
    s[:nh] = sinks_h.numpy()
    pos = None if kw.get("pos_ids") is None else kw["pos_ids"].numpy()
    cu = None if kw.get("cu_seqlens") is None else kw["cu_seqlens"].numpy()
    out, lse = oracle.attn_fwd(q, k, v, q_norm_w.numpy(), k_norm_w.numpy(), s, pos_ids=pos,
                               cu_seqlens=cu, window=kw["window"], use_rope=kw["use_rope"],
                               rope_theta=kw["rope_theta"], eps=kw["eps"], nthreads=1)
    return (torch.from_numpy(np.ascontiguousarray(out[:, :nh].reshape(T, nh * D))),
            torch.from_numpy(np.ascontiguousarray(lse[:, :nh].T)))


def _rank(rank, world, port, case, result_dir):
    import torch
    import torch.distributed as dist
    import oracle
    from full_gqa_learned_b200.cp import head_split_attention
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    w = case()
    T = w.T
    Tl = T // world
    f = lambda x: torch.from_numpy(np.ascontiguousarray(W.bf16_to_f64(x)))
    q, k, v = f(w.q), f(w.k), f(w.v)
    sl = slice(rank * Tl, (rank + 1) * Tl)
    kw = dict(window=w.window, use_rope=w.use_rope, rope_theta=w.rope_theta, eps=w.eps,
              pos_ids=None if w.pos_ids is None else torch.from_numpy(w.pos_ids),
              cu_seqlens=None if w.cu_seqlens is None else torch.from_numpy(w.cu_seqlens))
    out, lse = head_split_attention(q[sl], k[sl], v[sl], torch.from_numpy(w.q_norm_w.astype(np.float64)),
                                    torch.from_numpy(w.k_norm_w.astype(np.float64)),
                                    torch.from_numpy(np.asarray(w.sinks, np.float64)),
                                    attention=_oracle_slice, **kw)
    ref_o, ref_l = oracle.attn_fwd_workload(w, rows=np.arange(rank * Tl, (rank + 1) * Tl), nthreads=1)
    ok = (np.array_equal(out.numpy(), ref_o.reshape(Tl, HQ * D)) and
          np.array_equal(lse.numpy(), ref_l.T))
    with open(os.path.join(result_dir, "rank%d" % rank), "w") as fh:
        fh.write("ok" if ok else "mismatch")
    dist.barrier()
    dist.destroy_process_group()


def _case_sliding():
    return W.make_small(96, seed=21, window=13, use_rope=True)


def _case_docs():
    return W.make_small(64, seed=22, window=0, use_rope=True,
                        cu_seqlens=np.array([0, 5, 40, 41, 60], np.int32))


@pytest.mark.parametrize("world,case,port", [(2, _case_sliding, 29631), (4, _case_docs, 29632),
                                             (2, _case_docs, 29633)])
def test_head_split_matches_the_whole_sequence(tmp_path, world, case, port):
    import torch.multiprocessing as mp
    mp.start_processes(_rank, args=(world, port, case, str(tmp_path)), nprocs=world, start_method="spawn")
    for r in range(world):
        assert (tmp_path / ("rank%d" % r)).read_text() == "ok", r


def test_single_rank_is_the_whole_layer():
    import torch
    from full_gqa_learned_b200 import cp
    import torch.distributed as dist
    if dist.is_initialized():
        pytest.skip("a process group is already initialised")
    # one rank (no process group): the slice is all heads
    w = W.make_small(16, seed=23, window=0, use_rope=False)
    f = lambda x: torch.from_numpy(np.ascontiguousarray(W.bf16_to_f64(x)))
    out, lse = cp.head_split_attention(f(w.q), f(w.k), f(w.v), torch.from_numpy(w.q_norm_w.astype(np.float64)),
                                       torch.from_numpy(w.k_norm_w.astype(np.float64)),
                                       torch.from_numpy(np.asarray(w.sinks, np.float64)), window=0,
                                       use_rope=False, attention=_oracle_slice)
    import oracle
    ref_o, ref_l = oracle.attn_fwd_workload(w, rows=None, nthreads=1)
    assert np.array_equal(out.numpy(), ref_o.reshape(16, HQ * D))
    assert np.array_equal(lse.numpy(), ref_l.T)


@pytest.mark.gpu
@pytest.mark.parametrize("ng", [1, 2])
def test_head_slices_equal_the_full_call(ng):
    import torch
    import full_gqa_learned_b200 as fa
    from test_parity import to_device
    w = W.make_small(700, seed=24, window=129, use_rope=True,
                     cu_seqlens=np.array([0, 1, 200, 650], np.int32))
    t = to_device(w)
    kw = dict(cu_seqlens=t["cu_seqlens"], pos_ids=t["pos_ids"], window=w.window, use_rope=True)
    out, lse = fa.attn_fwd(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["sinks"], **kw)
    nh = 8 * ng
    for r in range(4 // ng):
        qs = t["q"][:, r * nh:(r + 1) * nh].contiguous()
        ks = t["k"][:, r * ng:(r + 1) * ng].contiguous()
        vs = t["v"][:, r * ng:(r + 1) * ng].contiguous()
        o, l = fa.attn_fwd_heads(qs, ks, vs, t["q_norm_w"], t["k_norm_w"],
                                 t["sinks"][r * nh:(r + 1) * nh].contiguous(), **kw)
        assert fa.device_status(fa.attn_fwd_heads.last_workspace) == 0
        torch.cuda.synchronize()
        assert torch.equal(o.view(torch.int16), out[:, r * nh * 128:(r + 1) * nh * 128].contiguous().view(torch.int16))
        assert torch.equal(l, lse[r * nh:(r + 1) * nh])


def _rank_bad(rank, world, port, result_dir):
    import torch
    import torch.distributed as dist
    from full_gqa_learned_b200.cp import head_split_attention
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    z = torch.zeros
    try:
        head_split_attention(z((4, 32, 128)), z((4, 4, 128)), z((4, 4, 128)), z(128), z(128), z(32),
                             window=0, use_rope=False, attention=_oracle_slice)
        msg = "no error"
    except ValueError as e:
        msg = "ValueError" if "1, 2 or 4" in str(e) else str(e)
    with open(os.path.join(result_dir, "rank%d" % rank), "w") as fh:
        fh.write(msg)
    dist.barrier()
    dist.destroy_process_group()


def test_group_of_three_is_rejected(tmp_path):
    """The 4 KV heads must divide the group: 3 ranks are refused on every rank
    before any exchange."""
    import torch.multiprocessing as mp
    mp.start_processes(_rank_bad, args=(3, 29634, str(tmp_path)), nprocs=3, start_method="spawn")
    for r in range(3):
        assert (tmp_path / ("rank%d" % r)).read_text() == "ValueError"
