"""Head-split context parallelism of the Flint attention (CP2 / CP4).

The "flint" model page ("Parallelism and backends") runs context parallelism
by splitting the attention heads over the CP group: both head counts must
divide the group size, so the 4 key/value heads permit CP2 or CP4, and the
learned sinks travel with their heads.  Each rank starts from a contiguous
sequence shard of the projections (tokens [r Tl, (r+1) Tl) of a T = N Tl
sequence, all heads) and must return the attention output and LSE of that
shard:

1. all-to-all: rank r receives, from every rank, that rank's tokens of KV
   heads [r g, (r+1) g) (g = 4 / N) and of their 8 g query heads, so it holds
   the whole sequence for its head slice;
2. the attention of the head slice over the whole sequence
   (flint_attn_fwd_heads), with the slice's sinks (the sinks are replicated
   parameters; each rank takes its heads' entries);
3. all-to-all back: the output rows and LSE entries of each sequence shard
   return to the shard's rank, head slices in rank order.

Positions and document boundaries (pos_ids, cu_seqlens) are those of the
whole sequence and are passed unchanged to every rank.  The exchange uses
NCCL's all-to-all on NCCL groups and paired point-to-point sends and receives
otherwise (gloo has no all-to-all).
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple

HQ, HKV, HEAD_DIM, GROUP = 32, 4, 128, 8


def _exchange(outs, ins, group):
    """out[j] <- what rank j sent to this rank in its ins[this rank]."""
    import torch.distributed as dist
    if len(ins) == 1:
        outs[0].copy_(ins[0])
        return
    rank = dist.get_rank(group)
    if dist.get_backend(group) == "nccl":
        dist.all_to_all(outs, ins, group=group)
        return
    reqs = []
    for j in range(len(ins)):
        if j == rank:
            outs[j].copy_(ins[j])
            continue
        peer = dist.get_global_rank(group, j) if group is not None else j
        reqs.append(dist.isend(ins[j].contiguous(), peer, group=group))
        reqs.append(dist.irecv(outs[j], peer, group=group))
    for r in reqs:
        r.wait()


def head_split_attention(q, k, v, q_norm_w, k_norm_w, sinks, *, group=None, pos_ids=None,
                         cu_seqlens=None, window: int = 513, use_rope: bool = True,
                         rope_theta: float = 10000.0, eps: float = 1e-6,
                         attention: Optional[Callable] = None) -> Tuple[object, object]:
    """Context-parallel attention forward with the heads split over `group`.

    q [Tl, 32, 128], k and v [Tl, 4, 128]: this rank's sequence shard (the
    group's shards in rank order make the sequence).  q_norm_w, k_norm_w
    [128], sinks [32]: replicated.  pos_ids [T] and cu_seqlens: of the whole
    sequence.  Returns (out [Tl, 4096], lse [32, Tl]) of this rank's shard.

    ``attention``: the per-slice forward, by default the library's
    flint_attn_fwd_heads; it is called as attention(q_h, k_h, v_h, q_norm_w,
    k_norm_w, sinks_h, pos_ids=..., cu_seqlens=..., window=..., use_rope=...,
    rope_theta=..., eps=...) and returns (out_h [T, 8 g x 128], lse_h [8 g, T]).
    """
    import torch
    import torch.distributed as dist
    n = dist.get_world_size(group) if dist.is_initialized() else 1
    r = dist.get_rank(group) if dist.is_initialized() else 0
    if n not in (1, 2, 4):
        raise ValueError("head-split context parallelism needs a group of 1, 2 or 4 ranks "
                         "(the 4 KV heads must divide it), got %d" % n)
    if attention is None:
        from . import attn_fwd_heads as attention
    Tl = int(q.shape[0])
    g = HKV // n                      # KV heads per rank
    nh = GROUP * g                    # query heads per rank
    # 1. sequence shards -> head slices
    qs = q.reshape(Tl, n, nh, HEAD_DIM)
    ks = k.reshape(Tl, n, g, HEAD_DIM)
    vs = v.reshape(Tl, n, g, HEAD_DIM)
    parts = []
    for x, h in ((qs, nh), (ks, g), (vs, g)):
        ins = [x[:, j].contiguous() for j in range(n)]
        outs = [torch.empty((Tl, h, HEAD_DIM), dtype=x.dtype, device=x.device) for _ in range(n)]
        _exchange(outs, ins, group)
        parts.append(torch.cat(outs, dim=0))          # [T, h, 128], tokens in rank order
    q_h, k_h, v_h = parts
    # 2. the head slice over the whole sequence
    out_h, lse_h = attention(q_h, k_h, v_h, q_norm_w, k_norm_w, sinks[r * nh:(r + 1) * nh].contiguous(),
                             pos_ids=pos_ids, cu_seqlens=cu_seqlens, window=window, use_rope=use_rope,
                             rope_theta=rope_theta, eps=eps)
    # 3. head slices -> sequence shards
    ins = [out_h[j * Tl:(j + 1) * Tl].contiguous() for j in range(n)]
    outs = [torch.empty((Tl, nh * HEAD_DIM), dtype=out_h.dtype, device=out_h.device) for _ in range(n)]
    _exchange(outs, ins, group)
    out = torch.stack(outs, dim=1).reshape(Tl, HQ * HEAD_DIM)
    ins = [lse_h[:, j * Tl:(j + 1) * Tl].contiguous() for j in range(n)]
    outs = [torch.empty((nh, Tl), dtype=lse_h.dtype, device=lse_h.device) for _ in range(n)]
    _exchange(outs, ins, group)
    lse = torch.cat(outs, dim=0)
    return out, lse
