"""Seeded synthetic inputs for the sink-aware GQA attention forward.

This module is shared by the oracle side and the CUDA side of the tests and
by ``bench.py``.  It draws random numbers and rounds them to BF16; it holds
none of the attention arithmetic (no normalisation, rotation, masking or
softmax).

Shapes follow the Flint attention layer described on the NeMo AutoModel
"flint" model page (section "Model Architecture": 32 query heads, 4 key/value
heads, head dimension 128, a 513-token sliding window that counts the current
token) and the ``FlintConfig`` API page (``rms_norm_eps`` 1e-6,
``max_position_embeddings`` 262,144).  The five named workloads are the
single-sliding-layer, full-layer, packed-THD, long-context and
massive-activation cases; their value distributions and seeds are stated in
``CONFIGS``.

Draw order for every workload: q, k, v, q_norm_w, k_norm_w, sinks, then the
structure (document cut points, padding lengths, outlier channels, sampled
rows), all from one ``numpy.random.default_rng(seed)`` stream.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

HQ = 32          # query heads
HKV = 4          # key/value heads
D = 128          # head dimension
WINDOW = 513     # sliding window, current token included
ROPE_THETA = 10000.0
EPS = 1e-6


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to BF16 (round to nearest, ties to even) and
    return the 16-bit patterns as uint16.  Inputs must be finite."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    out = np.empty(u.shape, dtype=np.uint16)
    # process in slabs to bound temporary memory on very large inputs
    flat_u = u.reshape(-1)
    flat_o = out.reshape(-1)
    step = 1 << 26
    for s in range(0, flat_u.size, step):
        b = flat_u[s:s + step]
        lsb = (b >> np.uint32(16)) & np.uint32(1)
        r = (b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
        flat_o[s:s + step] = r.astype(np.uint16)
    return out


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of BF16 bit patterns to float64."""
    u = bits.astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


@dataclasses.dataclass
class Workload:
    """One attention-layer invocation: tensors plus masking structure.

    q: uint16 [T,32,128] BF16 bits; k, v: uint16 [T,4,128] BF16 bits.
    q_norm_w, k_norm_w: float32 [128]; sinks: float32 [32].
    pos_ids: int32 [T] document-local positions (None: defaults).
    cu_seqlens: int32 [ndocs+1] for packed THD input, else None.
    pad_mask: uint8 [batch, seqlen] (1 = valid, trailing padding), else None.
    window: 513 for sliding layers, 0 for full causal layers.
    rows: query tokens the oracle evaluates for sampled checks (None = all).
    """
    name: str
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    q_norm_w: np.ndarray
    k_norm_w: np.ndarray
    sinks: np.ndarray
    pos_ids: Optional[np.ndarray]
    cu_seqlens: Optional[np.ndarray]
    pad_mask: Optional[np.ndarray]
    window: int
    use_rope: bool
    rope_theta: float = ROPE_THETA
    eps: float = EPS
    rows: Optional[np.ndarray] = None
    seed: int = 0

    @property
    def T(self) -> int:
        return int(self.q.shape[0])

    def valid_pairs(self) -> int:
        """Number of (query, key) pairs the causal/window/document mask keeps,
        per query head (counting only valid, non-padded queries)."""
        lens = segment_lengths(self)
        W = self.window
        tot = 0
        for L in lens:
            L = int(L)
            if W > 0 and L > W:
                tot += W * L - W * (W - 1) // 2
            else:
                tot += L * (L + 1) // 2
        return tot

    def flops(self) -> float:
        """Window-aware FLOPs: QK^T and PV, 2 flops per multiply-add,
        head_dim 128, 32 query heads: 4*128*32 per valid pair."""
        return 4.0 * D * HQ * self.valid_pairs()

    def algorithmic_bytes(self) -> int:
        """Q, K, V read once, out and LSE written once, plus the small
        per-token/per-segment metadata and weights."""
        T = self.T
        b = T * HQ * D * 2 + 2 * T * HKV * D * 2          # q, k, v
        b += T * HQ * D * 2 + T * HQ * 4                   # out, lse
        if self.use_rope:
            b += T * 4                                     # pos_ids
        if self.cu_seqlens is not None:
            b += self.cu_seqlens.size * 4
        if self.pad_mask is not None:
            b += self.pad_mask.size
        b += 2 * D * 4 + HQ * 4
        return int(b)


def segment_lengths(w: Workload) -> np.ndarray:
    if w.cu_seqlens is not None:
        return np.diff(w.cu_seqlens).astype(np.int64)
    if w.pad_mask is not None:
        return w.pad_mask.sum(axis=1).astype(np.int64)
    return np.array([w.T], dtype=np.int64)


def _local_positions(T: int, cu: np.ndarray) -> np.ndarray:
    pos = np.zeros(T, dtype=np.int32)
    for d in range(len(cu) - 1):
        a, b = int(cu[d]), int(cu[d + 1])
        pos[a:b] = np.arange(b - a, dtype=np.int32)
    return pos


def _normal(rng, shape, scale=1.0, dtype=np.float32):
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        x *= np.float32(scale)
    return x


def _draw_tensors(rng, T):
    q = bf16_bits(_normal(rng, (T, HQ, D)))
    k = bf16_bits(_normal(rng, (T, HKV, D)))
    v = bf16_bits(_normal(rng, (T, HKV, D)))
    wq = (1.0 + 0.1 * rng.standard_normal(D)).astype(np.float32)
    wk = (1.0 + 0.1 * rng.standard_normal(D)).astype(np.float32)
    sinks = rng.standard_normal(HQ).astype(np.float32)
    return q, k, v, wq, wk, sinks


def _sample_rows(rng, T, n, forced):
    n = min(n, T)
    forced = np.array(sorted({int(f) for f in forced if 0 <= f < T}), dtype=np.int64)
    rest = np.setdiff1d(np.arange(T, dtype=np.int64), forced)
    pick = rng.choice(rest, size=max(0, n - forced.size), replace=False)
    return np.sort(np.concatenate([forced, pick]))


def make_sliding(T=1024, seed=0, name="sliding_s1024", rows=None) -> Workload:
    rng = np.random.default_rng(seed)
    q, k, v, wq, wk, sinks = _draw_tensors(rng, T)
    return Workload(name, q, k, v, wq, wk, sinks,
                    pos_ids=np.arange(T, dtype=np.int32), cu_seqlens=None,
                    pad_mask=None, window=WINDOW, use_rope=True, rows=rows,
                    seed=seed)


def make_full(T=4096, seed=1, name="full_s4096") -> Workload:
    rng = np.random.default_rng(seed)
    q, k, v, wq, wk, sinks = _draw_tensors(rng, T)
    return Workload(name, q, k, v, wq, wk, sinks, pos_ids=None,
                    cu_seqlens=None, pad_mask=None, window=0, use_rope=False,
                    seed=seed)


def make_thd(T=32768, ndocs=8, seed=2, name="thd_8docs_32768",
             n_rows=4096) -> Workload:
    rng = np.random.default_rng(seed)
    q, k, v, wq, wk, sinks = _draw_tensors(rng, T)
    cuts = np.sort(rng.choice(np.arange(1, T), size=ndocs - 1, replace=False))
    cu = np.concatenate([[0], cuts, [T]]).astype(np.int32)
    forced = []
    for d in range(ndocs):
        a, b = int(cu[d]), int(cu[d + 1])
        forced += [a, a + 1, a + 511, a + 512, a + 513, b - 1]
    rows = _sample_rows(rng, T, n_rows, forced) if n_rows else None
    return Workload(name, q, k, v, wq, wk, sinks, pos_ids=_local_positions(T, cu),
                    cu_seqlens=cu, pad_mask=None, window=WINDOW, use_rope=True,
                    rows=rows, seed=seed)


def make_long(T=262144, seed=3, name="sliding_s262144", n_rows=4096) -> Workload:
    rng = np.random.default_rng(seed)
    q, k, v, wq, wk, sinks = _draw_tensors(rng, T)
    rows = _sample_rows(rng, T, n_rows, [0, 1, 511, 512, 513, T - 1])
    return Workload(name, q, k, v, wq, wk, sinks,
                    pos_ids=np.arange(T, dtype=np.int32), cu_seqlens=None,
                    pad_mask=None, window=WINDOW, use_rope=True, rows=rows,
                    seed=seed)


def make_stress(B=4, S=8192, max_pad=2048, seed=4,
                name="stress_full_4x8192_pad", n_rows=4096) -> Workload:
    """Massive-activation stress (HF discussion on RecursiveSI/flint, section
    "Numerics": residual magnitudes ~1e4): two outlier channels per KV group,
    shared by the group's 8 query heads and its key head, scaled by 1e4 in
    pre-norm Q/K; two value channels per KV head scaled by 1e3.  Sinks are
    drawn from {-20, 0, +20} plus N(0,1)."""
    rng = np.random.default_rng(seed)
    T = B * S
    qf = _normal(rng, (T, HQ, D))
    kf = _normal(rng, (T, HKV, D))
    vf = _normal(rng, (T, HKV, D))
    wq = (1.0 + 0.1 * rng.standard_normal(D)).astype(np.float32)
    wk = (1.0 + 0.1 * rng.standard_normal(D)).astype(np.float32)
    sinks = (rng.choice(np.array([-20.0, 0.0, 20.0]), size=HQ)
             + rng.standard_normal(HQ)).astype(np.float32)
    pads = rng.integers(0, max_pad + 1, size=B)
    qk_ch = np.stack([rng.choice(D, size=2, replace=False) for _ in range(HKV)])
    v_ch = np.stack([rng.choice(D, size=2, replace=False) for _ in range(HKV)])
    for g in range(HKV):
        for c in qk_ch[g]:
            qf[:, g * 8:(g + 1) * 8, c] *= np.float32(1e4)
            kf[:, g, c] *= np.float32(1e4)
        for c in v_ch[g]:
            vf[:, g, c] *= np.float32(1e3)
    q, k, v = bf16_bits(qf), bf16_bits(kf), bf16_bits(vf)
    del qf, kf, vf
    mask = np.zeros((B, S), dtype=np.uint8)
    for b in range(B):
        mask[b, :S - int(pads[b])] = 1
    pos = np.tile(np.arange(S, dtype=np.int32), B)
    forced = []
    for b in range(B):
        L = S - int(pads[b])
        forced += [b * S, b * S + 1, b * S + L - 1, b * S + L, (b + 1) * S - 1]
    rows = _sample_rows(rng, T, n_rows, forced) if n_rows else None
    return Workload(name, q, k, v, wq, wk, sinks, pos_ids=pos, cu_seqlens=None,
                    pad_mask=mask, window=0, use_rope=False, rows=rows,
                    seed=seed)


CONFIGS = {
    "sliding_s1024": make_sliding,
    "full_s4096": make_full,
    "thd_8docs_32768": make_thd,
    "sliding_s262144": make_long,
    "stress_full_4x8192_pad": make_stress,
}


# Smaller stand-ins with the structure of a named workload, sized for
# profiler captures (a few hundred MB on the device): the long-context
# sliding layer's per-tile chunk structure at 32,768 tokens.
PROFILE_CONFIGS = {
    "sliding_s32768": lambda: make_long(T=32768, seed=3, name="sliding_s32768"),
}


def make(name: str, **kw) -> Workload:
    if name in PROFILE_CONFIGS:
        return PROFILE_CONFIGS[name](**kw)
    return CONFIGS[name](**kw)


def make_small(T, seed, *, window=0, use_rope=False, cu_seqlens=None,
               pad_mask=None, sinks=None, pos_ids=None, name="small",
               qscale=1.0, kscale=1.0, vscale=1.0) -> Workload:
    """Small seeded case for edge tests; same distributions as the named
    workloads unless overridden."""
    rng = np.random.default_rng(seed)
    q = bf16_bits(_normal(rng, (T, HQ, D), qscale))
    k = bf16_bits(_normal(rng, (T, HKV, D), kscale))
    v = bf16_bits(_normal(rng, (T, HKV, D), vscale))
    wq = (1.0 + 0.1 * rng.standard_normal(D)).astype(np.float32)
    wk = (1.0 + 0.1 * rng.standard_normal(D)).astype(np.float32)
    s = rng.standard_normal(HQ).astype(np.float32)
    if sinks is not None:
        s = np.broadcast_to(np.asarray(sinks, dtype=np.float32), (HQ,)).copy()
    if pos_ids is None and use_rope:
        if cu_seqlens is not None:
            pos_ids = _local_positions(T, np.asarray(cu_seqlens))
        elif pad_mask is not None:
            pos_ids = np.tile(np.arange(pad_mask.shape[1], dtype=np.int32),
                              pad_mask.shape[0])
        else:
            pos_ids = np.arange(T, dtype=np.int32)
    return Workload(name, q, k, v, wq, wk, s, pos_ids=pos_ids,
                    cu_seqlens=None if cu_seqlens is None else np.asarray(cu_seqlens, np.int32),
                    pad_mask=pad_mask, window=window, use_rope=use_rope, seed=seed)


def make_small_f32(T, seed, *, window=0, use_rope=False, cu_seqlens=None, pad_mask=None,
                   name="small_f32") -> Workload:
    """Seeded case with FP32 projections (an FP32 model body, as the FP16
    attention-compute policy takes them): q, k, v float32 N(0,1), not
    rounded; the rest as make_small."""
    w = make_small(T, seed, window=window, use_rope=use_rope, cu_seqlens=cu_seqlens,
                   pad_mask=pad_mask, name=name)
    rng = np.random.default_rng(seed + 500)
    w.q = _normal(rng, (T, HQ, D))
    w.k = _normal(rng, (T, HKV, D))
    w.v = _normal(rng, (T, HKV, D))
    return w


@dataclasses.dataclass
class DecodeWorkload:
    """One decode step for B sequences: the new token's projections and a
    key/value cache of capacity cap (position j in slot j mod cap).  Cached
    keys stand in for normalised, rotated keys (N(0,1) BF16); values are
    N(0,1) BF16 like v."""
    name: str
    q: np.ndarray          # uint16 [B,32,128]
    k: np.ndarray          # uint16 [B,4,128]
    v: np.ndarray          # uint16 [B,4,128]
    k_cache: np.ndarray    # uint16 [B,4,cap,128] (head-major)
    v_cache: np.ndarray    # uint16 [B,4,cap,128]
    cache_len: np.ndarray  # int32 [B]: position of the new token
    q_norm_w: np.ndarray
    k_norm_w: np.ndarray
    sinks: np.ndarray
    window: int
    use_rope: bool
    rope_theta: float = ROPE_THETA
    eps: float = EPS

    @property
    def B(self) -> int:
        return int(self.q.shape[0])

    @property
    def cap(self) -> int:
        return int(self.k_cache.shape[2])          # [B, 4, cap, 128]

    def keys_per_sequence(self) -> np.ndarray:
        """Keys each new token attends to (its window, itself included)."""
        n = self.cache_len.astype(np.int64) + 1
        return np.minimum(n, self.window) if self.window > 0 else n

    def flops(self) -> float:
        return float(4 * D * HQ * self.keys_per_sequence().sum())

    def algorithmic_bytes(self) -> float:
        """Window keys and values read once per KV head, the new token's q, k,
        v read, its cache slot, out and lse written."""
        kv = 2 * HKV * D * 2 * self.keys_per_sequence().sum()
        return float(kv + self.B * (HQ * D * 2 + 2 * HKV * D * 2 + 2 * HKV * D * 2 + HQ * D * 2 + HQ * 4))


def make_decode(B, cap, seed, *, window, use_rope, max_len, min_len=0, name="decode",
                sinks=None) -> DecodeWorkload:
    """Seeded decode step: cache lengths uniform in [min_len, max_len)."""
    rng = np.random.default_rng(seed)
    q = bf16_bits(_normal(rng, (B, HQ, D), 1.0))
    k = bf16_bits(_normal(rng, (B, HKV, D), 1.0))
    v = bf16_bits(_normal(rng, (B, HKV, D), 1.0))
    wq = (1.0 + 0.1 * rng.standard_normal(D)).astype(np.float32)
    wk = (1.0 + 0.1 * rng.standard_normal(D)).astype(np.float32)
    s = rng.standard_normal(HQ).astype(np.float32)
    if sinks is not None:
        s = np.broadcast_to(np.asarray(sinks, dtype=np.float32), (HQ,)).copy()
    kc = bf16_bits(_normal(rng, (B, HKV, cap, D), 1.0))
    vc = bf16_bits(_normal(rng, (B, HKV, cap, D), 1.0))
    cache_len = rng.integers(min_len, max_len, size=B).astype(np.int32)
    return DecodeWorkload(name, q, k, v, kc, vc, cache_len, wq, wk, s, window=window, use_rope=use_rope)


# decode steps: a batch of sequences deep into a 262,144-token context on a
# sliding layer (ring cache of 513), and a full layer with a 4,096-token cache
DECODE_CONFIGS = {
    "decode_sliding_b128": dict(B=128, cap=513, seed=5, window=513, use_rope=True,
                                max_len=262144, min_len=513),
    "decode_full_b64_s4096": dict(B=64, cap=4096, seed=6, window=0, use_rope=False,
                                  max_len=4096, min_len=1),
    # a small batch of the sliding case, sized for profiler captures
    "decode_sliding_b16": dict(B=16, cap=513, seed=5, window=513, use_rope=True,
                               max_len=262144, min_len=513),
}


def make_decode_named(name: str) -> DecodeWorkload:
    return make_decode(name=name, **DECODE_CONFIGS[name])


# ---------------------------------------------------------------- whole layer

HIDDEN = 2048    # FlintConfig hidden size ("flint" model page, "Model Architecture")


@dataclasses.dataclass
class LayerWorkload:
    """Inputs of the whole attention layer: hidden states and the projection
    weights in the PyTorch Linear layout, plus the attention's own inputs.

    x: uint16 [T, hidden] BF16 bits, N(0,1).
    w_qkv: uint16 [5120, hidden]: W_q, W_k, W_v stacked, N(0, 1/hidden), so
      the projections are ~N(0,1) like the attention workloads' q, k, v.
    w_o: uint16 [hidden, 4096], N(0, 1/4096).
    attn: the attention part (norm weights, sinks, positions, masks, window;
      its q, k, v are unused)."""
    name: str
    x: np.ndarray
    w_qkv: np.ndarray
    w_o: np.ndarray
    attn: Workload

    @property
    def T(self) -> int:
        return int(self.x.shape[0])

    @property
    def hidden(self) -> int:
        return int(self.x.shape[1])

    def proj_flops(self) -> float:
        """QKV projection plus o_proj: 2 FLOPs per multiply-add."""
        return 2.0 * self.T * self.hidden * (HQ * D + 2 * HKV * D) + 2.0 * self.T * (HQ * D) * self.hidden

    def flops(self) -> float:
        return self.proj_flops() + self.attn.flops()


def make_layer(T, seed, *, hidden=HIDDEN, window=0, use_rope=False, cu_seqlens=None, pad_mask=None,
               name="layer") -> LayerWorkload:
    """Seeded whole-layer inputs; draw order x, w_qkv, w_o, then the attention
    part (make_small with seed + 1)."""
    rng = np.random.default_rng(seed)
    x = bf16_bits(_normal(rng, (T, hidden)))
    w_qkv = bf16_bits(_normal(rng, (HQ * D + 2 * HKV * D, hidden), 1.0 / np.sqrt(hidden)))
    w_o = bf16_bits(_normal(rng, (hidden, HQ * D), 1.0 / np.sqrt(HQ * D)))
    attn = make_small(T, seed + 1, window=window, use_rope=use_rope, cu_seqlens=cu_seqlens,
                      pad_mask=pad_mask, name=name)
    return LayerWorkload(name, x, w_qkv, w_o, attn)


# whole-layer workloads: the full layer at S=4096 and the sliding layer at
# S=1024, with the checkpoint's hidden size
LAYER_CONFIGS = {
    "layer_full_s4096": dict(T=4096, seed=41, window=0, use_rope=False),
    "layer_sliding_s1024": dict(T=1024, seed=42, window=WINDOW, use_rope=True),
}


def make_layer_named(name: str) -> LayerWorkload:
    return make_layer(name=name, **LAYER_CONFIGS[name])
