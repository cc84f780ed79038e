"""B200 (sm_100a) sink-aware GQA attention of the Flint decoder: forward,
gradient and decode step.

This package is a thin ctypes binding over ``libflint_attn.so``, whose C ABI
is declared in ``include/flint_attn.h``.  The binding only marshals
arguments: every step of the computation (key preparation, planning,
normalisation, rotation, attention, sink, masking, epilogue) runs in the
library's CUDA kernels.  PyTorch is used for device memory and streams.

There is no fallback: if the library is missing or the device is not an
sm_100 GPU, the call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Tuple

__all__ = ["attn_fwd", "attn_fwd_heads", "attn_fwd_fp16", "fp16_workspace_bytes", "attn_fwd_static", "static_status", "qkv_proj", "o_proj", "attn_layer_fwd",
           "attn_decode", "attn_bwd", "flint_attention", "workspace_bytes",
           "decode_workspace_bytes", "bwd_workspace_bytes", "device_status", "load_library",
           "FlintError", "LIB_PATH", "HQ", "HKV", "HEAD_DIM", "STATUS", "STATIC_SCRATCH_BYTES"]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libflint_attn.so")
HQ, HKV, HEAD_DIM = 32, 4, 128
STATIC_SCRATCH_BYTES = 16 << 20     # FLINT_STATIC_SCRATCH_BYTES
STATUS = {0: "FLINT_OK", 1: "FLINT_ERR_INVALID_ARG", 2: "FLINT_ERR_UNSUPPORTED",
          3: "FLINT_ERR_CUDA", 4: "FLINT_ERR_TIMEOUT", 5: "FLINT_ERR_WORKSPACE"}

_lock = threading.Lock()
_lib = None


class FlintError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__("%s: %s" % (STATUS.get(status, status), message))
        self.status = status


def load_library() -> ctypes.CDLL:
    """Load libflint_attn.so (built in-tree by ``full_gqa_learned_b200.build``)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise ImportError("libflint_attn.so is not built; run "
                              "`python -m full_gqa_learned_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        P, I32, F32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
        lib.flint_attn_abi_version.restype = I32
        lib.flint_attn_abi_version.argtypes = []
        lib.flint_attn_workspace_bytes.restype = ctypes.c_size_t
        lib.flint_attn_workspace_bytes.argtypes = [I32, I32]
        fwd_args = [P, P, P, P, P, P, P, P, I32, P, I32, I32, I32, I32, I32,
                    F32, F32, P, P, P, ctypes.c_size_t, P]
        for name in ("flint_attn_fwd", "flint_attn_prepare", "flint_attn_attend"):
            getattr(lib, name).restype = ctypes.c_int
            getattr(lib, name).argtypes = fwd_args
        lib.flint_attn_fwd_heads.restype = ctypes.c_int
        lib.flint_attn_fwd_heads.argtypes = fwd_args[:13] + [I32] + fwd_args[13:]
        lib.flint_attn_fwd_fp16.restype = ctypes.c_int
        lib.flint_attn_fwd_fp16.argtypes = fwd_args
        lib.flint_attn_fp16_workspace_bytes.restype = ctypes.c_size_t
        lib.flint_attn_fp16_workspace_bytes.argtypes = [I32, I32]
        lib.flint_attn_fwd_static.restype = ctypes.c_int
        lib.flint_attn_fwd_static.argtypes = fwd_args[:19] + [P]
        lib.flint_attn_fwd_static_status.restype = ctypes.c_int
        lib.flint_attn_fwd_static_status.argtypes = [P]
        lib.flint_attn_decode_workspace_bytes.restype = ctypes.c_size_t
        lib.flint_attn_decode_workspace_bytes.argtypes = [I32, I32, I32]
        lib.flint_attn_decode.restype = ctypes.c_int
        lib.flint_attn_decode.argtypes = [P, P, P, P, P, P, P, P, P, I32, I32, I32, I32, F32, F32,
                                          P, P, P, ctypes.c_size_t, P]
        lib.flint_attn_bwd_workspace_bytes.restype = ctypes.c_size_t
        lib.flint_attn_bwd_workspace_bytes.argtypes = [I32]
        lib.flint_attn_bwd.restype = ctypes.c_int
        lib.flint_attn_bwd.argtypes = [P, P, P, P, P, P, P, P, I32, P, I32, I32, I32, I32, I32,
                                       F32, F32, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        lib.flint_qkv_proj.restype = ctypes.c_int
        lib.flint_qkv_proj.argtypes = [P, P, I32, I32, P, P, P, P]
        lib.flint_o_proj.restype = ctypes.c_int
        lib.flint_o_proj.argtypes = [P, P, I32, I32, P, P]
        lib.flint_attn_layer_fwd.restype = ctypes.c_int
        lib.flint_attn_layer_fwd.argtypes = [P, P, P, P, P, P, P, P, I32, P, I32, I32, I32, I32, I32, I32,
                                             F32, F32, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        lib.flint_attn_device_status.restype = ctypes.c_int
        lib.flint_attn_device_status.argtypes = [P, P]
        lib.flint_attn_last_error.restype = ctypes.c_char_p
        lib.flint_attn_last_error.argtypes = []
        lib.flint_attn_status_string.restype = ctypes.c_char_p
        lib.flint_attn_status_string.argtypes = [ctypes.c_int]
        _lib = lib
        return lib


def workspace_bytes(T: int, num_segments: int = 1) -> int:
    return int(load_library().flint_attn_workspace_bytes(int(T), int(num_segments)))


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _check(t, name, dtype, shape=None):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))


def attn_fwd(q, k, v, q_norm_w, k_norm_w, sinks, *, pos_ids=None, cu_seqlens=None,
             pad_mask=None, window: int = 513, use_rope: bool = True,
             rope_theta: float = 10000.0, eps: float = 1e-6, out=None, lse=None,
             workspace=None, stream=None, want_lse: bool = True,
             stage: str = "both") -> Tuple[object, object]:
    """Sink-aware GQA attention forward (see include/flint_attn.h).

    q [T,32,128], k/v [T,4,128] bf16 CUDA tensors; q_norm_w, k_norm_w [128]
    and sinks [32] float32; pos_ids [T] int32 or None; cu_seqlens [n+1] int32
    (packed THD) or pad_mask [B,S] uint8 (trailing padding) or neither.
    window 0 = full causal.  Returns (out [T,4096] bf16, lse [32,T] f32 or
    None).  Asynchronous on ``stream`` (default: torch's current stream).
    ``stage``: "both" (flint_attn_fwd), or "prepare" / "attend" to enqueue
    the two kernels separately (same arguments and workspace for both).
    """
    import torch
    lib = load_library()
    T = int(q.shape[0]) if q.dim() >= 1 else 0
    _check(q, "q", torch.bfloat16, (T, HQ, HEAD_DIM))
    _check(k, "k", torch.bfloat16, (T, HKV, HEAD_DIM))
    _check(v, "v", torch.bfloat16, (T, HKV, HEAD_DIM))
    _check(q_norm_w, "q_norm_w", torch.float32, (HEAD_DIM,))
    _check(k_norm_w, "k_norm_w", torch.float32, (HEAD_DIM,))
    _check(sinks, "sinks", torch.float32, (HQ,))
    num_docs, batch, seqlen, nseg = 0, 0, 0, 1
    if pos_ids is not None:
        _check(pos_ids, "pos_ids", torch.int32, (T,))
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", torch.int32)
        num_docs = int(cu_seqlens.numel()) - 1
        nseg = max(num_docs, 1)
    if pad_mask is not None:
        _check(pad_mask, "pad_mask", torch.uint8)
        if pad_mask.dim() != 2:
            raise ValueError("pad_mask must be [batch, seqlen]")
        batch, seqlen = int(pad_mask.shape[0]), int(pad_mask.shape[1])
        nseg = batch
    dev = q.device
    if out is None:
        out = torch.empty((T, HQ * HEAD_DIM), dtype=torch.bfloat16, device=dev)
    _check(out, "out", torch.bfloat16, (T, HQ * HEAD_DIM))
    if lse is None and want_lse:
        lse = torch.empty((HQ, T), dtype=torch.float32, device=dev)
    if lse is not None:
        _check(lse, "lse", torch.float32, (HQ, T))
    need = workspace_bytes(T, nseg)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check(workspace, "workspace", torch.uint8)
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    sptr = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    with torch.cuda.device(dev):
        fn = {"both": lib.flint_attn_fwd, "prepare": lib.flint_attn_prepare,
              "attend": lib.flint_attn_attend}[stage]
        st = fn(
            _ptr(q), _ptr(k), _ptr(v), _ptr(q_norm_w), _ptr(k_norm_w), _ptr(sinks),
            _ptr(pos_ids), _ptr(cu_seqlens), num_docs, _ptr(pad_mask), batch, seqlen, T,
            int(window), int(bool(use_rope)), float(rope_theta), float(eps), _ptr(out),
            _ptr(lse), _ptr(workspace), int(workspace.numel()), sptr)
    if st != 0:
        raise FlintError(st, lib.flint_attn_last_error().decode())
    attn_fwd.last_workspace = workspace
    return out, lse


def decode_workspace_bytes(B: int, cap: int, window: int) -> int:
    return int(load_library().flint_attn_decode_workspace_bytes(int(B), int(cap), int(window)))


def attn_decode(q, k, v, q_norm_w, k_norm_w, sinks, k_cache, v_cache, cache_len, *,
                window: int = 513, use_rope: bool = True, rope_theta: float = 10000.0,
                eps: float = 1e-6, out=None, lse=None, workspace=None, stream=None,
                want_lse: bool = True) -> Tuple[object, object]:
    """One decode step (see include/flint_attn.h, flint_attn_decode).

    q [B,32,128], k/v [B,4,128] bf16: the new token of each sequence;
    k_cache, v_cache [B,4,cap,128] bf16, head-major (position j of KV head
    g in [b, g, j mod cap]; the step writes the new token into slot
    cache_len[b] mod cap); cache_len [B]
    int32.  Returns (out [B,4096] bf16, lse [32,B] f32 or None).
    """
    import torch
    lib = load_library()
    B = int(q.shape[0]) if q.dim() >= 1 else 0
    cap = int(k_cache.shape[2]) if k_cache.dim() >= 3 else 0
    _check(q, "q", torch.bfloat16, (B, HQ, HEAD_DIM))
    _check(k, "k", torch.bfloat16, (B, HKV, HEAD_DIM))
    _check(v, "v", torch.bfloat16, (B, HKV, HEAD_DIM))
    _check(q_norm_w, "q_norm_w", torch.float32, (HEAD_DIM,))
    _check(k_norm_w, "k_norm_w", torch.float32, (HEAD_DIM,))
    _check(sinks, "sinks", torch.float32, (HQ,))
    _check(k_cache, "k_cache", torch.bfloat16, (B, HKV, cap, HEAD_DIM))
    _check(v_cache, "v_cache", torch.bfloat16, (B, HKV, cap, HEAD_DIM))
    _check(cache_len, "cache_len", torch.int32, (B,))
    dev = q.device
    if out is None:
        out = torch.empty((B, HQ * HEAD_DIM), dtype=torch.bfloat16, device=dev)
    _check(out, "out", torch.bfloat16, (B, HQ * HEAD_DIM))
    if lse is None and want_lse:
        lse = torch.empty((HQ, B), dtype=torch.float32, device=dev)
    if lse is not None:
        _check(lse, "lse", torch.float32, (HQ, B))
    need = decode_workspace_bytes(B, max(cap, 1), window)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check(workspace, "workspace", torch.uint8)
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    sptr = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    with torch.cuda.device(dev):
        st = lib.flint_attn_decode(
            _ptr(q), _ptr(k), _ptr(v), _ptr(q_norm_w), _ptr(k_norm_w), _ptr(sinks), _ptr(k_cache),
            _ptr(v_cache), _ptr(cache_len), B, cap, int(window), int(bool(use_rope)),
            float(rope_theta), float(eps), _ptr(out), _ptr(lse), _ptr(workspace),
            int(workspace.numel()), sptr)
    if st != 0:
        raise FlintError(st, lib.flint_attn_last_error().decode())
    attn_decode.last_workspace = workspace
    return out, lse


def bwd_workspace_bytes(T: int) -> int:
    return int(load_library().flint_attn_bwd_workspace_bytes(int(T)))


def attn_bwd(q, k, v, q_norm_w, k_norm_w, sinks, out, lse, dout, *, pos_ids=None,
             cu_seqlens=None, pad_mask=None, window: int = 513, use_rope: bool = True,
             rope_theta: float = 10000.0, eps: float = 1e-6, grads=None, workspace=None,
             stream=None) -> dict:
    """Gradient of attn_fwd (see include/flint_attn.h, flint_attn_bwd).

    The forward's arguments, its out [T,4096] bf16 and lse [32,T] f32, and
    dout [T,4096] bf16.  Returns a dict of float32 CUDA tensors: dq
    [T,32,128], dk and dv [T,4,128], dq_norm_w and dk_norm_w [128], dsinks
    [32] (``grads``: the same dict to write into).  Asynchronous on ``stream``.
    """
    import torch
    lib = load_library()
    T = int(q.shape[0]) if q.dim() >= 1 else 0
    _check(q, "q", torch.bfloat16, (T, HQ, HEAD_DIM))
    _check(k, "k", torch.bfloat16, (T, HKV, HEAD_DIM))
    _check(v, "v", torch.bfloat16, (T, HKV, HEAD_DIM))
    _check(q_norm_w, "q_norm_w", torch.float32, (HEAD_DIM,))
    _check(k_norm_w, "k_norm_w", torch.float32, (HEAD_DIM,))
    _check(sinks, "sinks", torch.float32, (HQ,))
    _check(out, "out", torch.bfloat16, (T, HQ * HEAD_DIM))
    _check(lse, "lse", torch.float32, (HQ, T))
    _check(dout, "dout", torch.bfloat16, (T, HQ * HEAD_DIM))
    num_docs, batch, seqlen = 0, 0, 0
    if pos_ids is not None:
        _check(pos_ids, "pos_ids", torch.int32, (T,))
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", torch.int32)
        num_docs = int(cu_seqlens.numel()) - 1
    if pad_mask is not None:
        _check(pad_mask, "pad_mask", torch.uint8)
        if pad_mask.dim() != 2:
            raise ValueError("pad_mask must be [batch, seqlen]")
        batch, seqlen = int(pad_mask.shape[0]), int(pad_mask.shape[1])
    dev = q.device
    shapes = {"dq": (T, HQ, HEAD_DIM), "dk": (T, HKV, HEAD_DIM), "dv": (T, HKV, HEAD_DIM),
              "dq_norm_w": (HEAD_DIM,), "dk_norm_w": (HEAD_DIM,), "dsinks": (HQ,)}
    if grads is None:
        grads = {n: torch.empty(sh, dtype=torch.float32, device=dev) for n, sh in shapes.items()}
    for n, sh in shapes.items():
        _check(grads[n], n, torch.float32, sh)
    need = bwd_workspace_bytes(T)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check(workspace, "workspace", torch.uint8)
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    sptr = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    with torch.cuda.device(dev):
        st = lib.flint_attn_bwd(
            _ptr(q), _ptr(k), _ptr(v), _ptr(q_norm_w), _ptr(k_norm_w), _ptr(sinks),
            _ptr(pos_ids), _ptr(cu_seqlens), num_docs, _ptr(pad_mask), batch, seqlen, T,
            int(window), int(bool(use_rope)), float(rope_theta), float(eps), _ptr(out),
            _ptr(lse), _ptr(dout), _ptr(grads["dq"]), _ptr(grads["dk"]), _ptr(grads["dv"]),
            _ptr(grads["dq_norm_w"]), _ptr(grads["dk_norm_w"]), _ptr(grads["dsinks"]),
            _ptr(workspace), int(workspace.numel()), sptr)
    if st != 0:
        raise FlintError(st, lib.flint_attn_last_error().decode())
    attn_bwd.last_workspace = workspace
    return grads


def flint_attention(q, k, v, q_norm_w, k_norm_w, sinks, *, pos_ids=None, cu_seqlens=None,
                    pad_mask=None, window: int = 513, use_rope: bool = True,
                    rope_theta: float = 10000.0, eps: float = 1e-6):
    """Differentiable forward: returns (out [T,4096] bf16, lse [32,T] f32).

    Backpropagating a loss through ``out`` runs flint_attn_bwd and yields the
    gradients of q, k, v (cast to their dtype), q_norm_w, k_norm_w and sinks.
    lse is returned for inspection and receives no gradient.  Index and mask
    arguments are not differentiable.
    """
    return _FlintAttnFn.apply(q, k, v, q_norm_w, k_norm_w, sinks, pos_ids, cu_seqlens, pad_mask,
                              int(window), bool(use_rope), float(rope_theta), float(eps))


def _make_autograd_fn():
    import torch

    class FlintAttnFn(torch.autograd.Function):
        @staticmethod
        def forward(ctx, q, k, v, q_norm_w, k_norm_w, sinks, pos_ids, cu_seqlens, pad_mask, window,
                    use_rope, rope_theta, eps):
            cfg = dict(pos_ids=pos_ids, cu_seqlens=cu_seqlens, pad_mask=pad_mask, window=window,
                       use_rope=use_rope, rope_theta=rope_theta, eps=eps)
            out, lse = attn_fwd(q, k, v, q_norm_w, k_norm_w, sinks, **cfg)
            ctx.save_for_backward(q, k, v, q_norm_w, k_norm_w, sinks, out, lse)
            ctx.cfg = cfg
            ctx.mark_non_differentiable(lse)
            return out, lse

        @staticmethod
        def backward(ctx, dout, _dlse):
            q, k, v, q_norm_w, k_norm_w, sinks, out, lse = ctx.saved_tensors
            g = attn_bwd(q, k, v, q_norm_w, k_norm_w, sinks, out, lse,
                         dout.to(torch.bfloat16).contiguous(), **ctx.cfg)
            return (g["dq"].to(q.dtype), g["dk"].to(k.dtype), g["dv"].to(v.dtype),
                    g["dq_norm_w"].to(q_norm_w.dtype), g["dk_norm_w"].to(k_norm_w.dtype),
                    g["dsinks"].to(sinks.dtype), None, None, None, None, None, None, None)

    return FlintAttnFn


class _LazyFn:
    """Builds the autograd Function on first use, so importing the package
    does not import torch."""
    _fn = None

    def apply(self, *args):
        if _LazyFn._fn is None:
            _LazyFn._fn = _make_autograd_fn()
        return _LazyFn._fn.apply(*args)


_FlintAttnFn = _LazyFn()


def device_status(workspace, stream=None) -> int:
    """Synchronise and return the device-side status of the last call that
    used ``workspace`` (0 = FLINT_OK)."""
    import torch
    lib = load_library()
    if stream is None:
        stream = torch.cuda.current_stream(workspace.device)
    sptr = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    return int(lib.flint_attn_device_status(_ptr(workspace), sptr))


def attn_fwd_static(q, k, v, q_norm_w, k_norm_w, sinks, out, lse, *, pos_ids=None,
                    cu_seqlens=None, pad_mask=None, window: int = 513, use_rope: bool = True,
                    rope_theta: float = 10000.0, eps: float = 1e-6, stream=None) -> None:
    """flint_attn_fwd_static: the forward for callers that cannot allocate
    device memory when they run the layer.  The caller passes every buffer,
    outputs included; the kernels' scratch is a fixed device array inside the
    library (STATIC_SCRATCH_BYTES, about 16,000 tokens), shared by all calls,
    so calls that may overlap on the GPU must be serialised.  Nothing is
    allocated here."""
    import torch
    lib = load_library()
    T = int(q.shape[0])
    _check(q, "q", torch.bfloat16, (T, HQ, HEAD_DIM))
    _check(k, "k", torch.bfloat16, (T, HKV, HEAD_DIM))
    _check(v, "v", torch.bfloat16, (T, HKV, HEAD_DIM))
    _check(q_norm_w, "q_norm_w", torch.float32, (HEAD_DIM,))
    _check(k_norm_w, "k_norm_w", torch.float32, (HEAD_DIM,))
    _check(sinks, "sinks", torch.float32, (HQ,))
    _check(out, "out", torch.bfloat16, (T, HQ * HEAD_DIM))
    if lse is not None:
        _check(lse, "lse", torch.float32, (HQ, T))
    num_docs, batch, seqlen = 0, 0, 0
    if pos_ids is not None:
        _check(pos_ids, "pos_ids", torch.int32, (T,))
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", torch.int32)
        num_docs = int(cu_seqlens.numel()) - 1
    if pad_mask is not None:
        _check(pad_mask, "pad_mask", torch.uint8)
        batch, seqlen = int(pad_mask.shape[0]), int(pad_mask.shape[1])
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    sptr = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    with torch.cuda.device(q.device):
        st = lib.flint_attn_fwd_static(
            _ptr(q), _ptr(k), _ptr(v), _ptr(q_norm_w), _ptr(k_norm_w), _ptr(sinks),
            _ptr(pos_ids), _ptr(cu_seqlens), num_docs, _ptr(pad_mask), batch, seqlen, T,
            int(window), int(bool(use_rope)), float(rope_theta), float(eps), _ptr(out),
            _ptr(lse), sptr)
    if st != 0:
        raise FlintError(st, lib.flint_attn_last_error().decode())


def static_status(device=None, stream=None) -> int:
    """flint_attn_fwd_static_status: synchronise ``stream`` and return the
    device-side status of the last attn_fwd_static call that launched kernels
    (0 = FLINT_OK).  Reads one word; allocates nothing."""
    import torch
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    sptr = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    with torch.cuda.device(dev):
        return int(lib.flint_attn_fwd_static_status(sptr))


def _stream_ptr(stream, dev):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def qkv_proj(x, w_qkv, *, q=None, k=None, v=None, stream=None):
    """flint_qkv_proj: x [T, hidden] bf16, w_qkv [5120, hidden] bf16 (W_q, W_k,
    W_v stacked, Linear layout).  Returns (q [T,32,128], k [T,4,128],
    v [T,4,128]) bf16."""
    import torch
    lib = load_library()
    T, hidden = int(x.shape[0]), int(x.shape[1])
    _check(x, "x", torch.bfloat16, (T, hidden))
    _check(w_qkv, "w_qkv", torch.bfloat16, (HQ * HEAD_DIM + 2 * HKV * HEAD_DIM, hidden))
    dev = x.device
    q = torch.empty((T, HQ, HEAD_DIM), dtype=torch.bfloat16, device=dev) if q is None else q
    k = torch.empty((T, HKV, HEAD_DIM), dtype=torch.bfloat16, device=dev) if k is None else k
    v = torch.empty((T, HKV, HEAD_DIM), dtype=torch.bfloat16, device=dev) if v is None else v
    _check(q, "q", torch.bfloat16, (T, HQ, HEAD_DIM))
    _check(k, "k", torch.bfloat16, (T, HKV, HEAD_DIM))
    _check(v, "v", torch.bfloat16, (T, HKV, HEAD_DIM))
    with torch.cuda.device(dev):
        st = lib.flint_qkv_proj(_ptr(x), _ptr(w_qkv), T, hidden, _ptr(q), _ptr(k), _ptr(v),
                                _stream_ptr(stream, dev))
    if st != 0:
        raise FlintError(st, lib.flint_attn_last_error().decode())
    return q, k, v


def o_proj(attn_out, w_o, *, y=None, stream=None):
    """flint_o_proj: attn_out [T, 4096] bf16, w_o [hidden, 4096] bf16.
    Returns y [T, hidden] bf16."""
    import torch
    lib = load_library()
    T, hidden = int(attn_out.shape[0]), int(w_o.shape[0])
    _check(attn_out, "attn_out", torch.bfloat16, (T, HQ * HEAD_DIM))
    _check(w_o, "w_o", torch.bfloat16, (hidden, HQ * HEAD_DIM))
    dev = attn_out.device
    y = torch.empty((T, hidden), dtype=torch.bfloat16, device=dev) if y is None else y
    _check(y, "y", torch.bfloat16, (T, hidden))
    with torch.cuda.device(dev):
        st = lib.flint_o_proj(_ptr(attn_out), _ptr(w_o), T, hidden, _ptr(y), _stream_ptr(stream, dev))
    if st != 0:
        raise FlintError(st, lib.flint_attn_last_error().decode())
    return y


def attn_layer_fwd(x, w_qkv, w_o, q_norm_w, k_norm_w, sinks, *, pos_ids=None, cu_seqlens=None,
                   pad_mask=None, window: int = 513, use_rope: bool = True, rope_theta: float = 10000.0,
                   eps: float = 1e-6, out=None, workspace=None, stream=None, want_lse: bool = True) -> dict:
    """flint_attn_layer_fwd: the whole attention layer, x [T, hidden] -> y
    [T, hidden] (see include/flint_attn.h).  Returns a dict with y, the
    projections q, k, v, the attention output attn_out and lse.  ``out``: the
    same dict to write into."""
    import torch
    lib = load_library()
    T, hidden = int(x.shape[0]), int(x.shape[1])
    _check(x, "x", torch.bfloat16, (T, hidden))
    _check(w_qkv, "w_qkv", torch.bfloat16, (HQ * HEAD_DIM + 2 * HKV * HEAD_DIM, hidden))
    _check(w_o, "w_o", torch.bfloat16, (hidden, HQ * HEAD_DIM))
    _check(q_norm_w, "q_norm_w", torch.float32, (HEAD_DIM,))
    _check(k_norm_w, "k_norm_w", torch.float32, (HEAD_DIM,))
    _check(sinks, "sinks", torch.float32, (HQ,))
    num_docs, batch, seqlen, nseg = 0, 0, 0, 1
    if pos_ids is not None:
        _check(pos_ids, "pos_ids", torch.int32, (T,))
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", torch.int32)
        num_docs = int(cu_seqlens.numel()) - 1
        nseg = max(num_docs, 1)
    if pad_mask is not None:
        _check(pad_mask, "pad_mask", torch.uint8)
        batch, seqlen = int(pad_mask.shape[0]), int(pad_mask.shape[1])
        nseg = batch
    dev = x.device
    shapes = dict(q=(T, HQ, HEAD_DIM), k=(T, HKV, HEAD_DIM), v=(T, HKV, HEAD_DIM),
                  attn_out=(T, HQ * HEAD_DIM), y=(T, hidden))
    if out is None:
        out = {n: torch.empty(sh, dtype=torch.bfloat16, device=dev) for n, sh in shapes.items()}
        out["lse"] = torch.empty((HQ, T), dtype=torch.float32, device=dev) if want_lse else None
    for n, sh in shapes.items():
        _check(out[n], n, torch.bfloat16, sh)
    if out.get("lse") is not None:
        _check(out["lse"], "lse", torch.float32, (HQ, T))
    need = workspace_bytes(T, nseg)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check(workspace, "workspace", torch.uint8)
    with torch.cuda.device(dev):
        st = lib.flint_attn_layer_fwd(
            _ptr(x), _ptr(w_qkv), _ptr(w_o), _ptr(q_norm_w), _ptr(k_norm_w), _ptr(sinks), _ptr(pos_ids),
            _ptr(cu_seqlens), num_docs, _ptr(pad_mask), batch, seqlen, T, hidden, int(window),
            int(bool(use_rope)), float(rope_theta), float(eps), _ptr(out["q"]), _ptr(out["k"]),
            _ptr(out["v"]), _ptr(out["attn_out"]), _ptr(out["y"]), _ptr(out.get("lse")), _ptr(workspace),
            int(workspace.numel()), _stream_ptr(stream, dev))
    if st != 0:
        raise FlintError(st, lib.flint_attn_last_error().decode())
    attn_layer_fwd.last_workspace = workspace
    return out


def fp16_workspace_bytes(T: int, num_segments: int = 1) -> int:
    return int(load_library().flint_attn_fp16_workspace_bytes(int(T), int(num_segments)))


def attn_fwd_fp16(q, k, v, q_norm_w, k_norm_w, sinks, *, pos_ids=None, cu_seqlens=None,
                  pad_mask=None, window: int = 513, use_rope: bool = True,
                  rope_theta: float = 10000.0, eps: float = 1e-6, out=None, lse=None,
                  workspace=None, stream=None, want_lse: bool = True) -> Tuple[object, object]:
    """flint_attn_fwd_fp16, the FP16 attention-compute policy: q [T,32,128],
    k/v [T,4,128] float32 CUDA tensors; returns (out [T,4096] float16, lse
    [32,T] float32 or None).  Other arguments as for attn_fwd."""
    import torch
    lib = load_library()
    T = int(q.shape[0]) if q.dim() >= 1 else 0
    _check(q, "q", torch.float32, (T, HQ, HEAD_DIM))
    _check(k, "k", torch.float32, (T, HKV, HEAD_DIM))
    _check(v, "v", torch.float32, (T, HKV, HEAD_DIM))
    _check(q_norm_w, "q_norm_w", torch.float32, (HEAD_DIM,))
    _check(k_norm_w, "k_norm_w", torch.float32, (HEAD_DIM,))
    _check(sinks, "sinks", torch.float32, (HQ,))
    num_docs, batch, seqlen, nseg = 0, 0, 0, 1
    if pos_ids is not None:
        _check(pos_ids, "pos_ids", torch.int32, (T,))
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", torch.int32)
        num_docs = int(cu_seqlens.numel()) - 1
        nseg = max(num_docs, 1)
    if pad_mask is not None:
        _check(pad_mask, "pad_mask", torch.uint8)
        batch, seqlen = int(pad_mask.shape[0]), int(pad_mask.shape[1])
        nseg = batch
    dev = q.device
    if out is None:
        out = torch.empty((T, HQ * HEAD_DIM), dtype=torch.float16, device=dev)
    _check(out, "out", torch.float16, (T, HQ * HEAD_DIM))
    if lse is None and want_lse:
        lse = torch.empty((HQ, T), dtype=torch.float32, device=dev)
    if lse is not None:
        _check(lse, "lse", torch.float32, (HQ, T))
    if workspace is None:
        workspace = torch.empty(max(fp16_workspace_bytes(T, nseg), 256), dtype=torch.uint8, device=dev)
    _check(workspace, "workspace", torch.uint8)
    with torch.cuda.device(dev):
        st = lib.flint_attn_fwd_fp16(
            _ptr(q), _ptr(k), _ptr(v), _ptr(q_norm_w), _ptr(k_norm_w), _ptr(sinks), _ptr(pos_ids),
            _ptr(cu_seqlens), num_docs, _ptr(pad_mask), batch, seqlen, T, int(window),
            int(bool(use_rope)), float(rope_theta), float(eps), _ptr(out), _ptr(lse), _ptr(workspace),
            int(workspace.numel()), _stream_ptr(stream, dev))
    if st != 0:
        raise FlintError(st, lib.flint_attn_last_error().decode())
    attn_fwd_fp16.last_workspace = workspace
    return out, lse


def attn_fwd_heads(q, k, v, q_norm_w, k_norm_w, sinks, *, pos_ids=None, cu_seqlens=None,
                   pad_mask=None, window: int = 513, use_rope: bool = True, rope_theta: float = 10000.0,
                   eps: float = 1e-6, out=None, lse=None, workspace=None, stream=None,
                   want_lse: bool = True) -> Tuple[object, object]:
    """flint_attn_fwd_heads: the forward on a slice of kv_heads KV heads
    (q [T, 8 kv_heads, 128], k/v [T, kv_heads, 128], sinks [8 kv_heads]);
    returns (out [T, 8 kv_heads x 128] bf16, lse [8 kv_heads, T])."""
    import torch
    lib = load_library()
    T = int(q.shape[0]) if q.dim() >= 1 else 0
    ng = int(k.shape[1]) if k.dim() == 3 else 0
    nh = 8 * ng
    _check(q, "q", torch.bfloat16, (T, nh, HEAD_DIM))
    _check(k, "k", torch.bfloat16, (T, ng, HEAD_DIM))
    _check(v, "v", torch.bfloat16, (T, ng, HEAD_DIM))
    _check(q_norm_w, "q_norm_w", torch.float32, (HEAD_DIM,))
    _check(k_norm_w, "k_norm_w", torch.float32, (HEAD_DIM,))
    _check(sinks, "sinks", torch.float32, (nh,))
    num_docs, batch, seqlen, nseg = 0, 0, 0, 1
    if pos_ids is not None:
        _check(pos_ids, "pos_ids", torch.int32, (T,))
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", torch.int32)
        num_docs = int(cu_seqlens.numel()) - 1
        nseg = max(num_docs, 1)
    if pad_mask is not None:
        _check(pad_mask, "pad_mask", torch.uint8)
        batch, seqlen = int(pad_mask.shape[0]), int(pad_mask.shape[1])
        nseg = batch
    dev = q.device
    if out is None:
        out = torch.empty((T, nh * HEAD_DIM), dtype=torch.bfloat16, device=dev)
    _check(out, "out", torch.bfloat16, (T, nh * HEAD_DIM))
    if lse is None and want_lse:
        lse = torch.empty((nh, T), dtype=torch.float32, device=dev)
    if lse is not None:
        _check(lse, "lse", torch.float32, (nh, T))
    if workspace is None:
        workspace = torch.empty(max(workspace_bytes(T, nseg), 256), dtype=torch.uint8, device=dev)
    _check(workspace, "workspace", torch.uint8)
    with torch.cuda.device(dev):
        st = lib.flint_attn_fwd_heads(
            _ptr(q), _ptr(k), _ptr(v), _ptr(q_norm_w), _ptr(k_norm_w), _ptr(sinks), _ptr(pos_ids),
            _ptr(cu_seqlens), num_docs, _ptr(pad_mask), batch, seqlen, T, ng, int(window),
            int(bool(use_rope)), float(rope_theta), float(eps), _ptr(out), _ptr(lse), _ptr(workspace),
            int(workspace.numel()), _stream_ptr(stream, dev))
    if st != 0:
        raise FlintError(st, lib.flint_attn_last_error().decode())
    attn_fwd_heads.last_workspace = workspace
    return out, lse
