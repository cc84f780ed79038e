"""FP64 CPU oracle for the Flint sink-aware GQA attention forward.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check in the package
entry module and the CPU-baseline leg of the benchmark are the only callers.
The product path (the CUDA library and its binding) never imports this
package, and this package never imports the product.

The arithmetic lives in ``flint_oracle.c`` (plain C, double precision); this
module builds it with gcc, loads it with ctypes and widens BF16 inputs to
float64 exactly.  See the C file's header for the definition it follows and
the passages it cites.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "flint_oracle.c")
_LIB = os.path.join(_HERE, "libflint_oracle.so")
_lock = threading.Lock()
_lib = None

HQ, HKV, D = 32, 4, 128


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, IEEE semantics, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared",
                               "-pthread", "-D_GNU_SOURCE", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            lib.flint_oracle_attn_fwd.restype = ctypes.c_int
            lib.flint_oracle_attn_fwd.argtypes = [
                ctypes.c_int64, P, P, P, P, P, P, P, P,
                ctypes.c_int32, ctypes.c_int32, ctypes.c_double, ctypes.c_double,
                ctypes.c_int32, ctypes.c_int64, P, P, P, ctypes.c_int32]
            lib.flint_oracle_rmsnorm.restype = None
            lib.flint_oracle_rmsnorm.argtypes = [P, P, ctypes.c_double, P]
            lib.flint_oracle_rope.restype = None
            lib.flint_oracle_rope.argtypes = [P, ctypes.c_int64, ctypes.c_double, P]
            lib.flint_oracle_doc_ids_thd.restype = ctypes.c_int
            lib.flint_oracle_doc_ids_thd.argtypes = [ctypes.c_int64, P, ctypes.c_int32, P]
            lib.flint_oracle_doc_ids_padmask.restype = ctypes.c_int
            lib.flint_oracle_doc_ids_padmask.argtypes = [ctypes.c_int32, ctypes.c_int32, P, P]
            lib.flint_oracle_round_bf16.restype = ctypes.c_double
            lib.flint_oracle_round_bf16.argtypes = [ctypes.c_double]
            lib.flint_oracle_round_fp16.restype = ctypes.c_double
            lib.flint_oracle_round_fp16.argtypes = [ctypes.c_double]
            _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f64(x) -> np.ndarray:
    """BF16 bit patterns (uint16) widen exactly; float arrays pass through."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return np.ascontiguousarray(x, dtype=np.float64)


def rmsnorm(x, w, eps=1e-6) -> np.ndarray:
    """Step 1 on a single head row of 128 values."""
    lib = _load()
    x = _f64(x).reshape(D).copy()
    w = _f64(w).reshape(D).copy()
    y = np.empty(D, np.float64)
    lib.flint_oracle_rmsnorm(_ptr(x), _ptr(w), float(eps), _ptr(y))
    return y


def rope(x, pos: int, theta=10000.0) -> np.ndarray:
    """Step 2 on a single head row of 128 values."""
    lib = _load()
    x = _f64(x).reshape(D).copy()
    y = np.empty(D, np.float64)
    lib.flint_oracle_rope(_ptr(x), int(pos), float(theta), _ptr(y))
    return y


def round_bf16(x: float) -> float:
    return _load().flint_oracle_round_bf16(float(x))


def round_fp16(x: float) -> float:
    return _load().flint_oracle_round_fp16(float(x))


def doc_ids(T: int, cu_seqlens=None, pad_mask=None) -> np.ndarray:
    """Segment id per token (-1 = padding) from THD boundaries or a [B,S]
    attention mask; one segment when neither is given."""
    lib = _load()
    doc = np.empty(max(T, 1), np.int32)
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(cu_seqlens, np.int32)
        rc = lib.flint_oracle_doc_ids_thd(T, _ptr(cu), len(cu) - 1, _ptr(doc))
        if rc != 0:
            raise ValueError("invalid cu_seqlens")
    elif pad_mask is not None:
        m = np.ascontiguousarray(pad_mask, np.uint8)
        B, S = m.shape
        if B * S != T:
            raise ValueError("pad_mask shape does not match T")
        lib.flint_oracle_doc_ids_padmask(B, S, _ptr(m), _ptr(doc))
    else:
        doc[:] = 0
    return doc[:T]


def attn_fwd(q, k, v, q_norm_w, k_norm_w, sinks, *, pos_ids=None,
             cu_seqlens=None, pad_mask=None, window=0, use_rope=False,
             rope_theta=10000.0, eps=1e-6, rows=None, qk_round=0,
             nthreads=0):
    """Evaluate the attention forward for query tokens ``rows`` (all if None).

    q [T,32,128], k/v [T,4,128] as BF16 bit patterns (uint16) or floats;
    weights [128]; sinks [32].  Returns (out [n,32,128], lse [n,32]) in FP64.
    ``qk_round``: 0 exact, 1 round normalised Q/K to BF16, 2 to FP16
    (precision-floor studies only).
    """
    lib = _load()
    qf = _f64(q)
    T = qf.shape[0]
    if qf.shape != (T, HQ, D):
        raise ValueError("q must be [T,32,128]")
    kf, vf = _f64(k), _f64(v)
    if kf.shape != (T, HKV, D) or vf.shape != (T, HKV, D):
        raise ValueError("k, v must be [T,4,128]")
    wq = _f64(q_norm_w).reshape(D).copy()
    wk = _f64(k_norm_w).reshape(D).copy()
    sk = np.ascontiguousarray(np.asarray(sinks, np.float64).reshape(HQ))
    doc = doc_ids(T, cu_seqlens, pad_mask)
    pos = None if pos_ids is None else np.ascontiguousarray(pos_ids, np.int32).reshape(T)
    if rows is None:
        r = None
        n = T
    else:
        r = np.ascontiguousarray(rows, np.int64).reshape(-1)
        n = r.size
    out = np.empty((max(n, 1), HQ, D), np.float64)
    lse = np.empty((max(n, 1), HQ), np.float64)
    rc = lib.flint_oracle_attn_fwd(T, _ptr(qf), _ptr(kf), _ptr(vf), _ptr(wq), _ptr(wk),
                                   _ptr(sk), _ptr(pos), _ptr(doc), int(window),
                                   int(bool(use_rope)), float(rope_theta), float(eps),
                                   int(qk_round), n, _ptr(r), _ptr(out), _ptr(lse),
                                   int(nthreads))
    if rc != 0:
        raise RuntimeError("oracle failed (%d)" % rc)
    return out[:n], lse[:n]


def attn_fwd_workload(w, rows="workload", qk_round=0, nthreads=0):
    """Run the oracle on a ``workloads.Workload``.  rows="workload" uses the
    workload's sampled rows (all rows if it has none)."""
    if isinstance(rows, str):
        rows = w.rows
    return attn_fwd(w.q, w.k, w.v, w.q_norm_w, w.k_norm_w, w.sinks,
                    pos_ids=w.pos_ids, cu_seqlens=w.cu_seqlens, pad_mask=w.pad_mask,
                    window=w.window, use_rope=w.use_rope, rope_theta=w.rope_theta,
                    eps=w.eps, rows=rows, qk_round=qk_round, nthreads=nthreads)


class use_library:
    """Context manager that points this module at another build of the
    oracle source (used by the tests that plant a mistake in a copy of the
    oracle to show that the pins catch it)."""

    def __init__(self, so_path: str):
        self.so_path = so_path
        self._saved = None

    def __enter__(self):
        global _lib
        _load()
        self._saved = _lib
        lib = ctypes.CDLL(self.so_path)
        for name in ("flint_oracle_attn_fwd", "flint_oracle_rmsnorm", "flint_oracle_rope",
                     "flint_oracle_doc_ids_thd", "flint_oracle_doc_ids_padmask",
                     "flint_oracle_round_bf16", "flint_oracle_round_fp16"):
            src = getattr(self._saved, name)
            dst = getattr(lib, name)
            dst.restype = src.restype
            dst.argtypes = src.argtypes
        with _lock:
            _lib = lib
        return lib

    def __exit__(self, *exc):
        global _lib
        with _lock:
            _lib = self._saved
        return False


def source_path() -> str:
    return _SRC
