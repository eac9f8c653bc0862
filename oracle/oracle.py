"""Python face of the fp64 CPU attention oracle -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  It loads ``liboracle.so`` (built from
``attention_oracle.c`` by :func:`build`) and marshals arrays; all arithmetic is
in the C file, which states the definition it follows:

* the attention of the LTX-2 joint audio-video DiT block (video self, audio
  self with the key-padding mask on the zero-padded audio tail, v2a = audio
  queries over video keys/values, a2v = video queries over audio keys/values),
  "LTX-2: replicate audio stream across Ulysses ranks by default", Description;
* the merge of per-part softmax statistics over a key-range split,
  "feat(ltx2): tile-parallel video VAE and the two-stage pipeline", commit
  "Onboard Lightricks LTX-2.5".

Inputs are bf16 tensors (torch) or their raw uint16 bit patterns (numpy) in BSHD
layout; outputs are float64 numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attention_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``attention_oracle.c`` with gcc (IEEE fp64, no fast-math) and OpenMP."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", "-Wextra",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            u16p = ctypes.POINTER(ctypes.c_uint16)
            f64p = ctypes.POINTER(ctypes.c_double)
            i64p = ctypes.POINTER(ctypes.c_int64)
            ci = ctypes.c_int
            lib.oracle_attention.argtypes = [u16p, u16p, u16p, f64p, f64p, ci, ci, ci, ci, ci, ci,
                                             ctypes.c_double, i64p, ctypes.c_int64]
            lib.oracle_attention.restype = ci
            lib.oracle_attention_part.argtypes = [u16p, u16p, u16p, f64p, f64p, f64p, ci, ci, ci,
                                                  ci, ci, ci, ctypes.c_double, ci, ci]
            lib.oracle_attention_part.restype = ci
            lib.oracle_merge_partials.argtypes = [ci, ctypes.c_int64, ci, f64p, f64p, f64p, f64p,
                                                  f64p]
            lib.oracle_merge_partials.restype = ci
            lib.oracle_softmax_weights.argtypes = [u16p, u16p, f64p, ci, ci, ci, ci, ci, ci,
                                                   ctypes.c_double]
            lib.oracle_softmax_weights.restype = ci
            lib.oracle_num_threads.argtypes = []
            lib.oracle_num_threads.restype = ci
            _lib = lib
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle uses (``OMP_NUM_THREADS`` or all host cores)."""
    return int(_load().oracle_num_threads())


def _bits(x) -> np.ndarray:
    """bf16 tensor (torch) or uint16 bit array (numpy) -> contiguous uint16 numpy array."""
    if isinstance(x, np.ndarray):
        if x.dtype != np.uint16:
            raise TypeError("numpy inputs must be raw bf16 bit patterns (uint16)")
        return np.ascontiguousarray(x)
    import torch  # local: numpy-only callers need no torch
    if x.dtype != torch.bfloat16:
        raise TypeError("torch inputs must be bfloat16")
    return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _dims(q, k, v):
    if q.ndim != 4 or k.ndim != 4 or v.ndim != 4:
        raise ValueError("q, k, v must be [batch, len, heads, head_dim]")
    batch, q_len, heads, head_dim = q.shape
    if k.shape != v.shape or k.shape[0] != batch or k.shape[2:] != (heads, head_dim):
        raise ValueError("k and v must be [batch, kv_len, heads, head_dim] matching q")
    return batch, q_len, k.shape[1], heads, head_dim


def attention(q, k, v, scale: float, kv_valid_len: int | None = None, rows=None,
              return_lse: bool = False):
    """fp64 attention.  ``rows`` (optional): flat indices (b*q_len + i)*heads + h.

    Returns ``out`` as float64 [batch, q_len, heads, head_dim] (or [n_rows, head_dim]
    when ``rows`` is given), plus the natural-log LSE when ``return_lse``.
    """
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    batch, q_len, kv_len, heads, head_dim = _dims(qb, kb, vb)
    if kv_valid_len is None:
        kv_valid_len = kv_len
    if rows is None:
        out = np.empty((batch, q_len, heads, head_dim), dtype=np.float64)
        n = batch * q_len * heads
        rows_arr = None
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        n = rows_arr.size
        out = np.empty((n, head_dim), dtype=np.float64)
    lse = np.empty(n, dtype=np.float64) if return_lse else None
    rc = _load().oracle_attention(
        _ptr(qb, ctypes.c_uint16), _ptr(kb, ctypes.c_uint16), _ptr(vb, ctypes.c_uint16),
        _ptr(out, ctypes.c_double), _ptr(lse, ctypes.c_double) if lse is not None else None,
        batch, q_len, kv_len, int(kv_valid_len), heads, head_dim, float(scale),
        _ptr(rows_arr, ctypes.c_int64) if rows_arr is not None else None, int(n))
    if rc != 0:
        raise ValueError("oracle_attention rejected its arguments")
    if return_lse:
        return out, (lse if rows is not None else lse.reshape(batch, q_len, heads))
    return out


def attention_part(q, k, v, scale: float, j0: int, j1: int, kv_valid_len: int | None = None):
    """Attention over keys [j0, j1): (o_part BSHD, m_part [b,s,h], l_part [b,s,h])."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    batch, q_len, kv_len, heads, head_dim = _dims(qb, kb, vb)
    if kv_valid_len is None:
        kv_valid_len = kv_len
    o = np.empty((batch, q_len, heads, head_dim), dtype=np.float64)
    m = np.empty((batch, q_len, heads), dtype=np.float64)
    l = np.empty((batch, q_len, heads), dtype=np.float64)
    rc = _load().oracle_attention_part(
        _ptr(qb, ctypes.c_uint16), _ptr(kb, ctypes.c_uint16), _ptr(vb, ctypes.c_uint16),
        _ptr(o, ctypes.c_double), _ptr(m, ctypes.c_double), _ptr(l, ctypes.c_double),
        batch, q_len, kv_len, int(kv_valid_len), heads, head_dim, float(scale), int(j0), int(j1))
    if rc != 0:
        raise ValueError("oracle_attention_part rejected its arguments")
    return o, m, l


def merge_partials(o_parts, m_parts, l_parts, return_lse: bool = False):
    """Merge per-part (o, m, l) over a key-range split.  Shapes: o [P, rows, d], m/l [P, rows]."""
    o_parts = np.ascontiguousarray(o_parts, dtype=np.float64)
    m_parts = np.ascontiguousarray(m_parts, dtype=np.float64)
    l_parts = np.ascontiguousarray(l_parts, dtype=np.float64)
    n_parts, n_rows, head_dim = o_parts.shape
    if m_parts.shape != (n_parts, n_rows) or l_parts.shape != (n_parts, n_rows):
        raise ValueError("m_parts/l_parts must be [parts, rows]")
    out = np.empty((n_rows, head_dim), dtype=np.float64)
    lse = np.empty(n_rows, dtype=np.float64)
    rc = _load().oracle_merge_partials(n_parts, n_rows, head_dim, _ptr(o_parts, ctypes.c_double),
                                       _ptr(m_parts, ctypes.c_double),
                                       _ptr(l_parts, ctypes.c_double), _ptr(out, ctypes.c_double),
                                       _ptr(lse, ctypes.c_double))
    if rc != 0:
        raise ValueError("oracle_merge_partials rejected its arguments")
    return (out, lse) if return_lse else out


def softmax_weights(q, k, scale: float, kv_valid_len: int | None = None) -> np.ndarray:
    """The attention weights P [batch, heads, q_len, kv_len] (zero on masked keys)."""
    qb, kb = _bits(q), _bits(k)
    batch, q_len, heads, head_dim = qb.shape
    kv_len = kb.shape[1]
    if kv_valid_len is None:
        kv_valid_len = kv_len
    p = np.empty((batch, heads, q_len, kv_len), dtype=np.float64)
    rc = _load().oracle_softmax_weights(_ptr(qb, ctypes.c_uint16), _ptr(kb, ctypes.c_uint16),
                                        _ptr(p, ctypes.c_double), batch, q_len, kv_len,
                                        int(kv_valid_len), heads, head_dim, float(scale))
    if rc != 0:
        raise ValueError("oracle_softmax_weights rejected its arguments")
    return p
