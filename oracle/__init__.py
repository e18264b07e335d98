"""CPU oracle for exact attention (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import this package. The product library never does.

Two independent routes to the same result:

* :func:`attention` -- the plain definition in fp64 C (``attn_ref.c``): every
  score row is materialised in full and the softmax is taken in two passes.
  This follows "FlashAttention (UR)", section "Problem of standard attention".
* :func:`attention_bwd` -- the gradients dQ, dK, dV of the same definition for
  a given dO (chain rule through the row softmax, one query row at a time), in
  fp64 C. The pages state no backward algorithm; this is the exact gradient.
* :func:`attention_bwd_dq_rows` -- dQ of selected query rows only (the same
  definition; dQ row i depends on row i alone), for checks at full size.
* :func:`attention_bwd_kv_rows` -- dK and dV of selected key rows only (the
  same definition, every query row's softmax still taken in full), for
  checks at full size.
* :mod:`oracle.fp8` -- e4m3 decoding by the format's definition, feeding the
  fp64 attention of the dequantized tensors.
* :func:`online.attention_online` -- a blockwise online-softmax evaluation in
  numpy (running row max and running sum of exponentials, rescaled per key
  block), following section "Online softmax" of the same page. It exists only
  so the tests can check that the two evaluation orders agree.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_ref.c")
_LIB_PATH = os.path.join(_HERE, "_attn_ref.so")
_lock = threading.Lock()
_lib = None


def build(src: str = _SRC, out: str = _LIB_PATH, extra_flags=()) -> str:
    """Compile the oracle with gcc (fp64, OpenMP, no fast-math)."""
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
           *extra_flags, src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _bind(lib):
    dp = ctypes.POINTER(ctypes.c_double)
    i32p = ctypes.POINTER(ctypes.c_int32)
    u16p = ctypes.POINTER(ctypes.c_uint16)
    c_int, c_double = ctypes.c_int, ctypes.c_double
    lib.oracle_attn_general.argtypes = [dp, dp, dp, u16p, u16p, u16p, dp, dp, c_int, c_int,
                                         c_int, c_int, c_int, c_int, c_double, c_int, i32p,
                                         i32p, c_int, c_int]
    lib.oracle_attn_general.restype = c_int
    lib.oracle_attn_bwd.argtypes = [dp, dp, dp, dp, u16p, u16p, u16p, u16p, dp, dp, dp, c_int,
                                    c_int, c_int, c_int, c_int, c_double, c_int, i32p, c_int]
    lib.oracle_attn_bwd.restype = c_int
    lib.oracle_attn_bwd_dq_rows.argtypes = [u16p, u16p, u16p, u16p, dp, c_int, c_int, c_int,
                                            c_int, c_int, c_double, c_int, i32p, i32p, c_int,
                                            c_int]
    lib.oracle_attn_bwd_dq_rows.restype = c_int
    lib.oracle_attn_bwd_kv_rows.argtypes = [u16p, u16p, u16p, u16p, dp, dp, c_int, c_int, c_int,
                                            c_int, c_int, c_double, c_int, i32p, i32p, c_int,
                                            c_int]
    lib.oracle_attn_bwd_kv_rows.restype = c_int
    lib.oracle_max_threads.argtypes = []
    lib.oracle_max_threads.restype = c_int
    return lib


def load(path: str = _LIB_PATH):
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if path != _LIB_PATH:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            if (not os.path.exists(_LIB_PATH)
                    or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
                build()
            _lib = _bind(ctypes.CDLL(_LIB_PATH))
        return _lib


def max_threads() -> int:
    return int(load().oracle_max_threads())


def _as_numpy(x):
    """torch tensor or array -> (numpy array, is_bf16)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), True
            return x.to(torch.float64).numpy(), False
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(x)
    if a.dtype == np.uint16:
        return a, True
    return np.ascontiguousarray(a, dtype=np.float64), False


def attention(q, k, v, scale, causal=False, kv_len=None, rows=None,
              nthreads=0, lib=None):
    """Exact attention in fp64.

    q: [B, H, Nq, d]; k, v: [B, Hkv, Nk, d] with H a multiple of Hkv (query
    head h uses K/V head h // (H // Hkv); Hkv == H is plain multi-head
    attention) and Nq <= Nk (query row i stands at key position i + Nk - Nq;
    Nq == Nk is ordinary self-attention), as torch bf16 / float tensors or
    numpy arrays (uint16 arrays are read as bf16 bit patterns). kv_len: None
    or [B] ints. rows: None (all rows) or a list of query-row indices
    evaluated in every (b, h). Returns (o [B,H,R,d] float64, lse [B,H,R]
    float64), R = Nq or len(rows).
    """
    lib = lib or load()
    qa, qb16 = _as_numpy(q)
    ka, kb16 = _as_numpy(k)
    va, vb16 = _as_numpy(v)
    if not (qb16 == kb16 == vb16):
        raise TypeError("q, k, v must share one element type")
    if qa.ndim != 4 or ka.shape != va.shape or ka.ndim != 4:
        raise ValueError(f"bad shapes {qa.shape} {ka.shape} {va.shape}")
    B, H, Nq, d = qa.shape
    Hkv, N = ka.shape[1], ka.shape[2]
    if ka.shape != (B, Hkv, N, d) or Hkv < 1 or H % Hkv or Nq > N:
        raise ValueError(f"bad shapes {qa.shape} {ka.shape} {va.shape}")
    kvp = None
    if kv_len is not None:
        kvl = np.ascontiguousarray(np.asarray(
            kv_len.cpu().numpy() if hasattr(kv_len, "cpu") else kv_len,
            dtype=np.int32))
        if kvl.shape != (B,):
            raise ValueError("kv_len must have shape [B]")
        kvp = kvl.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    R = Nq if rows is None else len(rows)
    o = np.zeros((B, H, R, d), dtype=np.float64)
    lse = np.zeros((B, H, R), dtype=np.float64)
    dp = ctypes.POINTER(ctypes.c_double)
    u16p = ctypes.POINTER(ctypes.c_uint16)
    rp = None
    if rows is not None:
        ra = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
        rp = ra.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    if qb16:
        ptrs = (None, None, None, qa.ctypes.data_as(u16p), ka.ctypes.data_as(u16p),
                va.ctypes.data_as(u16p))
    else:
        ptrs = (qa.ctypes.data_as(dp), ka.ctypes.data_as(dp), va.ctypes.data_as(dp),
                None, None, None)
    rc = lib.oracle_attn_general(*ptrs, o.ctypes.data_as(dp), lse.ctypes.data_as(dp), B, H,
                                 Hkv, Nq, N, d, float(scale), int(bool(causal)), kvp, rp, R,
                                 int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle returned error {rc}")
    return o, lse


def attention_bwd(q, k, v, do, scale, causal=False, kv_len=None, nthreads=0, lib=None):
    """Exact gradients in fp64 of attention(q, k, v) for the output gradient do.

    q, do: [B, H, N, d]; k, v: [B, Hkv, N, d] (square, Nq == Nk == N; grouped
    heads as in :func:`attention`), all bf16 torch tensors / uint16 arrays or
    all float. Returns (dq [B,H,N,d], dk [B,Hkv,N,d], dv [B,Hkv,N,d]) float64;
    dk and dv of a shared K/V head sum over its group of query heads.
    """
    lib = lib or load()
    arrs = [_as_numpy(x) for x in (q, k, v, do)]
    if len({b for _, b in arrs}) != 1:
        raise TypeError("q, k, v, do must share one element type")
    (qa, bits), (ka, _), (va, _), (da, _) = arrs
    if qa.ndim != 4 or ka.shape != va.shape or da.shape != qa.shape:
        raise ValueError(f"bad shapes {qa.shape} {ka.shape} {va.shape} {da.shape}")
    B, H, N, d = qa.shape
    Hkv = ka.shape[1]
    if ka.shape != (B, Hkv, N, d) or Hkv < 1 or H % Hkv:
        raise ValueError(f"bad shapes {qa.shape} {ka.shape}")
    kvp = None
    if kv_len is not None:
        kvl = np.ascontiguousarray(np.asarray(
            kv_len.cpu().numpy() if hasattr(kv_len, "cpu") else kv_len, dtype=np.int32))
        if kvl.shape != (B,):
            raise ValueError("kv_len must have shape [B]")
        kvp = kvl.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    dq = np.zeros((B, H, N, d), dtype=np.float64)
    dk = np.zeros((B, Hkv, N, d), dtype=np.float64)
    dv = np.zeros((B, Hkv, N, d), dtype=np.float64)
    dp = ctypes.POINTER(ctypes.c_double)
    u16p = ctypes.POINTER(ctypes.c_uint16)
    if bits:
        ptrs = (None,) * 4 + tuple(a.ctypes.data_as(u16p) for a in (qa, ka, va, da))
    else:
        ptrs = tuple(a.ctypes.data_as(dp) for a in (qa, ka, va, da)) + (None,) * 4
    rc = lib.oracle_attn_bwd(*ptrs, dq.ctypes.data_as(dp), dk.ctypes.data_as(dp),
                             dv.ctypes.data_as(dp), B, H, Hkv, N, d, float(scale),
                             int(bool(causal)), kvp, int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle returned error {rc}")
    return dq, dk, dv


def attention_bwd_dq_rows(q, k, v, do, scale, rows, causal=False, kv_len=None, nthreads=0,
                          lib=None):
    """dQ of the given query rows of every (b, h), in fp64: [B, H, len(rows), d].
    Same definition as attention_bwd (dQ row i needs row i's P, dP and D only);
    bf16 torch tensors or uint16 arrays."""
    lib = lib or load()
    arrs = [_as_numpy(x) for x in (q, k, v, do)]
    if not all(b for _, b in arrs):
        raise TypeError("q, k, v, do must be bf16")
    (qa, _), (ka, _), (va, _), (da, _) = arrs
    B, H, N, d = qa.shape
    Hkv = ka.shape[1]
    if ka.shape != (B, Hkv, N, d) or va.shape != ka.shape or da.shape != qa.shape:
        raise ValueError("bad shapes")
    ra = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
    kvp = None
    if kv_len is not None:
        kvl = np.ascontiguousarray(np.asarray(
            kv_len.cpu().numpy() if hasattr(kv_len, "cpu") else kv_len, dtype=np.int32))
        kvp = kvl.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    out = np.zeros((B, H, len(ra), d), dtype=np.float64)
    u16p = ctypes.POINTER(ctypes.c_uint16)
    rc = lib.oracle_attn_bwd_dq_rows(*(a.ctypes.data_as(u16p) for a in (qa, ka, va, da)),
                                     out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), B, H,
                                     Hkv, N, d, float(scale), int(bool(causal)), kvp,
                                     ra.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                     len(ra), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle returned error {rc}")
    return out


def attention_bwd_kv_rows(q, k, v, do, scale, rows, causal=False, kv_len=None, nthreads=0,
                          lib=None):
    """dK and dV of the given key rows of every (b, K/V head), in fp64: two
    arrays [B, Hkv, len(rows), d]. Same definition as attention_bwd (each
    query row's softmax and D_i are computed over all its keys; only the sums
    into dK and dV are restricted to the selected keys); bf16 torch tensors
    or uint16 arrays, square (Nq == Nk)."""
    lib = lib or load()
    arrs = [_as_numpy(x) for x in (q, k, v, do)]
    if not all(b for _, b in arrs):
        raise TypeError("q, k, v, do must be bf16")
    (qa, _), (ka, _), (va, _), (da, _) = arrs
    B, H, N, d = qa.shape
    Hkv = ka.shape[1]
    if ka.shape != (B, Hkv, N, d) or va.shape != ka.shape or da.shape != qa.shape:
        raise ValueError("bad shapes")
    ra = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
    kvp = None
    if kv_len is not None:
        kvl = np.ascontiguousarray(np.asarray(
            kv_len.cpu().numpy() if hasattr(kv_len, "cpu") else kv_len, dtype=np.int32))
        kvp = kvl.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    dk = np.zeros((B, Hkv, len(ra), d), dtype=np.float64)
    dv = np.zeros((B, Hkv, len(ra), d), dtype=np.float64)
    u16p = ctypes.POINTER(ctypes.c_uint16)
    dp = ctypes.POINTER(ctypes.c_double)
    rc = lib.oracle_attn_bwd_kv_rows(*(a.ctypes.data_as(u16p) for a in (qa, ka, va, da)),
                                     dk.ctypes.data_as(dp), dv.ctypes.data_as(dp), B, H, Hkv, N,
                                     d, float(scale), int(bool(causal)), kvp,
                                     ra.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                     len(ra), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle returned error {rc}")
    return dk, dv
