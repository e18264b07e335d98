"""Exact, IO-aware fused attention forward for B200 (sm_100a).

Thin ctypes binding over ``libfa.so`` (C ABI declared in ``include/fa.h``).
Every function here only marshals arguments; all arithmetic runs in the CUDA
kernels of the library. There is no CPU fallback: if the library is missing
or the device is not an sm_100 GPU, calls fail loudly.

Names follow the C ABI: :func:`fa_fwd`, :func:`fa_fwd_kvlen`, :func:`fa_fwd_gqa`,
:func:`fa_fwd_splitkv`, :func:`fa_splitkv_workspace_bytes`,
:func:`fa_splitkv_default_splits`, :func:`fa_status_string`,
:func:`fa_last_device_error`, :func:`fa_watchdog_selftest`. :func:`attention`
is a convenience wrapper that allocates the outputs with torch and calls
:func:`fa_fwd` / :func:`fa_fwd_kvlen` / :func:`fa_fwd_gqa` on the current
stream; :func:`decode_attention` does the same for :func:`fa_fwd_splitkv`
(fewer queries than keys), allocating its workspace with torch.
"""
from __future__ import annotations

import ctypes
import math
import os
import re

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfa.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "fa.h")

FA_OK = 0
FA_ERR_INVALID_ARG = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_LAUNCH = 3
FA_ERR_TIMEOUT = 4

_lib = None


class FAError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}{': ' if what else ''}{fa_status_string(status)} ({status})")


def load_library(path: str = LIB_PATH):
    """Load libfa.so (raises if it has not been built)."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise ImportError(
            f"CUDA extension missing: {path} (build it with "
            "`python -m io_aware_exact_18_b200.build`)")
    lib = ctypes.CDLL(path)
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
    lib.fa_fwd.restype = i
    lib.fa_fwd_kvlen.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, vp]
    lib.fa_fwd_kvlen.restype = i
    lib.fa_fwd_gqa.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp, vp]
    lib.fa_fwd_gqa.restype = i
    sz = ctypes.c_size_t
    lib.fa_fwd_splitkv.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, i, vp, sz,
                                   vp]
    lib.fa_fwd_splitkv.restype = i
    lib.fa_fwd_splitkv_static.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, i,
                                          vp]
    lib.fa_fwd_splitkv_static.restype = i
    lib.fa_fwd_fp8.argtypes = [vp, vp, vp, f, f, f, vp, vp, i, i, i, i, i, f, i, vp, vp]
    lib.fa_fwd_fp8.restype = i
    lib.fa_fwd_splitkv_fp8.argtypes = [vp, vp, vp, f, f, f, vp, vp, i, i, i, i, i, i, f, i, vp,
                                       i, vp, sz, vp]
    lib.fa_fwd_splitkv_fp8.restype = i
    lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp, vp,
                           sz, vp]
    lib.fa_bwd.restype = i
    lib.fa_bwd_workspace_bytes.argtypes = [i, i, i]
    lib.fa_bwd_workspace_bytes.restype = sz
    lib.fa_splitkv_workspace_bytes.argtypes = [i, i, i, i, i]
    lib.fa_splitkv_workspace_bytes.restype = sz
    lib.fa_splitkv_default_splits.argtypes = [i, i, i, i, i, i]
    lib.fa_splitkv_default_splits.restype = i
    lib.fa_status_string.argtypes = [i]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_last_device_error.argtypes = [vp]
    lib.fa_last_device_error.restype = i
    lib.fa_watchdog_selftest.argtypes = [ctypes.c_uint64, vp]
    lib.fa_watchdog_selftest.restype = i
    if path == LIB_PATH:
        _lib = lib
    return lib


def declared_symbols(header: str = HEADER_PATH):
    """Function names declared in include/fa.h."""
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


def fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, stream) -> int:
    """C ABI fa_fwd; q,k,v,o,lse and stream are raw integers (device pointers, cudaStream_t)."""
    return load_library().fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, stream)


def fa_fwd_kvlen(q, k, v, o, lse, B, H, N, d, scale, causal, kv_len, stream) -> int:
    """C ABI fa_fwd_kvlen; kv_len is a device pointer to int32 [B] or 0/None."""
    return load_library().fa_fwd_kvlen(q, k, v, o, lse, B, H, N, d, scale, causal,
                                       kv_len, stream)


def fa_fwd_gqa(q, k, v, o, lse, B, H, H_kv, N, d, scale, causal, kv_len, stream) -> int:
    """C ABI fa_fwd_gqa: k, v have H_kv heads shared by groups of H / H_kv query heads."""
    return load_library().fa_fwd_gqa(q, k, v, o, lse, B, H, H_kv, N, d, scale, causal,
                                     kv_len, stream)


def fa_fwd_splitkv(q, k, v, o, lse, B, H, H_kv, Nq, Nk, d, scale, causal, kv_len,
                   num_splits, workspace, workspace_bytes, stream) -> int:
    """C ABI fa_fwd_splitkv: Nq query rows against Nk >= Nq keys, keys cut into
    num_splits ranges whose partial results are merged by log-sum-exp."""
    return load_library().fa_fwd_splitkv(q, k, v, o, lse, B, H, H_kv, Nq, Nk, d, scale,
                                         causal, kv_len, num_splits, workspace,
                                         workspace_bytes, stream)


def fa_fwd_splitkv_static(q, k, v, o, lse, B, H, H_kv, Nq, Nk, d, scale, causal, kv_len,
                          num_splits, stream) -> int:
    """C ABI fa_fwd_splitkv_static: fa_fwd_splitkv with the library's own
    per-device scratch (FA_STATIC_SCRATCH_BYTES), for callers that cannot
    allocate device memory at call time. Calls overlapping on the GPU race on
    the one scratch."""
    return load_library().fa_fwd_splitkv_static(q, k, v, o, lse, B, H, H_kv, Nq, Nk, d, scale,
                                                causal, kv_len, num_splits, stream)


FA_STATIC_SCRATCH_BYTES = 16 << 20


def fa_splitkv_workspace_bytes(B, H, Nq, d, num_splits) -> int:
    return int(load_library().fa_splitkv_workspace_bytes(B, H, Nq, d, num_splits))


def fa_splitkv_default_splits(B, H, H_kv, Nq, Nk, d) -> int:
    return int(load_library().fa_splitkv_default_splits(B, H, H_kv, Nq, Nk, d))


def fa_fwd_fp8(q, k, v, q_descale, k_descale, v_descale, o, lse, B, H, H_kv, N, d, scale,
               causal, kv_len, stream) -> int:
    """C ABI fa_fwd_fp8: e4m3 q, k, v with per-tensor descales; bf16 O, fp32 lse."""
    return load_library().fa_fwd_fp8(q, k, v, q_descale, k_descale, v_descale, o, lse, B, H,
                                     H_kv, N, d, scale, causal, kv_len, stream)


def fa_fwd_splitkv_fp8(q, k, v, q_descale, k_descale, v_descale, o, lse, B, H, H_kv, Nq, Nk,
                       d, scale, causal, kv_len, num_splits, workspace, workspace_bytes,
                       stream) -> int:
    """C ABI fa_fwd_splitkv_fp8: the split-KV forward on e4m3 q, k, v with
    per-tensor descales; bf16 O, fp32 lse."""
    return load_library().fa_fwd_splitkv_fp8(q, k, v, q_descale, k_descale, v_descale, o, lse,
                                             B, H, H_kv, Nq, Nk, d, scale, causal, kv_len,
                                             num_splits, workspace, workspace_bytes, stream)


def fa_bwd(q, k, v, o, lse, d_o, dq, dk, dv, B, H, H_kv, N, d, scale, causal, kv_len,
           workspace, workspace_bytes, stream) -> int:
    """C ABI fa_bwd: dq, dk, dv of the forward for the output gradient d_o."""
    return load_library().fa_bwd(q, k, v, o, lse, d_o, dq, dk, dv, B, H, H_kv, N, d, scale,
                                 causal, kv_len, workspace, workspace_bytes, stream)


def fa_bwd_workspace_bytes(B, H, N) -> int:
    return int(load_library().fa_bwd_workspace_bytes(B, H, N))


def fa_status_string(status: int) -> str:
    try:
        return load_library().fa_status_string(int(status)).decode()
    except ImportError:
        return f"status {status}"


def fa_last_device_error(stream) -> int:
    return load_library().fa_last_device_error(stream)


def fa_watchdog_selftest(limit_ns: int, stream) -> int:
    """C ABI fa_watchdog_selftest: one bounded wait that is made to run out."""
    return load_library().fa_watchdog_selftest(int(limit_ns), stream)


def _ptr(t):
    return None if t is None else t.data_ptr()


def attention(q, k, v, scale=None, causal=False, kv_len=None, out=None, lse=None,
              stream=None, check=True):
    """O, lse = attention(q, k, v) for bf16 CUDA tensors q [B, H, N, d] and
    k, v [B, H_kv, N, d] (H_kv == H, or H a multiple of H_kv for grouped /
    multi-query attention).

    Allocates O (bf16) and lse (fp32) unless given, calls the C ABI on the
    current torch stream (or `stream`), and raises FAError on a bad status.
    """
    import torch
    if q.dtype != torch.bfloat16 or k.dtype != torch.bfloat16 or v.dtype != torch.bfloat16:
        raise TypeError("q, k, v must be bfloat16")
    if not (q.is_cuda and k.is_cuda and v.is_cuda):
        raise ValueError("q, k, v must be CUDA tensors (no CPU fallback)")
    if q.dim() != 4 or k.dim() != 4 or k.shape != v.shape or \
            (q.shape[0], q.shape[2], q.shape[3]) != (k.shape[0], k.shape[2], k.shape[3]):
        raise ValueError(f"q [B,H,N,d] and k, v [B,H_kv,N,d] expected, got "
                         f"{q.shape} {k.shape} {v.shape}")
    if not (q.is_contiguous() and k.is_contiguous() and v.is_contiguous()):
        raise ValueError("q, k, v must be contiguous")
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    s = stream if stream is not None else torch.cuda.current_stream(q.device).cuda_stream
    H_kv = k.shape[1]
    if kv_len is not None and (kv_len.dtype != torch.int32 or not kv_len.is_cuda
                               or kv_len.shape != (B,)):
        raise ValueError("kv_len must be a CUDA int32 tensor of shape [B]")
    if H_kv != H:
        st = fa_fwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, H_kv, N, d,
                        float(scale), int(bool(causal)), _ptr(kv_len), s)
    elif kv_len is None:
        st = fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, N, d,
                    float(scale), int(bool(causal)), s)
    else:
        st = fa_fwd_kvlen(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, N, d,
                          float(scale), int(bool(causal)), _ptr(kv_len), s)
    if check and st != FA_OK:
        raise FAError(st, "fa_fwd")
    return out, lse


def decode_attention(q, k, v, scale=None, causal=False, kv_len=None, num_splits=None,
                     out=None, lse=None, workspace=None, stream=None, check=True):
    """O, lse for bf16 CUDA tensors q [B, H, Nq, d] and k, v [B, H_kv, Nk, d]
    with Nq <= Nk (query row i at key position i + Nk - Nq), through
    fa_fwd_splitkv. num_splits=None takes fa_splitkv_default_splits. The
    workspace (if any) is allocated with torch unless given as a CUDA uint8
    tensor of at least fa_splitkv_workspace_bytes bytes.
    """
    import torch
    if q.dtype != torch.bfloat16 or k.dtype != torch.bfloat16 or v.dtype != torch.bfloat16:
        raise TypeError("q, k, v must be bfloat16")
    if not (q.is_cuda and k.is_cuda and v.is_cuda):
        raise ValueError("q, k, v must be CUDA tensors (no CPU fallback)")
    if q.dim() != 4 or k.dim() != 4 or k.shape != v.shape or \
            (q.shape[0], q.shape[3]) != (k.shape[0], k.shape[3]):
        raise ValueError(f"q [B,H,Nq,d] and k, v [B,H_kv,Nk,d] expected, got "
                         f"{q.shape} {k.shape} {v.shape}")
    if not (q.is_contiguous() and k.is_contiguous() and v.is_contiguous()):
        raise ValueError("q, k, v must be contiguous")
    B, H, Nq, d = q.shape
    H_kv, Nk = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if num_splits is None:
        num_splits = fa_splitkv_default_splits(B, H, H_kv, Nq, Nk, d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    if kv_len is not None and (kv_len.dtype != torch.int32 or not kv_len.is_cuda
                               or kv_len.shape != (B,)):
        raise ValueError("kv_len must be a CUDA int32 tensor of shape [B]")
    need = fa_splitkv_workspace_bytes(B, H, Nq, d, num_splits)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    s = stream if stream is not None else torch.cuda.current_stream(q.device).cuda_stream
    st = fa_fwd_splitkv(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, H_kv, Nq, Nk,
                        d, float(scale), int(bool(causal)), _ptr(kv_len), int(num_splits),
                        _ptr(workspace), ws_bytes, s)
    if check and st != FA_OK:
        raise FAError(st, "fa_fwd_splitkv")
    return out, lse


def attention_bwd(q, k, v, o, lse, d_o, scale=None, causal=False, kv_len=None, dq=None,
                  dk=None, dv=None, workspace=None, stream=None, check=True):
    """dq, dk, dv for bf16 CUDA tensors of a forward call attention(q, k, v)
    that returned o and lse, and the output gradient d_o (bf16, like o).
    Allocates the gradients and the workspace with torch unless given."""
    import torch
    for t in (q, k, v, o, d_o):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v, o, d_o must be contiguous bf16 CUDA tensors")
    if lse.dtype != torch.float32 or not lse.is_cuda or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 CUDA tensor")
    B, H, N, d = q.shape
    H_kv = k.shape[1]
    if k.shape != (B, H_kv, N, d) or v.shape != k.shape or o.shape != q.shape or \
            d_o.shape != q.shape or lse.shape != (B, H, N):
        raise ValueError("shapes of q, k, v, o, lse, d_o do not match")
    if kv_len is not None and (kv_len.dtype != torch.int32 or not kv_len.is_cuda
                               or kv_len.shape != (B,)):
        raise ValueError("kv_len must be a CUDA int32 tensor of shape [B]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = fa_bwd_workspace_bytes(B, H, N)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    s = stream if stream is not None else torch.cuda.current_stream(q.device).cuda_stream
    st = fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(d_o), _ptr(dq), _ptr(dk),
                _ptr(dv), B, H, H_kv, N, d, float(scale), int(bool(causal)), _ptr(kv_len),
                _ptr(workspace), workspace.numel() * workspace.element_size(), s)
    if check and st != FA_OK:
        raise FAError(st, "fa_bwd")
    return dq, dk, dv


def attention_fp8(q8, k8, v8, q_descale, k_descale, v_descale, scale=None, causal=False,
                  kv_len=None, out=None, lse=None, stream=None, check=True):
    """O (bf16), lse for e4m3 CUDA tensors (torch.float8_e4m3fn or uint8 codes)
    q8 [B, H, N, d] and k8, v8 [B, H_kv, N, d] with per-tensor descales,
    through fa_fwd_fp8."""
    import torch
    for t in (q8, k8, v8):
        if t.element_size() != 1 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q8, k8, v8 must be contiguous one-byte CUDA tensors")
    B, H, N, d = q8.shape
    H_kv = k8.shape[1]
    if k8.shape != (B, H_kv, N, d) or v8.shape != k8.shape:
        raise ValueError(f"bad shapes {q8.shape} {k8.shape} {v8.shape}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q8.device)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q8.device)
    s = stream if stream is not None else torch.cuda.current_stream(q8.device).cuda_stream
    st = fa_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), float(q_descale), float(k_descale),
                    float(v_descale), _ptr(out), _ptr(lse), B, H, H_kv, N, d, float(scale),
                    int(bool(causal)), _ptr(kv_len), s)
    if check and st != FA_OK:
        raise FAError(st, "fa_fwd_fp8")
    return out, lse


def decode_attention_fp8(q8, k8, v8, q_descale, k_descale, v_descale, scale=None,
                         causal=False, kv_len=None, num_splits=None, out=None, lse=None,
                         workspace=None, stream=None, check=True):
    """O (bf16), lse for e4m3 CUDA tensors q8 [B, H, Nq, d] and k8, v8
    [B, H_kv, Nk, d] (Nq <= Nk) with per-tensor descales, through
    fa_fwd_splitkv_fp8 (key ranges merged by their log-sum-exp)."""
    import torch
    for t in (q8, k8, v8):
        if t.element_size() != 1 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q8, k8, v8 must be contiguous one-byte CUDA tensors")
    if q8.dim() != 4 or k8.dim() != 4 or k8.shape != v8.shape or \
            (q8.shape[0], q8.shape[3]) != (k8.shape[0], k8.shape[3]):
        raise ValueError(f"q [B,H,Nq,d] and k, v [B,H_kv,Nk,d] expected, got "
                         f"{q8.shape} {k8.shape} {v8.shape}")
    B, H, Nq, d = q8.shape
    H_kv, Nk = k8.shape[1], k8.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if num_splits is None:
        num_splits = fa_splitkv_default_splits(B, H, H_kv, Nq, Nk, d)
    if out is None:
        out = torch.empty((B, H, Nq, d), dtype=torch.bfloat16, device=q8.device)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q8.device)
    if kv_len is not None and (kv_len.dtype != torch.int32 or not kv_len.is_cuda
                               or kv_len.shape != (B,)):
        raise ValueError("kv_len must be a CUDA int32 tensor of shape [B]")
    need = fa_splitkv_workspace_bytes(B, H, Nq, d, num_splits)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q8.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    s = stream if stream is not None else torch.cuda.current_stream(q8.device).cuda_stream
    st = fa_fwd_splitkv_fp8(_ptr(q8), _ptr(k8), _ptr(v8), float(q_descale), float(k_descale),
                            float(v_descale), _ptr(out), _ptr(lse), B, H, H_kv, Nq, Nk, d,
                            float(scale), int(bool(causal)), _ptr(kv_len), int(num_splits),
                            _ptr(workspace), ws_bytes, s)
    if check and st != FA_OK:
        raise FAError(st, "fa_fwd_splitkv_fp8")
    return out, lse
