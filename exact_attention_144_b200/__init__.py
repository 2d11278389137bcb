"""Exact attention for NVIDIA B200 (sm_100a): thin Python binding of the C ABI.

The functions here carry the C entry points' names (``fa_fwd``, ``fa_fwd_f16``,
``fa_bwd``, ``fa_bwd_f16``, ...) and only marshal arguments: they check torch
tensors, allocate outputs when asked, and pass raw device pointers and the
current CUDA stream to ``libfa_b200.so``.  Every step of the computation runs
in the library's CUDA kernels; there is no other implementation to fall back
on: the first call fails loudly when the library has not been built.

Layout: q, k, v, o, dout, dq, dk, dv are contiguous [B, N, H, d] tensors of
bfloat16 (``fa_fwd``/``fa_bwd``) or float16 (``*_f16``); lse is a contiguous
[B, H, N] float32 tensor (natural log).
"""
from __future__ import annotations

import ctypes
import math
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfa_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "fa_b200.h")

_lib = None


class FwdPlan(ctypes.Structure):
    """fa_fwd_plan_t: how the forward decomposes a problem (see fa_fwd_plan)."""
    _fields_ = [("kernel", ctypes.c_int), ("unit_rows", ctypes.c_int),
                ("kv_tile_rows", ctypes.c_int), ("n_units", ctypes.c_int),
                ("n_kv_tiles", ctypes.c_int), ("n_split", ctypes.c_int), ("grid", ctypes.c_int),
                ("balanced", ctypes.c_int), ("scratch_bytes", ctypes.c_longlong)]

    def as_dict(self) -> dict:
        return {name: getattr(self, name) for name, _ in self._fields_}


def _load() -> ctypes.CDLL:
    """Load libfa_b200.so once; raise if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is not built; run `python -m exact_attention_144_b200.build` "
            "(nvcc, sm_100a). There is no fallback implementation.")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, vp]
    lib.fa_fwd_f16.argtypes = lib.fa_fwd.argtypes
    lib.fa_bwd.argtypes = [vp] * 9 + [i, i, i, i, f, vp]
    lib.fa_bwd_f16.argtypes = lib.fa_bwd.argtypes
    lib.fa_bwd_noalloc.argtypes = lib.fa_bwd.argtypes
    lib.fa_fwd_ex.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, ctypes.c_uint, vp]
    lib.fa_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, f, f, f, ctypes.c_uint, vp]
    lib.fa_bwd_ex.argtypes = [vp] * 9 + [i, i, i, i, f, i, ctypes.c_uint, vp]
    lib.fa_fwd_qkvpacked.argtypes = [vp, vp, vp, i, i, i, i, f, i, ctypes.c_uint, vp]
    lib.fa_bwd_qkvpacked.argtypes = [vp] * 5 + [i, i, i, i, f, i, ctypes.c_uint, vp]
    lib.fa_fwd_varlen.argtypes = [vp] * 6 + [i, i, i, i, i, f, i, ctypes.c_uint, vp]
    lib.fa_bwd_varlen.argtypes = [vp] * 10 + [i, i, i, i, i, f, i, ctypes.c_uint, vp]
    lib.fa_varlen_bounds.argtypes = [ctypes.POINTER(ctypes.c_int), i, i, i,
                                     ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
    lib.fa_varlen_bounds.restype = i
    for n in ("fa_fwd", "fa_fwd_f16", "fa_bwd", "fa_bwd_f16", "fa_bwd_noalloc", "fa_fwd_ex", "fa_fwd_fp8",
              "fa_bwd_ex", "fa_fwd_qkvpacked", "fa_bwd_qkvpacked", "fa_fwd_varlen",
              "fa_bwd_varlen"):
        getattr(lib, n).restype = i
    lib.fa_status_string.argtypes = [i]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_get_device_status.argtypes = [ctypes.POINTER(ctypes.c_ulonglong), i]
    lib.fa_get_device_status.restype = i
    lib.fa_selftest_bounded_wait.argtypes = [ctypes.c_uint, ctypes.POINTER(ctypes.c_ulonglong)]
    lib.fa_selftest_bounded_wait.restype = i
    lib.fa_version.restype = i
    lib.fa_set_kernel_events.argtypes = [vp, vp, vp, vp]
    lib.fa_set_kernel_events.restype = i
    lib.fa_kernel_launches.restype = ctypes.c_ulonglong
    lib.fa_scratch_allocs.restype = ctypes.c_ulonglong
    lib.fa_last_cuda_error.restype = i
    lib.fa_selftest_exp2.argtypes = [vp, vp, i, vp]
    lib.fa_selftest_exp2.restype = i
    lib.fa_fwd_plan.argtypes = [i, i, i, i, i, ctypes.POINTER(FwdPlan)]
    lib.fa_fwd_plan.restype = i
    lib.fa_fwd_plan_pieces.argtypes = [i, i, i, i, i, i, ctypes.POINTER(ctypes.c_int), i]
    lib.fa_fwd_plan_pieces.restype = i
    lib.fa_fwd_plan_ex.argtypes = [i, i, i, i, ctypes.c_uint, i, ctypes.POINTER(FwdPlan)]
    lib.fa_fwd_plan_ex.restype = i
    lib.fa_fwd_plan_pieces_ex.argtypes = [i, i, i, i, ctypes.c_uint, i, i,
                                          ctypes.POINTER(ctypes.c_int), i]
    lib.fa_fwd_plan_pieces_ex.restype = i
    lib.fa_bwd_plan.argtypes = [i, i, i, i, ctypes.c_uint, i, ctypes.POINTER(ctypes.c_int),
                                ctypes.POINTER(ctypes.c_int)]
    lib.fa_bwd_plan.restype = i
    _lib = lib
    return lib


FA_OK = 0
FA_ERR_NULL, FA_ERR_SHAPE, FA_ERR_HEADDIM, FA_ERR_ALIGN = -1, -2, -3, -4
FA_ERR_LAUNCH, FA_ERR_NOMEM, FA_ERR_DEVICE, FA_ERR_SCALE = -5, -6, -7, -8
FA_ERR_SCRATCH = -9
FA_ERR_FLAGS, FA_ERR_DTYPE = -10, -11
FA_BF16, FA_FP16 = 0, 1
FA_FLAG_CAUSAL = 1
_DTYPE_CODE = {torch.bfloat16: FA_BF16, torch.float16: FA_FP16}


class FAError(RuntimeError):
    def __init__(self, where: str, status: int):
        msg = f"{where}: {fa_status_string(status)} (status {status})"
        if status == FA_ERR_LAUNCH:
            msg += f", cudaError {_load().fa_last_cuda_error()}"
        super().__init__(msg)
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded C library (for callers that want the raw entry points)."""
    return _load()


def declared_functions() -> list[str]:
    """Names of the functions include/fa_b200.h declares."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^[A-Za-z_][\w \t\*]*?\b(fa_\w+)\s*\(", text, flags=re.M)


def fa_status_string(status: int) -> str:
    return _load().fa_status_string(int(status)).decode()


def fa_version() -> int:
    return int(_load().fa_version())


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check_bnhd(name: str, t: torch.Tensor, dtype: torch.dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _fwd(entry: str, dtype, q, k, v, o, lse, scale, stream, flags: int = 0):
    _check_bnhd("q", q, dtype)
    if q.dim() != 4:
        raise ValueError("q must be [B, N, H, d]")
    B, N, H, d = q.shape
    _check_bnhd("k", k, dtype, q.shape)
    _check_bnhd("v", v, dtype, q.shape)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _check_bnhd("o", o, dtype, q.shape)
    _check_bnhd("lse", lse, torch.float32, (B, H, N))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if flags:
        rc = _load().fa_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                               float(scale), _DTYPE_CODE[dtype], int(flags), _stream(stream))
        entry = "fa_fwd_ex"
    else:
        rc = getattr(_load(), entry)(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                                  float(scale), _stream(stream))
    if rc != FA_OK:
        raise FAError(entry, rc)
    return o, lse


def _bwd(entry: str, dtype, q, k, v, o, dout, lse, dq, dk, dv, scale, stream, flags: int = 0):
    _check_bnhd("q", q, dtype)
    if q.dim() != 4:
        raise ValueError("q must be [B, N, H, d]")
    B, N, H, d = q.shape
    for name, t in (("k", k), ("v", v), ("o", o), ("dout", dout)):
        _check_bnhd(name, t, dtype, q.shape)
    _check_bnhd("lse", lse, torch.float32, (B, H, N))
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _check_bnhd(name, t, dtype, q.shape)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if flags:
        rc = _load().fa_bwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                               _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, float(scale),
                               _DTYPE_CODE[dtype], int(flags), _stream(stream))
        entry = "fa_bwd_ex"
    else:
        rc = getattr(_load(), entry)(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                                  _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, float(scale),
                                  _stream(stream))
    if rc != FA_OK:
        raise FAError(entry, rc)
    return dq, dk, dv


def fa_fwd(q, k, v, o=None, lse=None, scale=None, stream=None):
    """bf16 forward: returns (o, lse); allocates them when not given."""
    return _fwd("fa_fwd", torch.bfloat16, q, k, v, o, lse, scale, stream)


def fa_fwd_f16(q, k, v, o=None, lse=None, scale=None, stream=None):
    """fp16 forward: returns (o, lse); allocates them when not given."""
    return _fwd("fa_fwd_f16", torch.float16, q, k, v, o, lse, scale, stream)


def fa_bwd(q, k, v, o, dout, lse, dq=None, dk=None, dv=None, scale=None, stream=None):
    """bf16 backward by recompute: returns (dq, dk, dv) (overwritten, not accumulated)."""
    return _bwd("fa_bwd", torch.bfloat16, q, k, v, o, dout, lse, dq, dk, dv, scale, stream)


def fa_bwd_f16(q, k, v, o, dout, lse, dq=None, dk=None, dv=None, scale=None, stream=None):
    """fp16 backward by recompute: returns (dq, dk, dv)."""
    return _bwd("fa_bwd_f16", torch.float16, q, k, v, o, dout, lse, dq, dk, dv, scale, stream)


def fa_bwd_noalloc(q, k, v, o, dout, lse, dq, dk, dv, scale=None, stream=None):
    """bf16 backward that allocates no device memory: the library's fixed
    64 MiB scratch buffer replaces the stream-ordered scratch of fa_bwd, for
    callers that must not allocate.  dq, dk, dv must be given (this wrapper
    allocates nothing either).  Calls that overlap on the GPU share the buffer
    and race; order them (for example on one stream)."""
    if dq is None or dk is None or dv is None:
        raise ValueError("fa_bwd_noalloc needs caller-provided dq, dk, dv")
    return _bwd("fa_bwd_noalloc", torch.bfloat16, q, k, v, o, dout, lse, dq, dk, dv, scale,
                stream)


_FWD = {torch.bfloat16: fa_fwd, torch.float16: fa_fwd_f16}
_BWD = {torch.bfloat16: fa_bwd, torch.float16: fa_bwd_f16}


def fa_fwd_fp8(q, k, v, descale_q=1.0, descale_k=1.0, descale_v=1.0, o=None, lse=None,
               scale=None, flags=0, stream=None):
    """Forward on E4M3 inputs (torch.float8_e4m3fn [B, N, H, 128]) with
    per-tensor descale factors: attention of (descale_q q, descale_k k,
    descale_v v).  Returns (o [B, N, H, d] bf16, lse [B, H, N] fp32)."""
    _check_bnhd("q", q, torch.float8_e4m3fn)
    if q.dim() != 4:
        raise ValueError("q must be [B, N, H, d]")
    B, N, H, d = q.shape
    for name, t in (("k", k), ("v", v)):
        _check_bnhd(name, t, torch.float8_e4m3fn, q.shape)
    o = torch.empty((B, N, H, d), dtype=torch.bfloat16, device=q.device) if o is None else o
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    _check_bnhd("o", o, torch.bfloat16, (B, N, H, d))
    _check_bnhd("lse", lse, torch.float32, (B, H, N))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rc = _load().fa_fwd_fp8(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                            float(scale), float(descale_q), float(descale_k), float(descale_v),
                            int(flags), _stream(stream))
    if rc != FA_OK:
        raise FAError("fa_fwd_fp8", rc)
    return o, lse


def fa_bwd_plan(B, H, N, d, sm_count, flags=0):
    """The backward's decomposition: {"n_split": blocks per key tile,
    "grid": blocks} (host only; same code as the launch)."""
    ns, grid = ctypes.c_int(), ctypes.c_int()
    rc = _load().fa_bwd_plan(B, H, N, d, int(flags), sm_count, ctypes.byref(ns), ctypes.byref(grid))
    if rc != FA_OK:
        raise FAError("fa_bwd_plan", rc)
    return {"n_split": ns.value, "grid": grid.value}


def fa_fwd_ex(q, k, v, o=None, lse=None, scale=None, flags=0, stream=None):
    """Forward with flags (FA_FLAG_CAUSAL); element type from q (bf16 / fp16)."""
    if q.dtype not in _DTYPE_CODE:
        raise TypeError(f"unsupported element type {q.dtype}")
    entry = "fa_fwd" if q.dtype == torch.bfloat16 else "fa_fwd_f16"
    if flags == 0:
        return _fwd(entry, q.dtype, q, k, v, o, lse, scale, stream)
    return _fwd(entry, q.dtype, q, k, v, o, lse, scale, stream, flags)


def fa_bwd_ex(q, k, v, o, dout, lse, dq=None, dk=None, dv=None, scale=None, flags=0, stream=None):
    """Backward with flags (FA_FLAG_CAUSAL: o and lse from the causal forward)."""
    if q.dtype not in _DTYPE_CODE:
        raise TypeError(f"unsupported element type {q.dtype}")
    entry = "fa_bwd" if q.dtype == torch.bfloat16 else "fa_bwd_f16"
    return _bwd(entry, q.dtype, q, k, v, o, dout, lse, dq, dk, dv, scale, stream, flags)


def _check_packed(qkv):
    if not isinstance(qkv, torch.Tensor) or not qkv.is_cuda or not qkv.is_contiguous():
        raise ValueError("qkv must be a contiguous CUDA tensor")
    if qkv.dim() != 5 or qkv.shape[2] != 3:
        raise ValueError("qkv must be [B, N, 3, H, d]")
    if qkv.dtype not in _DTYPE_CODE:
        raise TypeError(f"unsupported element type {qkv.dtype}")
    B, N, _, H, d = qkv.shape
    return B, N, H, d


def fa_fwd_qkvpacked(qkv, o=None, lse=None, scale=None, flags=0, stream=None):
    """Forward on a packed [B, N, 3, H, d] tensor; returns (o [B,N,H,d], lse)."""
    B, N, H, d = _check_packed(qkv)
    o = torch.empty((B, N, H, d), dtype=qkv.dtype, device=qkv.device) if o is None else o
    lse = torch.empty((B, H, N), dtype=torch.float32, device=qkv.device) if lse is None else lse
    _check_bnhd("o", o, qkv.dtype, (B, N, H, d))
    _check_bnhd("lse", lse, torch.float32, (B, H, N))
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    rc = _load().fa_fwd_qkvpacked(_ptr(qkv), _ptr(o), _ptr(lse), B, H, N, d, float(scale),
                                  _DTYPE_CODE[qkv.dtype], int(flags), _stream(stream))
    if rc != FA_OK:
        raise FAError("fa_fwd_qkvpacked", rc)
    return o, lse


def fa_bwd_qkvpacked(qkv, o, dout, lse, dqkv=None, scale=None, flags=0, stream=None):
    """Backward on a packed tensor; returns dqkv [B, N, 3, H, d] (dQ, dK, dV)."""
    B, N, H, d = _check_packed(qkv)
    for name, t in (("o", o), ("dout", dout)):
        _check_bnhd(name, t, qkv.dtype, (B, N, H, d))
    _check_bnhd("lse", lse, torch.float32, (B, H, N))
    dqkv = torch.empty_like(qkv) if dqkv is None else dqkv
    if tuple(dqkv.shape) != tuple(qkv.shape) or dqkv.dtype != qkv.dtype or \
            not dqkv.is_contiguous():
        raise ValueError("dqkv must match qkv")
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    rc = _load().fa_bwd_qkvpacked(_ptr(qkv), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dqkv), B, H, N,
                                  d, float(scale), _DTYPE_CODE[qkv.dtype], int(flags),
                                  _stream(stream))
    if rc != FA_OK:
        raise FAError("fa_bwd_qkvpacked", rc)
    return dqkv


def _check_varlen(q, cu_seqlens, max_seqlen):
    if q.dim() != 3:
        raise ValueError("varlen q must be [total, H, d]")
    if not (isinstance(cu_seqlens, torch.Tensor) and cu_seqlens.is_cuda and
            cu_seqlens.dtype == torch.int32 and cu_seqlens.dim() == 1 and
            cu_seqlens.is_contiguous() and cu_seqlens.numel() >= 2):
        raise ValueError("cu_seqlens must be a contiguous int32 CUDA tensor of B + 1 entries")
    if q.dtype not in _DTYPE_CODE:
        raise TypeError(f"unsupported element type {q.dtype}")
    total, H, d = q.shape
    return cu_seqlens.numel() - 1, total, H, d, int(max_seqlen)


def fa_fwd_varlen(q, k, v, cu_seqlens, max_seqlen, o=None, lse=None, scale=None, flags=0,
                  stream=None):
    """Forward over B sequences packed along the token axis: q, k, v are
    [total, H, d], cu_seqlens (int32, B + 1) their starts.  Returns (o [total,
    H, d], lse [H, total])."""
    B, total, H, d, ms = _check_varlen(q, cu_seqlens, max_seqlen)
    for name, t in (("k", k), ("v", v)):
        _check_bnhd(name, t, q.dtype, q.shape)
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty((H, total), dtype=torch.float32, device=q.device) if lse is None else lse
    _check_bnhd("o", o, q.dtype, q.shape)
    _check_bnhd("lse", lse, torch.float32, (H, total))
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    rc = _load().fa_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_seqlens), B,
                               total, ms, H, d, float(scale), _DTYPE_CODE[q.dtype], int(flags),
                               _stream(stream))
    if rc != FA_OK:
        raise FAError("fa_fwd_varlen", rc)
    return o, lse


def fa_bwd_varlen(q, k, v, o, dout, lse, cu_seqlens, max_seqlen, dq=None, dk=None, dv=None,
                  scale=None, flags=0, stream=None):
    """Backward of fa_fwd_varlen; returns (dq, dk, dv), each [total, H, d]."""
    B, total, H, d, ms = _check_varlen(q, cu_seqlens, max_seqlen)
    for name, t in (("k", k), ("v", v), ("o", o), ("dout", dout)):
        _check_bnhd(name, t, q.dtype, q.shape)
    _check_bnhd("lse", lse, torch.float32, (H, total))
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _check_bnhd(name, t, q.dtype, q.shape)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    rc = _load().fa_bwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                               _ptr(dq), _ptr(dk), _ptr(dv), _ptr(cu_seqlens), B, total, ms, H, d,
                               float(scale), _DTYPE_CODE[q.dtype], int(flags), _stream(stream))
    if rc != FA_OK:
        raise FAError("fa_bwd_varlen", rc)
    return dq, dk, dv


def fa_varlen_bounds(cu_seqlens, b: int, max_seqlen: int, total: int) -> tuple:
    """(first token, length) the varlen kernels use for sequence b, from a
    host list of cu_seqlens (the clamping rule, evaluated on the host)."""
    arr = (ctypes.c_int * len(cu_seqlens))(*cu_seqlens)
    t0, n = ctypes.c_int(0), ctypes.c_int(0)
    rc = _load().fa_varlen_bounds(arr, b, max_seqlen, total, ctypes.byref(t0), ctypes.byref(n))
    if rc != FA_OK:
        raise FAError("fa_varlen_bounds", rc)
    return t0.value, n.value


def forward(q, k, v, scale=None, o=None, lse=None, stream=None, causal=False):
    """fa_fwd or fa_fwd_f16 (fa_fwd_ex when causal), chosen by q's element type."""
    if q.dtype not in _FWD:
        raise TypeError(f"unsupported element type {q.dtype}")
    if causal:
        return fa_fwd_ex(q, k, v, o=o, lse=lse, scale=scale, flags=FA_FLAG_CAUSAL, stream=stream)
    return _FWD[q.dtype](q, k, v, o=o, lse=lse, scale=scale, stream=stream)


def backward(q, k, v, o, dout, lse, scale=None, dq=None, dk=None, dv=None, stream=None,
             causal=False):
    """fa_bwd or fa_bwd_f16 (fa_bwd_ex when causal), chosen by q's element type."""
    if q.dtype not in _BWD:
        raise TypeError(f"unsupported element type {q.dtype}")
    if causal:
        return fa_bwd_ex(q, k, v, o, dout, lse, dq=dq, dk=dk, dv=dv, scale=scale,
                         flags=FA_FLAG_CAUSAL, stream=stream)
    return _BWD[q.dtype](q, k, v, o, dout, lse, dq=dq, dk=dk, dv=dv, scale=scale, stream=stream)


def fa_fwd_plan(B: int, H: int, N: int, d: int, sm_count: int, flags: int = 0) -> dict:
    """The forward's work decomposition for a device with sm_count SMs (host
    logic only; needs no GPU)."""
    plan = FwdPlan()
    rc = _load().fa_fwd_plan_ex(B, H, N, d, flags, sm_count, ctypes.byref(plan))
    if rc != FA_OK:
        raise FAError("fa_fwd_plan", rc)
    return plan.as_dict()


def fa_fwd_plan_pieces(B: int, H: int, N: int, d: int, sm_count: int, block: int,
                       flags: int = 0) -> list:
    """The pieces one forward block processes, as (unit, first K/V tile, end
    K/V tile, kind, first peer, peer count) tuples; kind 0 = whole result,
    1 = partial rows, 2 = merge with the peers' partial rows."""
    lib_ = _load()
    n = lib_.fa_fwd_plan_pieces_ex(B, H, N, d, flags, sm_count, block, None, 0)
    if n < 0:
        raise FAError("fa_fwd_plan_pieces", n)
    buf = (ctypes.c_int * (6 * max(n, 1)))()
    got = lib_.fa_fwd_plan_pieces_ex(B, H, N, d, flags, sm_count, block, buf, n)
    if got != n:
        raise FAError("fa_fwd_plan_pieces", got if got < 0 else FA_ERR_SHAPE)
    return [tuple(buf[6 * i:6 * i + 6]) for i in range(n)]


def fa_get_device_status(clear: bool = False) -> int:
    """The device status word (0 = no bounded wait gave up).  Synchronises."""
    out = ctypes.c_ulonglong(0)
    rc = _load().fa_get_device_status(ctypes.byref(out), 1 if clear else 0)
    if rc != FA_OK:
        raise FAError("fa_get_device_status", rc)
    return int(out.value)


def fa_selftest_bounded_wait(limit_us: int = 20000) -> int:
    """Runs the bounded-wait self test; returns the status it recorded."""
    out = ctypes.c_ulonglong(0)
    rc = _load().fa_selftest_bounded_wait(int(limit_us), ctypes.byref(out))
    if rc != FA_OK:
        raise FAError("fa_selftest_bounded_wait", rc)
    return int(out.value)


def fa_selftest_exp2(x: torch.Tensor, stream=None) -> torch.Tensor:
    """2^x (float32 CUDA tensor) by the softmax's FMA-pipe exponential."""
    if not (isinstance(x, torch.Tensor) and x.is_cuda and x.dtype == torch.float32
            and x.is_contiguous()):
        raise TypeError("x must be a contiguous float32 CUDA tensor")
    y = torch.empty_like(x)
    rc = _load().fa_selftest_exp2(_ptr(x), _ptr(y), x.numel(), _stream(stream))
    if rc != FA_OK:
        raise FAError("fa_selftest_exp2", rc)
    return y


def _event_handle(ev):
    if ev is None:
        return None
    return ev.cuda_event if isinstance(ev, torch.cuda.Event) else int(ev)


def fa_set_kernel_events(fwd_start=None, fwd_stop=None, bwd_start=None, bwd_stop=None) -> None:
    """Arm torch.cuda.Event pairs (enable_timing=True) around the next forward
    and backward main kernels."""
    for ev in (fwd_start, fwd_stop, bwd_start, bwd_stop):
        if isinstance(ev, torch.cuda.Event) and ev.cuda_event == 0:
            ev.record()  # materialise the underlying CUDA event
    _load().fa_set_kernel_events(_event_handle(fwd_start), _event_handle(fwd_stop),
                                 _event_handle(bwd_start), _event_handle(bwd_stop))


def fa_kernel_launches() -> int:
    """Kernel launches this library has issued since it was loaded."""
    return int(_load().fa_kernel_launches())


def fa_scratch_allocs() -> int:
    """Scratch allocations this library has requested since it was loaded."""
    return int(_load().fa_scratch_allocs())


class _Attention(torch.autograd.Function):
    """Autograd glue over the C entry points: the forward saves only O and the
    LSE (the recompute strategy), the backward calls fa_bwd(_ex) with them."""

    @staticmethod
    def forward(ctx, q, k, v, scale, causal):
        o, lse = forward(q, k, v, scale=scale, causal=causal)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.scale, ctx.causal = scale, causal
        return o, lse

    @staticmethod
    def backward(ctx, do, dlse):
        if dlse is not None and bool(torch.any(dlse != 0)):
            raise NotImplementedError("gradients through the LSE output are not supported")
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = backward(q, k, v, o, do.contiguous(), lse, scale=ctx.scale,
                              causal=ctx.causal)
        return dq, dk, dv, None, None


def attention(q, k, v, scale=None, causal=False, return_lse=False):
    """Exact attention O = softmax(scale Q K^T [causal mask]) V with autograd.

    q, k, v: contiguous [B, N, H, d] CUDA tensors of bfloat16 or float16;
    scale defaults to 1/sqrt(d).  Returns O (and the fp32 LSE [B, H, N] when
    return_lse).  The backward recomputes P from O and the LSE in the
    library's kernels; no N x N matrix is ever stored.
    """
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    o, lse = _Attention.apply(q, k, v, float(scale), bool(causal))
    return (o, lse) if return_lse else o
