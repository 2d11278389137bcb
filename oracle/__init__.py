"""fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product library
(``exact_attention_144_b200``) never imports it, and it never imports the
product library: the two share no code.

The arithmetic lives in ``attn_oracle.c`` (plain C, fp64, sequential loops per
row, OpenMP only across independent rows or heads).  This module compiles it
with gcc on first use (or from ``build()``) and exposes numpy wrappers.

Parity status of each function (what pins it, in ``tests/test_oracle.py``):
  attn_fwd          closed forms (Q=0, N=1, constant V, hand-worked 1-d case),
                    shift and permutation invariances, one-hot dominance,
                    equality with the online recurrence and two-pass forms.
  attn_probs        rows sum to one; closed forms above.
  attn_fwd_rows     equal to attn_fwd on the sampled rows.
  attn_fwd_two_pass bit-equal to attn_fwd_online under the conditions where
                    every rescale factor is exactly one.
  attn_fwd_online   as above; otherwise within a rounding bound.
  attn_bwd          central finite differences of L = sum(O * dO); the
                    row-sum identity of dS; closed form at N=1.
  attn_bwd_rows     the row ranges of a split partition sum to attn_bwd.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "attn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_default = None

GCC_FLAGS = ["-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
             "-fno-fast-math", "-std=c11"]


def compile_source(src_path: str, out_path: str) -> str:
    """Compile an oracle C source into a shared library with the fixed flags.

    -ffp-contract=off keeps every multiply and add a separately rounded fp64
    operation, so the sequential sums are exactly the ones written in C.
    """
    subprocess.check_call(["gcc", *GCC_FLAGS, src_path, "-o", out_path + ".tmp", "-lm"])
    os.replace(out_path + ".tmp", out_path)
    return out_path


def build(force: bool = False) -> str:
    """Compile attn_oracle.c into liboracle.so next to it (if stale)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(SOURCE):
        compile_source(SOURCE, _LIB)
    return _LIB


def _c(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _shape(q):
    if q.ndim != 4:
        raise ValueError("expected [B, N, H, d]")
    return q.shape


class Oracle:
    """numpy front end over one compiled copy of the oracle C code."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int)
        i, f = ctypes.c_int, ctypes.c_double
        lib.oracle_attn_fwd.argtypes = [dp, dp, dp, dp, dp, i, i, i, i, f, i]
        lib.oracle_attn_fwd_two_pass.argtypes = [dp, dp, dp, dp, dp, i, i, i, i, f]
        lib.oracle_attn_fwd_online.argtypes = [dp, dp, dp, dp, dp, i, i, i, i, f, i, i]
        lib.oracle_attn_fwd_rows.argtypes = [dp, dp, dp, ip, i, dp, dp, i, i, i, i, f, i]
        lib.oracle_attn_probs.argtypes = [dp, dp, dp, i, i, i, i, f, i]
        lib.oracle_attn_bwd.argtypes = [dp, dp, dp, dp, dp, dp, dp, i, i, i, i, f, i]
        lib.oracle_attn_bwd_rows.argtypes = [dp, dp, dp, dp, dp, dp, dp, i, i, i, i, f, i, i, i]
        lib.oracle_attn_dscores.argtypes = [dp, dp, dp, dp, dp, i, i, i, i, f, i]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [i]
        self.lib = lib

    def num_threads(self) -> int:
        """OpenMP threads the oracle uses (OMP_NUM_THREADS, else all host cores)."""
        return int(self.lib.oracle_num_threads())

    def set_num_threads(self, n: int) -> None:
        """Use n OpenMP threads in later calls (timing only; no arithmetic changes)."""
        self.lib.oracle_set_num_threads(int(n))

    def attn_fwd(self, q, k, v, scale, causal=False):
        """O = softmax(scale Q K^T) V and LSE (natural log) by the definition;
        with causal, row i sees keys j <= i only.

        q, k, v: [B, N, H, d] arrays (any float dtype, widened to fp64).
        Returns o [B, N, H, d] fp64 and lse [B, H, N] fp64.
        """
        q, k, v = _c(q), _c(k), _c(v)
        B, N, H, d = _shape(q)
        o = np.empty_like(q)
        lse = np.empty((B, H, N), dtype=np.float64)
        self.lib.oracle_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                                 float(scale), int(bool(causal)))
        return o, lse

    def attn_fwd_rows(self, q, k, v, scale, rows, causal=False):
        """Forward pass for selected (b, h, i) rows; returns o [R, d], lse [R]."""
        q, k, v = _c(q), _c(k), _c(v)
        B, N, H, d = _shape(q)
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 3))
        R = rows.shape[0]
        o = np.empty((R, d), dtype=np.float64)
        lse = np.empty((R,), dtype=np.float64)
        self.lib.oracle_attn_fwd_rows(_ptr(q), _ptr(k), _ptr(v),
                                      rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), R,
                                      _ptr(o), _ptr(lse), B, H, N, d, float(scale),
                                      int(bool(causal)))
        return o, lse

    def attn_fwd_two_pass(self, q, k, v, scale):
        q, k, v = _c(q), _c(k), _c(v)
        B, N, H, d = _shape(q)
        o = np.empty_like(q)
        lse = np.empty((B, H, N), dtype=np.float64)
        self.lib.oracle_attn_fwd_two_pass(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                          B, H, N, d, float(scale))
        return o, lse

    def attn_fwd_online(self, q, k, v, scale, block_q, block_kv):
        q, k, v = _c(q), _c(k), _c(v)
        B, N, H, d = _shape(q)
        o = np.empty_like(q)
        lse = np.empty((B, H, N), dtype=np.float64)
        self.lib.oracle_attn_fwd_online(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                                        float(scale), int(block_q), int(block_kv))
        return o, lse

    def attn_probs(self, q, k, scale, causal=False):
        """P = softmax(scale Q K^T) as [B, H, N, N] (small N only)."""
        q, k = _c(q), _c(k)
        B, N, H, d = _shape(q)
        p = np.empty((B, H, N, N), dtype=np.float64)
        self.lib.oracle_attn_probs(_ptr(q), _ptr(k), _ptr(p), B, H, N, d, float(scale),
                                   int(bool(causal)))
        return p

    def attn_bwd(self, q, k, v, dout, scale, causal=False):
        """dQ, dK, dV of L = sum(O * dO) by recompute; each [B, N, H, d] fp64."""
        q, k, v, dout = _c(q), _c(k), _c(v), _c(dout)
        B, N, H, d = _shape(q)
        dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
        self.lib.oracle_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                                 B, H, N, d, float(scale), int(bool(causal)))
        return dq, dk, dv

    def attn_bwd_rows(self, q, k, v, dout, scale, row_begin, row_end, causal=False):
        """Backward pass restricted to query rows [row_begin, row_end): dq rows
        in the range are exact; dk, dv are those rows' contributions.  Rows of
        dq outside the range are returned as zeros."""
        q, k, v, dout = _c(q), _c(k), _c(v), _c(dout)
        B, N, H, d = _shape(q)
        if not 0 <= row_begin <= row_end <= N:
            raise ValueError("bad row range")
        dq, dk, dv = np.zeros_like(q), np.empty_like(q), np.empty_like(q)
        self.lib.oracle_attn_bwd_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk),
                                      _ptr(dv), B, H, N, d, float(scale), int(row_begin),
                                      int(row_end), int(bool(causal)))
        return dq, dk, dv

    def attn_dscores(self, q, k, v, dout, scale, causal=False):
        """dS = P * (dP - D) as [B, H, N, N] (small N only)."""
        q, k, v, dout = _c(q), _c(k), _c(v), _c(dout)
        B, N, H, d = _shape(q)
        ds = np.empty((B, H, N, N), dtype=np.float64)
        self.lib.oracle_attn_dscores(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(ds),
                                     B, H, N, d, float(scale), int(bool(causal)))
        return ds


def default() -> Oracle:
    """The oracle built from the committed attn_oracle.c."""
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def num_threads():
    return default().num_threads()


def set_num_threads(n: int) -> None:
    default().set_num_threads(n)


def attn_fwd(q, k, v, scale, causal=False):
    return default().attn_fwd(q, k, v, scale, causal)


def attn_fwd_rows(q, k, v, scale, rows, causal=False):
    return default().attn_fwd_rows(q, k, v, scale, rows, causal)


def attn_fwd_two_pass(q, k, v, scale):
    return default().attn_fwd_two_pass(q, k, v, scale)


def attn_fwd_online(q, k, v, scale, block_q, block_kv):
    return default().attn_fwd_online(q, k, v, scale, block_q, block_kv)


def attn_probs(q, k, scale, causal=False):
    return default().attn_probs(q, k, scale, causal)


def attn_bwd(q, k, v, dout, scale, causal=False):
    return default().attn_bwd(q, k, v, dout, scale, causal)


def attn_bwd_rows(q, k, v, dout, scale, row_begin, row_end, causal=False):
    return default().attn_bwd_rows(q, k, v, dout, scale, row_begin, row_end, causal)


def attn_dscores(q, k, v, dout, scale, causal=False):
    return default().attn_dscores(q, k, v, dout, scale, causal)
