"""fp64 CPU oracle for exact scaled-dot-product attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's ``cpu_baseline``
/ ``--impl reference`` legs may import this package.  The product path (the
CUDA library ``libattn`` and its Python binding) never imports it and shares
no code with it.

The arithmetic lives in ``attn_oracle.c`` (plain fp64 loops, OpenMP over
independent rows/heads); this module only builds it with gcc, loads it with
ctypes and converts numpy arrays.  Every function cites the passage it
follows in the C source.  Parity status of each function (what pins it) is
listed in ``tests/test_oracle_pins.py``; the byte model below is pinned by the
storage figures the pages print.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "attn_oracle.c"
_LIB = _HERE / "liboracle.so"

_c_dbl_p = ctypes.POINTER(ctypes.c_double)


def build(out: Path | str | None = None, mutant: int = 0, quiet: bool = True) -> Path:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math).

    ``mutant`` != 0 plants one of the known mistakes guarded by
    ``ORACLE_MUTANT`` (used only by the mutation tests).
    """
    out = Path(out) if out is not None else _LIB
    cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
           f"-DORACLE_MUTANT={int(mutant)}", str(_SRC), "-o", str(out), "-lm"]
    subprocess.run(cmd, check=True, capture_output=quiet)
    return out


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(_c_dbl_p)


def _f64(a) -> np.ndarray:
    """Widen (torch or numpy) input to a contiguous fp64 numpy array."""
    try:
        import torch

        if isinstance(a, torch.Tensor):
            a = a.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _window(window):
    """(left, right) window sizes as C ints; None or a negative side is unbounded."""
    if window is None:
        return -1, -1
    wl, wr = window
    return (-1 if wl is None else int(wl)), (-1 if wr is None else int(wr))


class Oracle:
    """ctypes wrapper around one build of ``attn_oracle.c``."""

    def __init__(self, lib_path: Path | str | None = None):
        path = Path(lib_path) if lib_path is not None else _LIB
        if lib_path is None and (not path.exists() or path.stat().st_mtime < _SRC.stat().st_mtime):
            build(path)
        self._lib = ctypes.CDLL(str(path))
        L = self._lib
        i, d, ll = ctypes.c_int, ctypes.c_double, ctypes.c_longlong
        P = _c_dbl_p
        L.oracle_attn_fwd.argtypes = [P, P, P, P, ll, P, P, i, i, i, i, i, i, i, d, i, i, i]
        L.oracle_attn_fwd_rows.argtypes = [P, P, P, P, ctypes.POINTER(ll), i, P, P, i, i, i, i, d, i, i, i]
        L.oracle_attn_fwd_varlen.argtypes = [P, P, P, ctypes.POINTER(ctypes.c_int),
                                             ctypes.POINTER(ctypes.c_int), i, P, P, i, i, i, d, i, i, i]
        L.oracle_attn_fwd_stream.argtypes = [P, P, P, P, ll, P, P, i, i, i, i, i, i, d, i, i, i, i,
                                             ctypes.POINTER(ll)]
        L.oracle_attn_bwd.argtypes = [P, P, P, P, ll, P, P, P, P, i, i, i, i, i, i, i, d, i, i, i]
        L.oracle_merge_partials.argtypes = [P, P, i, i, i, P, P]
        L.oracle_quantize_e4m3.argtypes = [P, ll, d, P]
        L.oracle_quantize_e4m3.restype = None
        L.oracle_quantize_e4m3_heads.argtypes = [P, i, i, i, i, P, P]
        L.oracle_quantize_e4m3_heads.restype = None
        for f in (L.oracle_attn_fwd, L.oracle_attn_fwd_rows, L.oracle_attn_fwd_varlen,
                  L.oracle_attn_fwd_stream, L.oracle_attn_bwd, L.oracle_merge_partials):
            f.restype = None

    # ------------------------------------------------------------------ forward
    @staticmethod
    def _bias(bias, Hq, Nq, Nk):
        if bias is None:
            return None, 0
        b = _f64(bias)
        per = Hq * Nq * Nk
        if b.size == per:
            return b, 0
        assert b.size % per == 0, "bias must be [Hq,Nq,Nk] or [B,Hq,Nq,Nk]"
        return b, per

    def fwd(self, q, k, v, bias=None, causal=False, scale=None, window=None):
        """O, LSE of softmax(scale*QK^T + B)V.  q [B,Nq,Hq,d], k/v [B,Nk,Hkv,d];
        returns o [B,Nq,Hq,d] and lse [B,Hq,Nq] (fp64).  window = (left, right):
        with a = i + Nk - Nq, keys a - left .. a + right are visible (negative:
        unbounded on that side)."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, Nq, Hq, d = q.shape
        Nk, Hkv, dv = k.shape[1], k.shape[2], v.shape[3]
        scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
        b, bstride = self._bias(bias, Hq, Nq, Nk)
        o = np.zeros((B, Nq, Hq, dv))
        lse = np.zeros((B, Hq, Nq))
        self._lib.oracle_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(b) if b is not None else None,
                                  bstride, _ptr(o), _ptr(lse), B, Hq, Hkv, Nq, Nk, d, dv, scale,
                                  int(bool(causal)), *_window(window))
        return o, lse

    def fwd_stream(self, q, k, v, bias=None, causal=False, scale=None, block=128, window=None):
        """Streaming (m, l, a) replay with key blocks of ``block``; returns o, lse, rescales."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, Nq, Hq, d = q.shape
        Nk, Hkv = k.shape[1], k.shape[2]
        scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
        b, bstride = self._bias(bias, Hq, Nq, Nk)
        o = np.zeros((B, Nq, Hq, d))
        lse = np.zeros((B, Hq, Nq))
        cnt = ctypes.c_longlong(0)
        self._lib.oracle_attn_fwd_stream(_ptr(q), _ptr(k), _ptr(v), _ptr(b) if b is not None else None,
                                         bstride, _ptr(o), _ptr(lse), B, Hq, Hkv, Nq, Nk, d, scale,
                                         int(bool(causal)), *_window(window), int(block), ctypes.byref(cnt))
        return o, lse, cnt.value

    def fwd_rows(self, q_rows, k_head, v_head, rows, Nq, bias_rows=None, causal=False, scale=None, window=None):
        """Forward of selected rows of one (batch, head).  q_rows [R,d], k/v_head [Nk,d],
        rows: query indices of q_rows; bias_rows [R,Nk] or None."""
        q_rows, k_head, v_head = _f64(q_rows), _f64(k_head), _f64(v_head)
        R, d = q_rows.shape
        Nk, dv = k_head.shape[0], v_head.shape[1]
        scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        br = _f64(bias_rows) if bias_rows is not None else None
        o = np.zeros((R, dv))
        lse = np.zeros(R)
        self._lib.oracle_attn_fwd_rows(_ptr(q_rows), _ptr(k_head), _ptr(v_head),
                                       _ptr(br) if br is not None else None,
                                       rows.ctypes.data_as(ctypes.POINTER(ctypes.c_longlong)), R,
                                       _ptr(o), _ptr(lse), int(Nq), Nk, d, dv, scale, int(bool(causal)),
                                       *_window(window))
        return o, lse

    def fwd_varlen(self, q, k, v, cu_q, cu_k, causal=False, scale=None, window=None):
        """Packed forward.  q [Tq,Hq,d], k/v [Tk,Hkv,d]; returns o [Tq,Hq,d], lse [Hq,Tq]."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        Tq, Hq, d = q.shape
        Hkv = k.shape[1]
        cq = np.ascontiguousarray(np.asarray(cu_q, dtype=np.int32))
        ck = np.ascontiguousarray(np.asarray(cu_k, dtype=np.int32))
        scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
        o = np.zeros((Tq, Hq, d))
        lse = np.zeros((Hq, Tq))
        ip = ctypes.POINTER(ctypes.c_int)
        self._lib.oracle_attn_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), cq.ctypes.data_as(ip),
                                         ck.ctypes.data_as(ip), len(cq) - 1, _ptr(o), _ptr(lse),
                                         Hq, Hkv, d, scale, int(bool(causal)), *_window(window))
        return o, lse

    # ----------------------------------------------------------------- backward
    def bwd(self, q, k, v, dout, bias=None, causal=False, scale=None, window=None):
        """dQ, dK, dV of the forward above for upstream gradient dout (fp64)."""
        q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
        B, Nq, Hq, d = q.shape
        Nk, Hkv, dvw = k.shape[1], k.shape[2], v.shape[3]
        scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
        b, bstride = self._bias(bias, Hq, Nq, Nk)
        dq = np.zeros_like(q)
        dk = np.zeros_like(k)
        dv = np.zeros_like(v)
        self._lib.oracle_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(b) if b is not None else None,
                                  bstride, _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                                  B, Hq, Hkv, Nq, Nk, d, dvw, scale, int(bool(causal)), *_window(window))
        return dq, dk, dv

    # --------------------------------------------------------------------- fp8
    def quantize_e4m3(self, x, scale=1.0):
        """Dequantised e4m3 values of x / scale, times scale (fp64, same shape)."""
        x = _f64(x)
        out = np.empty_like(x)
        self._lib.oracle_quantize_e4m3(_ptr(x), x.size, float(scale), _ptr(out))
        return out

    def quantize_e4m3_heads(self, x):
        """Per-(batch, head) e4m3 quantisation of x [B, N, H, d]: returns the
        dequantised values (fp64, same shape) and the fp32 scales [B, H]
        (amax / 448), the codes decided on the fp32 quotient x / scale."""
        x = _f64(x)
        B, N, H, d = x.shape
        out = np.empty_like(x)
        scales = np.empty((B, H))
        self._lib.oracle_quantize_e4m3_heads(_ptr(x), B, N, H, d, _ptr(out), _ptr(scales))
        return out, scales

    # -------------------------------------------------------------------- merge
    def merge_partials(self, o_parts, lse_parts):
        """Combine exact partial results over disjoint key shards.
        o_parts [T,R,d], lse_parts [T,R] -> o [R,d], lse [R]."""
        op, lp = _f64(o_parts), _f64(lse_parts)
        T, R, d = op.shape
        o = np.zeros((R, d))
        lse = np.zeros(R)
        self._lib.oracle_merge_partials(_ptr(op), _ptr(lp), T, R, d, _ptr(o), _ptr(lse))
        return o, lse


_default: Oracle | None = None


def get() -> Oracle:
    """The oracle built from ``attn_oracle.c`` (rebuilt when the source is newer)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default


# ---------------------------------------------------------------- byte model
def score_matrix_bytes(t_query: int, t_key: int, bytes_per_score: int) -> int:
    """Dense score-matrix payload of one head and one request:
    query positions x key positions x stored bytes per score
    ("Attention IO tiling" lesson card, Score storage)."""
    return int(t_query) * int(t_key) * int(bytes_per_score)


def score_matrix_entries(n_tokens: int) -> int:
    """Entries of the N x N score matrix of one head (self-attention)."""
    return int(n_tokens) * int(n_tokens)


def cpu_threads() -> int:
    """Threads the OpenMP runtime will use (OMP_NUM_THREADS or the core count)."""
    env = os.environ.get("OMP_NUM_THREADS")
    return int(env) if env else (os.cpu_count() or 1)
