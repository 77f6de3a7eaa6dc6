"""Exact IO-aware attention for B200: thin Python binding of the C-ABI library
``libattn.so`` (declared in ``include/attn.h``).

This module only marshals arguments: it checks shapes/dtypes, allocates the
output tensors with PyTorch (device memory and streams are PyTorch's), and
calls the C entry points of the same names.  Every step of the attention path
runs in the library's CUDA kernels; there is no fallback.  If the library is
missing, importing this module raises.
"""
from __future__ import annotations

import ctypes
import math
from pathlib import Path

import torch

_PKG = Path(__file__).resolve().parent
LIB_PATH = _PKG / "libattn.so"

ATTN_BF16 = 0
ATTN_F32 = 1
ATTN_OK = 0
ATTN_ERR_INVALID = -1
ATTN_ERR_UNSUPPORTED = -2
ATTN_ERR_WORKSPACE = -3
ATTN_ERR_CUDA = -4
ATTN_ERR_TIMEOUT = -5

# symbol -> (restype, argtypes)
_VP, _FP, _IP = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
_I, _LL, _F, _SZ = ctypes.c_int, ctypes.c_longlong, ctypes.c_float, ctypes.c_size_t
EXPORTS = {
    "attn_fwd": (_I, [_VP, _VP, _VP, _FP, _LL, _VP, _FP, _I, _I, _I, _I, _I, _I, _F, _I, _I, _VP]),
    "attn_fwd_alibi": (_I, [_VP, _VP, _VP, _FP, _VP, _FP, _I, _I, _I, _I, _I, _I, _F, _I, _I, _VP]),
    "attn_bwd_alibi": (_I, [_VP, _VP, _VP, _FP, _VP, _FP, _VP, _VP, _VP, _VP, _VP, _SZ, _I, _I, _I, _I, _I, _I,
                            _F, _I, _I, _VP]),
    "attn_fwd_local": (_I, [_VP, _VP, _VP, _FP, _VP, _FP, _I, _I, _I, _I, _I, _I, _F, _I, _I, _I, _I, _VP]),
    "attn_bwd_local": (_I, [_VP, _VP, _VP, _FP, _VP, _FP, _VP, _VP, _VP, _VP, _VP, _SZ, _I, _I, _I, _I, _I, _I,
                            _F, _I, _I, _I, _I, _VP]),
    "attn_bwd_varlen": (_I, [_VP, _VP, _VP, _VP, _FP, _VP, _VP, _VP, _VP, _IP, _IP, _I, _I, _I, _I, _I, _I, _I, _I,
                             _F, _I, _VP, _SZ, _I, _VP]),
    "attn_fwd_dv": (_I, [_VP, _VP, _VP, _VP, _FP, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _VP]),
    "attn_bwd_dv": (_I, [_VP, _VP, _VP, _VP, _FP, _VP, _VP, _VP, _VP, _VP, _SZ, _I, _I, _I, _I, _I, _I, _I, _F,
                         _I, _I, _VP]),
    "attn_selftest_wait_timeout": (_I, [ctypes.c_longlong, _VP]),
    "attn_selftest_ex2": (_I, [_VP, _VP, ctypes.c_longlong, _VP]),
    "attn_splitkv_num_splits": (_I, [_I, _I, _I, _I]),
    "attn_splitkv_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "attn_fwd_splitkv": (_I, [_VP, _VP, _VP, _VP, _FP, _I, _I, _I, _I, _I, _I, _F, _I, _I, _VP, _SZ, _I, _VP]),
    "attn_merge_partials": (_I, [_FP, _FP, _I, _VP, _FP, _I, _I, _I, _I, _I, _VP]),
    "attn_fwd_partial": (_I, [_VP, _VP, _VP, _FP, _FP, _I, _I, _I, _I, _I, _I, _F, _I, _I, _VP]),
    "attn_quantize_e4m3": (_I, [_VP, _VP, _FP, _I, _I, _I, _I, _VP]),
    "attn_fwd_fp8": (_I, [_VP, _FP, _VP, _FP, _VP, _VP, _FP, _I, _I, _I, _I, _I, _I, _F, _I, _VP]),
    "attn_bwd_workspace_size": (_SZ, [_I, _I, _I, _I]),
    "attn_bwd": (_I, [_VP, _VP, _VP, _FP, _LL, _VP, _FP, _VP, _VP, _VP, _VP, _VP, _SZ, _I, _I, _I, _I, _I,
                      _I, _F, _I, _I, _VP]),
    "attn_bwd_noalloc": (_I, [_VP, _VP, _VP, _FP, _LL, _VP, _FP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I,
                              _F, _I, _I, _VP]),
    "attn_fwd_varlen": (_I, [_VP, _VP, _VP, _VP, _FP, _IP, _IP, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I,
                             _VP]),
    "attn_naive_scratch_size": (_SZ, [_I, _I]),
    "attn_fwd_naive": (_I, [_VP, _VP, _VP, _VP, _FP, _VP, _SZ, _I, _I, _I, _I, _I, _I, _F, _I, _VP]),
    "attn_strerror": (ctypes.c_char_p, [_I]),
    "attn_device_status": (_I, [_VP]),
    "attn_launch_count": (_LL, [_I]),
    "attn_set_kernel_events": (_I, [_I, _VP, _VP]),
}

ATTN_KERNEL_FWD = 0
ATTN_KERNEL_BWD = 1


class AttnError(RuntimeError):
    pass


def _load() -> ctypes.CDLL:
    if not LIB_PATH.exists():
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m exact_io_aware_57_b200.build`")
    lib = ctypes.CDLL(str(LIB_PATH))
    for name, (res, args) in EXPORTS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def lib() -> ctypes.CDLL:
    return _lib


def _check(rc: int) -> None:
    if rc != ATTN_OK:
        raise AttnError(f"libattn error {rc}: {_lib.attn_strerror(rc).decode()}")


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return ATTN_BF16
    if t.dtype == torch.float32:
        return ATTN_F32
    raise AttnError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _dev(t: torch.Tensor, name: str) -> int:
    if not t.is_cuda:
        raise AttnError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise AttnError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _bias_args(bias, B, Hq, Nq, Nk):
    if bias is None:
        return None, 0
    if bias.dtype != torch.float32:
        raise AttnError("bias must be fp32")
    per = Hq * Nq * Nk
    if bias.numel() == per:
        return _dev(bias, "bias"), 0
    if bias.numel() == B * per:
        return _dev(bias, "bias"), per
    raise AttnError("bias must be [Hq,Nq,Nk] or [B,Hq,Nq,Nk]")


def _slopes(alibi_slopes, Hq):
    if alibi_slopes.dtype != torch.float32 or alibi_slopes.numel() != Hq:
        raise AttnError("alibi_slopes must be fp32 [h_q]")
    return _dev(alibi_slopes, "alibi_slopes")


def _window_args(window, bias):
    if bias is not None:
        raise AttnError("a local window takes alibi_slopes, not a dense bias")
    wl, wr = window
    return (-1 if wl is None else int(wl)), (-1 if wr is None else int(wr))


def attn_fwd(q, k, v, bias=None, causal=False, scale=None, out=None, lse=None, stream=None, alibi_slopes=None,
             window=None):
    """O, LSE = attention(q [B,Nq,Hq,d], k/v [B,Nk,Hkv,d]); o like q, lse fp32 [B,Hq,Nq].
    bias: dense fp32 [Hq,Nq,Nk] or [B,Hq,Nq,Nk]; alibi_slopes: fp32 [Hq] (bias
    -slope_h |j - (i + Nk - Nq)| formed in the kernel); at most one of the two.
    window = (left, right): local attention, keys a - left .. a + right of the
    key a = i + Nk - Nq aligned with row i (None or negative: unbounded)."""
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, Nq), device=q.device, dtype=torch.float32) if lse is None else lse
    if window is not None:
        wl, wr = _window_args(window, bias)
        _check(_lib.attn_fwd_local(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"),
                                   None if alibi_slopes is None else _slopes(alibi_slopes, Hq), _dev(o, "o"),
                                   _dev(lse, "lse"), B, Hq, Hkv, Nq, Nk, d, scale, int(bool(causal)), wl, wr,
                                   _dtype_code(q), _stream(stream)))
        return o, lse
    if alibi_slopes is not None:
        if bias is not None:
            raise AttnError("pass either bias or alibi_slopes")
        _check(_lib.attn_fwd_alibi(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _slopes(alibi_slopes, Hq),
                                   _dev(o, "o"), _dev(lse, "lse"), B, Hq, Hkv, Nq, Nk, d, scale, int(bool(causal)),
                                   _dtype_code(q), _stream(stream)))
        return o, lse
    bp, bs = _bias_args(bias, B, Hq, Nq, Nk)
    _check(_lib.attn_fwd(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), bp, bs, _dev(o, "o"), _dev(lse, "lse"),
                         B, Hq, Hkv, Nq, Nk, d, scale, int(bool(causal)), _dtype_code(q), _stream(stream)))
    return o, lse


def attn_fwd_dv(q, k, v, causal=False, scale=None, out=None, lse=None, stream=None):
    """Forward with V of its own width: q/k [..., d], v [B,Nk,Hkv,d_v] -> o [B,Nq,Hq,d_v]."""
    B, Nq, Hq, d = q.shape
    Nk, Hkv, dv = k.shape[1], k.shape[2], v.shape[3]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty((B, Nq, Hq, dv), device=q.device, dtype=q.dtype) if out is None else out
    lse = torch.empty((B, Hq, Nq), device=q.device, dtype=torch.float32) if lse is None else lse
    _check(_lib.attn_fwd_dv(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), _dev(lse, "lse"), B, Hq, Hkv,
                            Nq, Nk, d, dv, scale, int(bool(causal)), _dtype_code(q), _stream(stream)))
    return o, lse


def attn_bwd_dv(q, k, v, o, lse, dout, causal=False, scale=None, workspace=None, dq=None, dk=None, dv=None,
                stream=None):
    """Backward of attn_fwd_dv: q/k/dq/dk width d, v/o/dout/dv width d_v."""
    B, Nq, Hq, d = q.shape
    Nk, Hkv, d_v = k.shape[1], k.shape[2], v.shape[3]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = torch.empty(attn_bwd_workspace_size(B, Hq, Nq, d), device=q.device, dtype=torch.uint8)
    _check(_lib.attn_bwd_dv(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), _dev(lse, "lse"),
                            _dev(dout, "dout"), _dev(dq, "dq"), _dev(dk, "dk"), _dev(dv, "dv"),
                            _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(), B, Hq, Hkv,
                            Nq, Nk, d, d_v, scale, int(bool(causal)), _dtype_code(q), _stream(stream)))
    return dq, dk, dv


def attn_selftest_wait_timeout(limit_cycles=1_000_000, stream=None) -> None:
    """Launch the bounded-wait self-test (a wait that gives up after limit_cycles)."""
    _check(_lib.attn_selftest_wait_timeout(int(limit_cycles), _stream(stream)))


def attn_selftest_ex2(x, stream=None):
    """2^x by the kernels' FMA-pipe exponential (fp32 device tensor in, same out)."""
    if x.dtype != torch.float32 or not x.is_contiguous():
        raise ValueError("x must be a contiguous fp32 tensor")
    y = torch.empty_like(x)
    _check(_lib.attn_selftest_ex2(_dev(x, "x"), _dev(y, "y"), x.numel(), _stream(stream)))
    return y


def attn_splitkv_num_splits(batch, h_q, n_q, n_k) -> int:
    return int(_lib.attn_splitkv_num_splits(batch, h_q, n_q, n_k))


def attn_splitkv_workspace_size(batch, h_q, n_q, d, num_splits) -> int:
    return int(_lib.attn_splitkv_workspace_size(batch, h_q, n_q, d, num_splits))


def attn_fwd_splitkv(q, k, v, causal=False, scale=None, num_splits=0, out=None, lse=None, workspace=None,
                     stream=None):
    """attn_fwd computed over num_splits key ranges and merged (bf16, dense)."""
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, Nq), device=q.device, dtype=torch.float32) if lse is None else lse
    t = int(num_splits) if num_splits and num_splits > 0 else attn_splitkv_num_splits(B, Hq, Nq, Nk)
    if workspace is None:
        workspace = torch.empty(max(256, attn_splitkv_workspace_size(B, Hq, Nq, d, t)), device=q.device,
                                dtype=torch.uint8)
    _check(_lib.attn_fwd_splitkv(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), _dev(lse, "lse"), B, Hq,
                                 Hkv, Nq, Nk, d, scale, int(bool(causal)), t, _dev(workspace, "workspace"),
                                 workspace.numel() * workspace.element_size(), _dtype_code(q), _stream(stream)))
    return o, lse


def attn_fwd_partial(q, k, v, causal=False, scale=None, o_part=None, lse_part=None, stream=None):
    """Unmerged attention of q [B,Nq,Hq,d] over one key block k/v [B,Nk,Hkv,d] (bf16):
    o_part fp32 [B,Nq,Hq,d] (normalised over the block) and lse_part fp32 [B,Hq,Nq].
    Causal aligns the block bottom-right.  Partials of disjoint blocks combine
    with attn_merge_partials."""
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o_part = torch.empty((B, Nq, Hq, d), device=q.device, dtype=torch.float32) if o_part is None else o_part
    lse_part = torch.empty((B, Hq, Nq), device=q.device, dtype=torch.float32) if lse_part is None else lse_part
    if o_part.dtype != torch.float32 or lse_part.dtype != torch.float32:
        raise AttnError("partials are fp32")
    _check(_lib.attn_fwd_partial(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o_part, "o_part"),
                                 _dev(lse_part, "lse_part"), B, Hq, Hkv, Nq, Nk, d, scale, int(bool(causal)),
                                 _dtype_code(q), _stream(stream)))
    return o_part, lse_part


def attn_quantize_e4m3(x, x8=None, scales=None, stream=None):
    """Per-(batch, head) e4m3 quantisation of x bf16 [B,N,H,d]: returns x8 (uint8
    e4m3 bytes, same layout) and scales fp32 [B,H] (amax / 448)."""
    if x.dtype != torch.bfloat16:
        raise AttnError("x must be bf16")
    B, N, H, d = x.shape
    x8 = torch.empty(x.shape, device=x.device, dtype=torch.uint8) if x8 is None else x8
    scales = torch.empty((B, H), device=x.device, dtype=torch.float32) if scales is None else scales
    _check(_lib.attn_quantize_e4m3(_dev(x, "x"), _dev(x8, "x8"), _dev(scales, "scales"), B, N, H, d,
                                   _stream(stream)))
    return x8, scales


def attn_fwd_fp8(q8, q_scales, k8, k_scales, v, causal=False, scale=None, out=None, lse=None, stream=None):
    """Forward with S = Q8 K8^T on e4m3 tensor cores (see attn_quantize_e4m3), P V in
    bf16: o bf16 [B,Nq,Hq,d], lse fp32 [B,Hq,Nq].  d = 128."""
    B, Nq, Hq, d = q8.shape
    Nk, Hkv = k8.shape[1], k8.shape[2]
    if v.dtype != torch.bfloat16:
        raise AttnError("v must be bf16")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty((B, Nq, Hq, d), device=v.device, dtype=torch.bfloat16) if out is None else out
    lse = torch.empty((B, Hq, Nq), device=v.device, dtype=torch.float32) if lse is None else lse
    _check(_lib.attn_fwd_fp8(_dev(q8, "q8"), _dev(q_scales, "q_scales"), _dev(k8, "k8"), _dev(k_scales, "k_scales"),
                             _dev(v, "v"), _dev(o, "o"), _dev(lse, "lse"), B, Hq, Hkv, Nq, Nk, d, scale,
                             int(bool(causal)), _stream(stream)))
    return o, lse


def attn_merge_partials(o_parts, lse_parts, out=None, lse=None, out_dtype=torch.bfloat16, stream=None):
    """Merge fp32 partials o_parts [T,B,Nq,Hq,d], lse_parts [T,B,Hq,Nq] over disjoint key ranges."""
    if o_parts.dtype != torch.float32 or lse_parts.dtype != torch.float32:
        raise AttnError("partials must be fp32")
    T, B, Nq, Hq, d = o_parts.shape
    o = torch.empty((B, Nq, Hq, d), device=o_parts.device, dtype=out_dtype) if out is None else out
    lse = torch.empty((B, Hq, Nq), device=o_parts.device, dtype=torch.float32) if lse is None else lse
    code = 0 if o.dtype == torch.bfloat16 else 1 if o.dtype == torch.float32 else None
    if code is None:
        raise AttnError("merge output must be bf16 or fp32")
    _check(_lib.attn_merge_partials(_dev(o_parts, "o_parts"), _dev(lse_parts, "lse_parts"), T, _dev(o, "o"),
                                    _dev(lse, "lse"), B, Hq, Nq, d, code, _stream(stream)))
    return o, lse


def attn_bwd_workspace_size(batch, h_q, n_q, d) -> int:
    return int(_lib.attn_bwd_workspace_size(batch, h_q, n_q, d))


def attn_bwd(q, k, v, o, lse, dout, bias=None, causal=False, scale=None, workspace=None, dq=None, dk=None,
             dv=None, stream=None, alibi_slopes=None, window=None):
    """dq, dk, dv of attn_fwd for upstream gradient dout (layouts as q, k, v)."""
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = attn_bwd_workspace_size(B, Hq, Nq, d)
    if workspace is None:
        workspace = torch.empty(need, device=q.device, dtype=torch.uint8)
    if window is not None:
        wl, wr = _window_args(window, bias)
        _check(_lib.attn_bwd_local(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"),
                                   None if alibi_slopes is None else _slopes(alibi_slopes, Hq), _dev(o, "o"),
                                   _dev(lse, "lse"), _dev(dout, "dout"), _dev(dq, "dq"), _dev(dk, "dk"),
                                   _dev(dv, "dv"), _dev(workspace, "workspace"),
                                   workspace.numel() * workspace.element_size(), B, Hq, Hkv, Nq, Nk, d, scale,
                                   int(bool(causal)), wl, wr, _dtype_code(q), _stream(stream)))
        return dq, dk, dv
    if alibi_slopes is not None:
        if bias is not None:
            raise AttnError("pass either bias or alibi_slopes")
        _check(_lib.attn_bwd_alibi(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _slopes(alibi_slopes, Hq),
                                   _dev(o, "o"), _dev(lse, "lse"), _dev(dout, "dout"), _dev(dq, "dq"),
                                   _dev(dk, "dk"), _dev(dv, "dv"), _dev(workspace, "workspace"),
                                   workspace.numel() * workspace.element_size(), B, Hq, Hkv, Nq, Nk, d, scale,
                                   int(bool(causal)), _dtype_code(q), _stream(stream)))
        return dq, dk, dv
    bp, bs = _bias_args(bias, B, Hq, Nq, Nk)
    _check(_lib.attn_bwd(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), bp, bs, _dev(o, "o"), _dev(lse, "lse"),
                         _dev(dout, "dout"), _dev(dq, "dq"), _dev(dk, "dk"), _dev(dv, "dv"),
                         _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
                         B, Hq, Hkv, Nq, Nk, d, scale, int(bool(causal)), _dtype_code(q), _stream(stream)))
    return dq, dk, dv


def attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, causal=False, scale=None,
                    out=None, lse=None, stream=None):
    """Packed forward: q [Tq,Hq,d], k/v [Tk,Hkv,d], cu_seqlens int32 device; lse [Hq,Tq]."""
    Tq, Hq, d = q.shape
    Tk, Hkv = k.shape[0], k.shape[1]
    if cu_seqlens_q.dtype != torch.int32 or cu_seqlens_k.dtype != torch.int32:
        raise AttnError("cu_seqlens must be int32")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty_like(q) if out is None else out
    lse = torch.empty((Hq, Tq), device=q.device, dtype=torch.float32) if lse is None else lse
    _check(_lib.attn_fwd_varlen(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), _dev(lse, "lse"),
                                _dev(cu_seqlens_q, "cu_seqlens_q"), _dev(cu_seqlens_k, "cu_seqlens_k"),
                                cu_seqlens_q.numel() - 1, int(max_seqlen_q), int(max_seqlen_k), Tq, Tk, Hq, Hkv,
                                d, scale, int(bool(causal)), _dtype_code(q), _stream(stream)))
    return o, lse


def attn_bwd_varlen(q, k, v, o, lse, dout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, causal=False,
                    scale=None, workspace=None, dq=None, dk=None, dv=None, stream=None):
    """Backward of attn_fwd_varlen: dq like q [Tq,Hq,d], dk/dv like k/v [Tk,Hkv,d]."""
    Tq, Hq, d = q.shape
    Tk, Hkv = k.shape[0], k.shape[1]
    if cu_seqlens_q.dtype != torch.int32 or cu_seqlens_k.dtype != torch.int32:
        raise AttnError("cu_seqlens must be int32")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = torch.empty(attn_bwd_workspace_size(1, Hq, Tq, d), device=q.device, dtype=torch.uint8)
    _check(_lib.attn_bwd_varlen(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), _dev(lse, "lse"),
                                _dev(dout, "dout"), _dev(dq, "dq"), _dev(dk, "dk"), _dev(dv, "dv"),
                                _dev(cu_seqlens_q, "cu_seqlens_q"), _dev(cu_seqlens_k, "cu_seqlens_k"),
                                cu_seqlens_q.numel() - 1, int(max_seqlen_q), int(max_seqlen_k), Tq, Tk, Hq, Hkv, d,
                                scale, int(bool(causal)), _dev(workspace, "workspace"),
                                workspace.numel() * workspace.element_size(), _dtype_code(q), _stream(stream)))
    return dq, dk, dv


def attn_naive_scratch_size(n_q, n_k) -> int:
    return int(_lib.attn_naive_scratch_size(n_q, n_k))


def attn_fwd_naive(q, k, v, causal=False, scale=None, scratch=None, stream=None):
    """Materialising three-step forward (measurement comparator only)."""
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Nq), device=q.device, dtype=torch.float32)
    if scratch is None:
        scratch = torch.empty(attn_naive_scratch_size(Nq, Nk), device=q.device, dtype=torch.uint8)
    _check(_lib.attn_fwd_naive(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), _dev(lse, "lse"),
                               _dev(scratch, "scratch"), scratch.numel(), B, Hq, Hkv, Nq, Nk, d, scale,
                               int(bool(causal)), _stream(stream)))
    return o, lse


def attn_device_status(stream=None) -> int:
    """Synchronise and return/clear the device status word: 0, ATTN_ERR_TIMEOUT
    (a bounded wait gave up) or ATTN_ERR_INVALID (packed offsets rejected)."""
    return int(_lib.attn_device_status(_stream(stream)))


def attn_launch_count(reset: bool = False) -> int:
    return int(_lib.attn_launch_count(int(bool(reset))))


def attn_set_kernel_events(which: int, start=None, stop=None) -> None:
    """Record torch.cuda.Event pair (start, stop) around launches of kernel `which`
    (ATTN_KERNEL_FWD / ATTN_KERNEL_BWD) from this thread; None clears."""
    sp = None if start is None else start.cuda_event
    ep = None if stop is None else stop.cuda_event
    if (start is not None and not sp) or (stop is not None and not ep):
        raise AttnError("record the events once (torch creates them lazily) before registering them")
    _check(_lib.attn_set_kernel_events(int(which), sp, ep))
