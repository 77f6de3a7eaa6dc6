"""Seeded synthetic inputs shared by the tests, the benchmark and the smoke check.

This module draws random numbers and builds the input tensors only; it holds
none of the attention arithmetic.  Both the CUDA path and the fp64 oracle read
the tensors it returns (the oracle widens the same bf16/fp32 values to fp64).

Recipe: every tensor comes from a CPU ``torch.Generator`` seeded with
``seed`` (default 0) in a fixed order (q, k, v, dout), drawn as fp32
``randn * sigma`` and then cast to the working dtype.  The additive bias of
the grouped-query workload is the ALiBi-like slope matrix
``B[h, i, j] = -0.05 * |i - j| * (h + 1) / 32`` in fp32 (h = query head).
Variable lengths are drawn with ``numpy.random.default_rng(seed)`` uniformly
from an inclusive range and turned into int32 prefix offsets.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch


@dataclass
class Inputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    dout: torch.Tensor | None = None
    bias: torch.Tensor | None = None
    cu_seqlens: torch.Tensor | None = None  # int32 [num_seqs + 1] for packed inputs


def _randn(gen: torch.Generator, shape, sigma: float, dtype: torch.dtype) -> torch.Tensor:
    x = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if sigma != 1.0:
        x.mul_(sigma)
    return x.to(dtype)


def make_dense(batch: int, h_q: int, h_kv: int, n_q: int, n_k: int, d: int, *,
               dtype: torch.dtype = torch.bfloat16, seed: int = 0, sigma_qk: float = 1.0,
               sigma_v: float = 1.0, with_dout: bool = True) -> Inputs:
    """Q [B,Nq,Hq,d], K/V [B,Nk,Hkv,d] (and dO [B,Nq,Hq,d]) on the CPU."""
    g = torch.Generator().manual_seed(int(seed))
    q = _randn(g, (batch, n_q, h_q, d), sigma_qk, dtype)
    k = _randn(g, (batch, n_k, h_kv, d), sigma_qk, dtype)
    v = _randn(g, (batch, n_k, h_kv, d), sigma_v, dtype)
    dout = _randn(g, (batch, n_q, h_q, d), 1.0, dtype) if with_dout else None
    return Inputs(q, k, v, dout)


def alibi_like_bias(h_q: int, n_q: int, n_k: int, rows=None, heads=None,
                    device: str | torch.device = "cpu") -> torch.Tensor:
    """fp32 bias B[h, i, j] = -0.05 * |i - j| * (h + 1) / 32.

    ``heads`` / ``rows`` restrict the result to a subset (the full tensor is
    [h_q, n_q, n_k]).  Computed in fp32 with the same operation order on any
    device, so a subset equals the matching slice of the full tensor.
    """
    hs = torch.arange(h_q, device=device) if heads is None else torch.as_tensor(heads, device=device)
    ii = torch.arange(n_q, device=device) if rows is None else torch.as_tensor(rows, device=device)
    jj = torch.arange(n_k, device=device)
    dist = (ii[:, None] - jj[None, :]).abs().to(torch.float32)          # [R, Nk]
    slope = (hs.to(torch.float32) + 1.0) / 32.0                          # [H]
    return (-0.05 * dist)[None, :, :] * slope[:, None, None]


def alibi_like_slopes(h_q: int) -> torch.Tensor:
    """fp32 slopes (h + 1) * 0.05 / 32 of the grouped workload's bias."""
    return (torch.arange(h_q, dtype=torch.float32) + 1.0) * (0.05 / 32.0)


def bias_from_slopes(slopes, n_q: int, n_k: int) -> torch.Tensor:
    """Dense fp32 bias B[h, i, j] = -slope_h * |j - (i + n_k - n_q)| (fp32)."""
    i = torch.arange(n_q)[:, None]
    j = torch.arange(n_k)[None, :]
    dist = (j - (i + (n_k - n_q))).abs().to(torch.float32)
    return -torch.as_tensor(slopes, dtype=torch.float32)[:, None, None] * dist[None]


def varlen_lengths(num_seqs: int, lo: int, hi: int, seed: int = 0) -> np.ndarray:
    """Sequence lengths drawn uniformly from [lo, hi] (inclusive)."""
    return np.random.default_rng(int(seed)).integers(lo, hi + 1, size=int(num_seqs))


def cu_seqlens_of(lengths) -> torch.Tensor:
    """int32 prefix offsets [0, L0, L0+L1, ...]."""
    lengths = np.asarray(lengths, dtype=np.int64)
    cu = np.zeros(len(lengths) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(lengths)
    return torch.from_numpy(cu.astype(np.int32))


def make_packed(lengths, h_q: int, h_kv: int, d: int, *, dtype: torch.dtype = torch.bfloat16,
                seed: int = 0, sigma_qk: float = 1.0, with_dout: bool = False) -> Inputs:
    """Packed Q [T,Hq,d], K/V [T,Hkv,d] with cu_seqlens for the given lengths."""
    cu = cu_seqlens_of(lengths)
    total = int(cu[-1])
    g = torch.Generator().manual_seed(int(seed))
    q = _randn(g, (total, h_q, d), sigma_qk, dtype)
    k = _randn(g, (total, h_kv, d), sigma_qk, dtype)
    v = _randn(g, (total, h_kv, d), 1.0, dtype)
    dout = _randn(g, (total, h_q, d), 1.0, dtype) if with_dout else None
    return Inputs(q, k, v, dout, None, cu)
