"""The five attention workloads this library is measured and checked on, and the
matmul-only FLOP convention used to turn their timings into TFLOP/s.

FLOP convention: only the matrix products count.  The forward of one
(batch, query head) is 4*Nq*Nk*d (QK^T and PV, 2 FLOPs per multiply-add),
halved under causal masking with Nq == Nk; the backward performs five such
products (S recompute, dP, dV, dK, dQ), i.e. 2.5x the forward.
"""
from __future__ import annotations

from dataclasses import dataclass, field

from . import synth


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    h_q: int
    h_kv: int
    n: int
    d: int
    dtype: str            # "bf16" or "f32"
    causal: bool
    backward: bool
    sigma_qk: float = 1.0
    bias: bool = False
    varlen: bool = False
    num_seqs: int = 0
    len_lo: int = 0
    len_hi: int = 0
    n_q: int = 0              # query length when it differs from n (the key length)
    splitkv: bool = False     # forward through the split-KV path
    fp8: bool = False         # Q, K quantised to e4m3 per (batch, head); S on e4m3 tensor cores, P V in bf16
    description: str = field(default="", compare=False)


WORKLOADS = {
    "c1": Workload("single-head fp32 N=128 d=64 fwd+bwd", 1, 1, 1, 128, 64, "f32", False, True,
                   description="batch 1, 1 head, N=128, d=64, fp32 N(0,1), non-causal"),
    "c2": Workload("MHA bf16 B=4 H=16 N=2048 d=64 fwd", 4, 16, 16, 2048, 64, "bf16", False, False,
                   description="batch 4, 16 heads, N=2048, d=64, bf16 N(0,1), non-causal, forward"),
    "c3": Workload("causal bf16 B=2 H=32 N=8192 d=128 fwd+bwd", 2, 32, 32, 8192, 128, "bf16", True,
                   True, sigma_qk=3.0,
                   description="batch 2, 32 heads, N=8192, d=128, bf16, Q/K N(0,9), V/dO N(0,1), causal"),
    "c4": Workload("GQA 32:8 causal+bias bf16 B=4 N=4096 d=128 fwd+bwd", 4, 32, 8, 4096, 128, "bf16",
                   True, True, bias=True,
                   description="batch 4, 32 query / 8 KV heads, N=4096, d=128, causal, fp32 ALiBi-like bias"),
    "c5a": Workload("varlen causal bf16 16 seqs L~U[512,8192] H=32 d=128 fwd", 1, 32, 32, 0, 128, "bf16",
                    True, False, varlen=True, num_seqs=16, len_lo=512, len_hi=8192,
                    description="16 packed sequences, lengths uniform in [512, 8192] from the seed"),
    "kv1": Workload("split-KV: causal bf16 B=1 Hq=32 Hkv=8 Nq=512 Nk=65536 d=128 fwd", 1, 32, 8, 65536, 128,
                    "bf16", True, False, n_q=512, splitkv=True,
                    description="a 512-query block at the end of a 65536-key sequence (bottom-right causal), "
                                "GQA 32:8: 128 query-tile CTAs alone would not fill 148 SMs"),
    "c3fp8": Workload("FP8 causal B=2 H=32 N=8192 d=128 fwd (e4m3 Q/K, bf16 P V)", 2, 32, 32, 8192, 128, "e4m3+bf16",
                      True, False, sigma_qk=3.0, fp8=True,
                      description="the causal workload's forward with per-head e4m3 quantisation of Q and K "
                                  "inside the step"),
    "c5b": Workload("single sequence causal bf16 N=32768 H=16 d=128 fwd", 1, 16, 16, 32768, 128, "bf16",
                    True, False,
                    description="one sequence of 32768 tokens, 16 heads, causal, forward"),
}


def fwd_flops_pair(nq: int, nk: int, d: int, causal: bool) -> float:
    """Forward matmul FLOPs of one (batch, head) under the convention above."""
    return 4.0 * nq * nk * d * (0.5 if causal else 1.0)


def window_pairs(n: int, left: int) -> int:
    """Visible (query, key) pairs of causal self-attention over n tokens when
    each row also sees at most ``left`` earlier keys."""
    w = min(int(left), n - 1)
    # rows 0 .. w-1 see i + 1 keys, the other n - w rows see w + 1
    return w * (w + 1) // 2 + (n - w) * (w + 1) if n > 0 else 0


def flops(w: Workload, backward: bool | None = None, lengths=None, window: int | None = None) -> float:
    """Forward (+ backward when ``backward``) FLOPs of a whole workload.  With a
    causal sliding ``window`` (keys i - window .. i) the count is 4*d per
    visible pair, pairs counted exactly."""
    bwd = w.backward if backward is None else backward
    if w.n_q:
        nq, nk = w.n_q, w.n
        pairs = nq * (nk - nq) + nq * (nq + 1) // 2 if w.causal else nq * nk
        return 4.0 * w.d * pairs * w.batch * w.h_q * (3.5 if bwd else 1.0)
    if window is not None:
        assert not w.varlen and w.causal
        f = 4.0 * w.d * window_pairs(w.n, window) * w.batch * w.h_q
        return f * (3.5 if bwd else 1.0)
    if w.varlen:
        if lengths is None:
            lengths = synth.varlen_lengths(w.num_seqs, w.len_lo, w.len_hi)
        f = sum(fwd_flops_pair(int(L), int(L), w.d, w.causal) for L in lengths) * w.h_q
    else:
        f = fwd_flops_pair(w.n, w.n, w.d, w.causal) * w.batch * w.h_q
    return f * (3.5 if bwd else 1.0)
