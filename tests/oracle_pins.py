"""Pins that tie the fp64 oracle to facts fixed by the pages or by mathematics,
not to the oracle itself.  Each pin returns (ok, detail).  They are run on the
real oracle (test_oracle_pins.py) and on variants with planted mistakes
(test_oracle_mutants.py), which every pin set must reject.

Sources:
  * merge recurrence == one-shot softmax: "Softmax does not need the matrix",
    "Carry the Normalizer" (the carried (m, l, a) state suffices to resume the
    softmax without error) and its lab (materialised and streamed rows agree);
  * constant scores / single key / causal row 0 / permutation and shift
    invariance: closed forms of the softmax definition (same page and the
    handbook's 0.2 Notation);
  * library special case: scipy's logsumexp/softmax on the plain
    non-causal problem;
  * backward: central finite differences of the forward in fp64;
  * local (sliding-window) attention, named in the handbook's contents (4.2)
    without a definition: the reading a - left <= j <= a + right with
    a = i + Nk - Nq is checked against scipy's softmax over exactly that slice.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import logsumexp, softmax


def _rand(rng, *shape, scale=1.0):
    return rng.standard_normal(shape) * scale


def _rel(a, b):
    """Max relative error; a mismatch in non-finite entries (e.g. -inf against a
    finite value) counts as an infinite error."""
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    fa, fb = np.isfinite(a), np.isfinite(b)
    if not np.array_equal(fa, fb) or not np.array_equal(a[~fa], b[~fb]):
        return float("inf")
    if not fa.any():
        return 0.0
    return float(np.max(np.abs(a[fa] - b[fb])) / max(1e-300, np.max(np.abs(b[fb]))))


def pin_merge_every_split(orc):
    """Split the keys of a row at every point (and into random 3-4 shards):
    merging the exact per-shard (o, lse) equals the one-shot result."""
    rng = np.random.default_rng(11)
    worst = 0.0
    for nk in (1, 2, 5, 16):
        q = _rand(rng, 1, 3, 2, 4)
        k = _rand(rng, 1, nk, 2, 4, scale=2.0)
        v = _rand(rng, 1, nk, 2, 4)
        o_ref, l_ref = orc.fwd(q, k, v)
        splits = [[t] for t in range(1, nk)]
        for _ in range(4):
            if nk >= 4:
                splits.append(sorted(rng.choice(np.arange(1, nk), size=min(3, nk - 1), replace=False).tolist()))
        for sp in splits:
            bounds = [0] + list(sp) + [nk]
            parts_o, parts_l = [], []
            for a, b in zip(bounds[:-1], bounds[1:]):
                o_t, l_t = orc.fwd(q, k[:, a:b], v[:, a:b])
                parts_o.append(o_t.transpose(0, 2, 1, 3).reshape(-1, 4))   # rows (b,h,i)
                parts_l.append(l_t.reshape(-1))
            o_m, l_m = orc.merge_partials(np.stack(parts_o), np.stack(parts_l))
            worst = max(worst, _rel(o_m, o_ref.transpose(0, 2, 1, 3).reshape(-1, 4)),
                        _rel(l_m, l_ref.reshape(-1)))
    return worst <= 1e-13, f"max rel err {worst:.2e}"


def pin_stream_equals_oneshot(orc):
    """Streaming (m, l, a) replay with every block size equals the one-shot row
    (also under local windows, where a row's first block starts mid-sequence)."""
    rng = np.random.default_rng(12)
    worst = 0.0
    q = _rand(rng, 2, 16, 2, 8, scale=2.0)
    k = _rand(rng, 2, 16, 1, 8, scale=2.0)
    v = _rand(rng, 2, 16, 1, 8)
    bias = _rand(rng, 2, 16, 16)
    for causal, window in ((False, None), (True, None), (True, (5, None)), (False, (3, 2))):
        for b in (None, bias):
            o_ref, l_ref = orc.fwd(q, k, v, bias=b, causal=causal, window=window)
            for blk in range(1, 17):
                o_s, l_s, _ = orc.fwd_stream(q, k, v, bias=b, causal=causal, block=blk, window=window)
                worst = max(worst, _rel(o_s, o_ref), _rel(l_s, l_ref))
    return worst <= 1e-13, f"max rel err {worst:.2e}"


def pin_constant_scores(orc):
    """Equal scores (Q = 0, optional constant bias c): o is the mean of the
    visible values and LSE = c + ln(#visible)."""
    rng = np.random.default_rng(13)
    nq, nk, d = 6, 6, 4
    q = np.zeros((1, nq, 2, d))
    k = _rand(rng, 1, nk, 2, d)
    v = _rand(rng, 1, nk, 2, d)
    worst = 0.0
    for c in (0.0, 1.75, -3.0):
        bias = np.full((2, nq, nk), c)
        for causal in (False, True):
            o, l = orc.fwd(q, k, v, bias=bias, causal=causal)
            for i in range(nq):
                n = i + 1 if causal else nk
                for h in range(2):
                    worst = max(worst, _rel(o[0, i, h], v[0, :n, h].mean(axis=0)),
                                abs(l[0, h, i] - (c + math.log(n))))
    return worst <= 1e-13, f"max err {worst:.2e}"


def pin_single_key(orc):
    """One key: o = v_0 and LSE = s_0 = scale * q.k_0 + B."""
    rng = np.random.default_rng(14)
    d = 8
    q = _rand(rng, 2, 3, 2, d)
    k = _rand(rng, 2, 1, 2, d)
    v = _rand(rng, 2, 1, 2, d)
    bias = _rand(rng, 2, 3, 1)
    worst = 0.0
    for b in (None, bias):
        o, l = orc.fwd(q, k, v, bias=b)
        s0 = np.einsum("bihc,bhc->bhi", q, k[:, 0]) / math.sqrt(d)
        if b is not None:
            s0 = s0 + b[None, :, :, 0]
        worst = max(worst, _rel(o, np.broadcast_to(v, o.shape)), _rel(l, s0))
    return worst <= 1e-13, f"max rel err {worst:.2e}"


def pin_causal_prefix(orc):
    """Causal: row 0 returns v_0; row i equals the non-causal result over keys 0..i."""
    rng = np.random.default_rng(15)
    nq, d = 9, 4
    q = _rand(rng, 1, nq, 1, d, scale=2.0)
    k = _rand(rng, 1, nq, 1, d, scale=2.0)
    v = _rand(rng, 1, nq, 1, d)
    o, l = orc.fwd(q, k, v, causal=True)
    worst = _rel(o[0, 0, 0], v[0, 0, 0])
    for i in range(nq):
        o_i, l_i = orc.fwd(q[:, i:i + 1], k[:, :i + 1], v[:, :i + 1])
        worst = max(worst, _rel(o[0, i], o_i[0, 0]), abs(l[0, 0, i] - l_i[0, 0, 0]))
    return worst <= 1e-13, f"max err {worst:.2e}"


def pin_permutation(orc):
    """Non-causal O and LSE are invariant under one shared permutation of K/V rows."""
    rng = np.random.default_rng(16)
    q = _rand(rng, 2, 5, 4, 8)
    k = _rand(rng, 2, 7, 2, 8)
    v = _rand(rng, 2, 7, 2, 8)
    perm = rng.permutation(7)
    o1, l1 = orc.fwd(q, k, v)
    o2, l2 = orc.fwd(q, k[:, perm], v[:, perm])
    worst = max(_rel(o2, o1), _rel(l2, l1))
    return worst <= 1e-13, f"max rel err {worst:.2e}"


def pin_shift(orc):
    """Adding c to every bias entry of a row leaves o unchanged and shifts LSE by c."""
    rng = np.random.default_rng(17)
    q = _rand(rng, 1, 4, 2, 8)
    k = _rand(rng, 1, 6, 2, 8)
    v = _rand(rng, 1, 6, 2, 8)
    bias = _rand(rng, 2, 4, 6)
    shift = rng.standard_normal((2, 4, 1)) * 3
    worst = 0.0
    for causal in (False, True):
        o1, l1 = orc.fwd(q, k, v, bias=bias, causal=causal)
        o2, l2 = orc.fwd(q, k, v, bias=bias + shift, causal=causal)
        worst = max(worst, _rel(o2, o1), float(np.max(np.abs(l2 - l1 - shift[None, :, :, 0]))))
    return worst <= 1e-12, f"max err {worst:.2e}"


def pin_library_softmax(orc):
    """Non-causal, no bias, GQA 4:2: equals scipy softmax / logsumexp per head
    (query head h reads KV head h // 2)."""
    rng = np.random.default_rng(18)
    B, nq, nk, hq, hkv, d = 2, 5, 7, 4, 2, 8
    q = _rand(rng, B, nq, hq, d)
    k = _rand(rng, B, nk, hkv, d)
    v = _rand(rng, B, nk, hkv, d)
    o, l = orc.fwd(q, k, v, scale=0.3)
    worst = 0.0
    for b in range(B):
        for h in range(hq):
            s = 0.3 * (q[b, :, h] @ k[b, :, h // 2].T)
            worst = max(worst, _rel(o[b, :, h], softmax(s, axis=1) @ v[b, :, h // 2]),
                        _rel(l[b, h], logsumexp(s, axis=1)))
    return worst <= 1e-13, f"max rel err {worst:.2e}"


def _loss(orc, q, k, v, dout, bias, causal, window=None):
    o, _ = orc.fwd(q, k, v, bias=bias, causal=causal, window=window)
    return float(np.sum(o * dout))


def pin_backward_fd(orc):
    """Central finite differences (step 1e-6) of sum(dO * O) w.r.t. Q, K, V,
    including a value width d_v != d and local windows."""
    rng = np.random.default_rng(19)
    worst = 0.0
    # (B, Nq, Nk, Hq, Hkv, d, d_v, causal, bias, window)
    for (B, nq, nk, hq, hkv, d, dv_, causal, use_bias, window) in (
            (1, 5, 5, 2, 1, 4, 4, True, True, None),
            (1, 3, 6, 2, 2, 3, 3, False, False, None),
            (2, 4, 4, 1, 1, 2, 2, True, False, None),
            (1, 6, 6, 2, 1, 3, 3, True, True, (2, -1)),
            (1, 5, 7, 1, 1, 2, 2, False, False, (1, 1)),
            (1, 4, 5, 2, 1, 3, 5, True, False, None)):      # value width d_v != d
        q = _rand(rng, B, nq, hq, d)
        k = _rand(rng, B, nk, hkv, d)
        v = _rand(rng, B, nk, hkv, dv_)
        dout = _rand(rng, B, nq, hq, dv_)
        bias = _rand(rng, hq, nq, nk) if use_bias else None
        dq, dk, dv = orc.bwd(q, k, v, dout, bias=bias, causal=causal, window=window)
        for x, g in ((q, dq), (k, dk), (v, dv)):
            num = np.zeros_like(x)
            it = np.nditer(x, flags=["multi_index"])
            for _ in it:
                idx = it.multi_index
                old = x[idx]
                x[idx] = old + 1e-6
                lp = _loss(orc, q, k, v, dout, bias, causal, window)
                x[idx] = old - 1e-6
                lm = _loss(orc, q, k, v, dout, bias, causal, window)
                x[idx] = old
                num[idx] = (lp - lm) / 2e-6
            worst = max(worst, float(np.linalg.norm(g - num) / max(1e-300, np.linalg.norm(num))))
    return worst <= 1e-6, f"max rel Frobenius err {worst:.2e}"


def pin_gqa_sum(orc):
    """GQA gradients equal the MHA gradients of the same problem with K/V
    replicated per query head, summed over each group."""
    rng = np.random.default_rng(20)
    B, n, hq, hkv, d = 1, 6, 4, 2, 4
    q = _rand(rng, B, n, hq, d)
    k = _rand(rng, B, n, hkv, d)
    v = _rand(rng, B, n, hkv, d)
    dout = _rand(rng, B, n, hq, d)
    dq, dk, dv = orc.bwd(q, k, v, dout, causal=True)
    rep = np.repeat(np.arange(hkv), hq // hkv)
    dq2, dk2, dv2 = orc.bwd(q, k[:, :, rep], v[:, :, rep], dout, causal=True)
    dk_sum = dk2.reshape(B, n, hkv, hq // hkv, d).sum(axis=3)
    dv_sum = dv2.reshape(B, n, hkv, hq // hkv, d).sum(axis=3)
    worst = max(_rel(dq, dq2), _rel(dk, dk_sum), _rel(dv, dv_sum))
    return worst <= 1e-12, f"max rel err {worst:.2e}"


def pin_window_slices(orc):
    """Local attention: row i equals scipy's softmax over exactly the keys
    a - left .. a + right (a = i + Nk - Nq; causal caps the right side at a;
    a negative size is unbounded), and with left = 0 under causal the single
    key a is left, so o_i = v_a."""
    rng = np.random.default_rng(21)
    worst = 0.0
    d = 4
    for (nq, nk, wl, wr, causal) in ((9, 9, 2, -1, True), (9, 9, 0, -1, True), (7, 11, 3, 1, False),
                                     (11, 7, 1, 2, False), (8, 8, -1, 2, False), (6, 10, 4, 5, True),
                                     (10, 4, 1, -1, True)):
        q = _rand(rng, 1, nq, 2, d, scale=1.5)
        k = _rand(rng, 1, nk, 1, d, scale=1.5)
        v = _rand(rng, 1, nk, 1, d)
        bias = _rand(rng, 2, nq, nk)
        o, l = orc.fwd(q, k, v, bias=bias, causal=causal, window=(wl, wr))
        for h in range(2):
            for i in range(nq):
                a = i + nk - nq
                lo = 0 if wl < 0 else max(0, a - wl)
                hi = nk - 1 if wr < 0 else min(nk - 1, a + wr)
                if causal:
                    hi = min(hi, a)
                if hi < lo:
                    if not (np.all(o[0, i, h] == 0.0) and l[0, h, i] == -np.inf):
                        return False, f"row {i} has no visible key but o/LSE are not 0/-inf"
                    continue
                s = q[0, i, h] @ k[0, lo:hi + 1, 0].T / math.sqrt(d) + bias[h, i, lo:hi + 1]
                worst = max(worst, float(np.max(np.abs(o[0, i, h] - softmax(s) @ v[0, lo:hi + 1, 0]))),
                            abs(float(l[0, h, i] - logsumexp(s))))
        if causal and wl == 0 and nq == nk:
            worst = max(worst, float(np.max(np.abs(o[0, :, :, :] - v[0, :, 0, None, :]))))
    return worst <= 1e-13, f"max abs err {worst:.2e}"


def pin_value_width(orc):
    """V with its own width d_v != d (the handbook's 0.2 Notation gives V a
    separate width): every row equals scipy's softmax of its scaled scores
    times V, for d_v = 12 and 3 against d = 8, causal and not, GQA 4:2."""
    rng = np.random.default_rng(22)
    worst = 0.0
    B, nq, nk, hq, hkv, d = 2, 6, 9, 4, 2, 8
    for dv in (12, 3):
        for causal in (False, True):
            q = _rand(rng, B, nq, hq, d)
            k = _rand(rng, B, nk, hkv, d)
            v = _rand(rng, B, nk, hkv, dv)
            o, l = orc.fwd(q, k, v, causal=causal)
            if o.shape != (B, nq, hq, dv):
                return False, f"output shape {o.shape}"
            for b in range(B):
                for h in range(hq):
                    for i in range(nq):
                        last = nk - 1 if not causal else i + (nk - nq)
                        s_ = q[b, i, h] @ k[b, :last + 1, h // 2].T / math.sqrt(d)
                        worst = max(worst, float(np.max(np.abs(o[b, i, h] - softmax(s_) @ v[b, :last + 1, h // 2]))),
                                    abs(float(l[b, h, i] - logsumexp(s_))))
    return worst <= 1e-13, f"max abs err {worst:.2e}"


ALL_PINS = {
    "value_width": pin_value_width,
    "window_slices": pin_window_slices,
    "merge_every_split": pin_merge_every_split,
    "stream_equals_oneshot": pin_stream_equals_oneshot,
    "constant_scores": pin_constant_scores,
    "single_key": pin_single_key,
    "causal_prefix": pin_causal_prefix,
    "permutation": pin_permutation,
    "shift": pin_shift,
    "library_softmax": pin_library_softmax,
    "backward_fd": pin_backward_fd,
    "gqa_sum": pin_gqa_sum,
}
