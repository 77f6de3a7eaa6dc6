"""The oracle's e4m3 rounding (the input side of an FP8 forward: its oracle is
the exact attention of the dequantised inputs), pinned against what fixes it:
every finite e4m3 value decoded by torch is a fixed point, torch's own cast
agrees on random values and on every exact tie inside the finite range, values
beyond it saturate, and the rounding error respects the 3-bit mantissa bound."""
import numpy as np
import pytest
import torch


def _codes():
    v = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    return v[np.isfinite(v)]


def test_every_e4m3_value_is_a_fixed_point(orc):
    v = _codes()
    assert v.size == 254
    assert np.array_equal(orc.quantize_e4m3(v), v)


def test_matches_torch_cast_inside_the_finite_range(orc):
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-448, 448, 200000), rng.standard_normal(200000),
                        rng.standard_normal(100000) * 1e-2, rng.standard_normal(100000) * 1e-3])
    ref = torch.from_numpy(x).float().to(torch.float8_e4m3fn).double().numpy()
    # torch rounds from fp32: compare on the fp32 values it saw
    got = orc.quantize_e4m3(x.astype(np.float32).astype(np.float64))
    assert np.array_equal(got, ref)


def test_ties_go_to_even_mantissa(orc):
    v = np.sort(_codes())
    mids = (v[:-1] + v[1:]) / 2            # exact midpoints between neighbours (exact in fp64)
    ref = torch.from_numpy(mids).float().to(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(orc.quantize_e4m3(mids), ref)


def test_saturation_and_scale(orc):
    x = np.array([448.0, 449.0, 1e4, -1e4, -448.0])
    assert orc.quantize_e4m3(x).tolist() == [448.0, 448.0, 448.0, -448.0, -448.0]
    # a per-tensor scale maps amax onto 448 and back
    y = np.random.default_rng(1).standard_normal(1000) * 7.0
    s = np.abs(y).max() / 448.0
    q = orc.quantize_e4m3(y, s)
    assert np.abs(q).max() <= 448.0 * s * (1 + 1e-15)
    assert np.allclose(q, orc.quantize_e4m3(y / s) * s)


def test_relative_error_bound(orc):
    x = np.random.default_rng(2).uniform(2.0 ** -6, 440.0, 100000)   # normal range
    err = np.abs(orc.quantize_e4m3(x) - x) / x
    assert err.max() <= 2.0 ** -4 + 1e-15   # half a unit in the last of 3 mantissa bits


def test_attention_of_quantised_inputs_is_the_oracle_on_them(orc):
    """The FP8 forward's reference: the oracle fed the dequantised Q and K."""
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 5, 2, 8))
    k = rng.standard_normal((1, 7, 2, 8))
    v = rng.standard_normal((1, 7, 2, 8))
    sq, sk = np.abs(q).max() / 448, np.abs(k).max() / 448
    qq, kq = orc.quantize_e4m3(q, sq), orc.quantize_e4m3(k, sk)
    o, lse = orc.fwd(qq, kq, v)
    s_ = np.einsum("bihc,bjhc->bhij", qq, kq) / np.sqrt(8)
    p = np.exp(s_ - s_.max(-1, keepdims=True))
    p /= p.sum(-1, keepdims=True)
    assert np.allclose(o, np.einsum("bhij,bjhc->bihc", p, v), atol=1e-13)


def test_per_head_quantiser_against_numpy_and_torch(orc):
    """oracle_quantize_e4m3_heads: the scale of each (batch, head) is fp32 amax / 448
    (numpy's fp32 division), and every code is torch's fp32 -> e4m3 cast of the
    fp32 quotient (clamped to the finite range first: the oracle saturates)."""
    rng = np.random.default_rng(5)
    x = torch.from_numpy(rng.standard_normal((2, 37, 3, 64)) * 4.0).to(torch.bfloat16)
    x[1, :, 2] = 0                                     # an all-zero head: scale 1, codes 0
    x[0, 5, 1, 7] = 300.0                              # one large entry sets its head's scale
    got, scales = orc.quantize_e4m3_heads(x)
    xf = x.float()
    amax = xf.abs().amax(dim=(1, 3))                   # [B, H], exact
    a32 = amax.numpy().astype(np.float32)
    sc = torch.from_numpy(np.where(a32 > 0, a32 / np.float32(448.0), np.float32(1.0)).astype(np.float32))
    assert np.array_equal(scales, sc.double().numpy())
    quot = xf / sc[:, None, :, None]                   # fp32 IEEE division, as the kernel
    ref = quot.clamp(-448, 448).to(torch.float8_e4m3fn).double() * sc[:, None, :, None].double()
    assert np.array_equal(got, ref.numpy())
    assert not got[1, :, 2].any() and scales[1, 2] == 1.0
    # the largest magnitude of every head maps onto 448 * scale (up to the fp32 rounding of the scale)
    top = np.abs(got).max(axis=(1, 3))
    assert np.all(np.abs(top - amax.double().numpy()) <= 2.0 ** -4 * amax.double().numpy() + 1e-30)
