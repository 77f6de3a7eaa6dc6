"""The FMA-pipe exponential (ex2_poly) that the tensor-core kernels use for a
share of the probabilities' exponentials.

Host side: the coefficients compiled into the kernels are the ones the Remez
fit script produces, and the method (Cody-Waite reduction, degree-3 minimax
polynomial) meets its stated relative error of 7.6e-5 when evaluated in fp32.
GPU side: the kernels' function itself, through attn_selftest_ex2, against
exact 2^x in fp64 over its whole domain, its clamp and its special inputs.
"""
import importlib.util
import pathlib
import re

import numpy as np
import pytest
import torch

CSRC = pathlib.Path(__file__).resolve().parents[1] / "exact_io_aware_57_b200" / "csrc"
BOUND = 7.6e-5   # stated in include/attn.h; the bf16 P it feeds resolves 2^-9 = 1.95e-3


def _kernel_coefficients():
    src = (CSRC / "common.cuh").read_text()
    body = src[src.index("float ex2_poly(float x)"):]
    body = body[:body.index("\n}\n")]
    c = [float(v) for v in re.findall(r"(-?\d+\.\d+)f", body)]
    # fmaf(c3, f, c2) -> fmaf(p, f, c1) -> fmaf(p, f, c0): literals in that order
    assert len(c) >= 4
    c3, c2, c1, c0 = c[:4]
    return np.array([c0, c1, c2, c3], dtype=np.float32)


def _fit():
    spec = importlib.util.spec_from_file_location("ex2_poly_fit", CSRC / "ex2_poly_fit.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.remez(3).astype(np.float32)


def _fma32(a, b, c):
    # fp32 fused multiply-add: the fp64 product of two fp32 values is exact;
    # the single rounding of the sum to fp64 and then to fp32 agrees with one
    # rounding except in double-rounding ties, which the bound below absorbs
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _emulate(x):
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic).astype(np.float32)).astype(np.float32)
    c = _kernel_coefficients()
    p = _fma32(np.full_like(f, c[3]), f, np.full_like(f, c[2]))
    p = _fma32(p, f, np.full_like(f, c[1]))
    p = _fma32(p, f, np.full_like(f, c[0]))
    n = (t.view(np.int32) << 23).astype(np.int32)
    return (p.view(np.int32) + n).view(np.float32)


def test_kernel_coefficients_are_the_remez_fit():
    np.testing.assert_array_equal(_kernel_coefficients(), _fit())


def test_polynomial_error_on_the_reduced_range():
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    c = _kernel_coefficients()
    p = _fma32(np.full_like(f, c[3]), f, np.full_like(f, c[2]))
    p = _fma32(p, f, np.full_like(f, c[1]))
    p = _fma32(p, f, np.full_like(f, c[0]))
    rel = np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)
    assert rel.max() < BOUND
    # a minimax fit equioscillates: the error is spread, not concentrated at an end
    assert rel.max() > 0.5 * BOUND


def test_range_reduction_over_the_domain():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        -rng.uniform(0.0, 125.0, 400000),
        -np.linspace(0.0, 125.0, 400001),
        -np.arange(0, 126, dtype=np.float64),            # integers: f = 0
        -np.arange(0, 125, dtype=np.float64) - 0.5,       # halves: ties of the rounding
        [-1e-7, -0.25, -124.99],
    ]).astype(np.float32)
    y = _emulate(x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < BOUND
    assert _emulate(np.array([0.0], np.float32))[0] == pytest.approx(1.0, rel=BOUND)
    # the clamp: everything below -125 gives 2^-125 to the same error
    low = _emulate(np.array([-125.0, -126.0, -127.5, -1000.0, -np.inf], np.float32)).astype(np.float64)
    np.testing.assert_allclose(low, 2.0 ** -125, rtol=BOUND)


def test_planted_coefficient_error_is_caught():
    # a plausible slip (a coefficient of 2^f's Taylor series instead of the
    # minimax one) must break the stated bound
    f = np.linspace(-0.5, 0.5, 20001)
    c = _kernel_coefficients().astype(np.float64)
    c[1] = np.log(2.0)
    p = ((c[3] * f + c[2]) * f + c[1]) * f + c[0]
    assert np.abs(p / np.exp2(f) - 1.0).max() > BOUND


@pytest.mark.gpu
def test_kernel_ex2_against_exact():
    from exact_io_aware_57_b200 import attn
    g = torch.Generator().manual_seed(1)
    x = torch.cat([
        -torch.rand(1 << 22, generator=g, dtype=torch.float64) * 125.0,
        -torch.linspace(0.0, 125.0, 1 << 20, dtype=torch.float64),
        -torch.arange(0, 126, dtype=torch.float64),
        -torch.arange(0, 125, dtype=torch.float64) - 0.5,
        torch.tensor([0.0, -0.0, -1e-7, -124.99, -125.0]),
    ]).to(torch.float32)
    y = attn.attn_selftest_ex2(x.cuda()).cpu().double()
    exact = torch.exp2(x.double())
    rel = (y / exact - 1.0).abs()
    assert rel.max().item() < BOUND, rel.max().item()
    # ... and equal to the host emulation of the same steps up to the fma rounding
    emu = torch.from_numpy(_emulate(x.numpy()).astype(np.float64))
    assert ((y - emu).abs() <= 2.0 ** -22 * emu).all()


@pytest.mark.gpu
def test_kernel_ex2_clamp_and_ragged_lengths():
    from exact_io_aware_57_b200 import attn
    x = torch.tensor([-125.0, -126.0, -127.5, -1000.0, -float("inf")], dtype=torch.float32)
    y = attn.attn_selftest_ex2(x.cuda()).cpu().double()
    torch.testing.assert_close(y, torch.full((5,), 2.0 ** -125, dtype=torch.float64), rtol=BOUND, atol=0)
    for n in (0, 1, 255, 257, 148 * 8 * 256 + 3):   # empty, one, ragged, beyond one grid pass
        xs = -torch.rand(n, dtype=torch.float32) * 100.0
        ys = attn.attn_selftest_ex2(xs.cuda()).cpu().double()
        assert ys.shape == (n,)
        if n:
            assert ((ys / torch.exp2(xs.double()) - 1.0).abs().max() < BOUND)
