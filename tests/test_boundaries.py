"""Structural guarantees the parity claims rest on, checked on the CPU.

* The product package never imports, loads or calls the oracle (a product
  path through the oracle, or any CPU fallback, would void parity).
* The only module both sides share, the input generators, holds no attention
  arithmetic: it imports neither side.
* The slope form of the grouped-query workload's bias is exactly the dense
  workload bias when N_q == N_k (the slopes path is compared with the oracle
  through that dense tensor)."""
import ast
from pathlib import Path

import numpy as np
import torch

from exact_io_aware_57_b200 import synth

ROOT = Path(__file__).resolve().parents[1]
PKG = ROOT / "exact_io_aware_57_b200"


def _imports(path):
    tree = ast.parse(path.read_text())
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            for a in node.names:
                yield a.name
        elif isinstance(node, ast.ImportFrom):
            yield (node.module or "")


def test_product_package_never_touches_the_oracle():
    for path in PKG.rglob("*.py"):
        mods = list(_imports(path))
        assert not any(m == "oracle" or m.startswith("oracle.") for m in mods), f"{path} imports the oracle"
        text = path.read_text()
        assert "liboracle" not in text and "attn_oracle" not in text, f"{path} names the oracle library"
    for path in list((PKG / "csrc").glob("*.cu")) + list((PKG / "csrc").glob("*.cuh")) + list((PKG / "csrc").glob("*.h")):
        assert "oracle" not in path.read_text().lower(), f"{path} mentions the oracle"


def test_the_oracle_shares_no_code_with_the_cuda_path():
    for path in (ROOT / "oracle").glob("*"):
        if path.suffix in (".c", ".py"):
            text = path.read_text()
            assert "exact_io_aware_57_b200" not in text and "csrc" not in text, f"{path} reaches into the package"


def test_input_generators_import_neither_side():
    mods = list(_imports(PKG / "synth.py"))
    assert not any(m.startswith("oracle") or "attn" in m or m.startswith(".") for m in mods), mods


def test_slope_bias_equals_the_dense_workload_bias():
    h, n = 32, 300
    dense = synth.alibi_like_bias(h, n, n).numpy().astype(np.float64)
    from_slopes = synth.bias_from_slopes(synth.alibi_like_slopes(h), n, n).numpy().astype(np.float64)
    # both fp32: the same values up to fp32 rounding of slope * distance
    assert np.allclose(dense, from_slopes, rtol=2e-7, atol=1e-6)
    # bottom-right alignment when N_q != N_k: distance to the aligned key i + N_k - N_q
    b = synth.bias_from_slopes(torch.tensor([1.0]), 2, 5).numpy()[0]
    assert b.tolist() == [[-3.0, -2.0, -1.0, 0.0, -1.0], [-4.0, -3.0, -2.0, -1.0, 0.0]]
