"""The C-ABI library loads on a machine without a GPU, exports every symbol
include/attn.h declares, and rejects bad arguments before touching the GPU."""
import ctypes
import re
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]
HEADER = ROOT / "include" / "attn.h"


def declared_symbols():
    text = HEADER.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for s in ("attn_fwd", "attn_bwd", "attn_bwd_workspace_size", "attn_fwd_varlen", "attn_strerror"):
        assert s in syms


def test_library_exports_every_declared_symbol():
    from exact_io_aware_57_b200 import attn

    lib = ctypes.CDLL(str(attn.LIB_PATH))
    missing = [s for s in declared_symbols() if not hasattr(lib, s)]
    assert not missing, missing
    # the binding wraps exactly the declared boundary
    assert set(attn.EXPORTS) == set(declared_symbols())


def test_workspace_is_linear_in_n():
    from exact_io_aware_57_b200 import attn

    a = attn.attn_bwd_workspace_size(2, 32, 8192, 128)
    assert a == 2 * 8192 * 32 * 128 * 4 + 2 * 32 * 8192 * 4
    assert attn.attn_bwd_workspace_size(2, 32, 16384, 128) == 2 * a
    assert attn.attn_bwd_workspace_size(0, 1, 1, 64) == 0


def test_strerror_and_codes():
    from exact_io_aware_57_b200 import attn

    lib = attn.lib()
    for code in (0, -1, -2, -3, -4, -5):
        assert lib.attn_strerror(code)
    assert b"unknown" in lib.attn_strerror(123)


@pytest.mark.parametrize("case", ["null", "heads", "dim", "dtype", "nq"])
def test_invalid_arguments_rejected_without_launch(case):
    from exact_io_aware_57_b200 import attn

    lib = attn.lib()
    p = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    args = dict(q=p, k=p, v=p, o=p, lse=p, B=1, Hq=4, Hkv=2, Nq=128, Nk=128, d=128, dtype=0)
    expect = attn.ATTN_ERR_INVALID
    if case == "null":
        args["q"] = None
    elif case == "heads":
        args["Hkv"] = 3
    elif case == "dim":
        args["d"], expect = 96, attn.ATTN_ERR_UNSUPPORTED
    elif case == "dtype":
        args["dtype"], expect = 7, attn.ATTN_ERR_UNSUPPORTED
    elif case == "nq":
        args["Nq"] = 0
    rc = lib.attn_fwd(args["q"], args["k"], args["v"], None, 0, args["o"], args["lse"], args["B"], args["Hq"],
                      args["Hkv"], args["Nq"], args["Nk"], args["d"], 0.1, 0, args["dtype"], None)
    assert rc == expect
    assert attn.attn_launch_count() == 0


def test_bwd_workspace_checked_before_launch():
    from exact_io_aware_57_b200 import attn

    lib = attn.lib()
    p = ctypes.c_void_p(256)
    need = attn.attn_bwd_workspace_size(1, 2, 128, 64)
    rc = lib.attn_bwd(p, p, p, None, 0, p, p, p, p, p, p, p, need - 1, 1, 2, 2, 128, 128, 64, 0.1, 0, 0, None)
    assert rc == attn.ATTN_ERR_WORKSPACE
    rc = lib.attn_bwd(p, p, p, None, 0, p, p, p, p, p, p, None, need, 1, 2, 2, 128, 128, 64, 0.1, 0, 0, None)
    assert rc == attn.ATTN_ERR_WORKSPACE


def test_varlen_rejects_bad_bounds():
    from exact_io_aware_57_b200 import attn

    lib = attn.lib()
    p = ctypes.c_void_p(256)
    # max_seqlen larger than the total
    rc = lib.attn_fwd_varlen(p, p, p, p, p, p, p, 2, 300, 300, 256, 256, 4, 4, 128, 0.1, 1, 0, None)
    assert rc == attn.ATTN_ERR_INVALID
