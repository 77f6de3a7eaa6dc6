"""attn_bwd_noalloc, the backward for callers that cannot allocate device memory
when they run it (a framework that owns all device memory, or a loop that cannot
afford cudaMalloc's implicit synchronisation): it must give the same dQ, dK, dV
as attn_bwd with a caller-provided workspace, on consecutive calls that reuse its
built-in scratch, and reject problems larger than that scratch.

Collected last on purpose, so a stop-at-first-failure run has already run every
other test; it also passes alone in a fresh process."""
import ctypes
import math

import pytest
import torch

from exact_io_aware_57_b200 import synth
from parity import TOL_GRAD_BF16, rel_fro

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _noalloc(lib, t, causal, scale, bias=None):
    q, k, v, o, lse, do, dq, dk, dv = t
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    stream = torch.cuda.current_stream().cuda_stream
    return lib.attn_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                None if bias is None else bias.data_ptr(), 0, o.data_ptr(), lse.data_ptr(),
                                do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, Nq, Nk, d,
                                ctypes.c_float(scale), int(causal), 0, stream)


def _case(B, Hq, Hkv, N, d, seed):
    from exact_io_aware_57_b200 import attn

    inp = synth.make_dense(B, Hq, Hkv, N, N, d, seed=seed)
    q, k, v, do = (x.cuda() for x in (inp.q, inp.k, inp.v, inp.dout))
    o, lse = attn.attn_fwd(q, k, v, causal=True)
    return q, k, v, o, lse, do


def _free_bytes():
    free, _ = torch.cuda.mem_get_info()
    return free


def test_noalloc_matches_workspace_backward_twice(orc):
    from exact_io_aware_57_b200 import attn

    lib = attn.lib()
    # warm-up: the first call on a device looks up the array (and may load the
    # module that holds it); the calls measured below must allocate nothing
    w = _case(1, 2, 2, 130, 64, 4)
    wout = [torch.empty_like(w[0]), torch.empty_like(w[1]), torch.empty_like(w[2])]
    assert _noalloc(lib, (*w, *wout), True, 0.125) == 0
    torch.cuda.synchronize()
    assert attn.attn_device_status() == 0
    # a larger call first, then a smaller one that reuses the same scratch
    for (B, Hq, Hkv, N, d, seed) in ((2, 4, 2, 777, 128, 5), (1, 2, 1, 200, 64, 6)):
        q, k, v, o, lse, do = _case(B, Hq, Hkv, N, d, seed)
        scale = 1.0 / math.sqrt(d)
        ref = attn.attn_bwd(q, k, v, o, lse, do, causal=True)
        out = [torch.full_like(q, float("nan")), torch.full_like(k, float("nan")), torch.full_like(v, float("nan"))]
        torch.cuda.synchronize()
        held, free0 = torch.cuda.memory_allocated(), _free_bytes()
        rc = _noalloc(lib, (q, k, v, o, lse, do, *out), True, scale)
        assert rc == 0, lib.attn_strerror(rc)
        torch.cuda.synchronize()
        assert attn.attn_device_status() == 0
        # nothing was allocated: neither through torch nor behind its back
        assert torch.cuda.memory_allocated() == held
        assert _free_bytes() == free0
        for name, a, r in zip(("dq", "dk", "dv"), out, ref):
            e = rel_fro(a.cpu().double().numpy(), r.cpu().double().numpy())
            assert e <= TOL_GRAD_BF16, f"{name}: rel Frobenius {e:.3e}"
        if seed == 6:
            # the second call also stands on its own against the fp64 oracle
            inp = synth.make_dense(B, Hq, Hkv, N, N, d, seed=seed)
            dq_r, dk_r, dv_r = orc.bwd(inp.q, inp.k, inp.v, inp.dout, causal=True)
            for name, a, r in zip(("dq", "dk", "dv"), out, (dq_r, dk_r, dv_r)):
                e = rel_fro(a.cpu().double().numpy(), r)
                assert e <= TOL_GRAD_BF16, f"{name} vs oracle: rel Frobenius {e:.3e}"


def test_noalloc_rejects_problems_beyond_its_scratch():
    from exact_io_aware_57_b200 import attn

    lib = attn.lib()
    limit = 32 * 1024 * 1024
    # batch 2, 32 heads, N=8192, d=128 needs ~270 MB of scratch
    assert attn.attn_bwd_workspace_size(2, 32, 8192, 128) > limit
    p = ctypes.c_void_p(256)
    rc = lib.attn_bwd_noalloc(p, p, p, None, 0, p, p, p, p, p, p, 2, 32, 32, 8192, 8192, 128,
                              ctypes.c_float(0.088), 1, 0, None)
    assert rc == attn.ATTN_ERR_WORKSPACE
