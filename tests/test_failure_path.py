"""The failure path every kernel shares, made to run without a GPU fault: a
bounded mbarrier wait on a barrier that nothing arrives on gives up after a
short limit, the kernel returns, the host reads ATTN_ERR_TIMEOUT from the
device status word, and the context stays usable for normal work."""
import pytest
import torch

from parity import check_fwd

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def test_bounded_wait_gives_up_and_reports(orc):
    from exact_io_aware_57_b200 import attn

    assert attn.attn_device_status() == 0            # clean before
    attn.attn_selftest_wait_timeout(2_000_000)        # about a millisecond of SM cycles
    assert attn.attn_device_status() == attn.ATTN_ERR_TIMEOUT
    assert attn.attn_device_status() == 0            # reading clears it
    # the context is intact: a normal forward still meets the oracle
    check_fwd(orc, 1, 2, 2, 200, 200, 128, True)
    assert attn.attn_device_status() == 0
