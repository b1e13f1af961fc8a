"""Failure detection on the GPU without a fault: a bounded wait that nothing
satisfies must give up, be reported through the device status word, and
leave the context usable."""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tg():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import learned_token_pruning_rmsnorm_b200 as tg
    tg.load()
    return tg


def test_bounded_wait_times_out_and_reports(tg):
    from learned_token_pruning_rmsnorm_b200 import _lib
    st, _ = tg.tg_device_status(clear=True)
    assert st == _lib.TG_OK
    tg.tg_selftest_bounded_wait(20_000_000)  # 20 ms
    st, word = tg.tg_device_status(clear=False)
    assert st == _lib.TG_ERR_TIMEOUT
    assert word & 0x10000 and word & 0x4
    st, _ = tg.tg_device_status(clear=True)   # read-and-clear
    assert st == _lib.TG_ERR_TIMEOUT
    st, word = tg.tg_device_status(clear=False)
    assert st == _lib.TG_OK and word == 0


def test_context_usable_after_timeout(tg):
    from learned_token_pruning_rmsnorm_b200 import _lib
    tg.tg_selftest_bounded_wait(5_000_000)
    tg.tg_device_status(clear=True)
    # a real selection after the reported timeout still runs and is right
    s = torch.tensor([0.5, 3.0, -1.0, 2.0, 2.0, 0.0], dtype=torch.float32, device="cuda")
    keep = tg.tg_select_topk(s, [0, 6], [[0, 6]], [3]).cpu().numpy()
    np.testing.assert_array_equal(keep, [0, 1, 0, 1, 1, 0])
    st, word = tg.tg_device_status(clear=False)
    assert st == _lib.TG_OK and word == 0


def test_selftest_rejects_bad_timeout(tg):
    with pytest.raises(tg.TokenGateError):
        tg.tg_selftest_bounded_wait(0)
