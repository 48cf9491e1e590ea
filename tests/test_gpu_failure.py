"""Failure detection without a GPU fault: a bounded device wait that is sure
to expire (topk_selftest_wait_timeout) gives up, the expiry shows in the
device status, and the context stays usable for the next selection."""
import numpy as np
import pytest
import torch

import approximate_top_selection_b200 as atk
from approximate_top_selection_b200 import inputs

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_context_stays_usable(oracle_mod):
    if not torch.cuda.is_available():
        pytest.fail("these tests need a CUDA device")
    atk.load_library()
    assert atk.topk_device_status() == 0
    atk.topk_selftest_wait_timeout(2_000_000)  # 2 ms
    assert atk.topk_device_status() == 1       # TOPK_DEV_WAIT_TIMEOUT
    assert atk.topk_device_status() == 0       # reading clears it
    x = inputs.normal_rows(4, 10000, 31)
    v, i = atk.topk_bucketed(x.to("cuda:0"), 32, 64, 2)
    ov, oi = oracle_mod.bucketed(x.numpy(), 32, 64, 2)
    assert np.array_equal(i.cpu().numpy(), oi)
    assert atk.topk_device_status() == 0
