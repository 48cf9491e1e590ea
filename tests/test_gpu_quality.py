"""GPU: the assignment study's recall (quality.assignment_recall, CUDA
selection) equals the recall of the oracle's selections on the same AR(1)
rows, for interleaved and contiguous buckets."""
import numpy as np
import pytest
import torch

import approximate_top_selection_b200 as atk
from approximate_top_selection_b200 import inputs, quality
from oracle import recall as rc

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,n,k,b,kb,rho", [
    (32, 131072, 512, 256, 2, 0.99),
    (32, 65536, 100, 512, 1, 0.9),
    (16, 32768, 256, 128, 4, 0.999),
])
def test_assignment_recall_matches_oracle(oracle_mod, rows, n, k, b, kb, rho):
    if not torch.cuda.is_available():
        pytest.fail("these tests need a CUDA device")
    x = inputs.ar1_rows(rows, n, rho, 0x6A0 + n)
    gi, gc = quality.assignment_recall(x.to("cuda:0"), k, b, kb)
    _, ei = oracle_mod.exact(x.numpy(), k)
    _, ii = oracle_mod.bucketed(x.numpy(), k, b, kb)
    _, cp = oracle_mod.bucketed(quality.contiguous_view(x, b).numpy(), k, b, kb)
    ci = quality.contiguous_index(torch.from_numpy(cp).long(), n, b).numpy()
    assert np.array_equal(gi.cpu().numpy(), rc.recall(ii, ei))
    assert np.array_equal(gc.cpu().numpy(), rc.recall(ci, ei))
    assert atk.topk_device_status() == 0
