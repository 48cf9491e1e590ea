"""The allocation-free entry point, topk_bucketed_noalloc, on the GPU.

Some callers cannot allocate device memory at the moment they select -- a
serving loop where cudaMalloc could synchronise the device and stall other
streams, a framework that forbids allocations it does not account for, a
plugin that may only allocate at set-up.  For them topk_bucketed_noalloc takes
only inputs and outputs and keeps its scratch in a static buffer inside the
library.  These checks call it through the C ABI (ctypes, preallocated
outputs) and compare it, bit for bit, with the CPU oracle and with
topk_bucketed, on two calls in a row for each shape, including shapes whose
rows are split across CTAs (the case that needs scratch).  This file is
collected last so that a run stopping at the first failure has already run
every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import approximate_top_selection_b200 as atk
from approximate_top_selection_b200 import inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"

SHAPES = [
    # (rows, n, k, b, kb, kind)
    (8, 4096, 64, 128, 1, "normal"),        # one row per CTA: no scratch needed
    (3, 400000, 100, 512, 2, "normal"),     # long rows split across CTAs (fast path)
    (2500, 1001, 20, 50, 2, "uniform"),     # many rows per CTA, cut rows (general path)
    (2, 1 << 20, 300, 256, 4, "ties"),      # heavy ties, split rows
    (3, 600000, 512, 512, 4, "uniform"),    # the 16-warp k_b > 2 kernel, split rows
]


def _rows(rows, n, kind, seed):
    if kind == "normal":
        return inputs.normal_rows(rows, n, seed)
    if kind == "uniform":
        return inputs.uniform_rows(rows, n, seed)
    return inputs.integer_rows(rows, n, 50, seed)


def _noalloc(lib, x, k, b, kb, ov, oi):
    st = lib.topk_bucketed_noalloc(x.data_ptr(), x.shape[0], x.shape[1], k, b, kb, ov.data_ptr(),
                                   oi.data_ptr(), torch.cuda.current_stream().cuda_stream)
    return st


@pytest.mark.parametrize("rows,n,k,b,kb,kind", SHAPES)
def test_noalloc_matches_oracle_and_topk_bucketed(rows, n, k, b, kb, kind, oracle_mod):
    if not torch.cuda.is_available():
        pytest.fail("this test needs a CUDA device")
    lib = atk.load_library()
    for call in range(2):  # two calls in a row share (and must clear) the scratch
        xc = _rows(rows, n, kind, 9000 + 17 * call + n)
        x = xc.to(DEV)
        ov = torch.empty(rows, k, dtype=torch.float32, device=DEV)
        oi = torch.empty(rows, k, dtype=torch.int32, device=DEV)
        assert _noalloc(lib, x, k, b, kb, ov, oi) == atk.TOPK_OK
        rv, ri = atk.topk_bucketed(x, k, b, kb)
        torch.cuda.synchronize()
        wv, wi = oracle_mod.bucketed(xc.numpy(), k, b, kb)
        assert np.array_equal(oi.cpu().numpy(), wi), "indices differ from the oracle (call %d)" % call
        assert np.array_equal(ov.cpu().numpy().view(np.uint32), wv.view(np.uint32)), \
            "values differ from the oracle (call %d)" % call
        assert torch.equal(oi, ri), "indices differ from topk_bucketed (call %d)" % call
        assert torch.equal(ov.view(torch.int32), rv.view(torch.int32)), "values differ"
    assert atk.topk_device_status() == 0


def test_noalloc_rejects_oversized_scratch():
    """A call whose scratch need exceeds the built-in buffer is refused with
    TOPK_ESCRATCH before anything is queued."""
    if not torch.cuda.is_available():
        pytest.fail("this test needs a CUDA device")
    lib = atk.load_library()
    rows, n = 20_000_000, 4  # 80 MB of row tickets alone
    need = atk.topk_workspace_bytes(atk.TOPK_OP_BUCKETED, rows, n, 1, 2, 1)
    assert need > (32 << 20)
    dummy = torch.empty(16, dtype=torch.float32, device=DEV)  # never read: refused first
    st = lib.topk_bucketed_noalloc(dummy.data_ptr(), rows, n, 1, 2, 1, dummy.data_ptr(),
                                   dummy.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == atk.TOPK_ESCRATCH
    assert "built-in buffer" in atk.topk_status_string(st)
