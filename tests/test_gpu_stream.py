"""Calls made on a stream other than torch's current one.

The binding allocates the outputs and the zero-filled workspace it caches per
stream.  Those must be created (and the workspace zeroed) on the stream the
kernel runs on: a fill queued on the current stream behind other work would
let the kernel read tickets that are not yet zero.  Here the current stream is
kept busy by a spin kernel while the call runs on a side stream, on shapes
whose rows are split across CTAs (the case that reads the workspace), and the
results must still equal the oracle's bit for bit.
"""
import numpy as np
import pytest
import torch

import approximate_top_selection_b200 as atk
from approximate_top_selection_b200 import _binding, inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _busy_current_stream():
    torch.cuda._sleep(200_000_000)  # a bounded spin of ~0.1 s on the current stream


def test_side_stream_selection_and_sampling(oracle_mod):
    if not torch.cuda.is_available():
        pytest.fail("this test needs a CUDA device")
    atk.load_library()
    for it in range(2):
        side = torch.cuda.Stream()
        x = inputs.normal_rows(3, 400000, 61 + it)
        xd = x.to(DEV)
        u = torch.rand(3, generator=torch.Generator().manual_seed(it))
        ud = u.to(DEV)
        torch.cuda.synchronize()
        assert not any(key[1] == side.cuda_stream for key in _binding._ws_cache)
        _busy_current_stream()
        v, i = atk.topk_bucketed(xd, 100, 512, 2, stream=side)
        tok, sv, si = atk.topk_sample(xd, 64, 256, 1, 1.0, ud, stream=side)
        side.synchronize()
        ov, oi = oracle_mod.bucketed(x.numpy(), 100, 512, 2)
        assert np.array_equal(i.cpu().numpy(), oi)
        assert np.array_equal(v.cpu().numpy().view(np.uint32), ov.view(np.uint32))
        pv, pi = oracle_mod.bucketed(x.numpy(), 64, 256, 1)
        assert np.array_equal(si.cpu().numpy(), pi)
        otok, margin = oracle_mod.sample_rows(pv, pi, 1.0, u.numpy().astype(np.float64))
        assert np.all((tok.cpu().numpy() == otok) | (margin < 1e-5))
        torch.cuda.synchronize()
    assert atk.topk_device_status() == 0


def test_side_stream_fused_scoring(oracle_mod):
    if not torch.cuda.is_available():
        pytest.fail("this test needs a CUDA device")
    side = torch.cuda.Stream()
    q, K = inputs.decode_inputs(1, 2, 300000, 128, 62)  # long rows: split across CTAs
    qd, Kd = q.to(DEV), K.to(DEV)
    torch.cuda.synchronize()
    _busy_current_stream()
    v, i, s = atk.score_topk(qd, Kd, 512, 256, 2, return_scores=True, stream=side)
    side.synchronize()
    ov, oi = oracle_mod.bucketed(s.cpu().numpy(), 512, 256, 2)
    assert np.array_equal(i.cpu().numpy(), oi)
    assert np.array_equal(v.cpu().numpy().view(np.uint32), ov.view(np.uint32))
    torch.cuda.synchronize()
    assert atk.topk_device_status() == 0
