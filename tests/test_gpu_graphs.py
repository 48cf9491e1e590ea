"""The library's calls inside CUDA graphs: captured once, replayed on new
input data written into the captured buffers, bit-identical to eager calls
(the page's Fig. 9 measures the kernels with CUDA graphs)."""
import numpy as np
import pytest
import torch

import approximate_top_selection_b200 as atk
from approximate_top_selection_b200 import inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _capture(fn):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # workspace and kernel set-up for this stream
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        out = fn()
    return g, out


@pytest.mark.parametrize("rows,n,k,b,kb", [(8, 4096, 64, 128, 1), (300, 20000, 512, 256, 4),
                                            (3, 500000, 100, 512, 2)])
def test_bucketed_in_a_graph(rows, n, k, b, kb):
    x = inputs.normal_rows(rows, n, 1, device=DEV)
    g, (v, i) = _capture(lambda: atk.topk_bucketed(x, k, b, kb))
    for seed in (2, 3):
        x.copy_(inputs.normal_rows(rows, n, seed, device=DEV))
        g.replay()
        ev, ei = atk.topk_bucketed(x.clone(), k, b, kb)
        torch.cuda.synchronize()
        assert torch.equal(i, ei) and torch.equal(v.view(torch.int32), ev.view(torch.int32))
    assert atk.topk_device_status() == 0


def test_fused_scoring_and_sampling_in_a_graph():
    q, K = inputs.decode_inputs(2, 8, 8192, 128, 4, device=DEV)
    Ql, Kl = inputs.link_inputs(256, 16384, 256, 5, device=DEV)
    logits = inputs.vocab_logits(16, 32768, 6, device=DEV)
    u = torch.rand(16, device=DEV)

    def step():
        return (atk.score_topk(q, K, 512, 256, 2), atk.score_topk(Ql, Kl, 100, 1024, 1),
                atk.topk_sample(logits, 50, 512, 1, 1.0, u))
    g, out = _capture(step)
    q.copy_(inputs.decode_inputs(2, 8, 8192, 128, 7, device=DEV)[0])
    logits.copy_(inputs.vocab_logits(16, 32768, 8, device=DEV))
    u.copy_(torch.rand(16, device=DEV))
    g.replay()
    ref = step()
    torch.cuda.synchronize()
    for a, e in zip(out, ref):
        for ta, te in zip(a, e):
            assert torch.equal(ta, te)
    assert atk.topk_device_status() == 0
