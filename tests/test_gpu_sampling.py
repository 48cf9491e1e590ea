"""GPU parity of the vocabulary-sampling tail (topk_sample, topk_sample_rows)
through the C ABI against the oracle's draw (fp64 weights).  The kernel sums
fp32 weights in another order, so a draw may differ only where the oracle's
target lies within 1e-5 (relative) of a CDF boundary; the selection feeding
the draw is bit-exact."""
import numpy as np
import pytest
import torch

import approximate_top_selection_b200 as atk
from approximate_top_selection_b200 import inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
FRAGILE = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _gpu(oracle_mod):
    if not torch.cuda.is_available():
        pytest.fail("these tests need a CUDA device")
    atk.load_library()
    yield
    assert atk.topk_device_status() == 0


def _uniforms(rows, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.rand(rows, generator=g, dtype=torch.float32)


def _check(tok, otok, margin):
    tok = np.asarray(tok)
    ok = (tok == otok) | (margin < FRAGILE)
    assert ok.all(), np.nonzero(~ok)[0][:10]
    assert (tok == otok).mean() > 0.99


@pytest.mark.parametrize("rows,n,k,b,kb,T", [
    (64, 131072, 50, 512, 1, 1.0),
    (64, 131072, 50, 512, 1, 0.7),
    (32, 128256, 256, 256, 1, 1.0),
    (16, 50000, 100, 128, 2, 2.0),
])
def test_topk_sample_vs_oracle(oracle_mod, rows, n, k, b, kb, T):
    x = inputs.vocab_logits(rows, n, 0x5A + n + k)
    u = _uniforms(rows, k)
    tok, v, i = atk.topk_sample(x.to(DEV), k, b, kb, T, u.to(DEV))
    ov, oi = oracle_mod.bucketed(x.numpy(), k, b, kb)
    assert np.array_equal(i.cpu().numpy(), oi)
    otok, margin = oracle_mod.sample_rows(ov, oi, T, u.numpy().astype(np.float64))
    _check(tok.cpu().numpy(), otok, margin)


def test_sample_rows_special_values(oracle_mod):
    ninf, nan, inf = -np.inf, np.nan, np.inf
    v = np.array([[2.0, ninf, ninf, ninf], [nan, 1.0, 0.0, -1.0], [inf, 5.0, 1.0, 0.0],
                  [ninf, ninf, ninf, ninf], [0.0, -0.0, -1.0, ninf], [1.0, 1.0, 1.0, 1.0]],
                 np.float32)
    i = np.array([[4, 8, -1, -1], [6, 2, 1, 0], [9, 3, 0, 1], [-1, -1, -1, -1], [3, 1, 2, 0],
                  [1, -1, 2, 3]], np.int32)
    for u in (0.0, 0.3, 0.6, 0.9, 0.9999):
        uu = np.full(v.shape[0], u, np.float32)
        tok = atk.topk_sample_rows(torch.from_numpy(v).to(DEV), torch.from_numpy(i).to(DEV), 1.0,
                                   torch.from_numpy(uu).to(DEV))
        otok, margin = oracle_mod.sample_rows(v, i, 1.0, uu.astype(np.float64))
        _check(tok.cpu().numpy(), otok, margin)


def test_sample_rows_frequencies_follow_softmax(oracle_mod):
    N, k = 8192, 40
    g = np.random.default_rng(3)
    v = np.sort(g.normal(size=k).astype(np.float32) * 2)[::-1].copy()
    idx = g.permutation(100000)[:k].astype(np.int32)
    u = ((np.arange(N) + 0.5) / N).astype(np.float32)
    for T in (0.5, 1.0):
        tok = atk.topk_sample_rows(torch.from_numpy(np.repeat(v[None], N, 0)).to(DEV),
                                   torch.from_numpy(np.repeat(idx[None], N, 0)).to(DEV), T,
                                   torch.from_numpy(u).to(DEV)).cpu().numpy()
        p = np.exp((v.astype(np.float64) - v[0]) / T)
        p /= p.sum()
        for j in range(k):
            assert abs(int((tok == idx[j]).sum()) - N * p[j]) <= 2.0, (T, j)


def test_sample_rows_larger_k(oracle_mod):
    rows, k = 8, 5000
    x = inputs.normal_rows(rows, 20000, 77)
    v, i = atk.topk_exact(x.to(DEV), k)
    u = _uniforms(rows, 99)
    tok = atk.topk_sample_rows(v, i, 0.25, u.to(DEV))
    otok, margin = oracle_mod.sample_rows(v.cpu().numpy(), i.cpu().numpy(), 0.25,
                                          u.numpy().astype(np.float64))
    _check(tok.cpu().numpy(), otok, margin)


@pytest.mark.parametrize("rows,n,k,b,kb,T", [
    (64, 131072, 50, 512, 1, 1.0),
    (16, 128256, 256, 256, 1, 0.7),
    (8, 65536, 64, 512, 4, 1.0),   # the 16-warp k_b > 2 kernel with the draw
])
def test_topk_sample_bf16_vs_oracle(oracle_mod, rows, n, k, b, kb, T):
    """bf16 logits: the selection equals the oracle's on the exactly widened
    values, and the draw agrees away from CDF boundaries."""
    x = inputs.vocab_logits(rows, n, 0x5B + n + k).to(torch.bfloat16)
    u = _uniforms(rows, k + 1)
    tok, v, i = atk.topk_sample(x.to(DEV), k, b, kb, T, u.to(DEV))
    assert v.dtype == torch.bfloat16
    ov, oi = oracle_mod.bucketed(x.float().numpy(), k, b, kb)
    assert np.array_equal(i.cpu().numpy(), oi)
    got = v.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, (ov.view(np.uint32) >> 16).astype(np.uint16))
    otok, margin = oracle_mod.sample_rows(ov, oi, T, u.numpy().astype(np.float64))
    _check(tok.cpu().numpy(), otok, margin)
