"""GPU parity of the candidate re-ranking (score_rerank) through the C ABI.

(1) the selection the GPU made on its own per-slot scores equals the oracle's
exact top-k over those (score, index) pairs bit for bit; (2) the GPU scores are
within 2e-3 relative (floor 2^-10 |q| |K_i|) of the oracle's fp64 scores;
(3) the index sets equal the oracle's except at a near-tie (within twice the
tolerance) at the k-th/(k+1)-th boundary."""
import numpy as np
import pytest
import torch

import approximate_top_selection_b200 as atk
from approximate_top_selection_b200 import inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _gpu(oracle_mod):
    if not torch.cuda.is_available():
        pytest.fail("these tests need a CUDA device")
    atk.load_library()
    yield


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _supports(rows, n, c, seed, bad=False):
    """Union of four overlapping random supports per row (repeats kept), some empty slots."""
    g = np.random.default_rng(seed)
    if c < 4:
        return g.integers(0, n, size=(rows, c)).astype(np.int32)
    base = g.integers(0, n, size=(rows, c // 2))
    cand = np.concatenate([base, np.roll(base, 7, axis=1)[:, : c - c // 2]], axis=1)
    cand[:, 1::3] = g.integers(0, n, size=cand[:, 1::3].shape)
    cand[:, ::11] = -1
    if bad:
        cand[:, 5] = n + 3
    return cand.astype(np.int32)


def check_rerank(q, K, cand, k, oracle_mod):
    v, i, s = atk.score_rerank(q, K, torch.from_numpy(cand).to(DEV), k, return_scores=True)
    torch.cuda.synchronize()
    v, i, s = v.cpu().numpy(), i.cpu().numpy(), s.cpu().numpy()
    rows, c = cand.shape
    n = K.shape[-2]
    # exactly one slot per distinct valid index carries a score (which copy of
    # a repeated index does is up to the GPU); empty and invalid slots read -inf
    owned = ~np.isneginf(s)
    for r in range(rows):
        valid = (cand[r] >= 0) & (cand[r] < n)
        assert not np.any(owned[r] & ~valid), r
        got = cand[r][owned[r]]
        assert len(got) == len(set(got.tolist())) == len(set(cand[r][valid].tolist())), r
    # (1) selection on the GPU's own scores
    for r in range(rows):
        ov, oi = oracle_mod.bucketed_pairs(s[r][owned[r]], cand[r][owned[r]], k, 1, k)
        assert np.array_equal(i[r], oi), r
        assert np.array_equal(v[r].view(np.uint32), ov.view(np.uint32)), r
    # (2) scores against fp64
    qb, Kb = _bits(q), _bits(K)
    rv, ri = oracle_mod.rerank(qb, Kb, cand, k)
    qf = (qb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    Kf = (Kb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for r in range(rows):
        ids = cand[r][owned[r]].astype(np.int64)
        kr = Kf[r] if Kf.ndim == 3 else Kf
        ref = kr[ids] @ qf[r]
        scale = np.linalg.norm(qf[r]) * np.linalg.norm(kr[ids], axis=1)
        tol = 2e-3 * np.maximum(np.abs(ref), 2.0 ** -10 * scale)
        err = np.abs(s[r][owned[r]].astype(np.float64) - ref)
        assert np.all(err <= tol), (r, float((err / tol).max()))
        # (3) index sets
        a = set(ri[r][ri[r] >= 0].tolist())
        g = set(i[r][i[r] >= 0].tolist())
        diff = a ^ g
        if diff:
            srt = np.sort(ref)[::-1]
            T = 2 * float(tol.max())
            assert len(srt) > k and srt[k - 1] - srt[k] <= T, r
            for x in diff:
                sx = ref[list(ids).index(x)]
                assert srt[k] - T <= sx <= srt[k - 1] + T, (r, x)


@pytest.mark.parametrize("rows,n,d,c,k", [
    (32, 32768, 128, 2048, 512),
    (16, 8192, 256, 4096, 100),
    (8, 4000, 128, 300, 400),   # fewer distinct candidates than k: padding
    (4, 1000, 128, 1, 1),
])
def test_rerank_per_row_keys(oracle_mod, rows, n, d, c, k):
    q = inputs.bf16_normal((rows, d), 1.0, 0xB0 + n, device=DEV)
    K = inputs.bf16_normal((rows, n, d), d ** -0.5, 0xB1 + n, device=DEV)
    check_rerank(q, K, _supports(rows, n, c, n + c), k, oracle_mod)
    assert atk.topk_device_status() == 0


@pytest.mark.parametrize("rows,n,d,supports,size,k", [
    (64, 32768, 128, 4, 512, 512),   # ~960 distinct of 2048 slots: the k best selected, then 512 sorted
    (40, 32768, 256, 4, 512, 512),
    (48, 8192, 128, 2, 256, 200),    # ~330 distinct: select 200, sort 256
    (48, 8192, 128, 2, 256, 100),
])
def test_rerank_select_before_sort(oracle_mod, rows, n, d, supports, size, k):
    """Distinct-candidate counts whose sort shrinks to the next smaller power
    of two once only the k best are kept (the decode re-rank shape among them)."""
    q = inputs.bf16_normal((rows, d), 1.0, 0xB6 + d, device=DEV)
    K = inputs.bf16_normal((rows, n, d), d ** -0.5, 0xB7 + d, device=DEV)
    cand = inputs.support_union(rows, n, supports, size, 0xB8 + k).numpy()
    distinct = [len(set(r.tolist())) for r in cand]
    assert min(distinct) > k and max(distinct) <= 2 * max(k, 256) - 1, distinct[:4]
    check_rerank(q, K, cand, k, oracle_mod)
    assert atk.topk_device_status() == 0


@pytest.mark.parametrize("rows,n,d,c,k,shared", [
    (700, 1000, 128, 2048, 512, False),   # more rows than 4 CTAs x 148 SMs: a second wave
    (301, 100000, 256, 1000, 100, True),  # one key matrix for all rows; n > 32 * 2048: hash set
    (400, 1000, 128, 300, 64, False),
])
def test_rerank_many_rows(oracle_mod, rows, n, d, c, k, shared):
    """Hundreds of rows (one CTA each), per-row and shared key matrices, the
    bitmap and the hash-set listing."""
    q = inputs.bf16_normal((rows, d), 1.0, 0xB9 + d, device=DEV)
    shape = (n, d) if shared else (rows, n, d)
    K = inputs.bf16_normal(shape, d ** -0.5, 0xBA + d, device=DEV)
    check_rerank(q, K, _supports(rows, n, c, rows + c), k, oracle_mod)
    assert atk.topk_device_status() == 0


def test_rerank_shared_keys(oracle_mod):
    rows, n, d, c, k = 64, 65536, 256, 1000, 100
    q = inputs.bf16_normal((rows, d), d ** -0.5, 0xB2, device=DEV)
    K = inputs.bf16_normal((n, d), d ** -0.5, 0xB3, device=DEV)
    check_rerank(q, K, _supports(rows, n, c, 5), k, oracle_mod)
    assert atk.topk_device_status() == 0


def test_rerank_flags_out_of_range(oracle_mod):
    rows, n, d, c, k = 4, 2000, 128, 256, 32
    q = inputs.bf16_normal((rows, d), 1.0, 0xB4, device=DEV)
    K = inputs.bf16_normal((rows, n, d), d ** -0.5, 0xB5, device=DEV)
    check_rerank(q, K, _supports(rows, n, c, 9, bad=True), k, oracle_mod)
    assert atk.topk_device_status() == 2
