"""GPU parity of the candidate-list merge (topk_bucketed_merge) through the
C ABI: against the oracle's pair selection (bucket = index mod b) bit for bit,
and the split-and-merge property on one GPU -- rows cut into column slices at
arbitrary points, each slice selected on its own, the lists merged -- against
the single pass over the whole rows."""
from __future__ import annotations

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
    assert atk.topk_device_status() == 0


def bits(a):
    return np.ascontiguousarray(np.asarray(a, np.float32)).view(np.uint32)


def _rows(kind, rows, n, seed):
    if kind == "normal":
        return inputs.normal_rows(rows, n, seed)
    if kind == "uniform":
        return inputs.uniform_rows(rows, n, seed)
    if kind == "integer":
        return inputs.integer_rows(rows, n, 7, seed)
    return inputs.special_rows(rows, n, seed)


@pytest.mark.parametrize("rows,n,k,b,kb,kind,parts", [
    (6, 50000, 64, 128, 1, "normal", 2),
    (5, 40001, 100, 1000, 1, "uniform", 3),
    (4, 30000, 512, 256, 2, "uniform", 5),
    (4, 30000, 512, 512, 4, "uniform", 4),
    (3, 9999, 37, 7, 3, "integer", 3),
    (3, 5000, 200, 64, 2, "special", 2),
    (2, 131072, 50, 512, 1, "normal", 8),
])
def test_split_rows_merge_equals_single_pass(oracle_mod, rows, n, k, b, kb, kind, parts):
    x = _rows(kind, rows, n, 7000 + n + parts)
    g = np.random.default_rng(n + parts)
    cuts = np.sort(g.choice(np.arange(1, n), size=parts - 1, replace=False))
    starts = np.concatenate([[0], cuts])
    ends = np.concatenate([cuts, [n]])
    xd = x.to(DEV)
    vs, is_ = [], []
    for s, e in zip(starts, ends):
        v, i = atk.topk_bucketed(xd[:, s:e].contiguous(), k, b, kb)
        vs.append(v)
        is_.append(i)
    V, I = torch.stack(vs), torch.stack(is_)
    mv, mi = atk.topk_bucketed_merge(V, I, n, k, b, kb, part_offsets=starts.tolist())
    fv, fi = atk.topk_bucketed(xd, k, b, kb)
    torch.cuda.synchronize()
    assert np.array_equal(mi.cpu().numpy(), fi.cpu().numpy())
    assert np.array_equal(bits(mv.cpu()), bits(fv.cpu()))
    ov, oi = oracle_mod.bucketed(x.numpy(), k, b, kb)
    assert np.array_equal(mi.cpu().numpy(), oi)
    assert np.array_equal(bits(mv.cpu()), bits(ov))


def _pair_lists(parts, rows, m, n_total, seed, special=False):
    """Distinct global indices per row, spread over parts; some empty slots."""
    g = np.random.default_rng(seed)
    offs = np.sort(g.integers(0, n_total // 2, size=parts))
    vals = np.empty((parts, rows, m), np.float32)
    idx = np.empty((parts, rows, m), np.int32)
    for r in range(rows):
        glob = g.choice(n_total, size=parts * m, replace=False)
        for p in range(parts):
            gi = glob[p * m:(p + 1) * m]
            gi = np.where(gi >= offs[p], gi, gi + offs[p])  # >= offset; collisions dropped below
            idx[p, r] = gi - offs[p]
        v = g.integers(-5, 6, size=(parts, m)).astype(np.float32)
        if special:
            pick = g.random((parts, m))
            vu = v.view(np.uint32)
            vu[pick < 0.08] = 0x00000000                          # +0
            vu[(pick >= 0.08) & (pick < 0.16)] = 0x80000000       # -0
            vu[(pick >= 0.16) & (pick < 0.20)] = 0x7f800000       # +inf
            vu[(pick >= 0.20) & (pick < 0.24)] = 0xff800000       # -inf
            vu[(pick >= 0.24) & (pick < 0.28)] = 0x7fc00001       # NaN with a payload
            vu[(pick >= 0.28) & (pick < 0.30)] = 0xffc00002       # negative NaN
        vals[:, r] = v
        empty = g.random((parts, m)) < 0.1
        idx[:, r][empty] = -1
    # make the global indices of each row distinct after the offsets
    for r in range(rows):
        seen = set()
        for p in range(parts):
            for t in range(m):
                if idx[p, r, t] < 0:
                    continue
                gi = int(idx[p, r, t]) + int(offs[p])
                if gi in seen or gi >= n_total:
                    idx[p, r, t] = -1
                else:
                    seen.add(gi)
    return vals, idx, offs


def _oracle_merge(oracle_mod, vals, idx, offs, k, b, kb):
    parts, rows, m = vals.shape
    ov = np.empty((rows, k), np.float32)
    oi = np.empty((rows, k), np.int32)
    for r in range(rows):
        keep = idx[:, r] >= 0
        pv = vals[:, r][keep]
        pi = (idx[:, r] + offs[:, None].astype(np.int64))[keep].astype(np.int32)
        ov[r], oi[r] = oracle_mod.bucketed_pairs(pv, pi, k, b, kb)
    return ov, oi


@pytest.mark.parametrize("parts,rows,m,n_total,k,b,kb,special", [
    (1, 4, 300, 5000, 50, 16, 1, False),
    (3, 5, 200, 100000, 64, 128, 2, False),
    (4, 3, 512, 1 << 20, 512, 256, 4, False),
    (2, 4, 1000, 50000, 100, 1024, 3, False),
    (5, 3, 129, 7777, 700, 5, 4, False),
    (3, 4, 256, 20000, 128, 32, 2, True),
    (64, 2, 16, 100000, 200, 100, 1, True),
])
def test_merge_pairs_vs_oracle(oracle_mod, parts, rows, m, n_total, k, b, kb, special):
    vals, idx, offs = _pair_lists(parts, rows, m, n_total, 31 * parts + m, special)
    mv, mi = atk.topk_bucketed_merge(torch.from_numpy(vals).to(DEV), torch.from_numpy(idx).to(DEV),
                                     n_total, k, b, kb, part_offsets=offs.tolist())
    ov, oi = _oracle_merge(oracle_mod, vals, idx, offs, k, b, kb)
    assert np.array_equal(mi.cpu().numpy(), oi)
    assert np.array_equal(bits(mv.cpu()), bits(ov))


def test_merge_skips_and_flags_out_of_range_indices(oracle_mod):
    vals, idx, offs = _pair_lists(2, 3, 64, 1000, 5)
    bad = idx.copy()
    bad[1, 0, 3] = 5000  # global index beyond n_total
    mv, mi = atk.topk_bucketed_merge(torch.from_numpy(vals).to(DEV), torch.from_numpy(bad).to(DEV),
                                     1000, 20, 8, 2, part_offsets=offs.tolist())
    torch.cuda.synchronize()
    assert atk.topk_device_status() == 2
    clean = bad.copy()
    clean[1, 0, 3] = -1
    ov, oi = _oracle_merge(oracle_mod, vals, clean, offs, 20, 8, 2)
    assert np.array_equal(mi.cpu().numpy(), oi)
    assert np.array_equal(bits(mv.cpu()), bits(ov))


@pytest.mark.parametrize("shared", [False, True])
def test_split_keys_merge_equals_fused_single_pass(oracle_mod, shared):
    """Entity-parallel emulation on one GPU: the key matrices cut into slices,
    score_topk on each slice, then the merge.  The result equals the bucketed
    selection over the slices' own fp32 scores bit for bit (the oracle on those
    scores); a slice may sum a dot product in another fp32 order than the whole
    matrix does, so the scores themselves are checked against each other to
    the scoring tolerance."""
    rows, n, d, k, b, kb = (64, 65536, 256, 100, 1024, 1) if shared else (8, 20000, 128, 256, 128, 2)
    q = inputs.bf16_normal((rows, d), 1.0, 0xC0 + n, device=DEV)
    K = inputs.bf16_normal((n, d) if shared else (rows, n, d), d ** -0.5, 0xC1 + n, device=DEV)
    cuts = [0, n // 3, n // 3 + 4096 + 5, n] if not shared else [0, 16384, 40960, n]
    vs, is_, ss = [], [], []
    for s0, e0 in zip(cuts[:-1], cuts[1:]):
        Ks = K[s0:e0].contiguous() if shared else K[:, s0:e0].contiguous()
        v, i, sc = atk.score_topk(q, Ks, k, b, kb, return_scores=True)
        vs.append(v)
        is_.append(i)
        ss.append(sc)
    mv, mi = atk.topk_bucketed_merge(torch.stack(vs), torch.stack(is_), n, k, b, kb,
                                     part_offsets=cuts[:-1])
    torch.cuda.synchronize()
    slice_scores = torch.cat(ss, dim=1).cpu().numpy()
    ov, oi = oracle_mod.bucketed(slice_scores, k, b, kb)
    assert np.array_equal(mi.cpu().numpy(), oi)
    assert np.array_equal(bits(mv.cpu()), bits(ov))
    _, _, fs = atk.score_topk(q, K, k, b, kb, return_scores=True)
    full = fs.cpu().numpy().astype(np.float64)
    # fp32 sums of the same products in another order: a few ulps of sum(abs(terms))
    assert np.all(np.abs(slice_scores - full) <= 1e-5 + 1e-5 * np.abs(full))
