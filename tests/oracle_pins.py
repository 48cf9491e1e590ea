"""Checks that pin the CPU oracle to what the pages and mathematics fix.

Each function takes an `oracle.Oracle` instance and raises AssertionError when
the oracle disagrees with the pin.  They are collected as tests in
test_oracle_pins.py and re-run against oracle variants with planted mistakes in
test_oracle_mutants.py (each planted mistake must be caught by some pin).

Sources ("Approximate Top-k for Increased Parallelism", arXiv 2412.04358,
pith.science review page): the two-stage definition ("What carries the
argument"), Fig. 2 (n=11, k=4, b=3, k_b=2), Eq. (1) and Eq. (2) (same section),
and "What would settle it" (top values in one residue class mod b).
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch

from approximate_top_selection_b200 import inputs
from oracle import recall as rc

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "fig2_shape.txt")


# ---------------------------------------------------------------- brute force
def _rank_key(v: float, i: int):
    """Larger tuple ranks higher: NaN above every number, then value, then lower index."""
    if math.isnan(v):
        return (2, 0.0, -i)
    return (1, float(v), -i)


def brute_bucketed(x, k: int, b: int, kb: int):
    """Selection characterised by counting, not by sorting:
    element i survives stage 1 iff fewer than k_b elements of its bucket beat it;
    it is output iff it survives and fewer than k stage-1 survivors beat it."""
    n = len(x)
    keys = [_rank_key(float(x[i]), i) for i in range(n)]
    stage1 = [i for i in range(n)
              if sum(1 for j in range(i % b, n, b) if keys[j] > keys[i]) < kb]
    final = [i for i in stage1 if sum(1 for j in stage1 if keys[j] > keys[i]) < k]
    final.sort(key=lambda i: keys[i], reverse=True)
    return final, len(stage1)


def brute_exact(x, k: int):
    n = len(x)
    keys = [_rank_key(float(x[i]), i) for i in range(n)]
    sel = [i for i in range(n) if sum(1 for j in range(n) if keys[j] > keys[i]) < k]
    sel.sort(key=lambda i: keys[i], reverse=True)
    return sel


def _same_bits(a: np.ndarray, b: np.ndarray) -> bool:
    return np.array_equal(np.asarray(a, np.float32).view(np.uint32),
                          np.asarray(b, np.float32).view(np.uint32))


def _check_row(ov, oi, x, expect_idx, k):
    m = len(expect_idx)
    assert list(oi[:m]) == expect_idx, (list(oi[:m]), expect_idx)
    assert _same_bits(ov[:m], np.asarray(x, np.float32)[expect_idx])
    assert np.all(oi[m:] == -1)
    assert np.all(np.isneginf(ov[m:]))


def pin_brute_force_bucketed(orc, cases: int = 60, seed: int = 1):
    rng = np.random.default_rng(seed)
    for t in range(cases):
        n = int(rng.integers(1, 120))
        b = int(rng.integers(1, 17))
        kb = int(rng.integers(1, 5))
        k = int(rng.integers(1, 40))
        kind = t % 3
        if kind == 0:
            x = rng.integers(0, 5, n).astype(np.float32)  # heavy ties
        elif kind == 1:
            x = rng.standard_normal(n).astype(np.float32)
        else:
            x = inputs.special_rows(1, n, seed * 1000 + t).numpy()[0]
        ov, oi, oc = orc.bucketed(x, k, b, kb, return_candidates=True)
        want, c1 = brute_bucketed(x, k, b, kb)
        assert oc[0] == c1, (n, k, b, kb, oc[0], c1)
        _check_row(ov[0], oi[0], x, want, k)


def pin_brute_force_exact(orc, cases: int = 40, seed: int = 2):
    rng = np.random.default_rng(seed)
    for t in range(cases):
        n = int(rng.integers(1, 150))
        k = int(rng.integers(1, 60))
        if t % 2:
            x = inputs.special_rows(1, n, seed * 1000 + t).numpy()[0]
        else:
            x = rng.integers(0, 7, n).astype(np.float32)
        ov, oi = orc.exact(x, k)
        _check_row(ov[0], oi[0], x, brute_exact(x, k), k)


# ------------------------------------------------------- library special cases
def _numpy_exact_idx(x: np.ndarray, k: int):
    """numpy reference for NaN-free rows: sort by (-value, index), stable."""
    order = np.lexsort((np.arange(x.size), -x.astype(np.float64)))
    return [int(i) for i in order[:k]]


def pin_reductions_to_exact(orc, seed: int = 3):
    """b >= n with k_b = 1 (every bucket has at most one element) and b = 1
    with k_b >= k (one bucket keeps everything Stage 2 needs) are exact top-k."""
    rng = np.random.default_rng(seed)
    for t in range(30):
        n = int(rng.integers(2, 300))
        x = (rng.integers(0, 9, n) if t % 2 else rng.standard_normal(n)).astype(np.float32)
        k = int(rng.integers(1, 50))
        ov, oi = orc.bucketed(x, k, n + int(rng.integers(0, 3)), 1)
        _check_row(ov[0], oi[0], x, _numpy_exact_idx(x, k), k)
        k2 = int(rng.integers(1, 5))
        ov, oi = orc.bucketed(x, k2, 1, 4)
        _check_row(ov[0], oi[0], x, _numpy_exact_idx(x, k2), k2)
        ov, oi = orc.exact(x, k)
        _check_row(ov[0], oi[0], x, _numpy_exact_idx(x, k), k)


# ------------------------------------------------------------ Fig. 2 fixture
def load_golden():
    cases, cur = [], None
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        if line.startswith("case "):
            cur = {"name": line[5:].strip()}
            cases.append(cur)
            continue
        key, val = line.split(":", 1)
        cur[key.strip()] = val.strip()
    return cases


def pin_fig2_golden(orc):
    cases = load_golden()
    assert len(cases) == 3
    for c in cases:
        x = np.array([float(v) for v in c["x"].split()], np.float32)
        assert x.size == 11
        sizes = [len(range(j, 11, 3)) for j in range(3)]
        assert sizes == [int(v) for v in c["sizes"].split()]
        ov, oi, oc = orc.bucketed(x, 4, 3, 2, return_candidates=True)
        assert oc[0] == int(c["C"])
        assert list(oi[0]) == [int(v) for v in c["idx"].split()], c["name"]
        want_v = np.array([float(v) for v in c["val"].split()], np.float32)
        assert _same_bits(ov[0][~np.isnan(want_v)], want_v[~np.isnan(want_v)])
        assert np.array_equal(np.isnan(ov[0]), np.isnan(want_v))
        ev, ei = orc.exact(x, 4)
        assert list(ei[0]) == [int(v) for v in c["exact"].split()], c["name"]
        r = rc.recall(oi, ei)[0]
        assert abs(r - float(c["recall"])) < 1e-12


# ------------------------------------------------------- recall: Eq. (1)/(2)
def pin_recall_formulas_closed_forms():
    """Closed forms the formulas must meet."""
    for k in (1, 5, 64):
        # b = 1, k_b = 1: only the single largest element is retrieved.
        assert abs(rc.eq1_expected_recall(k, 1, 1) - 1.0 / k) < 1e-12
        assert abs(rc.expected_recall_exact(256, k, 1, 1) - 1.0 / k) < 1e-12
        # k_b >= k: nothing can be lost.
        assert rc.eq1_expected_recall(k, 7, max(k, 1)) == 1.0
    # every bucket a singleton (b = n): exact top-k.
    assert abs(rc.expected_recall_exact(64, 10, 64, 1) - 1.0) < 1e-12
    # k = 2, k_b = 1: the second element is lost iff it shares the first one's
    # bucket: with replacement 1/b, without replacement (s-1)/(n-1).
    n, b = 120, 8
    s = n // b
    assert abs(rc.eq1_expected_recall(2, b, 1) - (1 + (1 - 1 / b)) / 2) < 1e-12
    assert abs(rc.expected_recall_exact(n, 2, b, 1) - (1 + (1 - (s - 1) / (n - 1))) / 2) < 1e-12
    # worst case: k values in one bucket of size s >= k gives k_b / k.
    assert rc.eq2_worst_recall(4096, 16, 128, 2) == 2 / 16
    # ... and with s < k they fill ceil(k/s) buckets.
    assert rc.eq2_worst_recall(1024, 40, 64, 4) == (4 * 2 + 4) / 40


def pin_recall_formulas_monte_carlo(seed: int = 4):
    """Eq. (1) is the with-replacement model and the exact value the
    without-replacement one: simulate both models directly."""
    rng = np.random.default_rng(seed)
    n, k, b, kb = 256, 24, 16, 2
    s = n // b
    trials = 20000
    # with replacement: each of the top-k picks a bucket uniformly
    bk = rng.integers(0, b, (trials, k))
    kept = np.zeros(trials)
    for i in range(k):
        ahead = (bk[:, :i] == bk[:, i:i + 1]).sum(1)
        kept += ahead < kb
    mc1 = kept.mean() / k
    # without replacement: a random permutation of the n slots
    perm = np.argsort(rng.random((trials, n)), axis=1)[:, :k] // s
    kept = np.zeros(trials)
    for i in range(k):
        ahead = (perm[:, :i] == perm[:, i:i + 1]).sum(1)
        kept += ahead < kb
    mc2 = kept.mean() / k
    se = 0.5 / math.sqrt(trials)
    assert abs(mc1 - rc.eq1_expected_recall(k, b, kb)) < 4 * se
    assert abs(mc2 - rc.expected_recall_exact(n, k, b, kb)) < 4 * se


def recall_stats(orc, rows: int, n: int, k: int, b: int, kb: int, seed: int):
    x = inputs.uniform_rows(rows, n, seed).numpy()
    _, bi = orc.bucketed(x, k, b, kb)
    _, ei = orc.exact(x, k)
    r = rc.recall(bi, ei)
    mean = float(r.mean())
    se = float(r.std(ddof=1) / math.sqrt(rows))
    return mean, se


def pin_eq1_statistical(orc, configs=None):
    """Mean recall over iid uniform rows sits within 3 SE of the exact finite-n
    expectation and no more than 3 SE below Eq. (1) (a lower bound)."""
    if configs is None:
        configs = [(10000, 4096, 64, 128, 1, 11), (2000, 32768, 512, 256, 2, 12),
                   (2000, 8192, 256, 64, 4, 13)]
    for rows, n, k, b, kb, seed in configs:
        mean, se = recall_stats(orc, rows, n, k, b, kb, seed)
        e_exact = rc.expected_recall_exact(n, k, b, kb)
        e1 = rc.eq1_expected_recall(k, b, kb)
        assert abs(mean - e_exact) <= 3 * se, (n, k, b, kb, mean, e_exact, se)
        assert mean >= e1 - 3 * se, (n, k, b, kb, mean, e1, se)


def pin_adversarial(orc):
    """Top-k packed in the fewest residue classes mod b: recall is exactly the
    worst case of Eq. (2), row by row."""
    for (n, k, b, kb) in [(4096, 64, 128, 1), (4096, 64, 128, 2), (8192, 512, 64, 4),
                          (8192, 100, 256, 2), (2048, 40, 32, 1)]:
        x = inputs.adversarial_rows(8, n, k, b, seed=n + k + b + kb).numpy()
        _, bi = orc.bucketed(x, k, b, kb)
        _, ei = orc.exact(x, k)
        r = rc.recall(bi, ei)
        want = rc.eq2_worst_recall(n, k, b, kb)
        assert np.all(np.abs(r - want) < 1e-12), (n, k, b, kb, r, want)
        # and the expected classes are the ones holding the top values
        top = np.sort(ei, axis=1)
        assert np.all(x[np.arange(8)[:, None], top] >= 1.0)


def pin_split_merge(orc, cases: int = 200, seed: int = 5):
    """Splitting a row at any cut points, selecting on each slice with global
    indices (bucket = index mod b) and selecting again on the gathered results
    gives the single-pass answer.  (A property of the definition that the
    multi-block and multi-device merges rely on.)"""
    rng = np.random.default_rng(seed)
    for t in range(cases):
        n = int(rng.integers(2, 200))
        b = int(rng.integers(1, 20))
        kb = int(rng.integers(1, 5))
        k = int(rng.integers(1, 30))
        x = rng.integers(0, 4, n).astype(np.float32)
        cuts = sorted(set(int(c) for c in rng.integers(1, n, int(rng.integers(0, 5)))))
        bounds = [0] + cuts + [n]
        gv, gi = [], []
        for lo, hi in zip(bounds[:-1], bounds[1:]):
            v, i = orc.bucketed_pairs(x[lo:hi], np.arange(lo, hi, dtype=np.int32), k, b, kb)
            keep = i >= 0
            gv.append(v[keep])
            gi.append(i[keep])
        mv, mi = orc.bucketed_pairs(np.concatenate(gv), np.concatenate(gi), k, b, kb)
        sv, si = orc.bucketed(x, k, b, kb)
        assert np.array_equal(mi, si[0]) and _same_bits(mv, sv[0]), (n, k, b, kb, cuts)


# ------------------------------------------------------------------- scoring
def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def pin_scores_unit_vectors(orc, seed: int = 6):
    """q = e_j picks column j of K exactly (catches a transposed or shifted K)."""
    rows, n, d = 3, 37, 128
    K = inputs.bf16_normal((rows, n, d), 1.0, seed)
    q = torch.zeros(rows, d, dtype=torch.bfloat16)
    cols = [0, 77, d - 1]
    for r, j in enumerate(cols):
        q[r, j] = 1.0
    s = orc.scores(_bits(q), _bits(K))
    for r, j in enumerate(cols):
        assert np.array_equal(s[r], K[r, :, j].float().numpy())


def pin_scores_closed_form(orc):
    """q = c * 1 and K_i = a_i * 1 give d * c * a_i (all exactly representable)."""
    d, n = 256, 50
    c = 0.75
    a = np.arange(n, dtype=np.float32) - 20.0
    q = torch.full((2, d), c, dtype=torch.bfloat16)
    K = torch.tensor(np.repeat(a[:, None], d, 1), dtype=torch.bfloat16)
    s = orc.scores(_bits(q), _bits(K))  # shared K
    assert np.array_equal(s[0], (d * c * a).astype(np.float32))
    assert np.array_equal(s[1], s[0])
    q1 = torch.tensor([[3.0]], dtype=torch.bfloat16)
    K1 = torch.tensor([[[-2.5], [0.5]]], dtype=torch.bfloat16)
    assert np.array_equal(orc.scores(_bits(q1), _bits(K1))[0], np.array([-7.5, 1.5], np.float32))


def pin_scores_numpy_fp64(orc, seed: int = 7):
    """Against numpy's float64 matmul of the same bf16 values: the two exact
    up-to-rounding sums agree to one float32 ulp."""
    rows, n, d = 4, 300, 128
    q = inputs.bf16_normal((rows, d), 1.0, seed)
    K = inputs.bf16_normal((rows, n, d), d ** -0.5, seed + 1)
    s = orc.scores(_bits(q), _bits(K))
    ref = np.einsum("rd,rnd->rn", q.double().numpy(), K.double().numpy()).astype(np.float32)
    ulp = np.spacing(np.abs(ref)).astype(np.float32)
    assert np.all(np.abs(s - ref) <= ulp)
    Ks = inputs.bf16_normal((n, d), d ** -0.5, seed + 2)
    s2 = orc.scores(_bits(q), _bits(Ks))
    ref2 = (q.double().numpy() @ Ks.double().numpy().T).astype(np.float32)
    assert np.all(np.abs(s2 - ref2) <= np.spacing(np.abs(ref2)))


def pin_score_topk_selects_scores(orc, seed: int = 8):
    """The fused oracle is the bucketed oracle applied to its own scores."""
    q, K = inputs.decode_inputs(2, 2, 700, 128, seed)
    v, i, s = orc.score_topk(_bits(q), _bits(K), 64, 32, 2)
    v2, i2 = orc.bucketed(s, 64, 32, 2)
    assert np.array_equal(i, i2) and _same_bits(v, v2)
    for r in range(s.shape[0]):
        want, _ = brute_bucketed(s[r], 64, 32, 2)
        assert list(i[r]) == want


ALL_PINS = [
    pin_brute_force_bucketed, pin_brute_force_exact, pin_reductions_to_exact, pin_fig2_golden,
    pin_adversarial, pin_split_merge, pin_scores_unit_vectors, pin_scores_closed_form,
    pin_scores_numpy_fp64, pin_score_topk_selects_scores,
]


# ---------------------------------------------------------------- sampling tail
def pin_sampling_closed_forms(orc):
    """Inverse-CDF draws at hand-computed boundaries."""
    # two equal logits: the CDF boundary sits at exactly 1/2 (strictly above
    # the target picks), so u < 1/2 draws the first and u >= 1/2 the second
    v = np.array([[1.5, 1.5]], np.float32)
    i = np.array([[7, 3]], np.int32)
    for u, want in ((0.0, 7), (0.25, 7), (0.4999, 7), (0.5, 3), (0.75, 3), (0.9999, 3)):
        t, _ = orc.sample_rows(v, i, 1.0, [u])
        assert t[0] == want, (u, t[0], want)
    # logits ln 3, 0 at T = 1: probabilities 3/4, 1/4
    v = np.array([[math.log(3.0), 0.0]], np.float32)
    i = np.array([[0, 1]], np.int32)
    for u, want in ((0.74, 0), (0.76, 1)):
        assert orc.sample_rows(v, i, 1.0, [u])[0][0] == want
    # the same logits at T = 2 weigh sqrt(3) : 1, boundary sqrt(3)/(sqrt(3)+1) = 0.634
    for u, want in ((0.62, 0), (0.65, 1)):
        assert orc.sample_rows(v, i, 2.0, [u])[0][0] == want
    # at T = 1/2 they weigh 9 : 1, boundary 0.9
    for u, want in ((0.89, 0), (0.91, 1)):
        assert orc.sample_rows(v, i, 0.5, [u])[0][0] == want


def pin_sampling_frequencies(orc, N: int = 4000, seed: int = 11):
    """Stratified uniforms u_j = (j + 1/2) / N: each token is drawn
    round(N p_i) times up to one, p = softmax(v / T) over the selection."""
    g = np.random.default_rng(seed)
    for T in (0.5, 1.0, 3.0):
        k = 12
        v = np.sort(g.normal(size=k).astype(np.float32))[::-1].copy()
        idx = g.permutation(1000)[:k].astype(np.int32)
        rows_v = np.repeat(v[None], N, 0)
        rows_i = np.repeat(idx[None], N, 0)
        u = (np.arange(N) + 0.5) / N
        tok, _ = orc.sample_rows(rows_v, rows_i, T, u)
        p = np.exp((v.astype(np.float64) - v[0]) / T)
        p /= p.sum()
        for j in range(k):
            assert abs(int((tok == idx[j]).sum()) - N * p[j]) <= 1.0 + 1e-9, (T, j)


def pin_sampling_special(orc):
    """Padding and -inf weigh nothing; a NaN or +inf best entry is drawn;
    a row without candidates draws -1."""
    ninf = -np.inf
    v = np.array([[2.0, ninf, ninf], [np.nan, 1.0, 0.0], [np.inf, 5.0, 1.0], [ninf, ninf, ninf]],
                 np.float32)
    i = np.array([[4, 8, -1], [6, 2, 1], [9, 3, 0], [-1, -1, -1]], np.int32)
    for u in (0.0, 0.5, 0.999):
        t, _ = orc.sample_rows(v, i, 1.0, [u] * 4)
        assert list(t) == [4, 6, 9, -1], (u, list(t))
    # a padding slot in the middle of a list (whatever value it carries) moves
    # no boundary: three equal weights, boundaries at 1/3 and 2/3
    v = np.array([[1.0, 1.0, 1.0, 1.0]], np.float32)
    i = np.array([[1, -1, 2, 3]], np.int32)
    for u, want in ((0.3, 1), (0.6, 2), (0.9, 3)):
        assert orc.sample_rows(v, i, 1.0, [u])[0][0] == want, u


# ---------------------------------------------------------------- re-ranking
def _bf16_bits(x: torch.Tensor) -> np.ndarray:
    return x.to(torch.bfloat16).contiguous().view(torch.int16).numpy().view(np.uint16)


def pin_rerank_numpy(orc, seed: int = 12):
    """Re-ranking = numpy fp64 scores of the distinct valid candidates (rounded
    to float) + a lexsort top-k; repeats, -1 and out-of-range slots drop out."""
    g = np.random.default_rng(seed)
    rows, n, d, c, k = 5, 300, 128, 90, 20
    q = torch.from_numpy(g.normal(size=(rows, d)).astype(np.float32))
    K = torch.from_numpy((g.normal(size=(rows, n, d)) / np.sqrt(d)).astype(np.float32))
    qb, Kb = _bf16_bits(q), _bf16_bits(K)
    cand = g.integers(0, n, size=(rows, c)).astype(np.int32)  # repeats on purpose
    cand[:, ::7] = -1
    cand[:, 3] = n + 5  # out of range
    ov, oi = orc.rerank(qb, Kb, cand, k)
    qf = (qb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    Kf = (Kb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for r in range(rows):
        ids = np.array(sorted({int(i) for i in cand[r] if 0 <= i < n}), np.int64)
        s = (Kf[r, ids] @ qf[r]).astype(np.float32)
        order = np.lexsort((ids, -s.astype(np.float64)))[:k]
        assert list(oi[r, :len(order)]) == list(ids[order]), r
        assert np.array_equal(ov[r, :len(order)], s[order])
        assert np.all(oi[r, len(order):] == -1)


def pin_rerank_shared_keys_and_padding(orc):
    """A key matrix shared by all rows; fewer distinct candidates than k pads."""
    d, n = 128, 16
    K = torch.zeros(n, d)
    K[torch.arange(n), torch.arange(n)] = torch.arange(n, dtype=torch.float32)  # key i scores i*q_i
    q = torch.ones(2, d)
    cand = np.array([[3, 3, 9, -1, 1], [15, 0, 15, 15, 15]], np.int32)
    ov, oi = orc.rerank(_bf16_bits(q), _bf16_bits(K), cand, 4)
    assert list(oi[0]) == [9, 3, 1, -1] and list(ov[0, :3]) == [9.0, 3.0, 1.0]
    assert list(oi[1]) == [15, 0, -1, -1] and list(ov[1, :2]) == [15.0, 0.0]
