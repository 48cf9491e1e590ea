"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Selection (topk_bucketed, topk_exact) must match bit for bit: values and
indices.  Fused scoring (score_topk) must agree with the oracle's fp64 scores
within 2e-3 relative (floor 2^-10 * |q| |K_i|), the selection the GPU made on
its own fp32 scores must equal the oracle's selection on those same scores bit
for bit, and the index sets must match except where the oracle's decision is
fragile (a bucket's k_b-th/(k_b+1)-th gap or the k-th/(k+1)-th candidate gap
below the tolerance).
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import approximate_top_selection_b200 as atk
from approximate_top_selection_b200 import inputs
from oracle import recall as rc

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _gpu(oracle_mod):
    if not torch.cuda.is_available():
        pytest.fail("these tests need a CUDA device")
    atk.load_library()
    yield
    assert atk.topk_device_status() == 0


def same_bits(a, b) -> bool:
    a = np.ascontiguousarray(np.asarray(a, np.float32))
    b = np.ascontiguousarray(np.asarray(b, np.float32))
    return a.shape == b.shape and np.array_equal(a.view(np.uint32), b.view(np.uint32))


def check_bucketed(x_cpu: torch.Tensor, k, b, kb, oracle_mod, x_dev=None, rows_subset=None):
    x_dev = x_cpu.to(DEV) if x_dev is None else x_dev
    v, i = atk.topk_bucketed(x_dev, k, b, kb)
    torch.cuda.synchronize()
    v, i = v.cpu().numpy(), i.cpu().numpy()
    xs = x_cpu.numpy() if rows_subset is None else x_cpu.numpy()[rows_subset]
    ov, oi = oracle_mod.bucketed(xs, k, b, kb)
    if rows_subset is not None:
        v, i = v[rows_subset], i[rows_subset]
    bad = np.nonzero(~np.all(oi == i, axis=1))[0]
    assert bad.size == 0, "index mismatch in rows %s (k=%d b=%d kb=%d)" % (bad[:5], k, b, kb)
    assert same_bits(v, ov), "value bits differ"
    return v, i


# ------------------------------------------------------------------ bucketed
def test_tiny_config(oracle_mod):
    """8 rows x 4096 N(0,1), k=64, b=128, k_b=1 (final exact top-64 of 128)."""
    x = inputs.normal_rows(8, 4096, inputs.SEEDS["tiny"])
    check_bucketed(x, 64, 128, 1, oracle_mod)


@pytest.mark.parametrize("seed", range(6))
def test_random_shapes(oracle_mod, seed):
    """Random small shapes: ragged tails, b > n, k > C (padding), every k_b,
    fast (b | 1024, n % 4 == 0) and general paths."""
    rng = np.random.default_rng(100 + seed)
    for t in range(12):
        rows = int(rng.integers(1, 6))
        n = int(rng.integers(1, 9000))
        b = int(rng.choice([1, 2, 3, 8, 32, 100, 128, 256, 512, 1000, 1024]))
        kb = int(rng.integers(1, 5))
        k = int(rng.integers(1, 700))
        kind = t % 3
        if kind == 0:
            x = inputs.normal_rows(rows, n, seed * 100 + t)
        elif kind == 1:
            x = inputs.integer_rows(rows, n, 5, seed * 100 + t)
        else:
            x = inputs.special_rows(rows, n, seed * 100 + t)
        check_bucketed(x, k, b, kb, oracle_mod)


def test_special_values_fast_path(oracle_mod):
    """NaN, +-inf, +-0 and ties through the TMA path (n % 4 == 0, b | 1024)."""
    x = inputs.special_rows(16, 8192, 7)
    for (k, b, kb) in [(64, 128, 1), (100, 32, 4), (512, 256, 2), (30, 1, 4), (9, 1024, 3)]:
        check_bucketed(x, k, b, kb, oracle_mod)


def test_misaligned_rows_take_general_path(oracle_mod):
    """A base pointer that is not 16-byte aligned, and n % 4 != 0."""
    big = inputs.normal_rows(1, 4 * 3001 + 1, 9).reshape(-1)
    x = big[1:].reshape(4, 3001)
    xd = big.to(DEV)[1:].reshape(4, 3001)
    check_bucketed(x.contiguous(), 50, 64, 2, oracle_mod, x_dev=xd)


def test_split_rows_are_merged(oracle_mod):
    """Few long rows: each row is streamed by several CTAs and merged by the
    last one to finish (ticket in the workspace)."""
    x = inputs.normal_rows(3, 400000, 11)
    check_bucketed(x, 100, 512, 2, oracle_mod)
    x = inputs.integer_rows(2, 1 << 20, 50, 12)  # ties everywhere
    check_bucketed(x, 300, 256, 4, oracle_mod)
    x = inputs.normal_rows(1, 999999, 13)  # general path, split
    check_bucketed(x, 64, 100, 3, oracle_mod)


def test_many_rows_per_cta(oracle_mod):
    """More rows than resident CTAs: CTA ranges hold several rows and cut rows."""
    x = inputs.uniform_rows(3000, 2048, 14)
    check_bucketed(x, 16, 64, 1, oracle_mod)
    x = inputs.uniform_rows(2500, 1001, 15)
    check_bucketed(x, 20, 50, 2, oracle_mod)


def test_workspace_reuse_across_shapes(oracle_mod):
    """One workspace, calls of different shapes back to back: the tickets the
    merge uses are left at zero by every call."""
    nbytes = max(atk.topk_workspace_bytes(atk.TOPK_OP_BUCKETED, r, n, k, b, kb)
                 for (r, n, k, b, kb) in [(2, 300000, 50, 256, 2), (5, 100000, 64, 128, 1)])
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=DEV)
    for it in range(3):
        for (r, n, k, b, kb) in [(2, 300000, 50, 256, 2), (5, 100000, 64, 128, 1)]:
            x = inputs.normal_rows(r, n, 1000 * it + r)
            v, i = atk.topk_bucketed(x.to(DEV), k, b, kb, workspace=ws)
            ov, oi = oracle_mod.bucketed(x.numpy(), k, b, kb)
            assert np.array_equal(i.cpu().numpy(), oi) and same_bits(v.cpu().numpy(), ov)
    torch.cuda.synchronize()
    assert int(ws.count_nonzero()) <= nbytes  # slots may hold data; tickets must be zero
    tick = ws[:256].view(torch.int32)
    assert int(tick.abs().sum()) == 0


def test_vocab_config_full(oracle_mod):
    """256 rows x 131072 logits (N(0,1) + Zipf(1.1) rank offset), k=50, b=512, k_b=1."""
    x = inputs.vocab_logits(256, 131072, inputs.SEEDS["vocab"])
    check_bucketed(x, 50, 512, 1, oracle_mod)


@pytest.mark.parametrize("b", [128, 256, 512])
@pytest.mark.parametrize("kb", [1, 2, 4])
def test_long_context_sweep(oracle_mod, b, kb):
    """256 rows x 131072 iid U(0,1), k=512 (parity on a row sample), plus
    adversarial rows whose top-k sit in as few residue classes as possible:
    recall equals the worst case of Eq. (2) exactly."""
    seed = inputs.SEEDS["long"] + 16 * b + kb
    x = inputs.uniform_rows(256, 131072, seed)
    sample = np.arange(0, 256, 16)
    check_bucketed(x, 512, b, kb, oracle_mod, rows_subset=sample)
    adv = inputs.adversarial_rows(8, 131072, 512, b, seed + 1)
    _, gi = check_bucketed(adv, 512, b, kb, oracle_mod)
    _, ei = oracle_mod.exact(adv.numpy(), 512)
    r = rc.recall(gi, ei)
    assert np.all(np.abs(r - rc.eq2_worst_recall(131072, 512, b, kb)) < 1e-12)


@pytest.mark.parametrize("n,k,b,kb", [(4096, 64, 128, 1), (32768, 512, 256, 2),
                                      (8192, 256, 64, 4)])
def test_recall_band_on_gpu(oracle_mod, n, k, b, kb):
    """Recall of the GPU result over 10^4 iid uniform rows (2000 for the larger
    shapes): within 3 SE of the exact finite-n expectation, and not more than
    3 SE below Eq. (1)."""
    rows = 10000 if n <= 4096 else 2000
    x = inputs.uniform_rows(rows, n, 77 + n + kb).to(DEV)
    _, bi = atk.topk_bucketed(x, k, b, kb)
    _, ei = atk.topk_exact(x, k)
    bi, ei = bi.cpu().numpy(), ei.cpu().numpy()
    # the exact reference itself is checked against the oracle on a sample
    _, oi = oracle_mod.exact(x[:64].cpu().numpy(), k)
    assert np.array_equal(ei[:64], oi)
    r = rc.recall(bi, ei)
    mean, se = r.mean(), r.std(ddof=1) / math.sqrt(rows)
    assert abs(mean - rc.expected_recall_exact(n, k, b, kb)) <= 3 * se
    assert mean >= rc.eq1_expected_recall(k, b, kb) - 3 * se


# ------------------------------------------------------------------ exact
@pytest.mark.parametrize("rows,n,k", [(8, 4096, 64), (4, 1000, 1000), (3, 77, 200),
                                      (16, 8192, 512), (4, 8193, 50), (64, 131072, 50),
                                      (2, 131072, 16384), (5, 16000, 16000), (2, 20000, 16384),
                                      (3, 300001, 999)])
def test_exact_matches_oracle(oracle_mod, rows, n, k):
    x = inputs.normal_rows(rows, n, rows * 7 + n + k)
    v, i = atk.topk_exact(x.to(DEV), k)
    ov, oi = oracle_mod.exact(x.numpy(), k)
    assert np.array_equal(i.cpu().numpy(), oi) and same_bits(v.cpu().numpy(), ov)


def test_exact_ties_and_specials(oracle_mod):
    for (rows, n, k, levels) in [(4, 50000, 3000, 3), (2, 100000, 77, 1), (3, 40000, 5000, 2)]:
        x = inputs.integer_rows(rows, n, levels, n + k)
        v, i = atk.topk_exact(x.to(DEV), k)
        ov, oi = oracle_mod.exact(x.numpy(), k)
        assert np.array_equal(i.cpu().numpy(), oi) and same_bits(v.cpu().numpy(), ov)
    x = inputs.special_rows(4, 30000, 5)
    v, i = atk.topk_exact(x.to(DEV), 700)
    ov, oi = oracle_mod.exact(x.numpy(), 700)
    assert np.array_equal(i.cpu().numpy(), oi) and same_bits(v.cpu().numpy(), ov)


# ------------------------------------------------------------------ scoring
def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def check_scores(q: torch.Tensor, K: torch.Tensor, k, b, kb, oracle_mod, rows_subset=None):
    """q, K on the device.  Returns the GPU outputs after all checks."""
    v, i, s = atk.score_topk(q, K, k, b, kb, return_scores=True)
    torch.cuda.synchronize()
    rows = q.shape[0]
    sub = np.arange(rows) if rows_subset is None else np.asarray(rows_subset)
    if rows_subset is not None:  # copy back only the sampled rows
        keep = torch.as_tensor(sub, device=s.device)
        v = torch.zeros_like(v).index_copy_(0, keep, v[keep])
        i = torch.zeros_like(i).index_copy_(0, keep, i[keep])
        s = s[keep]
        s_full = np.zeros((rows, s.shape[1]), np.float32)
        s_full[sub] = s.cpu().numpy()
        s = s_full
    else:
        s = s.cpu().numpy()
    v, i = v.cpu().numpy(), i.cpu().numpy()
    # (1) the selection on the GPU's own scores is the oracle's, bit for bit
    ov, oi = oracle_mod.bucketed(s[sub], k, b, kb)
    assert np.array_equal(i[sub], oi) and same_bits(v[sub], ov)
    # (2) scores within tolerance of the fp64 oracle
    tsub = torch.as_tensor(sub, device=q.device)
    qs = q[tsub]
    Ks = K[tsub] if K.dim() == 3 else K
    ref = oracle_mod.scores(_bits(qs), _bits(Ks))
    qn = torch.linalg.vector_norm(qs.float().cpu(), dim=1).double().numpy()
    kn = torch.linalg.vector_norm(Ks.float().cpu(), dim=-1).double().numpy()
    scale = qn[:, None] * (kn if kn.ndim == 2 else kn[None, :])
    tol = 2e-3 * np.maximum(np.abs(ref), 2.0 ** -10 * scale)
    err = np.abs(s[sub].astype(np.float64) - ref)
    assert np.all(err <= tol), float((err / tol).max())
    # (3) index sets equal except at fragile decisions of the oracle: a near-tie
    # (within twice the tolerance) at a bucket's k_b-th/(k_b+1)-th boundary or at
    # the k-th/(k+1)-th candidate boundary, with the element inside that band.
    rv, ri = oracle_mod.bucketed(ref, k, b, kb)
    gi = i[sub]
    for row in range(len(sub)):
        a, g = set(ri[row][ri[row] >= 0].tolist()), set(gi[row][gi[row] >= 0].tolist())
        diff = a ^ g
        if not diff:
            continue
        sc = ref[row].astype(np.float64)
        T = 2 * float(tol[row].max())
        cols = [np.sort(sc[j::b])[::-1] for j in range(b)]
        cand = np.sort(np.concatenate([c[:kb] for c in cols]))[::-1]
        for idx in diff:
            col = cols[idx % b]
            near_bucket = (len(col) > kb and col[kb - 1] - col[kb] <= T
                           and col[kb] - T <= sc[idx] <= col[kb - 1] + T)
            near_stage2 = (len(cand) > k and cand[k - 1] - cand[k] <= T
                           and cand[k] - T <= sc[idx] <= cand[k - 1] + T)
            assert near_bucket or near_stage2, (row, idx)
    return v, i, s


def test_score_small_per_row_keys(oracle_mod):
    q, K = inputs.decode_inputs(2, 3, 5000, 128, 21)
    check_scores(q.to(DEV), K.to(DEV), 512, 256, 2, oracle_mod)


@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("kb", [1, 4])
def test_score_shapes(oracle_mod, d, kb):
    q, K = inputs.decode_inputs(1, 5, 3333, d, 22 + d + kb)
    check_scores(q.to(DEV), K.to(DEV), 100, 64, kb, oracle_mod)
    Q, Ks = inputs.link_inputs(7, 20001, d, 23 + d + kb)
    check_scores(Q.to(DEV), Ks.to(DEV), 100, 1024, kb, oracle_mod)


def test_score_long_rows_split(oracle_mod):
    q, K = inputs.decode_inputs(1, 2, 300000, 128, 24)
    check_scores(q.to(DEV), K.to(DEV), 512, 256, 2, oracle_mod)


def _cta_edge_rows(rows: int, n: int, ctas: int, extra: int, seed: int) -> list:
    """Sampled rows: the rows holding the first and the last element of CTA
    ranges when rows*n elements are cut into `ctas` equal ranges (the
    streaming kernels' split), plus `extra` rows drawn at random."""
    E = rows * n
    picked = set()
    for c in range(0, ctas, max(1, ctas // 24)):
        lo, hi = E * c // ctas, E * (c + 1) // ctas - 1
        picked.update((lo // n, hi // n))
    picked.update((0, rows - 1))
    rng = np.random.default_rng(seed)
    picked.update(int(r) for r in rng.choice(rows, size=extra, replace=False))
    return sorted(picked)


def test_decode_config_full(oracle_mod):
    """16 x 32 rows, 32768 keys of d=128: at least 64 sampled rows (the rows at
    the edges of CTA ranges among them) against the oracle."""
    q, K = inputs.decode_inputs(16, 32, 32768, 128, inputs.SEEDS["decode"], device=DEV)
    sub = _cta_edge_rows(512, 32768, 296, 24, 5)
    assert len(sub) >= 64
    check_scores(q, K, 512, 256, 2, oracle_mod, rows_subset=sub)


# ------------------------------------------------------------------ tensor-core scoring
@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("kb", [1, 2, 4])
def test_link_umma_shapes(oracle_mod, d, kb):
    """Shared key matrix, b | n and >= 32 queries: the tcgen05 path.  Ragged
    query tiles (not a multiple of 128) and stripe counts that are not a
    multiple of the 32-stripe tile are included."""
    for (rows, T, b, k) in [(32, 32, 64, 50), (200, 37, 64, 100), (130, 70, 256, 300)]:
        Q, K = inputs.link_inputs(rows, T * b, d, 31 + rows + d + kb)
        check_scores(Q.to(DEV), K.to(DEV), k, b, kb, oracle_mod)


@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("kb", [1, 2, 4])
def test_link_umma_pair_shapes(oracle_mod, d, kb):
    """256 queries or more: the CTA-pair selector (tcgen05 cta_group::2, one
    256-query tile per pair).  Ragged query tiles (the second CTA's rows past
    the end) and stripe counts that are not a multiple of the 32-stripe tile."""
    for (rows, T, b, k) in [(256, 32, 64, 50), (300, 37, 64, 100), (600, 70, 256, 300)]:
        Q, K = inputs.link_inputs(rows, T * b, d, 51 + rows + d + kb)
        check_scores(Q.to(DEV), K.to(DEV), k, b, kb, oracle_mod)


def test_link_umma_special_values(oracle_mod):
    """Scores that are +-inf or NaN (from inf / NaN inputs) take the exact
    queue update: the selection on the GPU's scores is still the oracle's."""
    Q, K = inputs.link_inputs(64, 64 * 32, 128, 41)
    K[5, :] = float("inf")
    K[77, 3] = float("nan")
    K[100, :] = -float("inf")
    v, i, s = atk.score_topk(Q.to(DEV), K.to(DEV), 40, 64, 2, return_scores=True)
    ov, oi = oracle_mod.bucketed(s.cpu().numpy(), 40, 64, 2)
    assert np.array_equal(i.cpu().numpy(), oi) and same_bits(v.cpu().numpy(), ov)


@pytest.mark.parametrize("rows", [64, 256])
def test_link_umma_kb1_special_values(oracle_mod, rows):
    """k_b = 1 takes each 32-score load's maximum before touching its queue:
    ties inside one load and across loads of a bucket, zero maxima (a zero
    query: every score is +0 or -0), +-inf and NaN scores must select exactly
    as the oracle does on the GPU's own scores (64 rows: one CTA per tile, 256:
    CTA pairs)."""
    b = 64
    Q, K = inputs.link_inputs(rows, 64 * b, 128, 43)   # 64 stripes per bucket: two loads each
    Q[1:4] = Q[0]                    # four queries share the tied maxima below
    Q[5] = 0.0                       # all scores +-0
    top = Q[0].float() * 8.0
    for key in (10, 10 + b, 10 + 2 * b, 20 + 3 * b, 20 + 40 * b):  # same load / across loads
        K[key] = top.to(K.dtype)
    K[7] = float("inf")
    K[8 + 33 * b] = -float("inf")
    K[9 + 5 * b, 3] = float("nan")
    v, i, s = atk.score_topk(Q.to(DEV), K.to(DEV), 40, b, 1, return_scores=True)
    ov, oi = oracle_mod.bucketed(s.cpu().numpy(), 40, b, 1)
    assert np.array_equal(i.cpu().numpy(), oi) and same_bits(v.cpu().numpy(), ov)
    assert atk.topk_device_status() == 0


def test_link_config_full(oracle_mod):
    """1024 queries x 2^20 entities, d = 256, k = 100, b = 1024, k_b = 1:
    sampled query rows against the fp64 oracle."""
    Q, K = inputs.link_inputs(1024, 1 << 20, 256, inputs.SEEDS["link"], device=DEV)
    # the first and last query of each 128-query tile, plus 48 drawn at random
    edges = {e for t in range(8) for e in (128 * t, 128 * t + 127)}
    rng = np.random.default_rng(6)
    rest = [int(r) for r in rng.permutation(1024) if int(r) not in edges][:48]
    sub = sorted(edges | set(rest))
    assert len(sub) == 64
    check_scores(Q, K, 100, 1024, 1, oracle_mod, rows_subset=sub)


# ------------------------------------------------------------------ bfloat16 rows
def _bf16_check(x_bf16: torch.Tensor, k, b, kb, oracle_mod, x_dev=None):
    """bf16 rows: the oracle selects on the exactly widened fp32 values; the
    GPU must return the same indices and the same bf16 bits."""
    x_dev = x_bf16.to(DEV) if x_dev is None else x_dev
    v, i = atk.topk_bucketed(x_dev, k, b, kb)
    assert v.dtype == torch.bfloat16
    torch.cuda.synchronize()
    xf = x_bf16.float().numpy()
    ov, oi = oracle_mod.bucketed(xf, k, b, kb)
    assert np.array_equal(i.cpu().numpy(), oi), "bf16 index mismatch (k=%d b=%d kb=%d)" % (k, b, kb)
    got = v.cpu().view(torch.int16).numpy().view(np.uint16)
    want = (ov.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(got, want), "bf16 value bits differ"


@pytest.mark.parametrize("kb", [1, 2, 3, 4])
def test_bf16_rows(oracle_mod, kb):
    """bf16 has 8 mantissa bits: rows are full of ties, the lowest index wins."""
    x = inputs.normal_rows(6, 65536, 300 + kb).to(torch.bfloat16)
    for (k, b) in [(64, 128), (512, 256), (50, 512), (100, 1024)]:
        _bf16_check(x, k, b, kb, oracle_mod)


def test_bf16_special_values_and_general_path(oracle_mod):
    x = inputs.special_rows(8, 8192, 71).to(torch.bfloat16)
    _bf16_check(x, 100, 64, 2, oracle_mod)
    x = inputs.normal_rows(3, 3001, 72).to(torch.bfloat16)  # n % 8 != 0: general path
    _bf16_check(x, 60, 100, 3, oracle_mod)
    x = inputs.normal_rows(2, 500000, 73).to(torch.bfloat16)  # split rows
    _bf16_check(x, 300, 512, 2, oracle_mod)


def test_bf16_vocab_config(oracle_mod):
    x = inputs.vocab_logits(256, 131072, inputs.SEEDS["vocab"]).to(torch.bfloat16)
    _bf16_check(x, 50, 512, 1, oracle_mod)


# ------------------------------------------------------------------ k_b > 2, b >= 512
@pytest.mark.parametrize("b", [512, 1024])
@pytest.mark.parametrize("kb", [3, 4])
def test_wide_kernel_shapes(oracle_mod, b, kb):
    """The 16-warp k_b > 2 kernel (b >= 512): whole rows, rows split across
    CTAs, ragged tails, special values, fp32 and bf16 rows, and its sampling
    variant."""
    for rows, n, k, kind in [(16, 65536, 512, "u"), (3, 400000, 700, "u"), (40, 8196, 100, "s"),
                             (300, 20000, 2000, "n"), (2, 4100, 4096, "i")]:
        seed = 900 + rows + n + b + kb
        if kind == "u":
            x = inputs.uniform_rows(rows, n, seed)
        elif kind == "n":
            x = inputs.normal_rows(rows, n, seed)
        elif kind == "i":
            x = inputs.integer_rows(rows, n, 9, seed)
        else:
            x = inputs.special_rows(rows, n, seed)
        check_bucketed(x, k, b, kb, oracle_mod)
        if kind != "s":
            _bf16_check(x.to(torch.bfloat16), k, b, kb, oracle_mod)
    x = inputs.vocab_logits(8, 65536, 77 + b + kb)
    u = torch.rand(8, generator=torch.Generator().manual_seed(kb))
    tok, v, i = atk.topk_sample(x.to(DEV), 64, b, kb, 1.0, u.to(DEV))
    ov, oi = oracle_mod.bucketed(x.numpy(), 64, b, kb)
    assert np.array_equal(i.cpu().numpy(), oi)
    otok, margin = oracle_mod.sample_rows(ov, oi, 1.0, u.numpy().astype(np.float64))
    assert np.all((tok.cpu().numpy() == otok) | (margin < 1e-5))


@pytest.mark.parametrize("b,kb,k", [(1024, 4, 3000), (1024, 4, 16384), (1024, 3, 2500), (1000, 4, 3500)])
def test_largest_candidate_sets_and_k(oracle_mod, b, kb, k):
    """The support limits: b = 1024 buckets of k_b = 4 (4096 candidates: the
    shared-memory sort of Stage 2), k up to 16384 (padding past the 4096
    candidates), b = 1000 (general kernel), one long row and rows split over
    CTAs, fp32 and bf16."""
    for rows, n in [(2, 1000000), (24, 65536)]:
        x = inputs.uniform_rows(rows, n, 4242 + b + kb + k + n)
        check_bucketed(x, k, b, kb, oracle_mod)
        _bf16_check(x.to(torch.bfloat16), k, b, kb, oracle_mod)


# ------------------------------------------------------------------ one row per CTA
@pytest.mark.parametrize("rows,n,k,b,kb", [(256, 65536, 50, 512, 1), (290, 32768, 512, 256, 2),
                                           (200, 65536, 700, 1024, 4), (160, 40000, 64, 128, 3),
                                           (148, 8192, 100, 64, 2)])
def test_one_row_per_cta_layout(oracle_mod, rows, n, k, b, kb):
    """A whole row per CTA: the queues' merge buffer and the Stage-2 buffer
    share the tile ring.  Called through the binding and through the C ABI
    with no workspace at all (none is needed), fp32 and bf16 rows, every
    kernel (float4 queues, survivor queues, the 16-warp kernel)."""
    lib = atk.load_library()
    x = inputs.uniform_rows(rows, n, 5000 + rows + kb)
    xd = x.to(DEV)
    check_bucketed(x, k, b, kb, oracle_mod, x_dev=xd)
    ov = torch.empty(rows, k, dtype=torch.float32, device=DEV)
    oi = torch.empty(rows, k, dtype=torch.int32, device=DEV)
    st = lib.topk_bucketed(xd.data_ptr(), rows, n, k, b, kb, ov.data_ptr(), oi.data_ptr(), None, 0,
                           torch.cuda.current_stream().cuda_stream)
    assert st == atk.TOPK_OK
    torch.cuda.synchronize()
    wv, wi = oracle_mod.bucketed(x.numpy(), k, b, kb)
    assert np.array_equal(oi.cpu().numpy(), wi) and same_bits(ov.cpu().numpy(), wv)
    _bf16_check(x.to(torch.bfloat16), k, b, kb, oracle_mod)


@pytest.mark.parametrize("b,kb", [(512, 1), (256, 2), (512, 4)])
def test_many_rows_sampling(oracle_mod, b, kb):
    """The sampling draw on a row per CTA over more rows than SMs, fp32 and
    bf16 logits."""
    x = inputs.vocab_logits(256, 32768, 88 + kb)
    u = torch.rand(256, generator=torch.Generator().manual_seed(9 + kb))
    for dt in (torch.float32, torch.bfloat16):
        xs = x.to(dt)
        tok, v, i = atk.topk_sample(xs.to(DEV), 50, b, kb, 0.7, u.to(DEV))
        ov, oi = oracle_mod.bucketed(xs.float().numpy(), 50, b, kb)
        assert np.array_equal(i.cpu().numpy(), oi)
        otok, margin = oracle_mod.sample_rows(ov, oi, 0.7, u.numpy().astype(np.float64))
        assert np.all((tok.cpu().numpy() == otok) | (margin < 1e-5))


# ------------------------------------------------------------------ bf16 order-key queues
def _bf16_from_bits(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.astype(np.uint16).view(np.int16)).view(torch.bfloat16)


@pytest.mark.parametrize("kb", [1, 2, 3, 4])
def test_bf16_key_queues_special_bits(oracle_mod, kb):
    """bf16 rows with k_b > 2 run on 32-bit order keys (value code and queue
    ordinal in one word), k_b <= 2 on packed bf16x2 queues.  Every special bit
    pattern must keep the total order: NaNs of any sign and payload tie above
    +inf, -0 ties +0, -inf is below every number, denormals order as numbers,
    equal values go by index -- whole rows, split rows and ragged tails; and
    with zeros and denormals only (no NaN or infinity), the packed compare of
    the k_b <= 2 fast path sees them too."""
    rng = np.random.default_rng(700 + kb)
    specials = np.array([0x7FC0, 0x7F81, 0xFFC1, 0x7FFF, 0xFF80, 0x7F80, 0x0000, 0x8000,
                         0x0001, 0x8001, 0x007F, 0x807F, 0x3F80, 0xBF80], np.uint16)
    for rows, n, k, b in [(6, 65536, 300, 256), (3, 400000, 700, 512), (40, 8200, 64, 1024),
                          (2, 4104, 4096, 128)]:
        bits = rng.integers(0x3E00, 0x4000, size=(rows, n)).astype(np.uint16)  # narrow: ties
        bits[rng.random((rows, n)) < 0.3] |= 0x8000                          # negatives
        pick = rng.random((rows, n)) < 0.02
        bits[pick] = rng.choice(specials, size=int(pick.sum()))
        x = _bf16_from_bits(bits)
        _bf16_check(x, k, b, kb, oracle_mod)
    finite = np.array([0x0000, 0x8000, 0x0001, 0x8001, 0x007F, 0x807F], np.uint16)
    for rows, n, k, b in [(6, 65536, 300, 256), (3, 400000, 700, 512)]:
        bits = rng.integers(0x0000, 0x0100, size=(rows, n)).astype(np.uint16)  # denormals, ties
        bits[rng.random((rows, n)) < 0.5] |= 0x8000
        pick = rng.random((rows, n)) < 0.05
        bits[pick] = rng.choice(finite, size=int(pick.sum()))
        _bf16_check(_bf16_from_bits(bits), k, b, kb, oracle_mod)
