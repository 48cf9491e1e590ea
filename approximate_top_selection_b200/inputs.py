"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no arithmetic of the method: it only draws numbers.  Both the
CUDA path and the CPU oracle read the same tensors it returns (device copies are
made by the caller), so a value drawn here is an input, never an expected result.

Workload shapes follow the pages the library implements:
  - "Approximate Top-k for Increased Parallelism" (arXiv 2412.04358),
    benchmark protocol in the appendix (rows of iid unit-normal values),
    Fig. 4 (vocabulary sampling; knowledge-graph link prediction), and the
    "What would settle it" test (top values placed in one residue class mod b).
  - "Recall Before You Rank" (ReTopK) abstract and the STARC page, Fig. 3:
    a decode query q in R^{1 x d_h} scored against a key cache K in R^{L x d_h}.
The pages' datasets (SQuAD, LLM vocabulary logits, PharMeBINet) are not used;
these seeded draws of the same shapes stand in for them.
"""
from __future__ import annotations

import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0xFFFFFFFFFFFF)
    return g


def normal_rows(rows: int, n: int, seed: int, device="cpu") -> torch.Tensor:
    """rows x n float32, iid N(0, 1)."""
    return torch.randn(rows, n, generator=_gen(seed, device), device=device, dtype=torch.float32)


def uniform_rows(rows: int, n: int, seed: int, device="cpu") -> torch.Tensor:
    """rows x n float32, iid U[0, 1)."""
    return torch.rand(rows, n, generator=_gen(seed, device), device=device, dtype=torch.float32)


def integer_rows(rows: int, n: int, levels: int, seed: int, device="cpu") -> torch.Tensor:
    """rows x n float32 holding small integers in [0, levels): heavy ties."""
    g = _gen(seed, device)
    return torch.randint(0, levels, (rows, n), generator=g, device=device).to(torch.float32)


def special_rows(rows: int, n: int, seed: int, with_nan: bool = True) -> torch.Tensor:
    """rows x n float32 mixing ties, +-0, +-inf and (optionally) NaN, on the CPU."""
    g = _gen(seed, "cpu")
    x = torch.randint(-3, 4, (rows, n), generator=g).to(torch.float32)
    pick = torch.randint(0, 16, (rows, n), generator=g)
    x[pick == 0] = 0.0
    x[pick == 1] = -0.0
    x[pick == 2] = float("inf")
    x[pick == 3] = float("-inf")
    if with_nan:
        x[pick == 4] = float("nan")
    return x


def ar1_rows(rows: int, n: int, rho: float, seed: int, device="cpu") -> torch.Tensor:
    """rows x n float32, a stationary AR(1) Gaussian process along each row:
    x_0 ~ N(0, 1), x_i = rho x_{i-1} + sqrt(1 - rho^2) e_i with e_i iid N(0, 1),
    so every x_i is N(0, 1) and corr(x_i, x_{i+l}) = rho^l.  The correlated
    inputs of the page's assignment study (Appendix A.1, Fig. 6: AR(1)
    multivariate-normal rows); |rho| < 1.
    """
    import numpy as np
    from scipy.signal import lfilter

    if not -1.0 < rho < 1.0:
        raise ValueError("need |rho| < 1")
    g = _gen(seed, "cpu")
    e = torch.randn(rows, n, generator=g, dtype=torch.float64).numpy()
    start = torch.randn(rows, 1, generator=g, dtype=torch.float64).numpy()  # x_{-1}
    c = float(np.sqrt(1.0 - rho * rho))
    x = lfilter([c], [1.0, -rho], e, axis=1, zi=rho * start)[0]
    return torch.from_numpy(x.astype(np.float32)).to(device)


def zipf_permutation(n: int, seed: int, device="cpu") -> torch.Tensor:
    """A seeded permutation rho of [0, n) (token id -> popularity rank)."""
    return torch.randperm(n, generator=_gen(seed ^ 0x5A5A, device), device=device)


def vocab_logits(rows: int, n: int, seed: int, exponent: float = 1.1, device="cpu") -> torch.Tensor:
    """Vocabulary-sampling logits: N(0,1) + a Zipf(exponent) rank-offset bias.

    Reading of "Zipf(1.1) rank-offset bias": token i has popularity rank
    rho(i) (a seeded permutation shared by all rows) and its logit is offset by
    -exponent * ln(1 + rho(i)), i.e. a Zipf law in probability space, with the
    popular tokens scattered over the vocabulary ids.
    """
    noise = normal_rows(rows, n, seed, device)
    rho = zipf_permutation(n, seed, device).to(torch.float32)
    return noise - exponent * torch.log1p(rho)[None, :]


def adversarial_rows(rows: int, n: int, k: int, b: int, seed: int, device="cpu") -> torch.Tensor:
    """Rows whose k largest values sit in as few residue classes mod b as possible.

    Background values are U(0,1); the k top values are 1 + U(0,1).  With
    s = n/b slots per class, classes r, r+1, ... (mod b) are filled in order:
    floor(k/s) classes completely and k mod s random slots of the next one.
    r is drawn per row from the seed.  Requires b | n.
    """
    if n % b:
        raise ValueError("adversarial rows need b | n")
    s = n // b
    g = _gen(seed, "cpu")
    x = torch.rand(rows, n, generator=g, dtype=torch.float32)
    top = 1.0 + torch.rand(rows, k, generator=g, dtype=torch.float32)
    full, rest = divmod(k, s)
    for r in range(rows):
        r0 = int(torch.randint(0, b, (1,), generator=g))
        pos = []
        for c in range(full):
            cls = (r0 + c) % b
            pos.extend(range(cls, n, b))
        if rest:
            cls = (r0 + full) % b
            slots = torch.randperm(s, generator=g)[:rest]
            pos.extend(int(cls + b * t) for t in slots)
        x[r, torch.tensor(pos, dtype=torch.long)] = top[r, : len(pos)]
    return x.to(device)


def bf16_normal(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    """bfloat16 tensor of iid N(0, std^2) draws (drawn in float32, rounded once)."""
    x = torch.randn(*shape, generator=_gen(seed, device), device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def decode_inputs(batch: int, heads: int, n: int, d: int, seed: int, device="cpu"):
    """Sparse-attention decode selection: one query per (batch, head) row.

    q: [batch*heads, d] bf16 N(0, 1) (the query's distribution is not stated on
    the pages; unit normal is a reading).  K: [batch*heads, n, d] bf16 with
    entries N(0, 1/d).
    """
    rows = batch * heads
    q = bf16_normal((rows, d), 1.0, seed, device)
    K = bf16_normal((rows, n, d), d ** -0.5, seed + 1, device)
    return q, K


def link_inputs(queries: int, entities: int, d: int, seed: int, device="cpu"):
    """Link-prediction scoring: Q [queries, d], K [entities, d], bf16 N(0, 1/d)."""
    Q = bf16_normal((queries, d), d ** -0.5, seed, device)
    K = bf16_normal((entities, d), d ** -0.5, seed + 1, device)
    return Q, K


# Seeds of the five workload families (one per family, fixed).
def support_union(rows: int, n: int, supports: int, size: int, seed: int, device="cpu") -> torch.Tensor:
    """rows x (supports * size) int32 candidate indices: the concatenation of
    `supports` index sets of `size` positions of [0, n) per row, each a shifted
    and partly redrawn copy of the first, so they overlap as the supports of
    similar queries do ("Recall Before You Rank", abstract).  Repeats stay in."""
    g = _gen(seed, "cpu")
    first = torch.randint(0, n, (rows, size), generator=g)
    parts = [first]
    for s in range(1, supports):
        p = torch.roll(first, shifts=7 * s, dims=1).clone()
        redraw = torch.rand(rows, size, generator=g) < 0.3
        p[redraw] = torch.randint(0, n, (int(redraw.sum()),), generator=g)
        parts.append(p)
    return torch.cat(parts, dim=1).to(torch.int32).to(device)


SEEDS = {"tiny": 0x70B00000, "decode": 0x70B00001, "vocab": 0x70B00002, "link": 0x70B00003,
         "long": 0x70B00004}
