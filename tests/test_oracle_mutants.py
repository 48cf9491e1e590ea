"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check that
the pins catch every one of them.  Nothing here touches the GPU or the shipped
oracle: each variant is a modified copy compiled into a temporary directory."""
import pytest

import oracle_pins as P

# (name, exact text in oracle.c, replacement, pins expected to catch it)
MUTANTS = [
    ("contiguous buckets",
     "for (int64_t i = j; i < n; i += b) {",
     "for (int64_t i = j * ((n + b - 1) / b); i < (j + 1) * ((n + b - 1) / b) && i < n; ++i) {",
     [P.pin_brute_force_bucketed, P.pin_adversarial]),
    ("tie-break by highest index",
     "return a->i < b->i; /* equal values",
     "return a->i > b->i; /* equal values",
     [P.pin_brute_force_bucketed, P.pin_fig2_golden]),
    ("NaN ranked below numbers",
     "return an; /* NaN is above every number */",
     "return bn; /* NaN is above every number */",
     [P.pin_brute_force_bucketed, P.pin_fig2_golden]),
    ("one candidate too few per bucket",
     "int64_t take = m < kb ? m : kb;",
     "int64_t take = m < kb ? m : kb - 1;",
     [P.pin_brute_force_bucketed, P.pin_fig2_golden]),
    ("Stage 2 skipped (candidates kept in bucket order)",
     "    qsort(cand, (size_t)C, sizeof(item), cmp_items);\n    int64_t keep = C < k ? C : k;",
     "    int64_t keep = C < k ? C : k;",
     [P.pin_brute_force_bucketed, P.pin_fig2_golden]),
    ("exact top-k off by one",
     "write_row(all, n < k ? n : k, k,",
     "write_row(all, n < k ? n : k - 1, k,",
     [P.pin_brute_force_exact, P.pin_reductions_to_exact]),
    ("transposed key matrix",
     "s += bf16_to_double(qr[t]) * bf16_to_double(Kr[i * d + t]);",
     "s += bf16_to_double(qr[t]) * bf16_to_double(Kr[t * n + i]);",
     [P.pin_scores_unit_vectors, P.pin_scores_numpy_fp64]),
    ("dropped last term of the dot product",
     "for (int64_t t = 0; t < d; ++t)\n                s +=",
     "for (int64_t t = 0; t < d - 1; ++t)\n                s +=",
     [P.pin_scores_unit_vectors, P.pin_scores_closed_form]),
    ("float accumulation",
     "double s = 0.0;",
     "float s = 0.0f;",
     [P.pin_scores_numpy_fp64]),
    ("per-row key matrices ignored (row 0's keys used for every row)",
     "const uint16_t *Kr = K + r * kstride;",
     "const uint16_t *Kr = K + 0 * kstride;",
     [P.pin_scores_unit_vectors, P.pin_scores_numpy_fp64]),
    ("sampling weights with the sign of the exponent flipped",
     "total += exp(((double)v[i] - (double)v[0]) * inv_t);",
     "total += exp(((double)v[0] - (double)v[i]) * inv_t);",
     [P.pin_sampling_closed_forms, P.pin_sampling_frequencies]),
    ("sampling boundary taken inclusively",
     "if (pick < 0 && run > target)",
     "if (pick < 0 && run >= target)",
     [P.pin_sampling_closed_forms]),
    ("temperature multiplied instead of divided",
     "const double w = exp(((double)v[i] - (double)v[0]) * inv_t);",
     "const double w = exp(((double)v[i] - (double)v[0]) / inv_t);",
     [P.pin_sampling_closed_forms, P.pin_sampling_frequencies]),
    ("padding entries given weight",
     "        if (idx[i] < 0)\n            continue;\n        const double w",
     "        const double w",
     [P.pin_sampling_special]),
    ("pair selection buckets by list position instead of index",
     "            if (all[t].i % b == j)",
     "            if (t % b == j)",
     [P.pin_split_merge]),
    ("re-ranking keeps repeated candidates",
     "                if (seen)\n                    continue;\n",
     "",
     [P.pin_rerank_numpy, P.pin_rerank_shared_keys_and_padding]),
    ("re-ranking drops the last candidate slot",
     "            for (int64_t j = 0; j < c; ++j) {\n                const int64_t i = cr[j];",
     "            for (int64_t j = 0; j < c - 1; ++j) {\n                const int64_t i = cr[j];",
     [P.pin_rerank_numpy, P.pin_rerank_shared_keys_and_padding]),
]


@pytest.mark.parametrize("name,old,new,pins", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(oracle_mod, tmp_path, name, old, new, pins):
    src = oracle_mod.source()
    assert src.count(old) == 1, "mutation anchor not found: %r" % old
    mutant = oracle_mod.variant(src.replace(old, new), str(tmp_path))
    caught = []
    for pin in pins:
        try:
            pin(mutant)
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, "no pin caught the planted mistake: " + name
