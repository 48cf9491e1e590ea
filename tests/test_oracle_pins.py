"""The CPU oracle against what the pages and mathematics fix (no GPU)."""
import pytest

import oracle_pins as P


def test_brute_force_bucketed(oracle_mod):
    P.pin_brute_force_bucketed(oracle_mod.default())


def test_brute_force_exact(oracle_mod):
    P.pin_brute_force_exact(oracle_mod.default())


def test_reductions_to_exact(oracle_mod):
    P.pin_reductions_to_exact(oracle_mod.default())


def test_fig2_golden(oracle_mod):
    P.pin_fig2_golden(oracle_mod.default())


def test_recall_formulas_closed_forms():
    P.pin_recall_formulas_closed_forms()


def test_recall_formulas_monte_carlo():
    P.pin_recall_formulas_monte_carlo()


def test_eq1_statistical(oracle_mod):
    P.pin_eq1_statistical(oracle_mod.default())


def test_adversarial_worst_case(oracle_mod):
    P.pin_adversarial(oracle_mod.default())


def test_split_merge(oracle_mod):
    P.pin_split_merge(oracle_mod.default())


def test_scores_unit_vectors(oracle_mod):
    P.pin_scores_unit_vectors(oracle_mod.default())


def test_scores_closed_form(oracle_mod):
    P.pin_scores_closed_form(oracle_mod.default())


def test_scores_numpy_fp64(oracle_mod):
    P.pin_scores_numpy_fp64(oracle_mod.default())


def test_score_topk_selects_scores(oracle_mod):
    P.pin_score_topk_selects_scores(oracle_mod.default())


def test_padding_when_few_candidates(oracle_mod):
    """C < k: all candidates are returned best-first, the rest is -inf / -1."""
    import numpy as np

    x = np.arange(10, dtype=np.float32)
    v, i, c = oracle_mod.bucketed(x, 8, 3, 1, return_candidates=True)
    assert c[0] == 3
    assert list(i[0]) == [9, 8, 7, -1, -1, -1, -1, -1]
    assert np.all(np.isneginf(v[0, 3:]))


def test_sampling_closed_forms(oracle_mod):
    P.pin_sampling_closed_forms(oracle_mod.default())


def test_sampling_frequencies(oracle_mod):
    P.pin_sampling_frequencies(oracle_mod.default())


def test_sampling_special(oracle_mod):
    P.pin_sampling_special(oracle_mod.default())


def test_rerank_numpy(oracle_mod):
    P.pin_rerank_numpy(oracle_mod.default())


def test_rerank_shared_keys_and_padding(oracle_mod):
    P.pin_rerank_shared_keys_and_padding(oracle_mod.default())
