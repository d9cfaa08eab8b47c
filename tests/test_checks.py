"""The parity checker must catch corrupted results (fault injection on the host).

Each test plants one plausible mistake in an otherwise correct (oracle)
result and requires the checker to report it, following the page
"2.4.1 · NSA" advice to corrupt an index and confirm that validation fires.
"""

import numpy as np

import oracle as O
from tests import checks


def _case(seed=0, n=64, topk=8, ints=True):
    rng = np.random.default_rng(seed)
    if ints:
        q = rng.integers(-3, 4, (1, n, 4, 8)).astype(float)
        k = rng.integers(-3, 4, (1, n, 8)).astype(float)
        w = rng.integers(-4, 5, (1, n, 4)) / 4.0
    else:
        q = rng.standard_normal((1, n, 4, 8))
        k = rng.standard_normal((1, n, 8))
        w = rng.standard_normal((1, n, 4))
    scores = O.indexer_scores(q, k, w)[0]
    idx = O.indexer_topk(q, k, w, topk)[0]
    return scores, idx


def test_clean_result_passes():
    scores, idx = _case()
    for t in range(idx.shape[0]):
        assert checks.topk_exact_errors(idx[t], idx[t], t, 8) == []
        errs, st = checks.topk_tolerant_errors(idx[t], scores[t], t, 8)
        assert errs == [] and st["overlap"] == 1.0


def test_slot_permutation_is_accepted():
    scores, idx = _case()
    t = 40
    row = idx[t].copy()
    row[:8] = row[:8][::-1]
    assert checks.topk_exact_errors(row, idx[t], t, 8) == []


def test_wrong_index_is_caught():
    scores, idx = _case()
    t = 50
    row = idx[t].copy()
    outside = [p for p in range(t + 1) if p not in row][0]
    row[3] = outside
    assert checks.topk_exact_errors(row, idx[t], t, 8)


def test_non_causal_index_is_caught():
    scores, idx = _case()
    t = 30
    row = idx[t].copy()
    row[0] = t + 1
    assert checks.row_structure_errors(row, t, 8)


def test_duplicate_and_padding_errors_are_caught():
    scores, idx = _case()
    t = 20
    row = idx[t].copy()
    row[1] = row[0]
    assert checks.row_structure_errors(row, t, 8)
    t = 3                       # short history: 4 valid entries then -1
    row = idx[t].copy()
    row[5] = 0
    assert checks.row_structure_errors(row, t, 8)
    row = idx[t].copy()
    row[2] = -1
    assert checks.row_structure_errors(row, t, 8)


def test_swapped_rows_are_caught():
    scores, idx = _case()
    assert checks.topk_exact_errors(idx[40], idx[41], 41, 8)


def test_tolerant_check_catches_a_low_score_swap():
    scores, idx = _case(ints=False)
    t = 60
    row = idx[t].copy()
    order = np.argsort(scores[t, : t + 1])
    row[0] = order[0]           # swap the best for the worst position
    errs, _ = checks.topk_tolerant_errors(row, scores[t], t, 8)
    assert errs


def test_close_errors():
    a = np.array([1.0, 2.0, 3.0])
    assert checks.close_errors(a, a + 1e-3, 2e-2, 1e-2) == []
    assert checks.close_errors(a, a + [0, 0, 0.2], 2e-2, 1e-2)
    assert checks.close_errors(np.array([-np.inf]), np.array([-np.inf]), 0, 0) == []
