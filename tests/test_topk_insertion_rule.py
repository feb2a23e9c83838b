"""The selection rule of the router GEMM's top-k epilogue (used when the
router's K is not split): one pass over the experts in index order keeping the
best 8 by insertion, where a value moves ahead of a kept one only if it is
strictly larger.  It must give the oracle's selection (value descending, lower
index first among equal values) for every k <= 8, ties included.  This
models the rule on the host; the kernel itself is checked on the GPU by
tests/test_gpu_parity.py (the unsplit router cases)."""
import numpy as np
import pytest

import oracle


def insertion_top8(row, shift=True):
    """The epilogue's rule (router.cu, topk_insert); shift=False is the form
    that re-compared a displaced pair instead of shifting it down."""
    sv = [0.0] * 8
    se = [-1] * 8
    for e, v in enumerate(row):
        if se[7] >= 0 and not v > sv[7]:
            continue
        shifting = False
        for i in range(8):
            if (shift and shifting) or se[i] < 0 or v > sv[i]:
                sv[i], v = v, sv[i]
                se[i], e = e, se[i]
                shifting = True
    return se


@pytest.mark.parametrize("E", [8, 9, 33, 64, 256])
def test_insertion_rule_matches_oracle_selection(E):
    rng = np.random.default_rng(E)
    T = 400
    logits = rng.normal(size=(T, E)).astype(np.float32)
    # many exact ties: values on a coarse grid, some rows constant
    logits[: T // 2] = np.round(logits[: T // 2] * 2) / 2
    logits[T // 2: T // 2 + 10] = 0.25
    sel = np.array([insertion_top8(r) for r in logits])
    for k in range(1, min(8, E) + 1):
        idx, _ = oracle.topk(logits, k)
        np.testing.assert_array_equal(sel[:, :k], idx)


def test_displaced_tie_keeps_its_place():
    """A larger value arriving later displaces a run of equal values: the run
    keeps its index order (the form without the shift put expert 0 behind 1-3)."""
    row = np.array([-0.0, -0.0, -0.0, 0.0, -2.0, 1.5, -1.0, -2.0], np.float32)
    assert insertion_top8(row)[:4] == [5, 0, 1, 2]
    assert insertion_top8(row, shift=False)[:2] == [5, 1]
    idx, _ = oracle.topk(row[None, :], 4)
    assert idx[0].tolist() == [5, 0, 1, 2]
