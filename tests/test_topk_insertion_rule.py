"""The router's two selection rules, modelled on the host, against the
oracle's selection (value descending, lower index first among equal values)
on tie-heavy rows, for every k <= 8:
  * the GEMM epilogue's (used when the router's K is not split): one pass over
    the experts in index order keeping the best 8 by insertion, a value moving
    ahead of a kept one only if it is strictly larger;
  * the split-K top-k kernel's: k rounds of a warp-wide arg-max.
The kernels themselves are checked on the GPU by tests/test_gpu_parity.py."""
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


def warp_argmax_topk(row, k, ep):
    """The split-K top-k kernel's rule (router.cu, router_topk_kernel): lane L
    holds experts L, L+32, ...; each of k rounds takes every lane's best live
    candidate (strictly larger replaces, so the lowest index wins within a
    lane), reduces over an xor butterfly preferring the larger value and, on
    equal values, the lower index, then retires the winner."""
    E = len(row)
    live = [[(lane + 32 * c) < E for c in range(ep // 32)] for lane in range(32)]
    out = []
    for _ in range(k):
        cand = []
        for lane in range(32):
            bv, be = 0.0, None
            for c in range(ep // 32):
                e = lane + 32 * c
                if live[lane][c] and (be is None or row[e] > bv):
                    bv, be = row[e], e
            cand.append((bv, be))
        off = 16
        while off:
            nxt = []
            for lane in range(32):
                bv, be = cand[lane]
                ov, oe = cand[lane ^ off]
                if oe is not None and (be is None or ov > bv or (ov == bv and oe < be)):
                    bv, be = ov, oe
                nxt.append((bv, be))
            cand = nxt
            off //= 2
        win = cand[0][1]
        out.append(win)
        live[win % 32][win // 32] = False
    return out


@pytest.mark.parametrize("E,ep", [(8, 32), (33, 64), (64, 64), (200, 256)])
def test_warp_argmax_rule_matches_oracle_selection(E, ep):
    rng = np.random.default_rng(E + 1)
    T = 150
    logits = np.round(rng.normal(size=(T, E)) * 2).astype(np.float32) / 2
    logits[:5] = 0.25
    logits[5, ::2] = -0.0
    k = min(8, E)
    idx, _ = oracle.topk(logits, k)
    for t in range(T):
        assert warp_argmax_topk(logits[t], k, ep) == idx[t].tolist(), t
