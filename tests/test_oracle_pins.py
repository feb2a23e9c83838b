"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each pin is chosen so that a plausible slip in the oracle (a transposed
operand, a dropped bias, a wrong tie-break, an off-by-one slot, a wrong sign in
silu, a missing gate weight, a renormalisation after drops) fails at least one
test here:
  * closed forms and special cases that reduce to a library routine
    (numpy matmul, scipy's softmax / expit, Python's sort);
  * brute force on tiny inputs (every token through every expert, then masked
    to its kept top-k pairs; slots counted by an O(T^2) scan);
  * invariants the pages fix (bucket counts, capacity, inverse permutation);
  * hand-derived cases in tests/golden/.
"""
import math
import os

import numpy as np
import pytest
from scipy.special import expit, softmax

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng_seed = 1234


def bf16_round(a):
    """Round fp32 values to bf16 bit patterns (round to nearest even)."""
    a = np.asarray(a, np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def rand_layer(T, d, E, f, seed, bias=False):
    r = np.random.default_rng(seed)
    x = bf16_round(r.standard_normal((T, d)))
    wr = (r.standard_normal((d, E)) / math.sqrt(d)).astype(np.float32)
    b = (r.standard_normal(E) * 0.5).astype(np.float32) if bias else None
    wg = bf16_round(r.standard_normal((E, d, f)) / math.sqrt(d))
    wu = bf16_round(r.standard_normal((E, d, f)) / math.sqrt(d))
    wd = bf16_round(r.standard_normal((E, f, d)) / math.sqrt(f))
    return x, wr, b, wg, wu, wd


# ----------------------------------------------------------------------------- capacity

@pytest.mark.parametrize("T,E,k,cf,C", [
    (64, 8, 2, 1.25, 20),          # tiny workload
    (8192, 256, 8, 1.25, 320),     # fine-grained workload
    (16384, 64, 6, 1.0, 1536),     # skewed workload
    (10, 3, 1, 1.0, 4),            # ceil of 3.33
    (10, 4, 2, 1.25, 7),           # ceil of 6.25
    (12, 4, 1, 1.0, 3),            # exact integer stays put
    (4096, 8, 2, 0.0, 4096),       # cf = 0: dropless, C = T
])
def test_capacity_formula(T, E, k, cf, C):
    assert oracle.capacity(T, E, k, cf) == C


# ----------------------------------------------------------------------------- router

def test_router_onehot_rows_pick_router_rows():
    d, E = 16, 5
    r = np.random.default_rng(0)
    wr = r.standard_normal((d, E)).astype(np.float32)
    bias = r.standard_normal(E).astype(np.float32)
    x = np.zeros((d, d), np.float32)
    x[np.arange(d), np.arange(d)] = 1.0
    l = oracle.router_logits(bf16_round(x), wr, bias)
    # token i is the unit vector e_i: its logits are row i of Wr plus the bias
    np.testing.assert_array_equal(l, wr.astype(np.float64) + bias.astype(np.float64))
    l0 = oracle.router_logits(bf16_round(x), wr, None)
    np.testing.assert_array_equal(l0, wr.astype(np.float64))


def test_router_two_hot_linear_combination():
    d, E = 32, 7
    r = np.random.default_rng(1)
    wr = r.standard_normal((d, E)).astype(np.float32)
    x = np.zeros((3, d), np.float32)
    x[0, 3], x[0, 17] = 2.0, -0.5
    x[1, :] = 1.0
    x[2, 31] = 0.25
    l = oracle.router_logits(bf16_round(x), wr)
    w64 = wr.astype(np.float64)
    np.testing.assert_allclose(l[0], 2.0 * w64[3] - 0.5 * w64[17], rtol=0, atol=1e-15)
    np.testing.assert_allclose(l[1], w64.sum(axis=0), rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(l[2], 0.25 * w64[31], rtol=0, atol=0)


def test_router_matches_library_matmul():
    x, wr, b, *_ = rand_layer(9, 40, 6, 8, seed=2, bias=True)
    l = oracle.router_logits(x, wr, b)
    ref = oracle.bits_to_f64(x) @ wr.astype(np.float64) + b.astype(np.float64)
    np.testing.assert_allclose(l, ref, rtol=1e-13, atol=1e-13)


# ----------------------------------------------------------------------------- top-k gating

def brute_topk(l32, k):
    T, E = l32.shape
    idx = np.empty((T, k), np.int32)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(l32[t, e]), e))
        idx[t] = order[:k]
    return idx


@pytest.mark.parametrize("E,k", [(8, 2), (64, 6), (256, 8), (5, 5), (3, 1)])
def test_topk_matches_full_sort(E, k):
    r = np.random.default_rng(E * 10 + k)
    l = r.standard_normal((50, E)).astype(np.float32)
    idx, w = oracle.topk(l, k)
    np.testing.assert_array_equal(idx, brute_topk(l, k))
    sel = np.take_along_axis(l.astype(np.float64), idx.astype(np.int64), axis=1)
    np.testing.assert_allclose(w, softmax(sel, axis=1), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    assert np.all(np.diff(w, axis=1) <= 0)  # descending weight order


def test_topk_ties_go_to_lower_index():
    # logits quantised to a few levels: many exact ties
    r = np.random.default_rng(7)
    l = r.integers(0, 3, size=(200, 16)).astype(np.float32)
    idx, w = oracle.topk(l, 4)
    np.testing.assert_array_equal(idx, brute_topk(l, 4))
    # a fully tied row selects experts 0..k-1 with equal weights
    idx1, w1 = oracle.topk(np.zeros((1, 10), np.float32), 3)
    assert idx1.tolist() == [[0, 1, 2]]
    np.testing.assert_allclose(w1, 1.0 / 3.0, rtol=1e-15)


def test_topk_k_equals_E_is_full_softmax():
    r = np.random.default_rng(3)
    l = (r.standard_normal((20, 6)) * 4).astype(np.float32)
    idx, w = oracle.topk(l, 6)
    full = softmax(l.astype(np.float64), axis=1)
    np.testing.assert_allclose(w, np.take_along_axis(full, idx.astype(np.int64), 1), rtol=1e-13)


def test_topk_large_logits_no_overflow():
    l = np.array([[1000.0, 999.0, -1000.0, 998.0]], np.float32)
    idx, w = oracle.topk(l, 2)
    assert idx.tolist() == [[0, 1]]
    np.testing.assert_allclose(w[0], [1 / (1 + math.exp(-1)), math.exp(-1) / (1 + math.exp(-1))])


# ----------------------------------------------------------------------------- permutation

def brute_permute(idx, E, C):
    """Slot of pair (t, j) = number of earlier tokens that also chose expert
    idx[t, j] (an O(T^2) count straight from the definition)."""
    T, k = idx.shape
    slot = np.empty((T, k), np.int32)
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            s = sum(1 for tp in range(t) if e in idx[tp])
            slot[t, j] = s if s < C else -1
    demand = np.bincount(idx.ravel(), minlength=E)
    counts = np.minimum(demand, C)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    return slot, counts.astype(np.int32), offsets, int((demand - counts).sum())


def random_routing(T, E, k, seed):
    r = np.random.default_rng(seed)
    # skewed popularity so that capacity bites
    p = 1.0 / np.arange(1, E + 1) ** 1.2
    p /= p.sum()
    idx = np.empty((T, k), np.int32)
    for t in range(T):
        idx[t] = r.choice(E, size=k, replace=False, p=p)
    return idx


@pytest.mark.parametrize("T,E,k,cf", [(64, 8, 2, 1.25), (40, 6, 3, 1.0), (33, 5, 2, 0.5),
                                      (50, 8, 2, 0.0), (20, 4, 4, 1.0), (1, 3, 2, 1.0)])
def test_permute_matches_bruteforce(T, E, k, cf):
    idx = random_routing(T, E, k, seed=T + E)
    C = oracle.capacity(T, E, k, cf)
    counts, offsets, slot, row_src, n_drop = oracle.permute(idx, E, C)
    bslot, bcounts, boffsets, bdrop = brute_permute(idx, E, C)
    np.testing.assert_array_equal(slot, bslot)
    np.testing.assert_array_equal(counts, bcounts)
    np.testing.assert_array_equal(offsets, boffsets)
    assert n_drop == bdrop
    # invariants: sum of bucket counts = kT - drops, buckets never exceed C,
    # and every kept pair appears exactly once in row_src
    assert counts.sum() == k * T - n_drop
    assert counts.max(initial=0) <= C
    kept = [(offsets[idx[t, j]] + slot[t, j], t) for t in range(T) for j in range(k)
            if slot[t, j] >= 0]
    rows = sorted(r for r, _ in kept)
    assert rows == list(range(offsets[E]))
    for r, t in kept:
        assert row_src[r] == t


def _read_golden(path):
    cases, cur = [], None
    with open(path) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, val = line.partition(" ")
            if key == "case":
                cur = {}
            elif key == "end":
                cases.append(cur)
            else:
                cur[key] = val
    return cases


def _rows(s):
    return np.array([[int(v) for v in r.split()] for r in s.split(";")], np.int32)


def _ints(s):
    return np.array([int(v) for v in s.split()], np.int32)


@pytest.mark.parametrize("case", _read_golden(os.path.join(GOLDEN, "permute_hand_cases.txt")))
def test_permute_hand_cases(case):
    T, E, k, cf = int(case["T"]), int(case["E"]), int(case["k"]), float(case["cf"])
    idx = _rows(case["topk"])
    assert idx.shape == (T, k)
    C = oracle.capacity(T, E, k, cf)
    assert C == int(case["C"])
    counts, offsets, slot, row_src, n_drop = oracle.permute(idx, E, C)
    np.testing.assert_array_equal(slot, _rows(case["slot"]))
    np.testing.assert_array_equal(counts, _ints(case["counts"]))
    np.testing.assert_array_equal(offsets, _ints(case["offsets"]))
    np.testing.assert_array_equal(row_src, _ints(case["row_src"]))
    assert n_drop == int(case["n_dropped"])


def test_dispatch_is_pure_copy():
    x, *_ = rand_layer(30, 24, 4, 8, seed=5)
    idx = random_routing(30, 4, 2, seed=5)
    C = oracle.capacity(30, 4, 2, 1.0)
    _, offsets, _, row_src, _ = oracle.permute(idx, 4, C)
    xp = oracle.dispatch(x, row_src)
    np.testing.assert_array_equal(xp, x[row_src])


# ----------------------------------------------------------------------------- expert MLP

def test_swiglu_closed_form_unit_rows():
    # x = e_i, Wd = identity (f = d): o_j = silu(Wg[i,j]) * Wu[i,j]
    d = f = 16
    r = np.random.default_rng(11)
    wg = bf16_round(r.standard_normal((d, f)) * 3)
    wu = bf16_round(r.standard_normal((d, f)))
    wd = bf16_round(np.eye(f))
    x = bf16_round(np.eye(d))
    h, o = oracle.swiglu_rows(x, wg, wu, wd, want_h=True, h_bf16=False)
    g, u = oracle.bits_to_f64(wg), oracle.bits_to_f64(wu)
    ref = g * expit(g) * u
    np.testing.assert_allclose(h, ref, rtol=1e-14, atol=1e-300)
    np.testing.assert_allclose(o, ref, rtol=1e-14, atol=1e-300)
    # with bf16 h (the GEMM operand precision) both outputs are the rounded value
    hr, orr = oracle.swiglu_rows(x, wg, wu, wd, want_h=True, h_bf16=True)
    np.testing.assert_array_equal(hr, np_round_bf16(h))
    np.testing.assert_array_equal(orr, np_round_bf16(h))


def np_round_bf16(a):
    """Nearest bf16 of fp64 values by bit manipulation (keep 7 of the 52
    stored mantissa bits, ties to even) — a different method from the
    oracle's frexp / nearbyint rounding."""
    a = np.ascontiguousarray(a, np.float64)
    b = a.view(np.uint64)
    drop = np.uint64(45)
    lsb = (b >> drop) & np.uint64(1)
    b = (b + (np.uint64(1) << np.uint64(44)) - np.uint64(1) + lsb) & ~((np.uint64(1) << drop)
                                                                     - np.uint64(1))
    return b.view(np.float64)


def np_swiglu(x64, wg64, wu64, wd64, h_bf16=False):
    g = x64 @ wg64
    u = x64 @ wu64
    h = g * expit(g) * u
    if h_bf16:
        h = np_round_bf16(h)
    return h @ wd64


def test_round_bf16_matches_library_conversion():
    import torch
    r = np.random.default_rng(31)
    v = (r.standard_normal(4000) * np.exp(r.uniform(-20, 20, 4000))).astype(np.float32)
    # exact ties: bf16 values plus half an ulp
    base = torch.from_numpy(v[:500]).to(torch.bfloat16).float().numpy()
    half_ulp = np.ldexp(np.ones_like(base), np.frexp(base)[1] - 9)
    ties = (base + np.sign(base) * half_ulp).astype(np.float32)
    v = np.concatenate([v, ties, -ties, np.float32([1.0, -1.0, 3.0, 1e-3])])
    want = torch.from_numpy(v).to(torch.bfloat16).double().numpy()
    got = np.array([oracle.round_bf16(float(a)) for a in v])
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(np_round_bf16(v.astype(np.float64)), want)


def test_single_expert_is_dense_swiglu_mlp():
    # E = 1, k = 1, dropless: the layer is one dense SwiGLU MLP (gate weight 1)
    T, d, f = 12, 32, 48
    x, wr, b, wg, wu, wd = rand_layer(T, d, 1, f, seed=12)
    for h_bf16 in (False, True):
        out = oracle.moe_forward(x, wr, b, wg, wu, wd, k=1, cf=0.0, h_bf16=h_bf16)
        ref = np_swiglu(oracle.bits_to_f64(x), *(oracle.bits_to_f64(a[0]) for a in (wg, wu, wd)),
                        h_bf16=h_bf16)
        np.testing.assert_allclose(out["y"], ref, rtol=1e-12, atol=1e-12)
    assert out["topk_idx"].ravel().tolist() == [0] * T
    np.testing.assert_array_equal(out["topk_w"], 1.0)


def dense_bruteforce(x, wr, b, wg, wu, wd, k, cf, h_bf16):
    """Every token through every expert, then masked to its kept top-k pairs.
    Routing by full sort, slots by the O(T^2) count."""
    T = x.shape[0]
    E = wg.shape[0]
    x64 = oracle.bits_to_f64(x)
    l64 = x64 @ wr.astype(np.float64) + (0 if b is None else b.astype(np.float64))
    l32 = l64.astype(np.float32)
    idx = brute_topk(l32, k)
    sel = np.take_along_axis(l32.astype(np.float64), idx.astype(np.int64), 1)
    w = softmax(sel, axis=1)
    C = T if cf == 0 else math.ceil(cf * k * T / E)
    slot, _, _, _ = brute_permute(idx, E, C)
    all_out = np.stack([np_swiglu(x64, *(oracle.bits_to_f64(a[e]) for a in (wg, wu, wd)),
                                  h_bf16=h_bf16) for e in range(E)])  # [E, T, d]
    y = np.zeros_like(x64)
    for t in range(T):
        kept = [j for j in range(k) if slot[t, j] >= 0]
        if not kept:
            y[t] = x64[t]
        for j in kept:
            y[t] += w[t, j] * all_out[idx[t, j], t]
    return y, idx, w, slot


@pytest.mark.parametrize("h_bf16", [False, True])
@pytest.mark.parametrize("T,d,E,k,f,cf,bias", [
    (64, 32, 8, 2, 48, 1.25, False),
    (48, 16, 6, 3, 32, 0.5, True),     # heavy dropping, some tokens fully dropped
    (30, 24, 4, 2, 16, 0.0, False),    # dropless
    (20, 16, 5, 5, 8, 0.0, True),      # k = E
])
def test_layer_matches_dense_bruteforce(T, d, E, k, f, cf, bias, h_bf16):
    x, wr, b, wg, wu, wd = rand_layer(T, d, E, f, seed=T * d + E, bias=bias)
    out = oracle.moe_forward(x, wr, b, wg, wu, wd, k=k, cf=cf, h_bf16=h_bf16)
    y, idx, w, slot = dense_bruteforce(x, wr, b, wg, wu, wd, k, cf, h_bf16)
    np.testing.assert_array_equal(out["topk_idx"], idx)
    np.testing.assert_array_equal(out["slot"], slot)
    np.testing.assert_allclose(out["topk_w"], w, rtol=1e-13, atol=1e-15)
    scale = np.sqrt(np.mean(y ** 2))
    np.testing.assert_allclose(out["y"], y, rtol=1e-12, atol=1e-12 * scale)


def test_k_equals_E_dropless_is_softmax_mixture():
    T, d, E, f = 10, 16, 4, 24
    x, wr, b, wg, wu, wd = rand_layer(T, d, E, f, seed=99, bias=True)
    out = oracle.moe_forward(x, wr, b, wg, wu, wd, k=E, cf=0.0, h_bf16=False)
    x64 = oracle.bits_to_f64(x)
    l = (x64 @ wr.astype(np.float64) + b).astype(np.float32).astype(np.float64)
    p = softmax(l, axis=1)
    ref = sum(p[:, e:e + 1] * np_swiglu(x64, *(oracle.bits_to_f64(a[e]) for a in (wg, wu, wd)))
              for e in range(E))
    np.testing.assert_allclose(out["y"], ref, rtol=1e-12, atol=1e-13)


def test_large_cf_equals_dropless():
    T, d, E, k, f = 40, 16, 4, 2, 16
    x, wr, b, wg, wu, wd = rand_layer(T, d, E, f, seed=5)
    a = oracle.moe_forward(x, wr, b, wg, wu, wd, k=k, cf=100.0)
    z = oracle.moe_forward(x, wr, b, wg, wu, wd, k=k, cf=0.0)
    assert a["n_dropped"] == 0 and z["n_dropped"] == 0
    np.testing.assert_array_equal(a["y"], z["y"])


# ----------------------------------------------------------------------------- combine

def test_combine_inverts_dispatch_with_identity_expert():
    # identity expert: y_perm = x_perm.  Dropless -> y = x (weights sum to 1);
    # with drops -> y[t] = (sum of kept weights) * x[t]; all dropped -> x[t].
    T, d, E, k = 60, 24, 6, 3
    x, wr, b, *_ = rand_layer(T, d, E, 8, seed=21)
    l32 = oracle.router_logits(x, wr).astype(np.float32)
    idx, w = oracle.topk(l32, k)
    x64 = oracle.bits_to_f64(x)
    for cf in (0.0, 0.5):
        C = oracle.capacity(T, E, k, cf)
        counts, offsets, slot, row_src, n_drop = oracle.permute(idx, E, C)
        y_perm = oracle.bits_to_f64(oracle.dispatch(x, row_src))
        y = oracle.combine(y_perm, x, idx, w, slot, offsets)
        kept_w = np.where(slot >= 0, w, 0.0).sum(axis=1)
        none_kept = (slot < 0).all(axis=1)
        expect = np.where(none_kept[:, None], x64, kept_w[:, None] * x64)
        np.testing.assert_allclose(y, expect, rtol=1e-14, atol=1e-14)
        if cf == 0.0:
            np.testing.assert_allclose(y, x64, rtol=1e-14, atol=1e-14)
        else:
            assert n_drop > 0 and none_kept.any() and (~none_kept).any()


@pytest.mark.parametrize("T,E,k,cf", [(40, 4, 2, 0.75), (64, 8, 2, 1.25), (10, 3, 3, 0.0)])
def test_dispatch_padded_bruteforce(T, E, k, cf):
    """The padded buffer from its definition: bucket e at rows e*C.., token
    rows at their slots, zero elsewhere; the kept rows are the ragged rows."""
    r = np.random.default_rng(T + E)
    x = r.integers(0, 1 << 16, size=(T, 6), dtype=np.uint16)
    idx = np.argsort(r.random((T, E)), axis=1)[:, :k].astype(np.int32)
    C = oracle.capacity(T, E, k, cf)
    counts, offsets, slot, row_src, _ = oracle.permute(idx, E, C)
    pad, src = oracle.dispatch_padded(x, idx, slot, E, C)
    want = np.zeros((E * C, 6), np.uint16)
    want_src = np.full(E * C, -1, np.int32)
    for e in range(E):
        n = 0
        for t in range(T):
            if e in idx[t]:
                if n < C:
                    want[e * C + n] = x[t]
                    want_src[e * C + n] = t
                n += 1
    np.testing.assert_array_equal(pad, want)
    np.testing.assert_array_equal(src, want_src)
    ragged = oracle.dispatch(x, row_src)
    for e in range(E):
        np.testing.assert_array_equal(pad[e * C:e * C + counts[e]],
                                      ragged[offsets[e]:offsets[e + 1]])
