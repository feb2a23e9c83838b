"""Pins for the oracle's FP8 (e4m3) weight quantization, against things other
than the oracle itself:
  * every e4m3 code decoded, and every value encoded, against PyTorch's own
    float8_e4m3fn conversion (round to nearest even);
  * ties between neighbouring codes resolved to the even code, by hand;
  * saturation at +-448 (the largest finite e4m3 value) and the subnormal step
    2^-9, by hand;
  * per-column scales equal to the fp32 max magnitude over 448, the column
    maximum mapping to the code of 448, and the dequantized weight within half
    an e4m3 step of the original;
  * the fp64-weight SwiGLU expert equal to the bf16-weight expert on weights
    that are exactly bf16, and to a numpy brute force on a tiny case;
  * row quantization of activations: scales from numpy's fp32 arithmetic and
    codes from PyTorch's conversion, as for the weight columns; the fp64
    gate/up and matmul steps against numpy / scipy on small cases.
"""
import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle

NAN_CODES = (0x7F, 0xFF)


def torch_e4m3_codes(v):
    t = torch.from_numpy(np.asarray(v, np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def finite_codes():
    return [c for c in range(256) if c not in NAN_CODES]


def test_decode_every_code_matches_library_type():
    codes = np.array(finite_codes(), np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_decode(int(c)) for c in codes])
    np.testing.assert_array_equal(got, ref)
    assert oracle.e4m3_decode(0x7E) == 448.0 and oracle.e4m3_decode(0x01) == 2.0 ** -9
    assert oracle.e4m3_decode(0x08) == 2.0 ** -6 and oracle.e4m3_decode(0x38) == 1.0


def test_encode_roundtrips_every_code():
    for c in finite_codes():
        v = oracle.e4m3_decode(c)
        want = c if v != 0.0 else (0x80 if c == 0x80 else 0x00)
        assert oracle.e4m3_encode(np.float32(v) if c != 0x80 else -0.0) == want, hex(c)


def test_encode_ties_go_to_even_code():
    pos = sorted({oracle.e4m3_decode(c) for c in range(0x00, 0x7F)})
    for lo, hi in zip(pos[:-1], pos[1:]):
        mid = np.float32((lo + hi) / 2)
        assert float(mid) == (lo + hi) / 2          # exactly representable in fp32
        c_lo, c_hi = oracle.e4m3_encode(lo), oracle.e4m3_encode(hi)
        even = c_lo if c_lo % 2 == 0 else c_hi
        assert oracle.e4m3_encode(mid) == even, (lo, hi)
        assert oracle.e4m3_encode(-mid) == even | 0x80


def test_encode_hand_cases():
    assert oracle.e4m3_encode(1.0) == 0x38
    assert oracle.e4m3_encode(-1.5) == 0xBC
    assert oracle.e4m3_encode(1.0625) == 0x38         # half a step above 1: tie -> even
    assert oracle.e4m3_encode(1.1875) == 0x3A         # tie between 1.125 and 1.25 -> 1.25
    assert oracle.e4m3_encode(2.0 ** -9) == 0x01
    assert oracle.e4m3_encode(2.0 ** -10) == 0x00     # tie between 0 and 2^-9 -> 0
    assert oracle.e4m3_encode(3 * 2.0 ** -10) == 0x02
    assert oracle.e4m3_encode(15.5 * 2.0 ** -10) == 0x08   # rounds up into the normals
    for big in (448.0, 449.0, 463.9, 500.0, 1e6, float("inf")):
        assert oracle.e4m3_encode(big) == 0x7E and oracle.e4m3_encode(-big) == 0xFE


def test_encode_matches_library_on_random_values():
    r = np.random.default_rng(7)
    mag = np.exp2(r.uniform(-13, np.log2(448.0), 20000)).astype(np.float32)
    v = np.where(r.random(mag.size) < 0.5, -mag, mag).astype(np.float32)
    got = np.array([oracle.e4m3_encode(x) for x in v], np.uint8)
    np.testing.assert_array_equal(got, torch_e4m3_codes(v))


def bf16_weights(E, K, N, seed):
    g = torch.Generator().manual_seed(seed)
    w = (torch.randn(E, K, N, generator=g) * 0.05).to(torch.bfloat16)
    w[0, :, 3] = 0                      # an all-zero column
    w[1, :, 5] = 0
    w[1, 7, 5] = -0.75                  # a column with one nonzero
    w[2, :, 0] = 2.0 ** -120            # tiny values: scale far below 1
    return w


def test_quantize_scales_codes_and_error_bound():
    E, K, N = 3, 64, 40
    w = bf16_weights(E, K, N, 3)
    q, s = oracle.quantize_fp8(oracle.bf16_bits(w))
    wf = w.float().numpy()
    mx = np.abs(wf).max(axis=1)                                       # [E, N], fp32
    want_s = np.where(mx > 0, mx / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    np.testing.assert_array_equal(s, want_s)
    assert s[0, 3] == 1.0 and np.all(q[0, :, 3] == 0)
    assert q[1, 7, 5] == 0xFE and np.all(np.delete(q[1, :, 5], 7) == 0)
    # the codes are the library's e4m3 conversion of the fp32 quotient
    quot = (wf / s[:, None, :]).astype(np.float32)
    np.testing.assert_array_equal(q, torch_e4m3_codes(quot))
    # each column's largest magnitude maps to the code of 448
    amax = np.abs(wf).argmax(axis=1)
    for e in range(E):
        for n in range(N):
            if mx[e, n] > 0:
                assert q[e, amax[e, n], n] & 0x7F == 0x7E
    # dequantized within half a step: 2^-4 relative (3 mantissa bits), or half
    # the subnormal spacing 2^-9 times the scale
    deq = oracle.dequant_fp8(q, s)
    bound = 2.0 ** -4 * np.abs(wf) * (1 + 2.0 ** -20) + 2.0 ** -10 * s[:, None, :]
    assert np.all(np.abs(deq - wf) <= bound)
    np.testing.assert_array_equal(
        deq, np.vectorize(oracle.e4m3_decode)(q) * s[:, None, :].astype(np.float64))


def test_swiglu_f64w_equals_bf16_expert_on_bf16_weights():
    g = torch.Generator().manual_seed(5)
    n, d, f = 7, 32, 48
    x = torch.randn(n, d, generator=g).to(torch.bfloat16)
    wg, wu = ((torch.randn(d, f, generator=g) / d ** 0.5).to(torch.bfloat16) for _ in range(2))
    wd = (torch.randn(f, d, generator=g) / f ** 0.5).to(torch.bfloat16)
    b = oracle.bf16_bits
    for h_bf16 in (True, False):
        h1, o1 = oracle.swiglu_rows(b(x), b(wg), b(wu), b(wd), want_h=True, h_bf16=h_bf16)
        h2, o2 = oracle.swiglu_rows_f64w(b(x), *(oracle.bits_to_f64(b(t)) for t in (wg, wu, wd)),
                                         want_h=True, h_bf16=h_bf16)
        np.testing.assert_allclose(h2, h1, rtol=1e-13, atol=1e-15)
        np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-14)


def test_swiglu_f64w_bruteforce():
    r = np.random.default_rng(9)
    n, d, f = 3, 8, 16
    x = torch.from_numpy(r.standard_normal((n, d)).astype(np.float32)).to(torch.bfloat16)
    wg, wu, wd = r.standard_normal((d, f)), r.standard_normal((d, f)), r.standard_normal((f, d))
    xb = oracle.bf16_bits(x)
    h, o = oracle.swiglu_rows_f64w(xb, wg, wu, wd, want_h=True, h_bf16=False)
    x64 = oracle.bits_to_f64(xb)
    for i in range(n):
        for j in range(f):
            gj = sum(x64[i, c] * wg[c, j] for c in range(d))
            uj = sum(x64[i, c] * wu[c, j] for c in range(d))
            assert h[i, j] == pytest.approx(gj * expit(gj) * uj, rel=1e-12, abs=1e-12)
        for c in range(d):
            assert o[i, c] == pytest.approx(sum(h[i, j] * wd[j, c] for j in range(f)),
                                            rel=1e-12, abs=1e-12)


def test_quantize_rows_scales_and_codes():
    g = torch.Generator().manual_seed(11)
    x = (torch.randn(37, 96, generator=g) * 3).to(torch.bfloat16)
    x[4] = 0                                        # all-zero row: scale 1, codes 0
    x[9, :] = 0
    x[9, 50] = 1e-30                                # tiny row: subnormal fp32 scale
    x[20, 3] = -2e5                                 # one large value: the rest small codes
    q, s = oracle.quantize_rows_fp8(oracle.bf16_bits(x))
    xf = x.float().numpy()
    mx = np.abs(xf).max(axis=1)
    want_s = np.where(mx > 0, mx / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    np.testing.assert_array_equal(s, want_s)
    np.testing.assert_array_equal(q, torch_e4m3_codes((xf / s[:, None]).astype(np.float32)))
    assert np.all(q[4] == 0) and q[20, 3] == 0xFE
    deq = oracle.dequant_rows_fp8(q, s)
    np.testing.assert_array_equal(
        deq, np.vectorize(oracle.e4m3_decode)(q) * s[:, None].astype(np.float64))
    bound = 2.0 ** -4 * np.abs(xf) * (1 + 2.0 ** -20) + 2.0 ** -10 * s[:, None]
    assert np.all(np.abs(deq - xf) <= bound)


def test_gate_up_f64_and_matmul_bruteforce():
    r = np.random.default_rng(13)
    n, d, f = 4, 12, 10
    a, wg, wu = r.standard_normal((n, d)), r.standard_normal((d, f)), r.standard_normal((d, f))
    h = oracle.gate_up_f64(a, wg, wu, h_bf16=False)
    g, u = a @ wg, a @ wu
    np.testing.assert_allclose(h, g * expit(g) * u, rtol=1e-12, atol=1e-12)
    hb = oracle.gate_up_f64(a, wg, wu, h_bf16=True)
    np.testing.assert_array_equal(hb, np.vectorize(oracle.round_bf16)(h))
    w = r.standard_normal((f, 7))
    np.testing.assert_allclose(oracle.matmul_f64(h, w), h @ w, rtol=1e-12, atol=1e-12)


def test_gate_up_f64_equals_bf16_expert():
    g = torch.Generator().manual_seed(17)
    n, d, f = 5, 32, 24
    x = torch.randn(n, d, generator=g).to(torch.bfloat16)
    wg, wu = ((torch.randn(d, f, generator=g) / d ** 0.5).to(torch.bfloat16) for _ in range(2))
    wd = (torch.randn(f, d, generator=g) / f ** 0.5).to(torch.bfloat16)
    b = oracle.bf16_bits
    h_ref, o_ref = oracle.swiglu_rows(b(x), b(wg), b(wu), b(wd), want_h=True)
    h = oracle.gate_up_f64(oracle.bits_to_f64(b(x)), oracle.bits_to_f64(b(wg)),
                           oracle.bits_to_f64(b(wu)))
    np.testing.assert_allclose(h, h_ref, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(oracle.matmul_f64(h, oracle.bits_to_f64(b(wd))), o_ref,
                               rtol=1e-12, atol=1e-14)
