"""GPU parity for the FP8 (e4m3) expert-weight variant, through the C ABI,
against the CPU oracle:
  * the weight quantizer: codes and scales bit-exact;
  * the grouped gate/up and down GEMMs on e4m3 weights against the oracle's
    expert evaluated on its own dequantized weights (same tolerances as the
    bf16 path: h within one bf16 rounding, y_perm within 2e-2 rms);
  * the whole layer with e4m3 experts, small workloads element by element and
    the decode-sized workloads on sampled tokens.
The oracle's quantization (codes and scales) is what the GPU GEMMs are fed, so
every expected value comes from the oracle alone.
"""
import numpy as np
import pytest
import torch

import oracle
import mixture_experts_layer_36_b200 as moe
from mixture_experts_layer_36_b200 import configs, synth
from moe_testlib import (WEIGHT_ATOL, assert_bf16_close, assert_bf16_rounding_close,
                         assert_logits_close, bits, cuda_inputs, f64, small)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    torch.cuda.synchronize()


def edge_weights(E, K, N, seed, std):
    g = torch.Generator().manual_seed(seed)
    w = (torch.randn(E, K, N, generator=g) * std).to(torch.bfloat16)
    w[0, :, min(3, N - 1)] = 0                       # all-zero column: scale 1, codes 0
    if E > 1:
        w[1, :, 0] = 0
        w[1, K // 2, 0] = -0.75                      # one nonzero: code 0xFE
        w[E - 1, :, N - 1] = 2.0 ** -120             # fp32-subnormal scale
        w[E - 1, 0, N - 2] = 3e4                     # one huge weight: the rest go subnormal
    return w


def quantize_oracle(w):
    q, s = oracle.quantize_fp8(bits(w))
    return torch.from_numpy(q), torch.from_numpy(s)


def dequant(q, s):
    return oracle.dequant_fp8(q.numpy(), s.numpy())


@pytest.mark.parametrize("E,K,N", [(3, 64, 40), (8, 256, 384), (2, 1000, 129)])
def test_quantizer_bit_exact(E, K, N):
    w = edge_weights(E, K, N, E + K + N, 0.05)
    q, s = moe.moe_quantize_weights_fp8(w.cuda())
    torch.cuda.synchronize()
    q_ref, s_ref = quantize_oracle(w)
    assert torch.equal(s.cpu(), s_ref)       # fp32 bit patterns (no NaN is possible)
    assert torch.equal(q.cpu(), q_ref)


MLP_CASES = [
    # (d, f, bucket sizes): ragged tails, M=64 tail tiles, empty and one-row
    # buckets, several row tiles, both down-GEMM tile widths (d % 256)
    (256, 384, [300, 0, 1, 129, 128, 257]),
    (128, 256, [5, 140, 0, 0, 64, 128]),
    (384, 128, [1, 1, 1, 400]),
    (512, 640, [129] * 3),
    (256, 256, [0, 0, 0]),
    (256, 256, [170, 0, 128, 129, 233, 256, 250, 131]),
]


@pytest.mark.parametrize("d,f,sizes", MLP_CASES)
def test_expert_mlp_fp8_matches_oracle(d, f, sizes):
    E = len(sizes)
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    N = int(offsets[-1])
    max_rows = N + 37
    g = torch.Generator().manual_seed(3 * d + f + E)
    x_perm = torch.randn(max_rows, d, generator=g).to(torch.bfloat16)
    wg = edge_weights(E, d, f, d + 1, d ** -0.5)
    wu = edge_weights(E, d, f, d + 2, d ** -0.5)
    wd = edge_weights(E, f, d, d + 3, f ** -0.5)
    (qg, sg), (qu, su), (qd, sd) = (quantize_oracle(w) for w in (wg, wu, wd))
    sentinel = -7.0
    h = torch.full((max_rows, f), sentinel, dtype=torch.bfloat16, device="cuda")
    y = torch.full((max_rows, d), sentinel, dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    off = torch.from_numpy(offsets).cuda()
    moe.moe_expert_gate_up_fp8(x_perm.cuda(), off, qg.cuda(), sg.cuda(), qu.cuda(), su.cuda(),
                               h=h, dev_status=status)
    moe.moe_expert_down_fp8(h, off, qd.cuda(), sd.cuda(), y_perm=y, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    g64, u64, d64 = dequant(qg, sg), dequant(qu, su), dequant(qd, sd)
    xb = bits(x_perm[:N])
    o_h, o_y = np.zeros((N, f)), np.zeros((N, d))
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        if b > a:
            o_h[a:b], o_y[a:b] = oracle.swiglu_rows_f64w(xb[a:b], g64[e], u64[e], d64[e],
                                                         want_h=True)
    assert_bf16_rounding_close(f64(h[:N]), o_h, "h")
    assert_bf16_close(f64(y[:N]), o_y, "y_perm")
    assert torch.all(h[N:] == sentinel) and torch.all(y[N:] == sentinel)


def oracle_layer_fp8(cpu, k, cf, gl, q):
    """The layer on the oracle's dequantized experts, routed on the GPU's fp32
    logits (the arg-max decision is taken in the kernel's precision)."""
    x_bits = bits(cpu["x"])
    T, d = x_bits.shape
    E = cpu["w_gate"].shape[0]
    o_idx, o_w = oracle.topk(gl, k)
    C = oracle.capacity(T, E, k, cf)
    counts, offsets, slot, row_src, n_drop = oracle.permute(o_idx, E, C)
    x_perm = oracle.dispatch(x_bits, row_src)
    f = cpu["w_gate"].shape[2]
    y_perm = np.zeros((int(offsets[-1]), d))
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        if b > a:
            wg, wu, wd = (oracle.dequant_fp8(q[n][0][e:e + 1].numpy(), q[n][1][e:e + 1].numpy())[0]
                          for n in ("w_gate", "w_up", "w_down"))
            _, y_perm[a:b] = oracle.swiglu_rows_f64w(x_perm[a:b], wg, wu, wd)
    y = oracle.combine(y_perm, x_bits, o_idx, o_w, slot, offsets)
    return dict(topk_idx=o_idx, topk_w=o_w, slot=slot, counts=counts, offsets=offsets,
                n_dropped=n_drop, y=y, f=f)


SMALL = [
    configs.TINY,
    small("mixtral_small", T=512, d=256, E=8, k=2, f=512, cf=0.0, seed=11),
    small("fine_small", T=512, d=256, E=256, k=8, f=256, cf=1.25, seed=12),
    small("decode_small", T=16, d=256, E=256, k=8, f=256, cf=0.0, seed=14),
    small("ragged_T", T=333, d=384, E=6, k=3, f=128, cf=0.5, seed=15),
]


def _ws(ws, name, cfg):
    return moe.workspace_view(ws, name, cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, cfg.cf)


@pytest.mark.parametrize("cfg", SMALL, ids=[c.name for c in SMALL])
def test_layer_forward_fp8_matches_oracle(cfg):
    inp, cpu = cuda_inputs(cfg)
    q = {n: quantize_oracle(cpu[n]) for n in ("w_gate", "w_up", "w_down")}
    qd = {n: (a.cuda(), b.cuda()) for n, (a, b) in q.items()}
    y, ws = moe.moe_layer_forward_fp8(inp["x"], inp["w_router"], inp["bias"], *qd["w_gate"],
                                      *qd["w_up"], *qd["w_down"], cfg.k, cfg.cf)
    torch.cuda.synchronize()
    assert _ws(ws, "status", cfg).item() == 0
    gl = _ws(ws, "logits", cfg).cpu().numpy()
    bias = None if cpu["bias"] is None else cpu["bias"].numpy()
    assert_logits_close(gl, oracle.router_logits(bits(cpu["x"]), cpu["w_router"].numpy(), bias))
    ref = oracle_layer_fp8(cpu, cfg.k, cfg.cf, gl, q)
    np.testing.assert_array_equal(_ws(ws, "topk_idx", cfg).cpu().numpy(), ref["topk_idx"])
    assert np.max(np.abs(_ws(ws, "topk_w", cfg).cpu().double().numpy() - ref["topk_w"])) \
        <= WEIGHT_ATOL
    np.testing.assert_array_equal(_ws(ws, "slot", cfg).cpu().numpy(), ref["slot"])
    np.testing.assert_array_equal(_ws(ws, "offsets", cfg).cpu().numpy(), ref["offsets"])
    assert _ws(ws, "n_dropped", cfg).item() == ref["n_dropped"]
    assert_bf16_close(f64(y), ref["y"], "y")
    dropped = (ref["slot"] < 0).all(axis=1)
    if dropped.any():
        np.testing.assert_array_equal(bits(y)[dropped], bits(cpu["x"])[dropped])


DECODE = [configs.DECODE.with_tokens(t) for t in configs.DECODE_T]


@pytest.mark.parametrize("cfg", DECODE, ids=[c.name for c in DECODE])
def test_decode_fp8_full_size_sampled(cfg):
    """Decode-sized layer with e4m3 experts quantized on the GPU: the
    quantizer bit-exact on the experts the sampled tokens use, routing exact
    for every token, outputs on sampled tokens from the oracle's own
    quantization of those experts."""
    torch.cuda.empty_cache()
    w = synth.make_weights(cfg, "cuda")
    x = synth.make_tokens(cfg, "cuda")
    qw = {n: moe.moe_quantize_weights_fp8(w[n]) for n in ("w_gate", "w_up", "w_down")}
    y, ws = moe.moe_layer_forward_fp8(x, w["w_router"], w["bias"], *qw["w_gate"], *qw["w_up"],
                                      *qw["w_down"], cfg.k, cfg.cf)
    torch.cuda.synchronize()
    assert _ws(ws, "status", cfg).item() == 0
    gl = _ws(ws, "logits", cfg).cpu().numpy()
    o_idx, o_w = oracle.topk(gl, cfg.k)
    np.testing.assert_array_equal(_ws(ws, "topk_idx", cfg).cpu().numpy(), o_idx)
    C = oracle.capacity(cfg.T, cfg.E, cfg.k, cfg.cf)
    _, offsets, slot, _, _ = oracle.permute(o_idx, cfg.E, C)
    np.testing.assert_array_equal(_ws(ws, "slot", cfg).cpu().numpy(), slot)

    rng = np.random.default_rng(cfg.seed + 1)
    toks = np.sort(rng.choice(cfg.T, size=2, replace=False))
    x_bits = bits(x)
    y_ref = np.zeros((len(toks), cfg.d))
    for i, t in enumerate(toks):
        for j in range(cfg.k):
            e = int(o_idx[t, j])
            mats = []
            for n in ("w_gate", "w_up", "w_down"):
                q_ref, s_ref = quantize_oracle(w[n][e:e + 1].cpu())
                assert torch.equal(qw[n][0][e:e + 1].cpu(), q_ref), (n, e)
                assert torch.equal(qw[n][1][e:e + 1].cpu(), s_ref), (n, e)
                mats.append(dequant(q_ref, s_ref)[0])
            _, o = oracle.swiglu_rows_f64w(x_bits[t:t + 1], *mats)
            y_ref[i] += o_w[t, j] * o[0]
    assert_bf16_close(f64(y[torch.from_numpy(toks).cuda().long()]), y_ref, "y (sampled)")
    del w, x, y, ws, qw
    torch.cuda.empty_cache()
