"""GPU parity for the FP8 expert variant (e4m3 activations and weights, fp32
row and column scales), through the C ABI, against the CPU oracle:
  * the weight quantizer and the row quantizer: codes and scales bit-exact
    (the weights come back K-major, the transpose of the oracle's layout);
  * the grouped gate/up and down GEMMs on e4m3 operands against the oracle's
    expert on the dequantized operands: h within one bf16 rounding, y_perm
    within 2e-2 rms (the bf16 path's tolerances);
  * the whole layer, small workloads element by element and the decode-sized
    workloads on sampled tokens.
Where floating point decides a code (the quantization of h), the oracle
quantizes the GPU's own h, after that h has been checked against the oracle's.
"""
import numpy as np
import pytest
import torch

import oracle
import mixture_experts_layer_36_b200 as moe
from mixture_experts_layer_36_b200 import configs, synth
from moe_testlib import (WEIGHT_ATOL, assert_bf16_close, assert_bf16_rounding_close,
                         assert_logits_close, bits, cuda_inputs, every_expert_rows, f64,
                         map_experts, small)

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


def quantize_w(w):
    """Oracle quantization of bf16 weights [E,K,N]: codes [E,K,N], scales [E,N]."""
    q, s = oracle.quantize_fp8(bits(w))
    return q, s


def kmajor(q):
    """Oracle codes [E,K,N] -> the GPU's K-major layout [E,N,K] on the device."""
    return torch.from_numpy(np.ascontiguousarray(q.transpose(0, 2, 1))).cuda()


@pytest.mark.parametrize("E,K,N", [(3, 64, 40), (8, 256, 384), (2, 1000, 129)])
def test_weight_quantizer_bit_exact(E, K, N):
    w = edge_weights(E, K, N, E + K + N, 0.05)
    q, s = moe.moe_quantize_weights_fp8(w.cuda())
    torch.cuda.synchronize()
    q_ref, s_ref = quantize_w(w)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    np.testing.assert_array_equal(q.cpu().numpy().transpose(0, 2, 1), q_ref)


@pytest.mark.parametrize("R,K,n_rows", [(37, 96, None), (300, 256, 211), (9, 7168, None),
                                         (6, 2048, 5), (5, 16384, None), (5, 16400, None),
                                         (7, 2064, None), (7, 8192, 6), (7, 8208, None)])
def test_row_quantizer_bit_exact(R, K, n_rows):
    g = torch.Generator().manual_seed(R + K)
    x = (torch.randn(R, K, generator=g) * 3).to(torch.bfloat16)
    x[1] = 0                                         # all-zero row
    x[2, :] = 0
    x[2, 5] = 1e-30                                  # fp32-subnormal scale
    x[3, 7] = -2e5                                   # the rest of the row: small codes
    x[4, :] = 460.0                                  # saturating quotients
    q = torch.full((R, K), 0x55, dtype=torch.uint8, device="cuda")
    s = torch.full((R,), -1.0, dtype=torch.float32, device="cuda")
    nr = None if n_rows is None else torch.tensor([n_rows], dtype=torch.int32, device="cuda")
    moe.moe_quantize_rows_fp8(x.cuda(), n_rows=nr, q=q, scale=s)
    torch.cuda.synchronize()
    n = R if n_rows is None else n_rows
    q_ref, s_ref = oracle.quantize_rows_fp8(bits(x[:n]))
    np.testing.assert_array_equal(s[:n].cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    np.testing.assert_array_equal(q[:n].cpu().numpy(), q_ref)
    assert torch.all(q[n:] == 0x55) and torch.all(s[n:] == -1.0)   # rows past n_rows untouched


@pytest.mark.parametrize("T,d,E,k,cf", [(333, 384, 6, 3, 0.5), (512, 256, 256, 8, 1.25),
                                        (64, 128, 8, 2, 0.0)])
def test_permute_fp8_matches_oracle(T, d, E, k, cf):
    """Codes and scales of each token, moved by the permutation: equal to the
    oracle's row quantization of its dispatched rows, bit for bit."""
    from moe_testlib import random_routing
    g = torch.Generator().manual_seed(T + E)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16)
    idx = random_routing(T, E, k, seed=T + d)
    xq_tok, sx_tok = moe.moe_quantize_rows_fp8(x.cuda())
    out = moe.moe_permute_fp8(xq_tok, sx_tok, torch.from_numpy(idx).cuda(), E, cf)
    torch.cuda.synchronize()
    C = oracle.capacity(T, E, k, cf)
    counts, offsets, slot, row_src, n_drop = oracle.permute(idx, E, C)
    np.testing.assert_array_equal(out["counts"].cpu().numpy(), counts)
    np.testing.assert_array_equal(out["offsets"].cpu().numpy(), offsets)
    np.testing.assert_array_equal(out["slot"].cpu().numpy(), slot)
    assert out["n_dropped"].item() == n_drop
    N = int(offsets[-1])
    np.testing.assert_array_equal(out["row_src"][:N].cpu().numpy(), row_src)
    xq, sx = oracle.quantize_rows_fp8(oracle.dispatch(bits(x), row_src))
    np.testing.assert_array_equal(out["xq"][:N].cpu().numpy(), xq)
    np.testing.assert_array_equal(out["sx"][:N].cpu().numpy().view(np.uint32), sx.view(np.uint32))


def deq_rows(q, s):
    return oracle.dequant_rows_fp8(q, s)


def run_mlp(xq, sx, offsets, qg, sg, qu, su, qd, sd, max_rows, d, f):
    """GPU: gate/up on (xq, sx), the row quantizer on h, down.  Inputs numpy
    (weights in the oracle's [E,K,N] layout).  Returns (h, hq, sh, y) on the host."""
    N = int(offsets[-1])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    off = torch.from_numpy(offsets).cuda()
    xq_d = torch.zeros(max_rows, d, dtype=torch.uint8, device="cuda")
    sx_d = torch.zeros(max_rows, dtype=torch.float32, device="cuda")
    xq_d[:N] = torch.from_numpy(xq).cuda()
    sx_d[:N] = torch.from_numpy(sx).cuda()
    sentinel = -7.0
    h = torch.full((max_rows, f), sentinel, dtype=torch.bfloat16, device="cuda")
    y = torch.full((max_rows, d), sentinel, dtype=torch.float32, device="cuda")
    moe.moe_expert_gate_up_fp8(xq_d, sx_d, off, kmajor(qg), torch.from_numpy(sg).cuda(),
                               kmajor(qu), torch.from_numpy(su).cuda(), h=h, dev_status=status)
    hq, sh = moe.moe_quantize_rows_fp8(h, n_rows=off[-1:])
    moe.moe_expert_down_fp8(hq, sh, off, kmajor(qd), torch.from_numpy(sd).cuda(), y_perm=y,
                            dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.all(h[N:] == sentinel) and torch.all(y[N:] == sentinel)
    return h[:N], hq[:N].cpu().numpy(), sh[:N].cpu().numpy(), y[:N]


def check_mlp(xq, sx, offsets, qg, sg, qu, su, qd, sd, h, hq, sh, y):
    """Oracle check of one GPU expert-MLP pass (see run_mlp)."""
    N, f = h.shape
    d = y.shape[1]
    E = len(offsets) - 1
    a = deq_rows(xq, sx)
    g64, u64, d64 = oracle.dequant_fp8(qg, sg), oracle.dequant_fp8(qu, su), \
        oracle.dequant_fp8(qd, sd)
    o_h = np.zeros((N, f))
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            o_h[lo:hi] = oracle.gate_up_f64(a[lo:hi], g64[e], u64[e])
    assert_bf16_rounding_close(f64(h), o_h, "h")
    # the codes of h: the oracle's quantizer on the GPU's h, bit for bit
    hq_ref, sh_ref = oracle.quantize_rows_fp8(bits(h))
    np.testing.assert_array_equal(sh.view(np.uint32), sh_ref.view(np.uint32))
    np.testing.assert_array_equal(hq, hq_ref)
    b = deq_rows(hq_ref, sh_ref)
    o_y = np.zeros((N, d))
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            o_y[lo:hi] = oracle.matmul_f64(b[lo:hi], d64[e])
    assert_bf16_close(f64(y), o_y, "y_perm")


MLP_CASES = [
    # (d, f, bucket sizes, pair): ragged tails, M=64 tail tiles, empty and
    # one-row buckets, several row tiles, both down-GEMM tile widths (d % 256);
    # pair=True gives a buffer of >= 512 rows per expert, which selects the
    # CTA-pair tiles (256 rows, half tiles of 128 at the tails)
    (256, 384, [300, 0, 1, 129, 128, 257], False),
    (128, 256, [5, 140, 0, 0, 64, 128], False),
    (384, 128, [1, 1, 1, 400], False),
    (512, 640, [129] * 3, False),
    (256, 256, [0, 0, 0], False),
    (256, 256, [170, 0, 128, 129, 233, 256, 250, 131], False),
    (256, 384, [300, 0, 1, 129, 128, 257, 700], True),
    (512, 256, [1, 256, 511, 513, 1024], True),
    (384, 256, [255, 257, 0], True),      # down GEMM: d % 256 != 0 keeps single-CTA tiles
    # several CTA-pair tiles per pair; long contractions
    (512, 384, [3000, 2999, 1, 2900], True),
    (256, 1024, [2048] * 4, True),
    (4096, 384, [300, 260, 255, 511, 0, 1], "mid"),
    (768, 8192, [600, 1, 300], True),
    # d, f multiples of 64 only: 64-wide K tails (half k-blocks) and N tails
    (192, 320, [300, 0, 1, 129], False),
    (320, 192, [3000, 1, 2900], True),
]


@pytest.mark.parametrize("d,f,sizes,pair", MLP_CASES)
def test_expert_mlp_fp8_matches_oracle(d, f, sizes, pair):
    E = len(sizes)
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    N = int(offsets[-1])
    g = torch.Generator().manual_seed(3 * d + f + E)
    x_perm = torch.randn(N, d, generator=g).to(torch.bfloat16)
    xq, sx = oracle.quantize_rows_fp8(bits(x_perm))
    qg, sg = quantize_w(edge_weights(E, d, f, d + 1, d ** -0.5))
    qu, su = quantize_w(edge_weights(E, d, f, d + 2, d ** -0.5))
    qd, sd = quantize_w(edge_weights(E, f, d, d + 3, f ** -0.5))
    if pair == "mid":
        max_rows = max(N + 37, 256 * E + 5)
    else:
        max_rows = max(N + 37, 512 * E + 5) if pair else N + 37
    out = run_mlp(xq, sx, offsets, qg, sg, qu, su, qd, sd, max_rows, d, f)
    check_mlp(xq, sx, offsets, qg, sg, qu, su, qd, sd, *out)


def random_codes(shape, rng):
    """Every finite e4m3 code, drawn uniformly (zero and subnormals included)."""
    q = rng.integers(0, 256, size=shape, dtype=np.uint8)
    q[(q & 0x7F) == 0x7F] -= 1                       # no NaN codes
    return q


def test_expert_mlp_fp8_every_code():
    d, f, sizes = 256, 384, [70, 0, 129, 1]
    E = len(sizes)
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    N = int(offsets[-1])
    rng = np.random.default_rng(31)
    xq = random_codes((N, d), rng)
    sx = rng.uniform(0.5, 2, N).astype(np.float32) / 64
    qg, qu, qd = random_codes((E, d, f), rng), random_codes((E, d, f), rng), \
        random_codes((E, f, d), rng)
    sg, su = (rng.uniform(0.5, 2, (E, f)).astype(np.float32) / (64 * d ** 0.5) for _ in range(2))
    sd = rng.uniform(0.5, 2, (E, d)).astype(np.float32) / (64 * f ** 0.5)
    assert ((qg & 0x78) == 0).any() and (qg == 0).any() and ((xq & 0x78) == 0).any()
    out = run_mlp(xq, sx, offsets, qg, sg, qu, su, qd, sd, N + 5, d, f)
    check_mlp(xq, sx, offsets, qg, sg, qu, su, qd, sd, *out)


SMALL = [
    configs.TINY,
    small("mixtral_small", T=512, d=256, E=8, k=2, f=512, cf=0.0, seed=11),
    small("fine_small", T=512, d=256, E=256, k=8, f=256, cf=1.25, seed=12),
    small("decode_small", T=16, d=256, E=256, k=8, f=256, cf=0.0, seed=14),
    small("ragged_T", T=333, d=384, E=6, k=3, f=128, cf=0.5, seed=15),
    small("pair_tiles", T=2048, d=256, E=4, k=2, f=256, cf=0.0, seed=19),
    small("pair_tiles_drops", T=3000, d=512, E=4, k=3, f=384, cf=0.8, seed=20),
    small("width64", T=300, d=192, E=8, k=2, f=320, cf=1.25, seed=23),
]


def _ws(ws, name, cfg):
    return moe.workspace_view(ws, name, cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, cfg.cf)


def gpu_quantized_weights(w, names=("w_gate", "w_up", "w_down")):
    return {n: moe.moe_quantize_weights_fp8(w[n]) for n in names}


@pytest.mark.parametrize("cfg", SMALL, ids=[c.name for c in SMALL])
def test_layer_forward_fp8_matches_oracle(cfg):
    inp, cpu = cuda_inputs(cfg)
    qw = gpu_quantized_weights(inp)
    y, ws = moe.moe_layer_forward_fp8(inp["x"], inp["w_router"], inp["bias"], *qw["w_gate"],
                                      *qw["w_up"], *qw["w_down"], cfg.k, cfg.cf)
    torch.cuda.synchronize()
    assert _ws(ws, "status", cfg).item() == 0
    gl = _ws(ws, "logits", cfg).cpu().numpy()
    bias = None if cpu["bias"] is None else cpu["bias"].numpy()
    x_bits = bits(cpu["x"])
    assert_logits_close(gl, oracle.router_logits(x_bits, cpu["w_router"].numpy(), bias))
    o_idx, o_w = oracle.topk(gl, cfg.k)
    C = oracle.capacity(cfg.T, cfg.E, cfg.k, cfg.cf)
    counts, offsets, slot, row_src, n_drop = oracle.permute(o_idx, cfg.E, C)
    np.testing.assert_array_equal(_ws(ws, "topk_idx", cfg).cpu().numpy(), o_idx)
    assert np.max(np.abs(_ws(ws, "topk_w", cfg).cpu().double().numpy() - o_w)) <= WEIGHT_ATOL
    np.testing.assert_array_equal(_ws(ws, "slot", cfg).cpu().numpy(), slot)
    np.testing.assert_array_equal(_ws(ws, "offsets", cfg).cpu().numpy(), offsets)
    assert _ws(ws, "n_dropped", cfg).item() == n_drop
    N = int(offsets[-1])
    # the weights' and x_perm's codes
    q = {n: quantize_w(cpu[n]) for n in ("w_gate", "w_up", "w_down")}
    for n in q:
        np.testing.assert_array_equal(qw[n][0].cpu().numpy().transpose(0, 2, 1), q[n][0])
    xq, sx = oracle.quantize_rows_fp8(oracle.dispatch(x_bits, row_src))
    np.testing.assert_array_equal(_ws(ws, "xq", cfg)[:N].cpu().numpy(), xq)
    np.testing.assert_array_equal(_ws(ws, "sx", cfg)[:N].cpu().numpy(), sx)
    h = _ws(ws, "h", cfg)[:N]
    hq = _ws(ws, "hq", cfg)[:N].cpu().numpy()
    sh = _ws(ws, "sh", cfg)[:N].cpu().numpy()
    y_perm = _ws(ws, "y_perm", cfg)[:N]
    (qg, sg), (qu, su), (qd, sd) = q["w_gate"], q["w_up"], q["w_down"]
    check_mlp(xq, sx, offsets, qg, sg, qu, su, qd, sd, h, hq, sh, y_perm)
    # the combine on the oracle's y_perm (from the GPU's h codes)
    hq_ref, sh_ref = oracle.quantize_rows_fp8(bits(h))
    b = deq_rows(hq_ref, sh_ref)
    d64 = oracle.dequant_fp8(qd, sd)
    o_y = np.zeros((N, cfg.d))
    for e in range(cfg.E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            o_y[lo:hi] = oracle.matmul_f64(b[lo:hi], d64[e])
    y_ref = oracle.combine(o_y, x_bits, o_idx, o_w, slot, offsets)
    assert_bf16_close(f64(y), y_ref, "y")
    dropped = (slot < 0).all(axis=1)
    if dropped.any():
        np.testing.assert_array_equal(bits(y)[dropped], x_bits[dropped])


FULL = [configs.MIXTRAL, configs.FINE, configs.SKEWED] + \
    [configs.DECODE.with_tokens(t) for t in configs.DECODE_T]


@pytest.mark.parametrize("cfg", FULL, ids=[c.name for c in FULL])
def test_fp8_full_size_sampled(cfg):
    """Full-size layer with FP8 experts quantized on the GPU, in the launch
    configuration the benchmark times: routing and slots exact for every
    token; for every expert that received rows, its weight codes bit-exact
    and two of its rows (the bucket's last, in the tail tile, and one more)
    through both GEMMs against the oracle; for two sampled tokens (and, where
    the capacity drops some, one whose every pair is dropped) the layer
    output from the oracle."""
    torch.cuda.empty_cache()
    w = synth.make_weights(cfg, "cuda")
    x = synth.make_tokens(cfg, "cuda")
    qw = gpu_quantized_weights(w)
    y, ws = moe.moe_layer_forward_fp8(x, w["w_router"], w["bias"], *qw["w_gate"], *qw["w_up"],
                                      *qw["w_down"], cfg.k, cfg.cf)
    torch.cuda.synchronize()
    assert _ws(ws, "status", cfg).item() == 0
    gl = _ws(ws, "logits", cfg).cpu().numpy()
    o_idx, o_w = oracle.topk(gl, cfg.k)
    np.testing.assert_array_equal(_ws(ws, "topk_idx", cfg).cpu().numpy(), o_idx)
    C = oracle.capacity(cfg.T, cfg.E, cfg.k, cfg.cf)
    counts, offsets, slot, row_src, n_drop = oracle.permute(o_idx, cfg.E, C)
    np.testing.assert_array_equal(_ws(ws, "slot", cfg).cpu().numpy(), slot)
    assert _ws(ws, "n_dropped", cfg).item() == n_drop
    x_bits = bits(x)

    # every expert with rows: codes of its weights, then two of its rows
    # through the gate/up GEMM (h) and the down GEMM (y_perm)
    picks = every_expert_rows(offsets, cfg.seed + 3)
    assert len(picks) == int((counts > 0).sum())
    h_all, yp_all = _ws(ws, "h", cfg), _ws(ws, "y_perm", cfg)

    def expert_ref(e):
        mats = []
        for n in ("w_gate", "w_up", "w_down"):
            q_ref, s_ref = quantize_w(w[n][e:e + 1].cpu())
            assert np.array_equal(qw[n][0][e].cpu().numpy().T, q_ref[0]), (n, e)
            assert np.array_equal(qw[n][1][e].cpu().numpy(), s_ref[0]), (n, e)
            mats.append(oracle.dequant_fp8(q_ref, s_ref)[0])
        rows = torch.tensor(picks[e], device="cuda").long()
        a = deq_rows(*oracle.quantize_rows_fp8(x_bits[row_src[picks[e]]]))
        h_ref = oracle.gate_up_f64(a, mats[0], mats[1])
        h_rows = h_all[rows]
        hq, sh = oracle.quantize_rows_fp8(bits(h_rows))
        return (f64(h_rows), h_ref, f64(yp_all[rows]),
                oracle.matmul_f64(deq_rows(hq, sh), mats[2]))
    refs = map_experts(expert_ref, picks)
    cat = lambda i: np.concatenate([refs[e][i] for e in picks])  # noqa: E731
    assert_bf16_rounding_close(cat(0), cat(1), f"h, {len(picks)} experts")
    assert_bf16_close(cat(2), cat(3), f"y_perm, {len(picks)} experts")

    rng = np.random.default_rng(cfg.seed + 1)
    toks = list(np.sort(rng.choice(cfg.T, size=2, replace=False)))
    all_dropped = np.flatnonzero((slot < 0).all(axis=1))
    if len(all_dropped):
        toks.append(int(all_dropped[0]))
    h_gpu = _ws(ws, "h", cfg)
    y_ref = np.zeros((len(toks), cfg.d))
    for i, t in enumerate(toks):
        if (slot[t] < 0).all():
            y_ref[i] = oracle.bits_to_f64(x_bits[t:t + 1])[0]
            continue
        xq, sx = oracle.quantize_rows_fp8(x_bits[t:t + 1])
        a = deq_rows(xq, sx)
        for j in range(cfg.k):
            if slot[t, j] < 0:
                continue
            e = int(o_idx[t, j])
            mats = []
            for n in ("w_gate", "w_up", "w_down"):
                q_ref, s_ref = quantize_w(w[n][e:e + 1].cpu())
                assert np.array_equal(qw[n][0][e].cpu().numpy().T, q_ref[0]), (n, e)
                assert np.array_equal(qw[n][1][e].cpu().numpy(), s_ref[0]), (n, e)
                mats.append(oracle.dequant_fp8(q_ref, s_ref)[0])
            h_ref = oracle.gate_up_f64(a, mats[0], mats[1])
            row = int(offsets[e] + slot[t, j])
            h_row = h_gpu[row:row + 1]
            assert_bf16_rounding_close(f64(h_row), h_ref, "h (sampled)")
            hq, sh = oracle.quantize_rows_fp8(bits(h_row))
            y_ref[i] += o_w[t, j] * oracle.matmul_f64(deq_rows(hq, sh), mats[2])[0]
    y_s = y[torch.tensor(toks, device="cuda").long()]
    moe_rows = np.array([not (slot[t] < 0).all() for t in toks])
    # the expert outputs against the oracle (tolerance from their own rms);
    # all-dropped tokens passed through bit for bit
    assert_bf16_close(f64(y_s)[moe_rows], y_ref[moe_rows], "y (sampled)")
    np.testing.assert_array_equal(bits(y_s)[~moe_rows], x_bits[np.array(toks)[~moe_rows]])
    del w, x, y, ws, qw
    torch.cuda.empty_cache()
