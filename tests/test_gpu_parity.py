"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle,
element by element on the same seeded inputs.

Sizes: small variants of every workload (same E, k, cf and routing structure,
smaller T / d / f so the oracle finishes in seconds while still spanning
several 128-row tiles, ragged bucket tails and every GEMM tile shape), plus the
full-size workloads checked on sampled tokens and on properties that hold at
any size.  Tolerances are in ``moe_testlib``.

The routing decision (an arg-max over fp32 logits) is compared the way the
method fixes it: the oracle selects on the GPU's own fp32 logits, after those
logits are themselves checked against the oracle's fp64 logits; and, as an
independent check, the oracle's own logits must select the same experts
wherever the top-k margin exceeds the logits tolerance.
"""
import numpy as np
import pytest
import torch

import oracle
import mixture_experts_layer_36_b200 as moe
from mixture_experts_layer_36_b200 import configs, synth
from moe_testlib import (H_MODES, WEIGHT_ATOL, LOGIT_RTOL, assert_bf16_close,
                         assert_bf16_rounding_close, assert_layer_close, assert_logits_close, bits,
                         cuda_inputs, every_expert_rows, f64, map_experts, random_routing, small)

pytestmark = pytest.mark.gpu

SMALL = [
    configs.TINY,
    small("mixtral_small", T=512, d=256, E=8, k=2, f=512, cf=0.0, seed=11),
    small("fine_small", T=512, d=256, E=256, k=8, f=256, cf=1.25, seed=12),
    small("skewed_small", T=1024, d=256, E=64, k=6, f=384, cf=1.0, seed=13, zipf_s=1.2),
    small("decode_small", T=16, d=256, E=256, k=8, f=256, cf=0.0, seed=14),
    small("ragged_T", T=333, d=384, E=6, k=3, f=128, cf=0.5, seed=15),
    small("single_expert", T=200, d=128, E=1, k=1, f=256, cf=0.0, seed=16),
    small("k_equals_E", T=100, d=128, E=4, k=4, f=128, cf=0.0, seed=17),
    small("one_token", T=1, d=128, E=8, k=2, f=128, cf=1.25, seed=18),
    # buffers of >= 512 rows per expert select the CTA-pair GEMM tiles
    small("pair_tiles", T=2048, d=256, E=4, k=2, f=256, cf=0.0, seed=19),
    small("pair_tiles_drops", T=3000, d=512, E=4, k=3, f=384, cf=0.8, seed=20),
    # 256 buffer rows per expert: CTA pairs with the expert tails inside full tiles
    small("medium_buckets", T=1024, d=256, E=16, k=4, f=384, cf=1.25, seed=22),
    # widths that are multiples of 64 but not of 128: ragged 64-column tails
    # in the router's K, the permuted rows, every GEMM tile shape and the combine
    small("width64", T=300, d=192, E=8, k=2, f=320, cf=1.25, seed=23),
    small("width64_pair", T=2048, d=320, E=4, k=2, f=192, cf=0.0, seed=24),
]
IDS = [c.name for c in SMALL]


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    torch.cuda.synchronize()


def independent_topk_check(ref64, gpu_idx, k):
    """Where the oracle's own logits separate the k-th and (k+1)-th experts by
    more than twice the logits tolerance, its selected set must equal the GPU's."""
    T, E = ref64.shape
    if k == E:
        return
    own_idx, _ = oracle.topk(ref64.astype(np.float32), k)
    srt = -np.sort(-ref64, axis=1)
    rms = np.sqrt(np.mean(ref64 ** 2))
    tol = LOGIT_RTOL * np.maximum(np.abs(srt[:, k - 1]), rms)
    clear = (srt[:, k - 1] - srt[:, k]) > 2 * tol
    assert clear.mean() > 0.9, "too few tokens with a clear top-k margin"
    for t in np.nonzero(clear)[0]:
        assert set(own_idx[t]) == set(gpu_idx[t]), t


# ----------------------------------------------------------------------------- stage: route

@pytest.mark.parametrize("cfg", SMALL, ids=IDS)
def test_route_matches_oracle(cfg):
    inp, cpu = cuda_inputs(cfg)
    logits, idx, w = moe.moe_route(inp["x"], inp["w_router"], inp["bias"], cfg.k)
    torch.cuda.synchronize()
    bias = None if cpu["bias"] is None else cpu["bias"].numpy()
    ref64 = oracle.router_logits(bits(cpu["x"]), cpu["w_router"].numpy(), bias)
    gl = logits.cpu().numpy()
    assert_logits_close(gl, ref64)
    o_idx, o_w = oracle.topk(gl, cfg.k)
    np.testing.assert_array_equal(idx.cpu().numpy(), o_idx)
    assert np.max(np.abs(w.cpu().double().numpy() - o_w)) <= WEIGHT_ATOL
    independent_topk_check(ref64, idx.cpu().numpy(), cfg.k)


def test_route_ties_take_lower_index():
    # every token sees exactly tied logits: x = 0 -> all logits equal the bias
    E, k, d, T = 16, 4, 128, 40
    x = torch.zeros(T, d, dtype=torch.bfloat16, device="cuda")
    wr = torch.randn(d, E, device="cuda")
    bias = torch.tensor([0.5, 1.0, 1.0, 0.5, 2.0, 1.0, 2.0, 0.0] * 2, device="cuda")
    _, idx, w = moe.moe_route(x, wr, bias, k)
    o_idx, o_w = oracle.topk(np.tile(bias.cpu().numpy(), (T, 1)), k)
    np.testing.assert_array_equal(idx.cpu().numpy(), o_idx)
    assert o_idx[0].tolist() == [4, 6, 12, 14]
    assert np.max(np.abs(w.cpu().double().numpy() - o_w)) <= WEIGHT_ATOL


# More row tiles (128 tokens each) than any B200 has SMs: the router GEMM runs
# without a K split and its epilogue does the top-k itself.
T_UNSPLIT = 148 * 128 + 37


@pytest.mark.parametrize("E,k,with_bias", [(8, 2, False), (64, 6, True), (200, 8, True),
                                            (256, 8, False), (33, 3, True)])
def test_route_unsplit_matches_oracle(E, k, with_bias):
    d = 128
    g = torch.Generator().manual_seed(E * 10 + k)
    x = torch.randn(T_UNSPLIT, d, generator=g).to(torch.bfloat16)
    wr = torch.randn(d, E, generator=g) / d ** 0.5
    bias = (torch.randn(E, generator=g) * 0.1) if with_bias else None
    logits, idx, w = moe.moe_route(x.cuda(), wr.cuda(), None if bias is None else bias.cuda(), k)
    torch.cuda.synchronize()
    ref64 = oracle.router_logits(bits(x), wr.numpy(), None if bias is None else bias.numpy())
    gl = logits.cpu().numpy()
    assert_logits_close(gl, ref64)
    o_idx, o_w = oracle.topk(gl, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), o_idx)
    assert np.max(np.abs(w.cpu().double().numpy() - o_w)) <= WEIGHT_ATOL
    independent_topk_check(ref64, idx.cpu().numpy(), k)


@pytest.mark.parametrize("pattern,k,want", [
    ([0.5, 1.0, 1.0, 0.5, 2.0, 1.0, 2.0, 0.0], 4, [4, 6, 12, 14]),
    # equal values displaced by a larger one arriving later keep their order
    ([1.0, 1.0, 1.0, 0.5, 2.0, 1.0, 2.0, 0.0], 8, [4, 6, 12, 14, 0, 1, 2, 5]),
    ([0.5, 1.0, 1.0, 0.5, 2.0, 1.0, 2.0, 0.0], 8, [4, 6, 12, 14, 1, 2, 5, 9]),
])
def test_route_unsplit_ties_take_lower_index(pattern, k, want):
    E, d = 16, 128
    x = torch.zeros(T_UNSPLIT, d, dtype=torch.bfloat16, device="cuda")
    x[::3] = torch.randn(x[::3].shape, device="cuda").to(torch.bfloat16)  # some untied rows
    wr = torch.randn(d, E, device="cuda")
    bias = torch.tensor(pattern * 2, device="cuda")
    logits, idx, w = moe.moe_route(x, wr, bias, k)
    gl = logits.cpu().numpy()
    o_idx, o_w = oracle.topk(gl, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), o_idx)
    assert o_idx[1].tolist() == want                      # an all-tied row
    assert np.max(np.abs(w.cpu().double().numpy() - o_w)) <= WEIGHT_ATOL


# Few tokens and a wide d: the router splits K 8 or more ways (one 128-token
# row tile, d / 64 k-blocks), and the top-k kernel then reduces one token's
# partial sums with all 8 warps.  E = 256 puts 8 experts on every lane, and the
# tied values below sit on different lanes and on different slots of one lane.
def _tie_bias(E):
    b = torch.zeros(E)
    b[[13, 77, 141, 200]] = 2.0            # lanes 13, 13, 13, 8: one value, four experts
    b[[0, 31, 32, 64, 255]] = 1.0          # lanes 0, 31, 0, 0, 31
    b[[1, 33, 254]] = 0.5
    return b


@pytest.mark.parametrize("d", [512, 1024, 4096])
def test_route_split_k_ties_across_lanes(d):
    E, k, T = 256, 8, 97
    g = torch.Generator().manual_seed(d)
    x = torch.zeros(T, d, dtype=torch.bfloat16)
    x[::4] = torch.randn(x[::4].shape, generator=g).to(torch.bfloat16)   # some untied rows
    wr = torch.randn(d, E, generator=g) / d ** 0.5
    bias = _tie_bias(E)
    logits, idx, w = moe.moe_route(x.cuda(), wr.cuda(), bias.cuda(), k)
    torch.cuda.synchronize()
    gl = logits.cpu().numpy()
    assert_logits_close(gl, oracle.router_logits(bits(x), wr.numpy(), bias.numpy()))
    o_idx, o_w = oracle.topk(gl, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), o_idx)
    # an all-tied row (x = 0): the four 2.0s, then the 1.0s by expert index
    assert o_idx[1].tolist() == [13, 77, 141, 200, 0, 31, 32, 64]
    assert np.max(np.abs(w.cpu().double().numpy() - o_w)) <= WEIGHT_ATOL


# ----------------------------------------------------------------------------- stage: permute

PERM_CASES = [(64, 128, 8, 2, 1.25), (1000, 256, 64, 6, 1.0), (777, 128, 256, 8, 1.25),
              (513, 128, 8, 2, 0.0), (300, 128, 5, 5, 0.3), (257, 384, 3, 1, 0.5),
              (4096, 256, 256, 8, 0.2), (4352, 128, 256, 8, 1.25), (65536, 128, 256, 8, 1.0)]


@pytest.mark.parametrize("T,d,E,k,cf", PERM_CASES)
def test_permute_matches_oracle(T, d, E, k, cf):
    g = torch.Generator().manual_seed(T * 7 + E)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16)
    idx = random_routing(T, E, k, seed=T + E)
    C = oracle.capacity(T, E, k, cf)
    assert moe.moe_capacity(T, E, k, cf) == C
    counts, offsets, slot, row_src, n_drop = oracle.permute(idx, E, C)
    N = int(offsets[E])
    out = moe.moe_permute(x.cuda(), torch.from_numpy(idx).cuda(), E, cf)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out["counts"].cpu().numpy(), counts)
    np.testing.assert_array_equal(out["offsets"].cpu().numpy(), offsets)
    np.testing.assert_array_equal(out["slot"].cpu().numpy(), slot)
    assert int(out["n_dropped"].item()) == n_drop
    np.testing.assert_array_equal(out["row_src"][:N].cpu().numpy(), row_src)
    np.testing.assert_array_equal(bits(out["x_perm"][:N]), oracle.dispatch(bits(x), row_src))
    # determinism: a second run gives the same bits
    out2 = moe.moe_permute(x.cuda(), torch.from_numpy(idx).cuda(), E, cf)
    for key in ("slot", "offsets", "row_src"):
        assert torch.equal(out[key][:N] if key == "row_src" else out[key],
                           out2[key][:N] if key == "row_src" else out2[key])
    assert torch.equal(out["x_perm"][:N], out2["x_perm"][:N])


# ----------------------------------------------------------------------------- stage: experts

MLP_CASES = [
    # (d, f, bucket sizes, pair): ragged tails, empty buckets, one-row buckets,
    # exact tile multiples, several row tiles; pair=True gives the buffer >= 512
    # rows per expert, which selects the CTA-pair tiles (256 rows, a half tile
    # at an expert's tail), "mid" 256-511 the CTA-pair tiles that compute an
    # expert's last <= 128 rows inside its last full tile; smaller buffers
    # select the single-CTA 128-row tiles
    (256, 384, [300, 0, 1, 129, 128, 257], False),
    (128, 256, [5, 140, 0, 0, 64, 128], False),
    (384, 128, [1, 1, 1, 400], False),
    (512, 640, [129] * 3, False),
    (256, 256, [0, 0, 0], False),
    (256, 384, [300, 0, 1, 129, 128, 257, 700], True),
    (512, 256, [1, 256, 511, 513, 1024], True),
    (384, 256, [255, 257, 0], True),      # down GEMM: d % 256 != 0 keeps single-CTA tiles
    (256, 256, [170, 0, 128, 129, 233, 256, 250, 131], False),
    (384, 128, [300, 301, 15, 16], False),
    # more CTA-pair tiles than pairs (several tiles per pair), K longer than
    # the ring (16 k-blocks) and shorter (2), a last N tile of 128 h-columns
    (1024, 1024, [2048] * 4, True),
    (512, 128, [6000] * 4, True),
    (256, 384, [3000, 2999, 1, 2900], True),
    # long contractions (K = 4096 with 256-511 buffer rows per expert, "mid";
    # K = 8192 on CTA-pair tiles)
    (4096, 384, [300, 260, 255, 511, 0, 1], "mid"),
    (768, 8192, [600, 1, 300], True),
    # d, f multiples of 64 only: 64-column N tails and K = 64 * odd
    (192, 320, [300, 0, 1, 129, 128, 257], False),
    (320, 192, [3000, 2999, 1, 2900], True),
    (64, 64, [70, 0, 129], False),
    # swapped tail tiles of every width (N = 32, 64, 96, 128: tails of 1-32,
    # 33-64, 65-96, 97-128 rows, alone or after full 256-row tiles), tails of
    # more than 128 rows (a full pair tile), 64-column N tails of h (f = 320)
    (256, 320, [257, 289, 320, 353, 1, 97, 128, 129, 200, 0, 511, 384], "mid"),
    (512, 256, [33, 64, 65, 96, 300, 416, 480, 32, 31], "mid"),
    (256, 448, [260, 272, 288, 304], "mid"),
]


def mlp_buffer_rows(N, E, pair):
    """Rows of the permuted buffer for a bucket layout: pair=True gives >= 512
    per expert (CTA-pair tiles), "mid" 256-511 (bf16: CTA pairs with the
    expert tails inside full tiles; e4m3: single-CTA tiles) and False fewer
    (single-CTA tiles)."""
    if pair == "mid":
        rows = max(N + 37, 256 * E + 5)
        assert rows < 512 * E
        return rows
    return max(N + 37, 512 * E + 5) if pair else N + 37


@pytest.mark.parametrize("d,f,sizes,pair", MLP_CASES)
def test_expert_mlp_matches_oracle(d, f, sizes, pair):
    E = len(sizes)
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    N = int(offsets[-1])
    max_rows = mlp_buffer_rows(N, E, pair)
    g = torch.Generator().manual_seed(d + f + E)
    x_perm = torch.randn(max_rows, d, generator=g).to(torch.bfloat16)
    wg = (torch.randn(E, d, f, generator=g) / d ** 0.5).to(torch.bfloat16)
    wu = (torch.randn(E, d, f, generator=g) / d ** 0.5).to(torch.bfloat16)
    wd = (torch.randn(E, f, d, generator=g) / f ** 0.5).to(torch.bfloat16)
    sentinel = -7.0
    h = torch.full((max_rows, f), sentinel, dtype=torch.bfloat16, device="cuda")
    y = torch.full((max_rows, d), sentinel, dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.moe_expert_mlp(x_perm.cuda(), torch.from_numpy(offsets).cuda(), wg.cuda(), wu.cuda(),
                       wd.cuda(), h=h, y_perm=y, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    o_h, o_y = oracle.expert_mlp(bits(x_perm[:N]), offsets, bits(wg), bits(wu), bits(wd),
                                 want_h=True)
    assert_bf16_rounding_close(f64(h[:N]), o_h, "h")
    assert_bf16_close(f64(y[:N]), o_y, "y_perm")
    # rows outside every bucket are not written
    assert torch.all(h[N:] == sentinel) and torch.all(y[N:] == sentinel)


# ----------------------------------------------------------------------------- stage: combine

@pytest.mark.parametrize("T,d,E,k,cf", [(64, 128, 8, 2, 1.25), (500, 256, 16, 4, 0.4),
                                        (300, 128, 4, 4, 0.0)])
def test_combine_matches_oracle(T, d, E, k, cf):
    g = torch.Generator().manual_seed(T + d)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16)
    logits = torch.randn(T, E, generator=g).numpy()
    idx, w64 = oracle.topk(logits, k)
    w32 = w64.astype(np.float32)
    C = oracle.capacity(T, E, k, cf)
    counts, offsets, slot, row_src, n_drop = oracle.permute(idx, E, C)
    rows = max(int(offsets[E]), 1)
    y_perm = torch.randn(rows, d, generator=g)
    y = moe.moe_combine(y_perm.cuda(), x.cuda(), torch.from_numpy(idx).cuda(),
                        torch.from_numpy(w32).cuda(), torch.from_numpy(slot).cuda(),
                        torch.from_numpy(offsets).cuda())
    torch.cuda.synchronize()
    ref = oracle.combine(f64(y_perm), bits(x), idx, w32.astype(np.float64), slot, offsets)
    assert_bf16_close(f64(y), ref, "y")
    dropped = (slot < 0).all(axis=1)
    if dropped.any():
        np.testing.assert_array_equal(bits(y)[dropped], bits(x)[dropped])


@pytest.mark.parametrize("T,d,E,k,cf", [(64, 128, 8, 2, 1.25), (500, 256, 16, 4, 0.4)])
def test_combine_bf16rows_matches_oracle(T, d, E, k, cf):
    """The combine on bf16 expert-output rows (the expert-parallel return in
    bf16) against the oracle's combine on the same bf16 values."""
    g = torch.Generator().manual_seed(T + d + 1)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16)
    logits = torch.randn(T, E, generator=g).numpy()
    idx, w64 = oracle.topk(logits, k)
    w32 = w64.astype(np.float32)
    C = oracle.capacity(T, E, k, cf)
    counts, offsets, slot, row_src, n_drop = oracle.permute(idx, E, C)
    rows = max(int(offsets[E]), 1)
    y_rows = torch.randn(rows, d, generator=g).to(torch.bfloat16)
    y = moe.moe_combine_bf16rows(y_rows.cuda(), x.cuda(), torch.from_numpy(idx).cuda(),
                                 torch.from_numpy(w32).cuda(), torch.from_numpy(slot).cuda(),
                                 torch.from_numpy(offsets).cuda())
    torch.cuda.synchronize()
    ref = oracle.combine(f64(y_rows), bits(x), idx, w32.astype(np.float64), slot, offsets)
    assert_bf16_close(f64(y), ref, "y")
    dropped = (slot < 0).all(axis=1)
    if dropped.any():
        np.testing.assert_array_equal(bits(y)[dropped], bits(x)[dropped])


def test_rows_to_bf16_rounds_like_the_oracle():
    """fp32 -> bf16, bit for bit the oracle's rounding (nearest, ties to
    even), on random values of several magnitudes and on exact ties."""
    g = torch.Generator().manual_seed(77)
    rows, d = 37, 192
    v = torch.randn(rows, d, generator=g) * torch.exp2(torch.randint(-30, 30, (rows, d),
                                                                     generator=g).float())
    u = v.view(torch.int32)
    # every fourth value halfway between two bf16 values (low 16 bits 0x8000)
    tie = (u & ~0xFFFF) | 0x8000
    u = torch.where(torch.arange(rows * d).view(rows, d) % 4 == 0, tie, u)
    v = u.view(torch.float32)
    got = moe.moe_rows_to_bf16(v.cuda())
    torch.cuda.synchronize()
    ref = np.vectorize(oracle.round_bf16)(v.numpy().astype(np.float64))
    want = (ref.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    np.testing.assert_array_equal(bits(got), want)


# ----------------------------------------------------------------------------- whole layer

def _ws(ws, name, cfg):
    return moe.workspace_view(ws, name, cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, cfg.cf)


@pytest.mark.parametrize("h_bf16", H_MODES, ids=["h_fp64", "h_bf16"])
@pytest.mark.parametrize("cfg", SMALL, ids=IDS)
def test_layer_forward_matches_oracle(cfg, h_bf16):
    """The whole layer against the oracle: h_fp64 is the plain definition
    (the MLP in fp64 throughout), h_bf16 the oracle with h rounded to bf16
    like the GEMMs' operand (tolerances in moe_testlib.H_MODES)."""
    inp, cpu = cuda_inputs(cfg)
    y, ws = moe.moe_layer_forward(inp["x"], inp["w_router"], inp["bias"], inp["w_gate"],
                                  inp["w_up"], inp["w_down"], cfg.k, cfg.cf)
    torch.cuda.synchronize()
    assert _ws(ws, "status", cfg).item() == 0
    gl = _ws(ws, "logits", cfg).cpu().numpy()
    bias = None if cpu["bias"] is None else cpu["bias"].numpy()
    ref = oracle.moe_forward(bits(cpu["x"]), cpu["w_router"].numpy(), bias, bits(cpu["w_gate"]),
                             bits(cpu["w_up"]), bits(cpu["w_down"]), cfg.k, cfg.cf,
                             decision_logits=gl, h_bf16=h_bf16)
    assert_logits_close(gl, ref["logits64"])
    np.testing.assert_array_equal(_ws(ws, "topk_idx", cfg).cpu().numpy(), ref["topk_idx"])
    assert np.max(np.abs(_ws(ws, "topk_w", cfg).cpu().double().numpy() - ref["topk_w"])) \
        <= WEIGHT_ATOL
    np.testing.assert_array_equal(_ws(ws, "slot", cfg).cpu().numpy(), ref["slot"])
    np.testing.assert_array_equal(_ws(ws, "counts", cfg).cpu().numpy(), ref["counts"])
    np.testing.assert_array_equal(_ws(ws, "offsets", cfg).cpu().numpy(), ref["offsets"])
    C = oracle.capacity(cfg.T, cfg.E, cfg.k, cfg.cf)
    counts = ref["counts"]
    assert counts.max() <= C and counts.sum() == cfg.k * cfg.T - ref["n_dropped"]
    assert _ws(ws, "n_dropped", cfg).item() == ref["n_dropped"]
    assert_layer_close(f64(y), ref["y"], h_bf16, "y")
    dropped = (ref["slot"] < 0).all(axis=1)
    if dropped.any():
        np.testing.assert_array_equal(bits(y)[dropped], bits(cpu["x"])[dropped])
    independent_topk_check(ref["logits64"], ref["topk_idx"], cfg.k)


@pytest.mark.parametrize("cfg", SMALL[:4], ids=IDS[:4])
def test_stages_equal_one_shot(cfg):
    inp, _ = cuda_inputs(cfg)
    y1, _ = moe.moe_layer_forward(inp["x"], inp["w_router"], inp["bias"], inp["w_gate"],
                                  inp["w_up"], inp["w_down"], cfg.k, cfg.cf)
    logits, idx, w = moe.moe_route(inp["x"], inp["w_router"], inp["bias"], cfg.k)
    p = moe.moe_permute(inp["x"], idx, cfg.E, cfg.cf)
    _, y_perm = moe.moe_expert_mlp(p["x_perm"], p["offsets"], inp["w_gate"], inp["w_up"],
                                   inp["w_down"])
    y2 = moe.moe_combine(y_perm, inp["x"], idx, w, p["slot"], p["offsets"])
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("cfg", [configs.TINY, SMALL[3]], ids=["tiny", "skewed_small"])
def test_layer_forward_ex_writes_routing_outputs(cfg):
    """moe_layer_forward_ex: the caller's routing tensors receive exactly what
    moe_layer_forward leaves in its workspace, and y is bit-identical."""
    inp, _ = cuda_inputs(cfg)
    args = (inp["x"], inp["w_router"], inp["bias"], inp["w_gate"], inp["w_up"], inp["w_down"],
            cfg.k, cfg.cf)
    y1, ws = moe.moe_layer_forward(*args)
    T, E, k = cfg.T, cfg.E, cfg.k
    fill = lambda *shape, dt: torch.full(shape, -5, dtype=dt, device="cuda")  # noqa: E731
    outs = {"logits": fill(T, E, dt=torch.float32), "topk_idx": fill(T, k, dt=torch.int32),
            "topk_w": fill(T, k, dt=torch.float32), "slot": fill(T, k, dt=torch.int32),
            "counts": fill(E, dt=torch.int32)}
    y2, ws2 = moe.moe_layer_forward_ex(*args, **outs)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    for name, t in outs.items():
        assert torch.equal(t, _ws(ws, name, cfg)), name
    assert _ws(ws2, "status", cfg).item() == 0


def test_hot_expert_many_row_tiles():
    # a bias that sends every token to experts 0 and 1: two buckets of T rows
    cfg = small("hot", T=1500, d=256, E=8, k=2, f=256, cf=0.0, seed=21)
    inp, cpu = cuda_inputs(cfg)
    bias = torch.tensor([50.0, 40.0] + [0.0] * 6)
    y, ws = moe.moe_layer_forward(inp["x"], inp["w_router"], bias.cuda(), inp["w_gate"],
                                  inp["w_up"], inp["w_down"], cfg.k, cfg.cf)
    torch.cuda.synchronize()
    counts = _ws(ws, "counts", cfg).cpu().numpy()
    assert counts[0] == cfg.T and counts[1] == cfg.T
    gl = _ws(ws, "logits", cfg).cpu().numpy()
    ref = oracle.moe_forward(bits(cpu["x"]), cpu["w_router"].numpy(), bias.numpy(),
                             bits(cpu["w_gate"]), bits(cpu["w_up"]), bits(cpu["w_down"]), cfg.k,
                             cfg.cf, decision_logits=gl)
    assert_bf16_close(f64(y), ref["y"], "y")


def test_empty_batch_is_noop():
    cfg = small("empty", T=0, d=128, E=8, k=2, f=128, cf=1.25, seed=0)
    x = torch.empty(0, 128, dtype=torch.bfloat16, device="cuda")
    w = synth.make_weights(cfg, "cuda")
    y, _ = moe.moe_layer_forward(x, w["w_router"], None, w["w_gate"], w["w_up"], w["w_down"],
                                 cfg.k, cfg.cf)
    assert y.shape == (0, 128)


# ----------------------------------------------------------------------------- full sizes

FULL = [configs.MIXTRAL, configs.FINE, configs.SKEWED] + \
    [configs.DECODE.with_tokens(t) for t in configs.DECODE_T]


@pytest.mark.parametrize("cfg", FULL, ids=[c.name for c in FULL])
def test_full_size_sampled(cfg):
    """Full-size workload in the benchmark's launch configuration: routing,
    capacity and permutation checked for every token; logits, x_perm rows and
    outputs checked on a seeded sample the oracle computes one by one; the
    down GEMM's rows checked for every expert that received rows (its
    bucket's last row, in the tail tile, and one more)."""
    torch.cuda.empty_cache()
    w = synth.make_weights(cfg, "cuda")
    x = synth.make_tokens(cfg, "cuda")
    y, ws = moe.moe_layer_forward(x, w["w_router"], w["bias"], w["w_gate"], w["w_up"],
                                  w["w_down"], cfg.k, cfg.cf)
    torch.cuda.synchronize()
    assert _ws(ws, "status", cfg).item() == 0
    gl = _ws(ws, "logits", cfg).cpu().numpy()
    o_idx, o_w = oracle.topk(gl, cfg.k)
    np.testing.assert_array_equal(_ws(ws, "topk_idx", cfg).cpu().numpy(), o_idx)
    assert np.max(np.abs(_ws(ws, "topk_w", cfg).cpu().double().numpy() - o_w)) <= WEIGHT_ATOL
    C = oracle.capacity(cfg.T, cfg.E, cfg.k, cfg.cf)
    counts, offsets, slot, row_src, n_drop = oracle.permute(o_idx, cfg.E, C)
    np.testing.assert_array_equal(_ws(ws, "counts", cfg).cpu().numpy(), counts)
    np.testing.assert_array_equal(_ws(ws, "offsets", cfg).cpu().numpy(), offsets)
    np.testing.assert_array_equal(_ws(ws, "slot", cfg).cpu().numpy(), slot)
    assert _ws(ws, "n_dropped", cfg).item() == n_drop
    N = int(offsets[-1])
    np.testing.assert_array_equal(_ws(ws, "row_src", cfg)[:N].cpu().numpy(), row_src)

    rng = np.random.default_rng(cfg.seed)
    x_bits = bits(x)
    # sampled permuted rows are exact copies of their token rows
    rows = rng.choice(N, size=min(N, 256), replace=False)
    xp = _ws(ws, "x_perm", cfg)
    np.testing.assert_array_equal(bits(xp[torch.from_numpy(rows).cuda().long()]),
                                  x_bits[row_src[rows]])
    # every expert with rows: y_perm (fp32) rows against the oracle's expert,
    # with h in fp64 (the definition) and rounded to bf16 (the GEMM operand)
    picks = every_expert_rows(offsets, cfg.seed)
    assert len(picks) == int((counts > 0).sum())

    def expert_ref(e):
        wg, wu, wd = (bits(w[n][e]) for n in ("w_gate", "w_up", "w_down"))
        xr = x_bits[row_src[picks[e]]]
        return {hb: oracle.swiglu_rows(xr, wg, wu, wd, h_bf16=hb)[1] for hb in H_MODES}
    refs = map_experts(expert_ref, picks)
    rows_all = np.concatenate([picks[e] for e in picks])
    got = f64(_ws(ws, "y_perm", cfg)[torch.from_numpy(rows_all).cuda().long()])
    for hb in H_MODES:
        assert_bf16_close(got, np.concatenate([refs[e][hb] for e in picks]),
                          f"y_perm, {len(picks)} experts, h_bf16={hb}")

    # sampled tokens: logits and outputs from the oracle, one token at a time
    n_tok = 4 if cfg.E >= 64 else 8
    toks = np.sort(rng.choice(cfg.T, size=min(n_tok, cfg.T), replace=False))
    if (slot < 0).all(axis=1).any():
        toks = np.unique(np.concatenate([toks, np.nonzero((slot < 0).all(axis=1))[0][:2]]))
    wr = w["w_router"].cpu().numpy()
    bias = None if w["bias"] is None else w["bias"].cpu().numpy()
    assert_logits_close(gl[toks], oracle.router_logits(x_bits[toks], wr, bias))
    by_expert = {}
    for i, t in enumerate(toks):
        for j in range(cfg.k):
            if slot[t, j] >= 0:
                by_expert.setdefault(int(o_idx[t, j]), []).append((i, t, j))
    y_s = y[torch.from_numpy(toks).cuda().long()]
    moe_rows = ~(slot[toks] < 0).all(axis=1)
    for hb in H_MODES:
        y_ref = np.zeros((len(toks), cfg.d))
        for i, t in enumerate(toks):
            if not moe_rows[i]:
                y_ref[i] = oracle.bits_to_f64(x_bits[t])
        for e, users in by_expert.items():
            wg, wu, wd = (bits(w[n][e]) for n in ("w_gate", "w_up", "w_down"))
            _, o = oracle.swiglu_rows(x_bits[[t for _, t, _ in users]], wg, wu, wd, h_bf16=hb)
            for (i, t, j), orow in zip(users, o):
                y_ref[i] += o_w[t, j] * orow
        # the expert outputs against the oracle (tolerance from their own rms)
        assert_layer_close(f64(y_s)[moe_rows], y_ref[moe_rows], hb, "y (sampled)")
    # all-dropped tokens passed through bit for bit
    np.testing.assert_array_equal(bits(y_s)[~moe_rows], x_bits[toks[~moe_rows]])
    del w, x, y, ws
    torch.cuda.empty_cache()
