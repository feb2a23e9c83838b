"""GPU parity for the fused path, through the C ABI, against the oracle and
against the unfused entry points: the permutation with row_pair and the zeroed
fp32 token accumulator (with and without the row copy), the gate/up GEMM
gathering its rows from x (no x_perm), the down GEMM adding the gate-weighted
rows into the accumulator, and the finishing pass.

The gathered GEMM computes from the same row values with the same tiles as
the permuted one, so its h must be identical bit for bit.  The scatter sums a
token's k terms in the order the GEMM tiles finish, so y is compared with the
oracle at the usual tolerance (not bit for bit with the unfused combine).
"""
import numpy as np
import pytest
import torch

import oracle
import mixture_experts_layer_36_b200 as moe
from mixture_experts_layer_36_b200 import configs, synth
from moe_testlib import (H_MODES, WEIGHT_ATOL, assert_bf16_close, assert_bf16_rounding_close,
                         assert_layer_close, bits, cuda_inputs, every_expert_rows, f64,
                         map_experts, random_routing, small)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    torch.cuda.synchronize()


@pytest.mark.parametrize("copy_rows", [True, False])
@pytest.mark.parametrize("T,d,E,k,cf", [(333, 384, 6, 3, 0.5), (512, 256, 256, 8, 1.25),
                                        (64, 128, 8, 2, 0.0)])
def test_permute_fused_matches_oracle(T, d, E, k, cf, copy_rows):
    g = torch.Generator().manual_seed(T + d)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16)
    idx = random_routing(T, E, k, seed=T + E + 1)
    out = moe.moe_permute_fused(x.cuda(), torch.from_numpy(idx).cuda(), E, cf,
                                copy_rows=copy_rows)
    torch.cuda.synchronize()
    C = oracle.capacity(T, E, k, cf)
    counts, offsets, slot, row_src, n_drop = oracle.permute(idx, E, C)
    np.testing.assert_array_equal(out["counts"].cpu().numpy(), counts)
    np.testing.assert_array_equal(out["offsets"].cpu().numpy(), offsets)
    np.testing.assert_array_equal(out["slot"].cpu().numpy(), slot)
    assert out["n_dropped"].item() == n_drop
    N = int(offsets[-1])
    np.testing.assert_array_equal(out["row_src"][:N].cpu().numpy(), row_src)
    pair = out["row_pair"][:N].cpu().numpy()
    t, j = pair // k, pair % k
    np.testing.assert_array_equal(t, row_src)
    bucket = np.repeat(np.arange(E), np.diff(offsets))
    np.testing.assert_array_equal(idx[t, j], bucket)
    np.testing.assert_array_equal(offsets[bucket] + slot[t, j], np.arange(N))
    assert torch.all(out["y32"] == 0)
    if copy_rows:
        np.testing.assert_array_equal(bits(out["x_perm"][:N]), oracle.dispatch(bits(x), row_src))


SMALL = [
    configs.TINY,
    small("mixtral_small", T=512, d=256, E=8, k=2, f=512, cf=0.0, seed=11),
    small("fine_small", T=512, d=256, E=256, k=8, f=256, cf=1.25, seed=12),
    small("skewed_small", T=1024, d=256, E=64, k=6, f=384, cf=1.0, seed=13, zipf_s=1.2),
    small("decode_small", T=16, d=256, E=256, k=8, f=256, cf=0.0, seed=14),
    small("ragged_T", T=333, d=384, E=6, k=3, f=128, cf=0.5, seed=15),
    small("pair_tiles", T=2048, d=256, E=4, k=2, f=256, cf=0.0, seed=19),
    small("pair_tiles_drops", T=3000, d=512, E=4, k=3, f=384, cf=0.8, seed=20),
    small("down_d384", T=700, d=384, E=4, k=2, f=256, cf=0.0, seed=23),
    # 256 buffer rows per expert: the gate/up GEMM on CTA pairs with the
    # expert tails inside full tiles (also gathering its rows); the
    # scattering down GEMM keeps single-CTA tiles there
    small("tails", T=1024, d=256, E=16, k=4, f=256, cf=1.25, seed=25),
]
IDS = [c.name for c in SMALL]


@pytest.mark.parametrize("cfg", SMALL, ids=IDS)
def test_gather_gate_up_equals_permuted(cfg):
    inp, _ = cuda_inputs(cfg)
    _, idx, _ = moe.moe_route(inp["x"], inp["w_router"], inp["bias"], cfg.k)
    p = moe.moe_permute(inp["x"], idx, cfg.E, cfg.cf)
    rows = p["x_perm"].shape[0]
    h_perm = moe.moe_expert_gate_up(p["x_perm"], p["offsets"], inp["w_gate"], inp["w_up"])
    h_gath = moe.moe_expert_gate_up_gather(inp["x"], p["row_src"], p["offsets"], inp["w_gate"],
                                           inp["w_up"], rows)
    torch.cuda.synchronize()
    N = int(p["offsets"][-1].item())
    assert torch.equal(h_gath[:N], h_perm[:N])


@pytest.mark.parametrize("cfg", SMALL, ids=IDS)
def test_layer_forward_fused_matches_oracle(cfg):
    inp, cpu = cuda_inputs(cfg)
    y, ws = moe.moe_layer_forward_fused(inp["x"], inp["w_router"], inp["bias"], inp["w_gate"],
                                        inp["w_up"], inp["w_down"], cfg.k, cfg.cf)
    torch.cuda.synchronize()
    view = lambda n: moe.workspace_view(ws, n, cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, cfg.cf)  # noqa
    assert view("status").item() == 0
    gl = view("logits").cpu().numpy()
    bias = None if cpu["bias"] is None else cpu["bias"].numpy()
    for hb in H_MODES:       # h in fp64 (the definition) and rounded to bf16
        ref = oracle.moe_forward(bits(cpu["x"]), cpu["w_router"].numpy(), bias,
                                 bits(cpu["w_gate"]), bits(cpu["w_up"]), bits(cpu["w_down"]),
                                 cfg.k, cfg.cf, decision_logits=gl, h_bf16=hb)
        assert_layer_close(f64(y), ref["y"], hb, "y")
    np.testing.assert_array_equal(view("topk_idx").cpu().numpy(), ref["topk_idx"])
    assert np.max(np.abs(view("topk_w").cpu().double().numpy() - ref["topk_w"])) <= WEIGHT_ATOL
    np.testing.assert_array_equal(view("slot").cpu().numpy(), ref["slot"])
    np.testing.assert_array_equal(view("offsets").cpu().numpy(), ref["offsets"])
    assert view("n_dropped").item() == ref["n_dropped"]
    dropped = (ref["slot"] < 0).all(axis=1)
    if dropped.any():
        np.testing.assert_array_equal(bits(y)[dropped], bits(cpu["x"])[dropped])
    # the same layer unfused: equal up to the summation order of each token's terms
    y2, _ = moe.moe_layer_forward(inp["x"], inp["w_router"], inp["bias"], inp["w_gate"],
                                  inp["w_up"], inp["w_down"], cfg.k, cfg.cf)
    torch.cuda.synchronize()
    assert_bf16_close(f64(y), f64(y2), "y (fused vs unfused)")


FULL = [configs.MIXTRAL, configs.DECODE.with_tokens(64)]


@pytest.mark.parametrize("cfg", FULL, ids=[c.name for c in FULL])
def test_fused_full_size_sampled(cfg):
    """Full-size fused layer against the unfused one on every token (same
    routing and rows; only the order of each token's k-term sum differs),
    its gate/up rows against the oracle for every expert that received rows
    (the bucket's last row and one more), and its output against the oracle
    on sampled tokens."""
    torch.cuda.empty_cache()
    w = synth.make_weights(cfg, "cuda")
    x = synth.make_tokens(cfg, "cuda")
    y, ws = moe.moe_layer_forward_fused(x, w["w_router"], w["bias"], w["w_gate"], w["w_up"],
                                        w["w_down"], cfg.k, cfg.cf)
    y2, _ = moe.moe_layer_forward(x, w["w_router"], w["bias"], w["w_gate"], w["w_up"],
                                  w["w_down"], cfg.k, cfg.cf)
    torch.cuda.synchronize()
    view = lambda n: moe.workspace_view(ws, n, cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, cfg.cf)  # noqa
    assert view("status").item() == 0
    assert_bf16_close(f64(y), f64(y2), "y (fused vs unfused)")
    gl = view("logits").cpu().numpy()
    o_idx, o_w = oracle.topk(gl, cfg.k)
    C = oracle.capacity(cfg.T, cfg.E, cfg.k, cfg.cf)
    counts, offsets, slot, row_src, _ = oracle.permute(o_idx, cfg.E, C)
    np.testing.assert_array_equal(view("row_src")[:int(offsets[-1])].cpu().numpy(), row_src)
    x_bits = bits(x)
    # every expert with rows: h rows of the gathering-free gate/up GEMM
    picks = every_expert_rows(offsets, cfg.seed + 5)
    assert len(picks) == int((counts > 0).sum())
    h_all = view("h")

    def expert_h(e):
        h_ref, _ = oracle.swiglu_rows(x_bits[row_src[picks[e]]], bits(w["w_gate"][e]),
                                      bits(w["w_up"][e]), bits(w["w_down"][e]), want_h=True)
        return f64(h_all[torch.tensor(picks[e], device="cuda").long()]), h_ref
    refs = map_experts(expert_h, picks)
    assert_bf16_rounding_close(np.concatenate([refs[e][0] for e in picks]),
                               np.concatenate([refs[e][1] for e in picks]),
                               f"h, {len(picks)} experts")
    rng = np.random.default_rng(cfg.seed + 2)
    toks = np.sort(rng.choice(cfg.T, size=3, replace=False))
    if (slot < 0).all(axis=1).any():          # and a token whose every pair is dropped
        toks = np.unique(np.append(toks, np.nonzero((slot < 0).all(axis=1))[0][0]))
    y_s = y[torch.from_numpy(toks).cuda().long()]
    moe_rows = ~(slot[toks] < 0).all(axis=1)
    for hb in H_MODES:       # h in fp64 (the definition) and rounded to bf16
        y_ref = np.zeros((len(toks), cfg.d))
        for i, t in enumerate(toks):
            for j in range(cfg.k):
                if slot[t, j] < 0:
                    continue
                e = int(o_idx[t, j])
                _, o = oracle.swiglu_rows(x_bits[t:t + 1], bits(w["w_gate"][e]),
                                          bits(w["w_up"][e]), bits(w["w_down"][e]), h_bf16=hb)
                y_ref[i] += o_w[t, j] * o[0]
        assert_layer_close(f64(y_s)[moe_rows], y_ref[moe_rows], hb, "y (sampled)")
    np.testing.assert_array_equal(bits(y_s)[~moe_rows], x_bits[toks[~moe_rows]])
    del w, x, y, y2, ws
    torch.cuda.empty_cache()
