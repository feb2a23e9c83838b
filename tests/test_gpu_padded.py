"""GPU parity for the padded [E, C, d] layout (moe_permute_padded followed by
the unchanged grouped GEMM and combine entry points), against the oracle:
the padded buffer, its row_src and the routing outputs bit-exact; the layer
output within the bf16 path's tolerance; padding rows computed to exact zeros.
"""
import numpy as np
import pytest
import torch

import oracle
import mixture_experts_layer_36_b200 as moe
from moe_testlib import (H_MODES, WEIGHT_ATOL, assert_layer_close, bits,
                         cuda_inputs, f64, random_routing, small)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    torch.cuda.synchronize()


@pytest.mark.parametrize("T,d,E,k,cf", [(333, 384, 6, 3, 0.5), (512, 256, 256, 8, 1.25),
                                        (64, 128, 8, 2, 0.0), (1000, 256, 16, 4, 1.0)])
def test_permute_padded_matches_oracle(T, d, E, k, cf):
    g = torch.Generator().manual_seed(T + d)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16)
    idx = random_routing(T, E, k, seed=T + E)
    out = moe.moe_permute_padded(x.cuda(), torch.from_numpy(idx).cuda(), E, cf)
    torch.cuda.synchronize()
    C = oracle.capacity(T, E, k, cf)
    counts, _, slot, _, n_drop = oracle.permute(idx, E, C)
    np.testing.assert_array_equal(out["counts"].cpu().numpy(), counts)
    np.testing.assert_array_equal(out["offsets"].cpu().numpy(), np.arange(E + 1) * C)
    np.testing.assert_array_equal(out["slot"].cpu().numpy(), slot)
    assert out["n_dropped"].item() == n_drop
    pad, src = oracle.dispatch_padded(bits(x), idx, slot, E, C)
    np.testing.assert_array_equal(bits(out["x_pad"]), pad)
    np.testing.assert_array_equal(out["row_src"].cpu().numpy(), src)


PADDED = [
    small("fine_small", T=512, d=256, E=256, k=8, f=256, cf=1.25, seed=12),
    small("skewed_small", T=1024, d=256, E=64, k=6, f=384, cf=1.0, seed=13, zipf_s=1.2),
    small("ragged_T", T=333, d=384, E=6, k=3, f=128, cf=0.5, seed=15),
    small("pair_tiles_drops", T=3000, d=512, E=4, k=3, f=384, cf=0.8, seed=20),
    small("dropless", T=200, d=128, E=4, k=2, f=256, cf=0.0, seed=21),
    # buckets of C = 320 rows: a 64-row tail inside every expert's full tile
    small("tails", T=1024, d=256, E=16, k=4, f=256, cf=1.25, seed=25),
]


@pytest.mark.parametrize("cfg", PADDED, ids=[c.name for c in PADDED])
def test_layer_padded_matches_oracle(cfg):
    inp, cpu = cuda_inputs(cfg)
    logits, idx, w = moe.moe_route(inp["x"], inp["w_router"], inp["bias"], cfg.k)
    p = moe.moe_permute_padded(inp["x"], idx, cfg.E, cfg.cf)
    h, y_pad = moe.moe_expert_mlp(p["x_pad"], p["offsets"], inp["w_gate"], inp["w_up"],
                                  inp["w_down"])
    y = moe.moe_combine(y_pad, inp["x"], idx, w, p["slot"], p["offsets"])
    torch.cuda.synchronize()
    gl = logits.cpu().numpy()
    bias = None if cpu["bias"] is None else cpu["bias"].numpy()
    for hb in H_MODES:       # h in fp64 (the definition) and rounded to bf16
        ref = oracle.moe_forward(bits(cpu["x"]), cpu["w_router"].numpy(), bias,
                                 bits(cpu["w_gate"]), bits(cpu["w_up"]), bits(cpu["w_down"]),
                                 cfg.k, cfg.cf, decision_logits=gl, h_bf16=hb)
        assert_layer_close(f64(y), ref["y"], hb, "y")
    np.testing.assert_array_equal(idx.cpu().numpy(), ref["topk_idx"])
    assert np.max(np.abs(w.cpu().double().numpy() - ref["topk_w"])) <= WEIGHT_ATOL
    np.testing.assert_array_equal(p["slot"].cpu().numpy(), ref["slot"])
    # padding rows: zero inputs, so exactly zero h and y_pad
    pad_rows = torch.from_numpy(p["row_src"].cpu().numpy() < 0).cuda()
    assert torch.all(h[pad_rows] == 0) and torch.all(y_pad[pad_rows] == 0)
    dropped = (ref["slot"] < 0).all(axis=1)
    if dropped.any():
        np.testing.assert_array_equal(bits(y)[dropped], bits(cpu["x"])[dropped])
