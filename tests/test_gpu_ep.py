"""GPU parity for the expert-parallel pieces on one GPU: the bucket MLP
(slots mapped to experts b % E_w, only each slot's received rows) against the
oracle, and the expert-parallel layer over a one-rank NCCL group (its
exchanges are then copies) against the oracle layer.  The multi-rank exchange
logic is covered on CPU ranks (tests/test_ep_gloo.py).
"""
import datetime
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
import mixture_experts_layer_36_b200 as moe
from mixture_experts_layer_36_b200 import ep
from moe_testlib import (H_MODES, assert_bf16_close, assert_bf16_rounding_close,
                         assert_layer_close, bits, cuda_inputs, f64, small)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    torch.cuda.synchronize()


@pytest.mark.parametrize("E_w,P,C,d,f", [(2, 2, 200, 256, 384), (4, 3, 130, 128, 256),
                                         (1, 4, 600, 256, 256)])
def test_mlp_buckets_matches_oracle(E_w, P, C, d, f):
    B = E_w * P
    g = torch.Generator().manual_seed(B + C)
    rng = np.random.default_rng(B + C)
    rows = rng.integers(0, C + 1, size=B).astype(np.int32)
    rows[0] = C                                          # a full slot
    rows[-1] = 0                                         # an empty one
    x = torch.randn(B * C, d, generator=g).to(torch.bfloat16)
    wg = (torch.randn(E_w, d, f, generator=g) / d ** 0.5).to(torch.bfloat16)
    wu = (torch.randn(E_w, d, f, generator=g) / d ** 0.5).to(torch.bfloat16)
    wd = (torch.randn(E_w, f, d, generator=g) / f ** 0.5).to(torch.bfloat16)
    offsets = torch.arange(B + 1, dtype=torch.int32) * C
    sentinel = -7.0
    h = torch.full((B * C, f), sentinel, dtype=torch.bfloat16, device="cuda")
    y = torch.full((B * C, d), sentinel, dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.moe_expert_mlp_buckets(x.cuda(), offsets.cuda(), torch.from_numpy(rows).cuda(), wg.cuda(),
                               wu.cuda(), wd.cuda(), h=h, y_rows=y, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    xb = bits(x)
    for b in range(B):
        lo, n, e = b * C, int(rows[b]), b % E_w
        if n:
            o_h, o_y = oracle.swiglu_rows(xb[lo:lo + n], bits(wg[e]), bits(wu[e]), bits(wd[e]),
                                          want_h=True)
            assert_bf16_rounding_close(f64(h[lo:lo + n]), o_h, f"h bucket {b}")
            assert_bf16_close(f64(y[lo:lo + n]), o_y, f"y bucket {b}")
        assert torch.all(h[lo + n:lo + C] == sentinel) and torch.all(y[lo + n:lo + C] == sentinel)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture(scope="module")
def one_rank_group():
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=120),
                            device_id=torch.device("cuda", 0))
    yield
    dist.destroy_process_group()


EP = [
    small("ep_fine", T=512, d=256, E=16, k=4, f=256, cf=1.25, seed=31),
    small("ep_drops", T=333, d=384, E=6, k=3, f=128, cf=0.5, seed=32),
    small("ep_pair", T=2048, d=256, E=4, k=2, f=256, cf=1.0, seed=33),
    # slots of C = 320 rows, of which only the received counts are real: the
    # expert-tail pair tiles with per-bucket row counts
    small("ep_tails", T=1024, d=256, E=8, k=2, f=256, cf=1.25, seed=34),
]


@pytest.mark.parametrize("cfg", EP, ids=[c.name for c in EP])
def test_expert_parallel_one_rank_matches_oracle(cfg, one_rank_group):
    inp, cpu = cuda_inputs(cfg)
    layer = ep.ExpertParallelMoE(inp["w_router"], inp["bias"], inp["w_gate"], inp["w_up"],
                                 inp["w_down"], cfg.k, cfg.cf)
    y = layer(inp["x"])
    logits, _, _ = moe.moe_route(inp["x"], inp["w_router"], inp["bias"], cfg.k)
    torch.cuda.synchronize()
    bias = None if cpu["bias"] is None else cpu["bias"].numpy()
    for hb in H_MODES:       # h in fp64 (the definition) and rounded to bf16
        ref = oracle.moe_forward(bits(cpu["x"]), cpu["w_router"].numpy(), bias,
                                 bits(cpu["w_gate"]), bits(cpu["w_up"]), bits(cpu["w_down"]),
                                 cfg.k, cfg.cf, decision_logits=logits.cpu().numpy(), h_bf16=hb)
        assert_layer_close(f64(y), ref["y"], hb, "y")
    dropped = (ref["slot"] < 0).all(axis=1)
    if dropped.any():
        np.testing.assert_array_equal(bits(y)[dropped], bits(cpu["x"])[dropped])


@pytest.mark.parametrize("cfg", [EP[0], EP[-1]], ids=[EP[0].name, EP[-1].name])
def test_expert_parallel_bf16_return_matches_oracle(cfg, one_rank_group):
    """The return exchange in bf16: the layer against the oracle's combine of
    its expert outputs rounded to bf16, and half the return bytes."""
    inp, cpu = cuda_inputs(cfg)
    layer = ep.ExpertParallelMoE(inp["w_router"], inp["bias"], inp["w_gate"], inp["w_up"],
                                 inp["w_down"], cfg.k, cfg.cf, return_bf16=True)
    y = layer(inp["x"])
    logits, _, _ = moe.moe_route(inp["x"], inp["w_router"], inp["bias"], cfg.k)
    torch.cuda.synchronize()
    assert dict(layer.exchange_log)["combine_bf16"] == 0       # one rank sends nothing away
    bias = None if cpu["bias"] is None else cpu["bias"].numpy()
    xb = bits(cpu["x"])
    ref = oracle.moe_forward(xb, cpu["w_router"].numpy(), bias, bits(cpu["w_gate"]),
                             bits(cpu["w_up"]), bits(cpu["w_down"]), cfg.k, cfg.cf,
                             decision_logits=logits.cpu().numpy())
    C = oracle.capacity(cfg.T, cfg.E, cfg.k, cfg.cf)
    _, offsets, slot, row_src, _ = oracle.permute(ref["topk_idx"], cfg.E, C)
    _, rows = oracle.expert_mlp(oracle.dispatch(xb, row_src), offsets, bits(cpu["w_gate"]),
                                bits(cpu["w_up"]), bits(cpu["w_down"]))
    rows_b = np.vectorize(oracle.round_bf16)(rows)
    y_ref = oracle.combine(rows_b, xb, ref["topk_idx"], ref["topk_w"], slot, offsets)
    assert_bf16_close(f64(y), y_ref, "y")
