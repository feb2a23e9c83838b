"""Device-side robustness: time-limited waits end with a status word (no
hang), and the whole layer replays inside a CUDA graph."""
import time

import pytest
import torch

import mixture_experts_layer_36_b200 as moe
from mixture_experts_layer_36_b200 import configs, synth
from moe_testlib import cuda_inputs, small

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_bounded_wait_times_out_and_reports():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    moe.moe_selftest_bounded_wait(status, 50_000_000)       # 50 ms, nothing ever arrives
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert status.item() == moe.binding.DEV_ERR_WAIT_TIMEOUT
    assert 0.04 < elapsed < 5.0
    # the context is still usable: a full layer runs and reports no error
    cfg = configs.TINY
    inp, _ = cuda_inputs(cfg)
    y, ws = moe.moe_layer_forward(inp["x"], inp["w_router"], inp["bias"], inp["w_gate"],
                                  inp["w_up"], inp["w_down"], cfg.k, cfg.cf)
    torch.cuda.synchronize()
    st = moe.workspace_view(ws, "status", cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, cfg.cf)
    assert st.item() == 0 and torch.isfinite(y.float()).all()


@pytest.mark.parametrize("cfg", [configs.TINY,
                                 small("graph_pairs", T=2048, d=256, E=4, k=2, f=256, cf=0.0,
                                       seed=23),
                                 # 256 buffer rows per expert: the expert-tail pair tiles,
                                 # whose tile counter must be back at zero for every replay
                                 small("graph_tails", T=1024, d=256, E=16, k=4, f=256,
                                       cf=1.25, seed=25)],
                         ids=["tiny", "pair_tiles", "expert_tails"])
def test_layer_forward_replays_in_cuda_graph(cfg):
    inp, _ = cuda_inputs(cfg)
    x = inp["x"].clone()
    y = torch.empty_like(x)
    ws = torch.empty(moe.moe_workspace_size(cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, cfg.cf),
                     dtype=torch.uint8, device="cuda")
    args = (inp["w_router"], inp["bias"], inp["w_gate"], inp["w_up"], inp["w_down"], cfg.k, cfg.cf)
    moe.moe_layer_forward(x, *args, y=y, ws=ws)                 # first call outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        moe.moe_layer_forward(x, *args, y=y, ws=ws)
    for seed in (5, 6):
        x.copy_(synth.make_tokens(cfg, "cuda", seed=seed))
        g.replay()
        torch.cuda.synchronize()
        ref, _ = moe.moe_layer_forward(x.clone(), *args)
        torch.cuda.synchronize()
        assert torch.equal(y, ref)


def _replay_check(cfg, forward, ws_size, compare):
    """Capture forward(x, y, ws) in a CUDA graph after one eager call, replay it
    on new tokens and compare y with a fresh eager call via compare(y, ref)."""
    inp, _ = cuda_inputs(cfg)
    x = inp["x"].clone()
    y = torch.empty_like(x)
    ws = torch.empty(ws_size, dtype=torch.uint8, device="cuda")
    forward(inp, x, y, ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        forward(inp, x, y, ws)
    for seed in (7, 8):
        x.copy_(synth.make_tokens(cfg, "cuda", seed=seed))
        g.replay()
        torch.cuda.synchronize()
        ref = torch.empty_like(x)
        forward(inp, x.clone(), ref, torch.empty_like(ws))
        torch.cuda.synchronize()
        compare(y, ref)


GRAPH_CFG = small("graph_drops", T=700, d=256, E=8, k=2, f=256, cf=0.75, seed=24)


def test_fp8_layer_replays_in_cuda_graph():
    cfg = GRAPH_CFG
    q = {}

    def forward(inp, x, y, ws):
        if not q:
            q.update({n: moe.moe_quantize_weights_fp8(inp[n]) for n in ("w_gate", "w_up",
                                                                         "w_down")})
        moe.moe_layer_forward_fp8(x, inp["w_router"], inp["bias"], *q["w_gate"], *q["w_up"],
                                  *q["w_down"], cfg.k, cfg.cf, y=y, ws=ws)

    size = moe.moe_workspace_size_fp8(cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, cfg.cf)
    _replay_check(cfg, forward, size, lambda a, b: torch.equal(a, b) or pytest.fail("y differs"))


def test_fused_layer_replays_in_cuda_graph():
    from moe_testlib import assert_bf16_close, f64
    cfg = GRAPH_CFG

    def forward(inp, x, y, ws):
        moe.moe_layer_forward_fused(x, inp["w_router"], inp["bias"], inp["w_gate"], inp["w_up"],
                                    inp["w_down"], cfg.k, cfg.cf, y=y, ws=ws)

    size = moe.moe_workspace_size_fused(cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, cfg.cf)
    # the fused sums run in tile-completion order: equal up to fp32 rounding
    _replay_check(cfg, forward, size, lambda a, b: assert_bf16_close(f64(a), f64(b), "y"))


def test_permute_out_of_range_expert_ids_are_dropped_and_reported():
    """A caller-given top-k table with expert ids outside [0, E): the kernels'
    bounds checks treat those pairs as dropped (slot -1, no bucket place, no
    row written) and set status bit 4; every other pair is placed exactly as
    the oracle places the valid pairs."""
    import numpy as np
    import oracle
    from moe_testlib import bits, random_routing
    T, d, E, k, cf = 300, 128, 8, 2, 0.75
    idx = random_routing(T, E, k, seed=41)
    bad = np.zeros_like(idx, dtype=bool)
    bad[5, 0], bad[17, 1], bad[250, 0] = True, True, True
    idx_bad = idx.copy()
    idx_bad[5, 0], idx_bad[17, 1], idx_bad[250, 0] = -1, E, 1 << 20
    g = torch.Generator().manual_seed(42)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = moe.moe_permute(x.cuda(), torch.from_numpy(idx_bad).cuda(), E, cf, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 4
    # expected: the invalid pairs moved to an extra expert E, which is then dropped
    C = oracle.capacity(T, E, k, cf)
    idx_ref = np.where(bad, E, idx).astype(np.int32)
    counts, offsets, slot, row_src, _ = oracle.permute(idx_ref, E + 1, C)
    slot = np.where(bad, -1, slot)
    N = int(offsets[E])
    np.testing.assert_array_equal(out["slot"].cpu().numpy(), slot)
    np.testing.assert_array_equal(out["counts"].cpu().numpy(), counts[:E])
    np.testing.assert_array_equal(out["offsets"].cpu().numpy(), offsets[:E + 1])
    np.testing.assert_array_equal(out["row_src"][:N].cpu().numpy(), row_src[:N])
    np.testing.assert_array_equal(bits(out["x_perm"][:N]), oracle.dispatch(bits(x), row_src[:N]))
    valid_drops = int(((slot < 0) & ~bad).sum())
    assert out["n_dropped"].item() == valid_drops
