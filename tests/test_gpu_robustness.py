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
                                       seed=23)], ids=["tiny", "pair_tiles"])
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
