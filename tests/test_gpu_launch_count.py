"""The benchmark's launch count (its gpu_launches figure) against the libmoe
kernels the CUDA profiler records for one layer step, in every mode of the
step, with and without a K split in the router, and for the one-shot layer
call its end-to-end leg times."""
import pytest
import torch

import bench
from mixture_experts_layer_36_b200 import configs
from mixture_experts_layer_36_b200.configs import MoEConfig

pytestmark = pytest.mark.gpu

# more 128-token row tiles than SMs: the router runs without a K split
UNSPLIT = MoEConfig("unsplit", T=148 * 128 + 37, d=128, E=16, k=2, f=256, cf=1.25, seed=9)
# more than 4096 chunk-histogram counters (17 chunks x 256 experts): the
# permutation runs its scan kernel
SCANNED = MoEConfig("scanned", T=4352, d=128, E=256, k=8, f=128, cf=1.25, seed=10)
MODES = {"bf16": {}, "fp8": {"fp8": True}, "fused": {"fused": True}, "padded": {"padded": True}}


def _libmoe_kernels(fn):
    from torch.autograd import DeviceType
    from torch.profiler import ProfilerActivity, profile
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CPU, ProfilerActivity.CUDA]) as prof:
        fn()
        torch.cuda.synchronize()
    return [e.name for e in prof.events()
            if e.device_type == DeviceType.CUDA and "moe::" in e.name]


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("cfg", [configs.TINY, UNSPLIT, SCANNED],
                         ids=["tiny", "unsplit", "scanned"])
def test_launch_count_matches_profiler(cfg, mode):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda", 0)
    layer = bench.Layer(cfg, dev, token_seed=cfg.seed, **MODES[mode])
    layer.step()                                   # first call sets kernel attributes
    torch.cuda.synchronize()
    names = _libmoe_kernels(layer.step)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    want = bench.launches_per_step(cfg, sms, fp8=mode == "fp8", padded=mode == "padded",
                                   fused=mode == "fused")
    assert len(names) == want, names
    assert any("router_topk_kernel" in n for n in names) == (cfg is not UNSPLIT)
    assert any("permute_scan_kernel" in n for n in names) == (cfg is SCANNED)
    one_shot = _libmoe_kernels(lambda: layer.layer_forward(layer.x, layer.y))
    assert sorted(one_shot) == sorted(names)
    assert int(layer.status.item()) == 0
