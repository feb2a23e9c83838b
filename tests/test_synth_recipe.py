"""The seeded synthetic inputs follow their stated recipe (synth.py): x drawn
N(0, 1) in fp32 and rounded to bf16 (nearest even), router weights N(0, 1/d),
gate / up weights N(0, 1/d) and down weights N(0, 1/f) in bf16, the skewed
workload's router bias -s ln(e + 1), one independent reproducible stream per
tensor and seed."""
import math

import numpy as np
import torch

from mixture_experts_layer_36_b200 import configs, synth
from mixture_experts_layer_36_b200.configs import MoEConfig

CFG = MoEConfig("recipe", T=512, d=256, E=4, k=2, f=384, cf=1.0, seed=11)


def _std_ok(t, want, n_sigma=5.0):
    v = t.double().flatten()
    n = v.numel()
    # sample std of n normals: relative standard error ~ 1/sqrt(2n)
    assert abs(v.std().item() / want - 1.0) < n_sigma / math.sqrt(2 * n)
    assert abs(v.mean().item()) < n_sigma * want / math.sqrt(n)


def test_tokens_are_rounded_normal_draws():
    x = synth.make_tokens(CFG, "cpu")
    assert x.dtype == torch.bfloat16 and tuple(x.shape) == (CFG.T, CFG.d)
    g = synth._gen("cpu", CFG.seed, "x")
    x32 = torch.randn(CFG.T, CFG.d, generator=g, dtype=torch.float32)
    assert torch.equal(x, x32.to(torch.bfloat16))          # round to nearest even
    _std_ok(x32, 1.0)


def test_weight_scales():
    w = synth.make_weights(CFG, "cpu")
    assert w["w_router"].dtype == torch.float32 and tuple(w["w_router"].shape) == (CFG.d, CFG.E)
    _std_ok(w["w_router"], 1 / math.sqrt(CFG.d))
    for n, shape, fan_in in (("w_gate", (CFG.E, CFG.d, CFG.f), CFG.d),
                             ("w_up", (CFG.E, CFG.d, CFG.f), CFG.d),
                             ("w_down", (CFG.E, CFG.f, CFG.d), CFG.f)):
        assert w[n].dtype == torch.bfloat16 and tuple(w[n].shape) == shape
        _std_ok(w[n], 1 / math.sqrt(fan_in))
    assert w["bias"] is None


def test_skewed_bias_is_log_zipf_rank_weight():
    b = synth.router_bias(configs.SKEWED)
    e = np.arange(configs.SKEWED.E, dtype=np.float64)
    want = (-configs.SKEWED.zipf_s * np.log(e + 1.0)).astype(np.float32)
    np.testing.assert_array_equal(b.numpy(), want)
    assert b[0].item() == 0.0 and np.all(np.diff(b.numpy()) < 0)   # expert 0 hottest
    assert synth.router_bias(configs.MIXTRAL) is None


def test_streams_reproducible_and_independent():
    a, b = synth.make_weights(CFG, "cpu"), synth.make_weights(CFG, "cpu")
    for n in ("w_router", "w_gate", "w_up", "w_down"):
        assert torch.equal(a[n], b[n])
    # gate and up come from different streams: uncorrelated
    g, u = a["w_gate"].double().flatten(), a["w_up"].double().flatten()
    corr = torch.corrcoef(torch.stack([g, u]))[0, 1].item()
    assert abs(corr) < 5 / math.sqrt(g.numel())
    # a token seed gives another batch; the default seed is the config's
    assert torch.equal(synth.make_tokens(CFG, "cpu"), synth.make_tokens(CFG, "cpu", seed=CFG.seed))
    assert not torch.equal(synth.make_tokens(CFG, "cpu"), synth.make_tokens(CFG, "cpu", seed=12))
