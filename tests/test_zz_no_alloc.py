"""moe_permute_noalloc: the permutation for callers that cannot allocate device
memory (or pass any scratch buffer) — for instance an operator plugin that only
receives its declared tensors, or a runtime that plans all device memory up
front.  It must give exactly what moe_permute gives, call after call, although
every call reuses the same library-owned scratch array.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import pytest
import torch

import mixture_experts_layer_36_b200 as moe
from moe_testlib import random_routing


def _outputs(T, d, E, k, cf, device="cuda", fill=-3):
    rows = max(moe.moe_max_rows(T, E, k, cf), 1)
    z = lambda *s, dt: torch.full(s, fill, dtype=dt, device=device)  # noqa: E731
    return {"counts": z(E, dt=torch.int32), "offsets": z(E + 1, dt=torch.int32),
            "slot": z(T, k, dt=torch.int32), "row_src": z(rows, dt=torch.int32),
            "x_perm": torch.zeros(rows, d, dtype=torch.bfloat16, device=device),
            "n_dropped": z(1, dt=torch.int32)}


@pytest.mark.gpu
def test_noalloc_permute_matches_moe_permute_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    cases = [(4096, 256, 256, 8, 1.25, 1), (1000, 128, 64, 6, 1.0, 2)]
    for T, d, E, k, cf, seed in cases:          # two calls in a row, different shapes
        g = torch.Generator().manual_seed(seed)
        x = torch.randn(T, d, generator=g).to(torch.bfloat16).cuda()
        idx = torch.from_numpy(random_routing(T, E, k, seed=seed)).cuda()
        ref = moe.moe_permute(x, idx, E, cf)
        got = moe.moe_permute_noalloc(x, idx, E, cf, out=_outputs(T, d, E, k, cf))
        torch.cuda.synchronize()
        N = int(ref["offsets"][E].item())
        for key in ("counts", "offsets", "slot", "n_dropped"):
            assert torch.equal(got[key], ref[key]), key
        assert torch.equal(got["row_src"][:N], ref["row_src"][:N])
        assert torch.equal(got["x_perm"][:N], ref["x_perm"][:N])


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = moe.lib()
    fake = ctypes.c_void_p(1 << 20)
    args = [fake, fake]
    # E = 256: ceil(T/256) * 256 counters; T = 65536 fits, T = 65537 does not
    too_big = lib.moe_permute_noalloc(*args, 65537, 128, 256, 8, 1.0, *([fake] * 6), None)
    assert too_big == 2  # MOE_ERR_WORKSPACE
    assert lib.moe_permute_noalloc(*args, 0, 128, 256, 8, 1.0, *([fake] * 6), None) == 0
    assert lib.moe_permute_noalloc(*args, 10, 100, 8, 2, 1.0, *([fake] * 6), None) == 4
