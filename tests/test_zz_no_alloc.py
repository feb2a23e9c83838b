"""moe_permute_noalloc: the permutation for callers that cannot allocate device
memory (or pass any scratch buffer) — for instance an operator plugin that only
receives its declared tensors, or a runtime that plans all device memory up
front.  It must give exactly what moe_permute gives, call after call, although
every call reuses the same library-owned scratch array, and it must accept and
reject exactly the arguments moe_permute accepts and rejects.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import mixture_experts_layer_36_b200 as moe
from moe_testlib import bits, random_routing


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
    # two calls in a row with different shapes, the second at the scratch limit
    cases = [(4096, 256, 256, 8, 1.25, 1), (1000, 128, 64, 6, 1.0, 2),
             (65536, 128, 256, 8, 1.0, 3)]
    for T, d, E, k, cf, seed in cases:
        g = torch.Generator().manual_seed(seed)
        x = torch.randn(T, d, generator=g).to(torch.bfloat16)
        idx_np = random_routing(T, E, k, seed=seed)
        xd, idx = x.cuda(), torch.from_numpy(idx_np).cuda()
        ref = moe.moe_permute(xd, idx, E, cf)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        got = moe.moe_permute_noalloc(xd, idx, E, cf, out=_outputs(T, d, E, k, cf),
                                      dev_status=status)
        torch.cuda.synchronize()
        assert status.item() == 0
        N = int(ref["offsets"][E].item())
        for key in ("counts", "offsets", "slot", "n_dropped"):
            assert torch.equal(got[key], ref[key]), key
        assert torch.equal(got["row_src"][:N], ref["row_src"][:N])
        assert torch.equal(got["x_perm"][:N], ref["x_perm"][:N])
        # and directly against the oracle's permutation and dispatch
        C = oracle.capacity(T, E, k, cf)
        counts, offsets, slot, row_src, n_drop = oracle.permute(idx_np, E, C)
        np.testing.assert_array_equal(got["counts"].cpu().numpy(), counts)
        np.testing.assert_array_equal(got["offsets"].cpu().numpy(), offsets)
        np.testing.assert_array_equal(got["slot"].cpu().numpy(), slot)
        assert int(got["n_dropped"].item()) == n_drop
        np.testing.assert_array_equal(got["row_src"][:N].cpu().numpy(), row_src)
        np.testing.assert_array_equal(bits(got["x_perm"][:N]), oracle.dispatch(bits(x), row_src))


@pytest.mark.gpu
def test_noalloc_reports_out_of_range_experts_like_moe_permute():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    T, d, E, k, cf = 300, 128, 8, 2, 1.0
    idx = torch.from_numpy(random_routing(T, E, k, seed=5)).cuda()
    idx[7, 1] = E              # outside [0, E): dropped and reported (bit 4)
    idx[100, 0] = -1
    x = torch.randn(T, d, device="cuda").to(torch.bfloat16)
    st_ref = torch.zeros(1, dtype=torch.int32, device="cuda")
    st_got = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref = moe.moe_permute(x, idx, E, cf, dev_status=st_ref)
    got = moe.moe_permute_noalloc(x, idx, E, cf, out=_outputs(T, d, E, k, cf), dev_status=st_got)
    torch.cuda.synchronize()
    assert st_ref.item() == 4 and st_got.item() == 4
    assert got["slot"][7, 1].item() == -1 and got["slot"][100, 0].item() == -1
    for key in ("counts", "offsets", "slot", "n_dropped"):
        assert torch.equal(got[key], ref[key]), key


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = moe.lib()
    fake = ctypes.c_void_p(1 << 20)
    outs = [fake] * 6
    # E = 256: (ceil(T/256) + 1) * 256 counters; T = 65536 fits, T = 65537 does not
    too_big = lib.moe_permute_noalloc(fake, fake, 65537, 128, 256, 8, 1.0, *outs, None, None)
    assert too_big == 2  # MOE_ERR_WORKSPACE
    assert lib.moe_permute_noalloc(fake, fake, 0, 128, 256, 8, 1.0, *outs, None, None) == 0
    assert lib.moe_permute_noalloc(fake, fake, 10, 100, 8, 2, 1.0, *outs, None, None) == 4


# (T, d, E, k, cf, which pointer is null or misaligned): every case fails the
# host-side checks, so neither call reaches the GPU
BAD_ARGS = [
    (-1, 128, 8, 2, 1.0, None), (10, 128, 0, 1, 1.0, None), (10, 128, 257, 2, 1.0, None),
    (10, 128, 8, 0, 1.0, None), (10, 128, 8, 9, 1.0, None), (10, 128, 4, 5, 1.0, None),
    (1 << 28, 128, 256, 8, 1.0, None), (10, 0, 8, 2, 1.0, None), (10, 100, 8, 2, 1.0, None),
    (10, 96, 8, 2, 1.0, None), (10, 128, 8, 2, -1.0, None), (10, 128, 8, 2, float("inf"), None),
    (10, 128, 8, 2, float("nan"), None), (0, 128, 8, 2, 1.0, None),
    (10, 128, 8, 2, 1.0, "x"), (10, 128, 8, 2, 1.0, "topk_idx"), (10, 128, 8, 2, 1.0, "counts"),
    (10, 128, 8, 2, 1.0, "offsets"), (10, 128, 8, 2, 1.0, "slot"), (10, 128, 8, 2, 1.0, "row_src"),
    (10, 128, 8, 2, 1.0, "x_perm"), (10, 128, 8, 2, 1.0, "n_dropped"),
    (10, 128, 8, 2, 1.0, "x+8"), (10, 128, 8, 2, 1.0, "x_perm+8"),
]


@pytest.mark.parametrize("T,d,E,k,cf,bad", BAD_ARGS)
def test_noalloc_validates_like_moe_permute(T, d, E, k, cf, bad):
    lib = moe.lib()
    names = ["x", "topk_idx", "counts", "offsets", "slot", "row_src", "x_perm", "n_dropped"]
    ptrs = {n: ctypes.c_void_p((1 << 20) * (i + 1)) for i, n in enumerate(names)}
    if bad and bad.endswith("+8"):
        ptrs[bad[:-2]] = ctypes.c_void_p(ptrs[bad[:-2]].value + 8)
    elif bad:
        ptrs[bad] = None
    args = [ptrs[n] for n in names[:2]], [ptrs[n] for n in names[2:]]
    ws = ctypes.c_void_p(1 << 30)
    want = lib.moe_permute(*args[0], T, d, E, k, cf, *args[1], ws, ctypes.c_size_t(1 << 40),
                           None, None)
    got = lib.moe_permute_noalloc(*args[0], T, d, E, k, cf, *args[1], None, None)
    assert got == want, (got, want)
    assert want != 0 or T == 0
