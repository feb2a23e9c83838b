"""The C-ABI library without a GPU: it loads, exports every entry point that
include/moe.h declares, and its host-side arithmetic and validation behave as
documented (no kernel is launched by any call here)."""
import ctypes
import os
import re

import pytest

import oracle
import mixture_experts_layer_36_b200 as moe
from mixture_experts_layer_36_b200 import binding, configs

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "moe.h")

OK, INVALID, WORKSPACE, CUDA, UNSUPPORTED = 0, 1, 2, 3, 4
FAKE = ctypes.c_void_p(1 << 20)   # aligned non-null pointer; never dereferenced on these paths


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 14
    lib = ctypes.CDLL(binding.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(binding.EXPORTED) == names


def test_version_and_status_strings():
    assert moe.lib().moe_version() >> 16 == 1
    assert moe.moe_status_string(0) == "MOE_OK"
    assert moe.moe_status_string(4) == "MOE_ERR_UNSUPPORTED"
    assert moe.moe_status_string(99) == "MOE_ERR_UNKNOWN"


@pytest.mark.parametrize("T,E,k,cf", [(64, 8, 2, 1.25), (8192, 256, 8, 1.25), (16384, 64, 6, 1.0),
                                      (4096, 8, 2, 0.0), (10, 3, 1, 1.0), (7, 5, 2, 3.3),
                                      (0, 4, 2, 1.0)])
def test_capacity_agrees_with_oracle(T, E, k, cf):
    assert moe.moe_capacity(T, E, k, cf) == oracle.capacity(T, E, k, cf)
    C = oracle.capacity(T, E, k, cf)
    assert moe.moe_max_rows(T, E, k, cf) == min(T * k, E * C)


def test_capacity_rejects_bad_args():
    assert moe.moe_capacity(10, 0, 1, 1.0) == -1
    assert moe.moe_capacity(10, 4, 0, 1.0) == -1
    assert moe.moe_capacity(10, 4, 1, -1.0) == -1
    assert moe.moe_capacity(10, 4, 1, float("nan")) == -1


@pytest.mark.parametrize("cfg", list(configs.ALL.values()), ids=list(configs.ALL))
def test_workspace_layout(cfg):
    T, d, E, k, f, cf = cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, cfg.cf
    total = moe.moe_workspace_size(T, d, E, k, f, cf)
    offs = [moe.moe_workspace_field_offset(i, T, d, E, k, f, cf) for i in range(14)]
    assert offs[0] == 0 and all(o % 256 == 0 for o in offs)
    assert offs == sorted(offs)
    rows = moe.moe_max_rows(T, E, k, cf)
    ends = offs[1:] + [total]
    need = {1: T * E * 4, 2: T * k * 4, 3: T * k * 4, 4: T * k * 4, 5: E * 4, 6: (E + 1) * 4,
            8: rows * 4, 9: moe.moe_permute_workspace_size(T, E, k), 10: rows * d * 2,
            11: rows * f * 2, 12: rows * d * 4, 13: moe.moe_route_workspace_size(T, d, E, k)}
    for i, n in need.items():
        assert ends[i] - offs[i] >= n, binding.WS_FIELDS[i]
    assert moe.moe_route_workspace_size(T, d, E, k) >= 2 * d * ((E + 63) // 64 * 64) * 2
    # the FP8 layer's extra fields follow the standard ones
    total8 = moe.moe_workspace_size_fp8(T, d, E, k, f, cf)
    offs8 = [moe.moe_workspace_field_offset(i, T, d, E, k, f, cf) for i in range(14, 20)]
    assert offs8[0] == total and all(o % 256 == 0 for o in offs8) and offs8 == sorted(offs8)
    ends8 = offs8[1:] + [total8]
    for i, n in enumerate((rows * d, rows * 4, rows * f, rows * 4, T * d, T * 4)):
        assert ends8[i] - offs8[i] >= n, binding.WS_FIELDS[14 + i]
    # and so do the fused layer's (independently of the FP8 ones)
    o_pair = moe.moe_workspace_field_offset(20, T, d, E, k, f, cf)
    o_y32 = moe.moe_workspace_field_offset(21, T, d, E, k, f, cf)
    assert o_pair == total and o_y32 >= o_pair + rows * 4 and o_y32 % 256 == 0
    assert moe.moe_workspace_size_fused(T, d, E, k, f, cf) >= o_y32 + T * d * 4
    assert moe.moe_workspace_field_offset(22, T, d, E, k, f, cf) == -1
    assert moe.moe_workspace_field_offset(-1, T, d, E, k, f, cf) == -1


def test_validation_codes_without_launch():
    L = moe.lib()
    s = ctypes.c_void_p(0)
    # route: bad E, bad k, k > E, unsupported width, empty batch, small workspace
    R = moe.moe_route_workspace_size(4, 128, 8, 2)
    W = [FAKE, R, None, s]
    assert L.moe_route(FAKE, FAKE, None, 4, 128, 0, 1, FAKE, FAKE, FAKE, *W) == INVALID
    assert L.moe_route(FAKE, FAKE, None, 4, 128, 300, 2, FAKE, FAKE, FAKE, *W) == INVALID
    assert L.moe_route(FAKE, FAKE, None, 4, 128, 8, 9, FAKE, FAKE, FAKE, *W) == INVALID
    assert L.moe_route(FAKE, FAKE, None, 4, 128, 2, 3, FAKE, FAKE, FAKE, *W) == INVALID
    assert L.moe_route(FAKE, FAKE, None, 4, 100, 8, 2, FAKE, FAKE, FAKE, *W) == UNSUPPORTED
    assert L.moe_route(None, FAKE, None, 4, 128, 8, 2, FAKE, FAKE, FAKE, *W) == INVALID
    assert L.moe_route(FAKE, FAKE, None, 0, 128, 8, 2, FAKE, FAKE, FAKE, *W) == OK
    assert L.moe_route(FAKE, FAKE, None, 4, 128, 8, 2, FAKE, FAKE, FAKE, FAKE, R - 1, None, s) \
        == WORKSPACE
    misaligned = ctypes.c_void_p((1 << 20) + 2)
    assert L.moe_route(misaligned, FAKE, None, 4, 128, 8, 2, FAKE, FAKE, FAKE, *W) == INVALID
    # permute: workspace too small
    need = moe.moe_permute_workspace_size(100, 8, 2)
    assert need > 0
    args = [FAKE, FAKE, 100, 128, 8, 2, 1.25, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE]
    assert L.moe_permute(*args, need - 1, None, s) == WORKSPACE
    assert L.moe_permute(*args[:6], -1.0, *args[7:], need, None, s) == INVALID
    # experts: widths must be multiples of 64
    assert L.moe_expert_gate_up(FAKE, FAKE, 8, 200, 256, 100, FAKE, FAKE, FAKE, None, s) \
        == UNSUPPORTED
    assert L.moe_expert_gate_up(FAKE, FAKE, 8, 256, 96, 100, FAKE, FAKE, FAKE, None, s) \
        == UNSUPPORTED
    assert L.moe_expert_down(FAKE, FAKE, 8, 256, 200, 100, FAKE, FAKE, None, s) == UNSUPPORTED
    assert L.moe_expert_mlp(FAKE, FAKE, 8, 256, 256, 0, FAKE, FAKE, FAKE, FAKE, FAKE, None, s) \
        == OK
    # tile counts that would overflow the kernels' 32-bit tile indices
    assert L.moe_expert_gate_up(FAKE, FAKE, 8, 1 << 20, 1 << 20, (1 << 31) - 1, FAKE, FAKE, FAKE,
                                None, s) == UNSUPPORTED
    # combine / layer
    assert L.moe_combine(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 10, 128, 9, FAKE, s) == INVALID
    assert L.moe_combine_bf16rows(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 10, 128, 9, FAKE, s) \
        == INVALID
    assert L.moe_combine_bf16rows(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 10, 96, 2, FAKE, s) \
        == UNSUPPORTED
    assert L.moe_combine_bf16rows(None, FAKE, FAKE, FAKE, FAKE, FAKE, 10, 128, 2, FAKE, s) \
        == INVALID
    assert L.moe_combine_bf16rows(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 128, 2, FAKE, s) == OK
    # fp32 -> bf16 rows
    assert L.moe_rows_to_bf16(FAKE, FAKE, 10, 100, s) == UNSUPPORTED
    assert L.moe_rows_to_bf16(FAKE, FAKE, -1, 128, s) == INVALID
    assert L.moe_rows_to_bf16(FAKE, FAKE, 1 << 31, 128, s) == INVALID
    assert L.moe_rows_to_bf16(None, FAKE, 10, 128, s) == INVALID
    assert L.moe_rows_to_bf16(FAKE, ctypes.c_void_p((1 << 20) + 8), 10, 128, s) == INVALID
    assert L.moe_rows_to_bf16(FAKE, FAKE, 0, 128, s) == OK
    ws_need = moe.moe_workspace_size(64, 128, 8, 2, 256, 1.25)
    assert L.moe_layer_forward(FAKE, FAKE, None, FAKE, FAKE, FAKE, 64, 128, 8, 2, 256, 1.25, FAKE,
                               FAKE, ws_need - 1, s) == WORKSPACE
    assert L.moe_layer_forward(FAKE, FAKE, None, FAKE, FAKE, FAKE, 64, 128, 8, 2, 250, 1.25, FAKE,
                               FAKE, ws_need, s) == UNSUPPORTED
    assert L.moe_layer_forward(FAKE, FAKE, None, FAKE, FAKE, FAKE, 0, 128, 8, 2, 256, 1.25, FAKE,
                               FAKE, 0, s) == OK
    outs = [None] * 5
    assert L.moe_layer_forward_ex(FAKE, FAKE, None, FAKE, FAKE, FAKE, 64, 128, 8, 2, 250, 1.25,
                                  FAKE, *outs, FAKE, ws_need, s) == UNSUPPORTED
    assert L.moe_layer_forward_ex(FAKE, FAKE, None, FAKE, FAKE, FAKE, 64, 128, 8, 2, 256, 1.25,
                                  FAKE, *outs, FAKE, ws_need - 1, s) == WORKSPACE
    assert L.moe_layer_forward_ex(FAKE, FAKE, None, FAKE, FAKE, FAKE, 0, 128, 8, 2, 256, 1.25,
                                  FAKE, *outs, FAKE, 0, s) == OK


def test_validation_codes_of_the_variants_without_launch():
    """FP8, padded, fused and bucket entry points: each case below fails (or
    returns early on an empty input) before anything reaches the GPU."""
    L = moe.lib()
    s = ctypes.c_void_p(0)
    F = FAKE
    odd = ctypes.c_void_p((1 << 20) + 4)          # not 16-byte aligned
    # ---- FP8
    assert L.moe_quantize_weights_fp8(F, 0, 64, 64, F, F, s) == INVALID
    assert L.moe_quantize_weights_fp8(None, 2, 64, 64, F, F, s) == INVALID
    assert L.moe_quantize_rows_fp8(F, 10, 24, None, F, F, s) == INVALID       # K % 16
    assert L.moe_quantize_rows_fp8(F, 0, 64, None, F, F, s) == OK
    assert L.moe_quantize_rows_fp8(odd, 10, 64, None, F, F, s) == INVALID
    assert L.moe_quantize_rows_fp8(F, 10, 64, None, None, F, s) == INVALID
    need = moe.moe_permute_workspace_size(100, 8, 2)
    p8 = [F, F, F, 100, 128, 8, 2, 1.25, F, F, F, F, F, F, F, F]
    assert L.moe_permute_fp8(*p8, need - 1, None, s) == WORKSPACE
    assert L.moe_permute_fp8(*p8[:7], -1.0, *p8[8:], need, None, s) == INVALID
    assert L.moe_permute_fp8(None, *p8[1:], need, None, s) == INVALID
    assert L.moe_permute_fp8(*p8[:3], 0, *p8[4:], 0, None, s) == OK
    g8 = [F, F, F, 8, 256, 256, 100, F, F, F, F, F, None, s]
    assert L.moe_expert_gate_up_fp8(*g8[:4], 200, *g8[5:]) == UNSUPPORTED
    assert L.moe_expert_gate_up_fp8(*g8[:6], 0, *g8[7:]) == OK
    assert L.moe_expert_gate_up_fp8(None, *g8[1:]) == INVALID
    d8 = [F, F, F, 8, 256, 256, 100, F, F, F, None, s]
    assert L.moe_expert_down_fp8(*d8[:5], 200, *d8[6:]) == UNSUPPORTED
    assert L.moe_expert_down_fp8(*d8[:9], odd, *d8[10:]) == INVALID
    ws8 = moe.moe_workspace_size_fp8(64, 128, 8, 2, 256, 1.25)
    assert ws8 > moe.moe_workspace_size(64, 128, 8, 2, 256, 1.25)
    l8 = [F] * 9
    assert L.moe_layer_forward_fp8(*l8, 64, 128, 8, 2, 256, 1.25, F, F, ws8 - 1, s) == WORKSPACE
    assert L.moe_layer_forward_fp8(*l8, 64, 128, 8, 2, 250, 1.25, F, F, ws8, s) == UNSUPPORTED
    assert L.moe_layer_forward_fp8(*l8, 0, 128, 8, 2, 256, 1.25, F, F, 0, s) == OK
    # ---- padded layout
    pp = [F, F, 100, 128, 8, 2, 1.25, F, F, F, F, F, F, F]
    assert L.moe_permute_padded(*pp, need - 1, None, s) == WORKSPACE
    assert moe.moe_padded_rows(1 << 27, 256, 8, 0.0) == -1                    # E*C >= 2^31
    assert L.moe_permute_padded(F, F, 1 << 27, 128, 256, 8, 0.0, *pp[7:], need, None, s) \
        == INVALID
    # ---- buckets (expert parallelism)
    bk = [F, F, None, 6, 4, 256, 256, 100, F, F, F, F, F, None, s]
    assert L.moe_expert_mlp_buckets(*bk) == INVALID                           # 6 % 4 != 0
    assert L.moe_expert_mlp_buckets(*bk[:4], 0, *bk[5:]) == INVALID
    assert L.moe_expert_mlp_buckets(*bk[:3], 8, 4, 256, 256, 0, *bk[8:]) == OK
    # ---- fused path
    pf = [F, F, 100, 128, 8, 2, 1.25, F, F, F, F, F, F, F, F, F]
    assert L.moe_permute_fused(*pf, need - 1, None, s) == WORKSPACE
    assert L.moe_permute_fused(*pf[:12], None, *pf[13:], need, None, s) == INVALID  # x w/o x_perm
    assert L.moe_permute_fused(*pf[:14], odd, F, need, None, s) == INVALID          # y32 aligned
    ga = [F, 5, F, F, 8, 256, 256, 100, F, F, F, None, s]
    assert L.moe_expert_gate_up_gather(ga[0], 0, *ga[2:]) == INVALID
    assert L.moe_expert_gate_up_gather(*ga[:7], 0, *ga[8:]) == OK
    ds = [F, F, 8, 256, 256, 100, F, F, F, 2, F, None, s]
    assert L.moe_expert_down_scatter(*ds[:9], 0, *ds[10:]) == INVALID
    assert L.moe_expert_down_scatter(*ds[:9], 9, *ds[10:]) == INVALID
    assert L.moe_expert_down_scatter(*ds[:10], None, *ds[11:]) == INVALID
    assert L.moe_combine_finalize(F, F, F, 10, 128, 0, F, s) == INVALID
    assert L.moe_combine_finalize(F, F, F, 10, 100, 2, F, s) == UNSUPPORTED
    assert L.moe_combine_finalize(F, F, F, 0, 128, 2, F, s) == OK
    wsf = moe.moe_workspace_size_fused(64, 128, 8, 2, 256, 1.25)
    assert wsf > moe.moe_workspace_size(64, 128, 8, 2, 256, 1.25)
    lf = [F] * 6
    assert L.moe_layer_forward_fused(*lf, 64, 128, 8, 2, 256, 1.25, F, F, wsf - 1, s) == WORKSPACE
    assert L.moe_layer_forward_fused(*lf, 0, 128, 8, 2, 256, 1.25, F, F, 0, s) == OK


def test_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(4, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        moe.moe_route(x, torch.zeros(128, 8), None, 2)
