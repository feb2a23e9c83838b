"""Shared helpers for the parity tests: seeded inputs, oracle calls on them,
and the tolerances every comparison uses.

Tolerances (written once, used everywhere):
  * integer / index results (top-k indices, counts, offsets, slots, drop mask,
    row_src, n_dropped) and pure copies (x_perm, passthrough rows): bit-exact;
  * fp32 logits: |gpu - ref| <= 1e-4 * max(|ref|, rms(ref)) elementwise;
  * fp32 gate weights: |gpu - ref| <= 1e-6 absolute;
  * the layer output y (bf16) and the down GEMM's fp32 rows y_perm:
    max |gpu - ref| <= 2e-2 * rms(ref);
  * the bf16 intermediate h = silu(g) * u, against the oracle's h rounded to
    bf16 as well: elementwise |gpu - ref| <= 2^-7 * |ref| + 1e-3 * rms(ref).
    Both sides round a value to bf16; when the fp32 (GPU) and fp64 (oracle)
    values straddle a rounding boundary the results differ by one bf16 ulp,
    which is at most 2^-7 of the value; the absolute term covers the fp32
    accumulation order and the exponential in silu near zero.  (h is
    heavy-tailed, so a max-relative-to-rms bound would not describe it.)
"""
import numpy as np
import torch

import oracle
from mixture_experts_layer_36_b200 import synth
from mixture_experts_layer_36_b200.configs import MoEConfig

LOGIT_RTOL = 1e-4
WEIGHT_ATOL = 1e-6
BF16_RMS_TOL = 2e-2


def bits(t):
    return oracle.bf16_bits(t)


def f64(t):
    """torch tensor (bf16 or float) -> fp64 numpy, exactly."""
    if t.dtype == torch.bfloat16:
        return oracle.bits_to_f64(bits(t))
    return t.detach().cpu().double().numpy()


def assert_logits_close(gpu, ref64):
    ref = np.asarray(ref64, np.float64)
    g = np.asarray(gpu, np.float64)
    rms = np.sqrt(np.mean(ref ** 2)) if ref.size else 0.0
    bound = LOGIT_RTOL * np.maximum(np.abs(ref), rms)
    err = np.abs(g - ref)
    assert np.all(err <= bound), f"logits: worst excess {np.max(err - bound):.3e}"


def assert_bf16_close(gpu, ref64, what):
    ref = np.asarray(ref64, np.float64)
    g = np.asarray(gpu, np.float64)
    assert g.shape == ref.shape, (what, g.shape, ref.shape)
    if ref.size == 0:
        return
    rms = np.sqrt(np.mean(ref ** 2))
    err = np.max(np.abs(g - ref))
    assert err <= BF16_RMS_TOL * rms, f"{what}: max|err| {err:.4e} > {BF16_RMS_TOL} * rms {rms:.4e}"


H_REL_TOL = 2.0 ** -7
H_ABS_RMS_TOL = 1e-3


def assert_bf16_rounding_close(gpu, ref64, what):
    ref = np.asarray(ref64, np.float64)
    g = np.asarray(gpu, np.float64)
    assert g.shape == ref.shape, (what, g.shape, ref.shape)
    if ref.size == 0:
        return
    rms = np.sqrt(np.mean(ref ** 2))
    bound = H_REL_TOL * np.abs(ref) + H_ABS_RMS_TOL * rms
    excess = np.abs(g - ref) - bound
    i = np.unravel_index(np.argmax(excess), excess.shape)
    assert excess[i] <= 0, (f"{what}: at {i} gpu {g[i]:.6g} ref {ref[i]:.6g} "
                            f"exceeds the bf16-rounding bound by {excess[i]:.3e}")


def small(name, T, d, E, k, f, cf, seed, zipf_s=None):
    return MoEConfig(name, T=T, d=d, E=E, k=k, f=f, cf=cf, seed=seed, zipf_s=zipf_s)


def cuda_inputs(cfg, device="cuda"):
    """Seeded inputs drawn on the CPU (small shapes) and copied to the GPU."""
    cpu = synth.make_inputs(cfg, "cpu")
    return {k: (None if v is None else v.to(device)) for k, v in cpu.items()}, cpu


def random_routing(T, E, k, seed, skew=1.2):
    """A seeded (token -> k distinct experts) table with Zipf-skewed
    popularity so that capacity limits bite."""
    r = np.random.default_rng(seed)
    p = 1.0 / np.arange(1, E + 1) ** skew
    p /= p.sum()
    keys = r.random((T, E)) ** (1.0 / p)      # weighted sampling without replacement
    return np.argsort(-keys, axis=1)[:, :k].astype(np.int32)
