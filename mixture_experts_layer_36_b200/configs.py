"""The five seeded synthetic MoE-layer workloads, by shape.

Shapes follow the pages' own examples where they give one: Mixtral's 8 experts
with top-2 routing ("Expert parallelism vs tensor parallelism", section "Expert
parallelism vs tensor parallelism in one layer"), and the fine-grained
d=7168 / T=8192 / top-8 layer of the dispatch-volume table ("Expert Parallelism
& All-to-All", section "The bandwidth bill").  The capacity factor cf=1.25 is
the glossary's example value ("Expert Parallelism" glossary, capacity entry).

This module holds sizes only: no arithmetic of the method.
"""
from dataclasses import dataclass, replace
from typing import Optional


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int          # tokens in the batch
    d: int          # model width
    E: int          # experts
    k: int          # experts per token (top-k)
    f: int          # expert hidden width (SwiGLU)
    cf: float       # capacity factor; 0 means dropless
    seed: int
    zipf_s: Optional[float] = None  # per-expert router bias -s*ln(rank) when set

    def with_tokens(self, T: int) -> "MoEConfig":
        return replace(self, T=T, name=f"{self.name.split('@')[0]}@T{T}")


TINY = MoEConfig("tiny", T=64, d=128, E=8, k=2, f=256, cf=1.25, seed=0)
MIXTRAL = MoEConfig("mixtral", T=4096, d=4096, E=8, k=2, f=14336, cf=0.0, seed=1)
FINE = MoEConfig("fine_grained", T=8192, d=7168, E=256, k=8, f=2048, cf=1.25, seed=2)
SKEWED = MoEConfig("skewed", T=16384, d=2048, E=64, k=6, f=1408, cf=1.0, seed=3, zipf_s=1.2)
DECODE = MoEConfig("decode", T=256, d=7168, E=256, k=8, f=2048, cf=0.0, seed=4)
DECODE_T = (16, 64, 256)

# Profiling slice of the Mixtral-shaped layer: 2 of its experts with the same
# rows per expert (T*k/E = 1024), so a full ncu capture of the expert GEMMs
# holds under 1 GB on the device while the per-expert GEMM shape is unchanged.
MIXTRAL_SLICE = MoEConfig("mixtral_slice", T=1024, d=4096, E=2, k=2, f=14336, cf=0.0, seed=1)
# Same idea for the fine-grained layer: 16 of its 256 experts, 320 rows each.
FINE_SLICE = MoEConfig("fine_slice", T=512, d=7168, E=16, k=8, f=2048, cf=1.25, seed=2)

# And for the decode layer: 32 of its 256 experts with 8 rows each (as at
# T = 256), about 4 GB of bf16 + e4m3 expert weights on the device.
DECODE_SLICE = MoEConfig("decode_slice", T=32, d=7168, E=32, k=8, f=2048, cf=0.0, seed=4)

# The fine-grained layer's token side (T, d, k, cf: the same x and permuted
# rows, 1.06 GB moved by the permutation) with 16 of its experts, so that a
# capture of the permutation and combine holds a few GB on the device.
FINE_ROWS_SLICE = MoEConfig("fine_rows_slice", T=8192, d=7168, E=16, k=8, f=2048, cf=1.25,
                            seed=2)

ALL = {c.name: c for c in (TINY, MIXTRAL, FINE, SKEWED, DECODE, MIXTRAL_SLICE, FINE_SLICE,
                           DECODE_SLICE, FINE_ROWS_SLICE)}


def by_name(name: str) -> MoEConfig:
    """`name` or `name@T<tokens>` (the decode sweep uses decode@T16 etc.)."""
    base, _, tok = name.partition("@T")
    cfg = ALL[base]
    return cfg.with_tokens(int(tok)) if tok else cfg
