"""Workload shapes of the routed-branch forward (sizes only, no arithmetic).

Each entry names a layer by what it is.  L tokens of width d, an N_r x N_c grid
of atomic experts (N = N_r * N_c), K experts per token, groups of B experts.
"""
from __future__ import annotations

from dataclasses import dataclass, asdict


@dataclass(frozen=True)
class LayerConfig:
    name: str
    L: int
    d: int
    N_r: int
    N_c: int
    K: int
    B: int
    zipf: bool = False          # additive Zipf(s=1.1) log-bias on router rows/columns

    @property
    def N(self) -> int:
        return self.N_r * self.N_c

    @property
    def G(self) -> int:
        return (self.N + self.B - 1) // self.B

    @property
    def M(self) -> int:
        return self.L * self.K

    def with_L(self, L: int) -> "LayerConfig":
        return LayerConfig(f"{self.name.split('_L')[0]}_L{L}", L, self.d, self.N_r, self.N_c,
                           self.K, self.B, self.zipf)

    def asdict(self) -> dict:
        out = asdict(self)
        out["N"] = self.N
        return out


TINY = LayerConfig("tiny_L256_d256_N4096_K16_B32", 256, 256, 64, 64, 16, 32)
SMALL = LayerConfig("small_L4096_d768_N262144_K64_B64", 4096, 768, 512, 512, 64, 64)
HEADLINE = LayerConfig("headline_L4096_d1024_N1700416_K64_B128", 4096, 1024, 1304, 1304, 64, 128)
SKEW = LayerConfig("skew_L16384_d2048_N1048576_K128_B128_zipf", 16384, 2048, 1024, 1024, 128, 128,
                   zipf=True)
SWEEP_BASE = LayerConfig("sweep_d2048_N1700416_K64_B128", 4096, 2048, 1304, 1304, 64, 128)
SWEEP_L = (1, 16, 256, 4096, 65536)


def sweep(L: int) -> LayerConfig:
    return LayerConfig(f"sweep_L{L}_d2048_N1700416_K64_B128", L, 2048, 1304, 1304, 64, 128)


# Headline task structure at a size small enough for full profiler captures:
# the same L, d, K, tasks (M = 262,144) and tasks per group (L*K*B/N = 20),
# with W and V of 512 MB each (N = 512^2) instead of 3.5 GB.
PROFILE = LayerConfig("profile_L4096_d1024_N262144_K64_B20", 4096, 1024, 512, 512, 64, 20)

# The skewed layer's router (1024 x 1024 grid, K = 128, Zipf bias) at 4096
# tokens, for profiler captures of the router stage (which never touches W, V).
SKEW_ROUTER_PROFILE = LayerConfig("skew_router_profile_L4096_d2048_N1048576_K128_B128_zipf", 4096,
                                  2048, 1024, 1024, 128, 128, zipf=True)


def mlp_hidden(d: int) -> int:
    """Hidden width F of the shared dense MLP beside a layer of width d: 8d/3
    rounded up to a multiple of 64 (the width at which a gated MLP has the
    weights of a plain two-matrix MLP of width 4d)."""
    return -(-8 * d // (3 * 64)) * 64


# One decode token at the sweep's width on a 512 x 512 grid (W and V of 1 GB
# each), for profiler captures of the fused decode step.
DECODE_PROFILE = LayerConfig("decode_profile_L1_d2048_N262144_K64_B128", 1, 2048, 512, 512, 64, 128)

ALL = [TINY, SMALL, HEADLINE, SKEW] + [sweep(L) for L in SWEEP_L] + [PROFILE, SKEW_ROUTER_PROFILE,
                                                                    DECODE_PROFILE]
BY_NAME = {c.name: c for c in ALL}
