"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This module holds only random-number generation and the bf16 storage
rounding of the draws; none of the quantization or GEMM arithmetic lives
here. Both the CUDA path and the CPU oracle receive the same host bytes.

Workload shapes follow the projections the pages quote (dispatch_proj.rs,
`cublas_fp8_proj`; fp8_act_quant_floor.rs, header tables): decode widths
M in {16, 17, 25} and prefill widths M in {1168, 4576}, with K in
{5120, 6144, 17408}. The pages publish no dataset; these draws stand in:

  X  bf16 [M, K]:  N(0, 1); each entry independently replaced, with
                   probability p, by a draw from N(0, sigma)  (outliers)
  W  bf16 [N, K]:  N(0, 0.02)

The dense FFN (dispatch_proj.rs, doc of `cublas_fp8_proj_prequant`) is
taken at hidden size D = 5120 and intermediate size I = 17408, the two
projection shapes above (gate/up: N = 17408, K = 5120; down: N = 5120,
K = 17408); its gate and up weights are one [2I, D] draw, gate rows first.
For the SiLU-and-multiply step alone, gate and up are drawn like the
projections' outputs: N(0, 3) (sqrt(5120) * 0.02 * rms(X) ~ 3), bf16.

Generator: numpy PCG64 seeded with (1000 + config number, tag, M, K) so
every shape has its own stream; fp32 draws are rounded to bf16 with
round-to-nearest-even.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

_TAG_X = 1
_TAG_W = 2
_TAG_GATE = 3
_TAG_UP = 4


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round finite fp32 values to bf16 (nearest, ties to even); return the uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (np.ascontiguousarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(seed: int, tag: int, a: int, b: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(tag), int(a), int(b)])


def activations(m: int, k: int, seed: int, outlier_p: float = 0.01,
                outlier_sigma: float = 20.0) -> np.ndarray:
    """X bf16 bits [m, k]: N(0,1) with a fraction `outlier_p` of N(0, outlier_sigma) outliers."""
    rng = _rng(seed, _TAG_X, m, k)
    x = rng.standard_normal((m, k), dtype=np.float32)
    if outlier_p > 0.0 and m * k > 0:
        mask = rng.random((m, k), dtype=np.float32) < np.float32(outlier_p)
        cnt = int(mask.sum())
        x[mask] = rng.standard_normal(cnt, dtype=np.float32) * np.float32(outlier_sigma)
    return f32_to_bf16_bits(x)


def weights(n: int, k: int, seed: int, sigma: float = 0.02) -> np.ndarray:
    """W bf16 bits [n, k]: N(0, sigma)."""
    rng = _rng(seed, _TAG_W, n, k)
    w = rng.standard_normal((n, k), dtype=np.float32) * np.float32(sigma)
    return f32_to_bf16_bits(w)


def gate_up(m: int, i: int, seed: int, sigma: float = 3.0) -> tuple[np.ndarray, np.ndarray]:
    """gate, up bf16 bits [m, i]: independent N(0, sigma) draws."""
    g = _rng(seed, _TAG_GATE, m, i).standard_normal((m, i), dtype=np.float32) * np.float32(sigma)
    u = _rng(seed, _TAG_UP, m, i).standard_normal((m, i), dtype=np.float32) * np.float32(sigma)
    return f32_to_bf16_bits(g), f32_to_bf16_bits(u)


@dataclass(frozen=True)
class Workload:
    """One projection shape of the pages' workloads."""
    name: str
    number: int            # config number 1..5
    m: int
    n: int
    k: int
    outlier_p: float = 0.01
    outlier_sigma: float = 20.0

    @property
    def seed(self) -> int:
        return 1000 + self.number

    def x(self) -> np.ndarray:
        return activations(self.m, self.k, self.seed, self.outlier_p, self.outlier_sigma)

    def w(self) -> np.ndarray:
        return weights(self.n, self.k, self.seed)


def _mk(number, name, ms, n, ks, p=0.01, sigma=20.0):
    return [Workload(f"{name}_m{m}_n{n}_k{k}", number, m, n, k, p, sigma) for m in ms for k in ks]


# The five workload families (tiny; decode K=5120; decode K=17408; prefill
# M=1168; prefill M=4576), each expanded over its M and K values.
CONFIGS: dict[int, list[Workload]] = {
    1: _mk(1, "tiny", [16], 512, [512]),
    2: _mk(2, "decode", [16, 17, 25], 6144, [5120]),
    3: _mk(3, "decode_widek", [16, 17, 25], 5120, [17408]),
    4: _mk(4, "prefill", [1168], 17408, [5120]),
    5: _mk(5, "prefill", [4576], 6144, [6144, 17408], p=0.001, sigma=50.0),
}


def all_workloads() -> list[Workload]:
    return [w for n in sorted(CONFIGS) for w in CONFIGS[n]]


@dataclass(frozen=True)
class FfnWorkload:
    """One dense-FFN shape: x [M, D] -> gate|up [M, 2I] -> h [M, I] -> y [M, D]."""
    name: str
    m: int
    d: int
    i: int
    seed: int = 1100

    def x(self) -> np.ndarray:
        return activations(self.m, self.d, self.seed)

    def w_gate_up(self) -> np.ndarray:
        return weights(2 * self.i, self.d, self.seed)

    def w_down(self) -> np.ndarray:
        return weights(self.d, self.i, self.seed + 1)


FFN_CONFIGS: list[FfnWorkload] = [
    FfnWorkload("ffn_m25_d5120_i17408", 25, 5120, 17408),
    FfnWorkload("ffn_m1168_d5120_i17408", 1168, 5120, 17408),
]
