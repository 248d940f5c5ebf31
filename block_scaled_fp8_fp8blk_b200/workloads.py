"""Named workloads for the block-FP8 linear ``y[M,N] = x[M,K] . dequant(W)[N,K]^T``.

Shapes follow the decoder of the pages' 32B-class text encoder (hidden 5120,
fused QKV 8192 + 1024 + 1024, o_proj 8192 -> 5120, MLP 25600); the largest
linear, 25600 x 5120, matches the size of the BF16 temporary that the Hopper
route materializes per call, about a quarter of a gigabyte (FastVideo PR
#1829, "Checklist").
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import synth


@dataclass(frozen=True)
class Workload:
    name: str
    M: int
    K: int
    N: int
    row_gain_sigma: float = 0.0   # per-output-row LogNormal(0, sigma) weight gain
    outlier_frac: float = 0.01    # fraction of K channels of x scaled x20
    seed: int = 0

    @property
    def flops(self) -> int:
        return 2 * self.M * self.N * self.K

    @property
    def weight_bytes(self) -> int:
        nb, kb = -(-self.N // 128), -(-self.K // 128)
        return self.N * self.K + 4 * nb * kb

    def with_m(self, M: int) -> "Workload":
        return Workload(f"{self.name.split('_m')[0]}_m{M}_k{self.K}_n{self.N}", M, self.K, self.N,
                        self.row_gain_sigma, self.outlier_frac, self.seed)

    # --- inputs (float32 draws, rounded to BF16 by torch) -------------------
    def weight_bf16(self):
        return synth.to_bf16(synth.weight_f32(self.seed, self.N, self.K, self.row_gain_sigma))

    def x_bf16(self):
        return synth.to_bf16(synth.activation_f32(self.seed, self.M, self.K, self.outlier_frac))

    def checked_rows(self, count: int = 256) -> np.ndarray:
        if self.M <= count:
            return np.arange(self.M, dtype=np.int64)
        return synth.sample_rows(self.seed, self.M, count)


TINY = Workload("tiny_m64_k256_n384", 64, 256, 384, outlier_frac=0.0)
RAGGED = Workload("ragged_m77_k1000_n1000", 77, 1000, 1000, row_gain_sigma=0.5)
QKV = Workload("qkv_m512_k5120_n10240", 512, 5120, 10240)
O_PROJ = Workload("o_proj_m512_k8192_n5120", 512, 8192, 5120)
GATE_UP = Workload("gate_up_m512_k5120_n51200", 512, 5120, 51200)
DOWN = Workload("down_m512_k25600_n5120", 512, 25600, 5120)
LINEAR_512 = Workload("linear_m512_k5120_n25600", 512, 5120, 25600)
LARGE_4096 = Workload("linear_m4096_k5120_n25600", 4096, 5120, 25600)
LARGE_16384 = Workload("linear_m16384_k5120_n25600", 16384, 5120, 25600)

DECODER_SHAPES = (QKV, O_PROJ, GATE_UP, DOWN)
SMALL_M = (1, 16, 64)

ALL = {w.name: w for w in (TINY, RAGGED, QKV, O_PROJ, GATE_UP, DOWN, LINEAR_512,
                           LARGE_4096, LARGE_16384)}
for _w in DECODER_SHAPES:
    for _m in SMALL_M:
        _s = _w.with_m(_m)
        ALL[_s.name] = _s

HEADLINE = LINEAR_512
