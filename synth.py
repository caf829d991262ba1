"""Seeded synthetic inputs for the W8A8 int8-dynamic linear layer.

This module is shared by the tests, the smoke check and the benchmark.  It
holds input distributions only -- none of the method's arithmetic -- so both
the CUDA path and the CPU oracle can be fed the same bytes without sharing any
computation.

No real model weights or prompts are available, so seeded random tensors with
the shapes of a Qwen-Image-class diffusion transformer stand in for them
(hidden ~3072, MLP ~12288, ~4096 image + 256 text tokens; the AdaLN modulation
projection 3072 -> 18432 computed at M = batch).  Values are drawn in float64
with ``numpy.random.default_rng``, rounded to float32 and then to bf16 (round
to nearest even both times, via torch's CPU conversion).  bf16 tensors are
returned as their uint16 bit patterns.

Distributions:
  * ``outlier20``  x ~ N(0, 1) with 4 seeded channels multiplied by 20.
  * ``studentt``   x ~ N(0, 1) with round(1% of K) seeded channels replaced by
                   Student-t (nu = 3) samples (unscaled): heavy-tailed channels.
  * ``gelu``       x = gelu_tanh(z), z ~ N(0, 1): non-negative-skewed, long
                   right tail, minimum about -0.17 (input of a down-projection).
  * ``normal``     x ~ N(0, 1).
  * weights        W ~ N(0, 0.02);  bias ~ N(0, 0.01).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

# Independent random streams per tensor role, so changing one shape never
# changes another tensor's values.
_TAG_X, _TAG_W, _TAG_BIAS, _TAG_CHAN = 11, 22, 33, 44


def _rng(seed: int, tag: int, extra: int = 0) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(tag), int(extra)])


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float64/float32 array -> bf16 bit patterns (uint16), nearest-even."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> exact float64 values."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def make_x(M: int, K: int, kind: str, seed: int) -> np.ndarray:
    rng = _rng(seed, _TAG_X, M * 1_000_003 + K)
    if kind == "gelu":
        z = rng.standard_normal((M, K))
        x = 0.5 * z * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (z + 0.044715 * z ** 3)))
        return to_bf16_bits(x)
    x = rng.standard_normal((M, K))
    crng = _rng(seed, _TAG_CHAN, K)
    if kind == "outlier20":
        ch = crng.choice(K, size=min(4, K), replace=False)
        x[:, ch] *= 20.0
    elif kind == "studentt":
        n = max(1, int(round(0.01 * K)))
        ch = crng.choice(K, size=min(n, K), replace=False)
        x[:, ch] = rng.standard_t(3.0, size=(M, len(ch)))
    elif kind != "normal":
        raise ValueError(f"unknown activation distribution {kind!r}")
    return to_bf16_bits(x)


def make_w(N: int, K: int, seed: int) -> np.ndarray:
    rng = _rng(seed, _TAG_W, N * 1_000_003 + K)
    return to_bf16_bits(rng.normal(0.0, 0.02, size=(N, K)))


def make_bias(N: int, seed: int) -> np.ndarray:
    rng = _rng(seed, _TAG_BIAS, N)
    return to_bf16_bits(rng.normal(0.0, 0.01, size=(N,)))


@dataclass(frozen=True)
class LayerCase:
    """One linear-layer call: x [M, K] against W [N, K] (+ bias [N])."""
    name: str
    M: int
    K: int
    N: int
    x_kind: str
    seed: int = 0
    bias: bool = True

    def x(self) -> np.ndarray:
        return make_x(self.M, self.K, self.x_kind, self.seed)

    def w(self) -> np.ndarray:
        return make_w(self.N, self.K, self.seed)

    def b(self):
        return make_bias(self.N, self.seed) if self.bias else None

    @property
    def ops(self) -> int:
        return 2 * self.M * self.N * self.K


# The workloads: a tiny layer the oracle runs in well under a second, the
# fused QKV projection (4096 image + 256 text tokens), the FFN pair, and the
# AdaLN modulation projection as a GEMV at M = 1 and 2 (CFG batch).
TINY = LayerCase("tiny", 64, 256, 128, "outlier20", 0)
QKV = LayerCase("qkv", 4352, 3072, 9216, "studentt", 0)
FFN_UP = LayerCase("ffn_up", 4352, 3072, 12288, "studentt", 0)
FFN_DOWN = LayerCase("ffn_down", 4352, 12288, 3072, "gelu", 0)
ADALN_M1 = LayerCase("adaln_m1", 1, 3072, 18432, "normal", 0)
ADALN_M2 = LayerCase("adaln_m2", 2, 3072, 18432, "normal", 0)
# the same projection for a batch of 16 conditioning vectors
ADALN_M16 = LayerCase("adaln_m16", 16, 3072, 18432, "normal", 0)

# One DiT block's quantized linears at CFG batch 2 (the conditional and
# unconditional branches batched: M = 2 x 4352 tokens): the fused q|k|v
# projection, the attention output projection, the fused FFN proj|gate
# projection (two 3072 -> 12288 linears on the same input), the FFN output
# projection, and the AdaLN modulation projection as a GEMV at M = 2.
DIT_BLOCK = (
    LayerCase("blk_qkv", 8704, 3072, 9216, "studentt", 10),
    LayerCase("blk_to_out", 8704, 3072, 3072, "studentt", 11),
    LayerCase("blk_proj_gate", 8704, 3072, 24576, "studentt", 12),
    LayerCase("blk_ffn_out", 8704, 12288, 3072, "gelu", 13),
    LayerCase("blk_adaln", 2, 3072, 18432, "normal", 14),
)

SWEEP_M = (1, 16, 17, 256, 1024, 4352, 8704, 16384)
SWEEP_KN = ((3072, 9216), (3072, 3072), (3072, 12288), (12288, 3072))
SWEEP_SEEDS = (0, 1, 2, 3)


def sweep_cases(ms=SWEEP_M, kns=SWEEP_KN, seeds=SWEEP_SEEDS):
    """The M sweep over one DiT block's linear set (K=12288 takes GELU inputs)."""
    out = []
    for seed in seeds:
        for K, N in kns:
            for M in ms:
                kind = "gelu" if K == 12288 else "studentt"
                out.append(LayerCase(f"sweep_m{M}_k{K}_n{N}_s{seed}", M, K, N, kind, seed))
    return out


NAMED = {c.name: c for c in (TINY, QKV, FFN_UP, FFN_DOWN, ADALN_M1, ADALN_M2, ADALN_M16)}
