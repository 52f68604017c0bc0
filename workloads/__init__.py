"""Seeded synthetic inputs for the ternary-weight FWHT-1024 path.

This module only draws random numbers and lays them out as arrays. It holds
none of the method's arithmetic (no packing, no rotation, no matmul), so the
oracle and the CUDA library can both be fed from it without sharing code.

Distributions follow the workloads the pages measure on (a 27B ternary model,
decode tg128 and prefill pp512, in the Ternary Bonsai 2 27B release summary,
sections 三值权重怎么压缩到 1.76 bit and 实测吞吐). The model itself and its
datasets are not available, so these seeded arrays stand in for them:

* trits   i.i.d. with P(-1) = 0.3, P(0) = 0.4, P(+1) = 0.3, int8 [N, K]
* scales  fp16(|N(0,1)| * 0.02), rounded to nearest, [N, K/128]
* sign    S = +-1 with p = 1/2, one 1024-vector, seed 1024
* x       bf16(N(0,1)) [M, K]; where outliers are asked for, exactly
          ceil(0.001 * M * K) distinct positions are multiplied by 20 before
          the bf16 rounding.

All generators use numpy's PCG64 with the stated seed.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

GROUP = 128          # weights per FP16 scale (g128)
BLOCK = 1024         # rotation block length
SIGN_SEED = 1024


@dataclass(frozen=True)
class Layer:
    name: str
    K: int
    N: int


# The decode triple: K x N with W stored row-major [N][K].
TRIPLE = (Layer("L1", 5120, 5120), Layer("L2", 5120, 17408), Layer("L3", 17408, 5120))
TINY = Layer("L0", 1024, 256)

CONFIGS = {
    "C0": dict(seed=1, M=1, layers=(TINY,), outliers=False,
               text="tiny single layer: x bf16 [1,1024], W [256,1024]"),
    "C1": dict(seed=2, M=1, layers=TRIPLE, outliers=True,
               text="decode GEMV M=1 on the 5120x5120 / 5120x17408 / 17408x5120 triple"),
    "C2": dict(seed=3, M=(1, 4, 16), layers=TRIPLE, outliers=True, stacks=64, triples_per_stack=2,
               text="27B-equivalent decode sweep: 64 stacks x 2 triples = 384 matrices"),
    "C3": dict(seed=4, M=512, layers=TRIPLE, outliers=True,
               text="prefill pp512: X bf16 [512,K] on the triple shapes"),
    "C4": dict(seed=5, M=(1, 512), layers=TRIPLE, outliers=True,
               fwht_M=(1, 16, 512), fwht_K=(1024, 5120, 17408),
               text="layout A/B (2-bit vs base-3) plus a standalone FWHT sweep"),
}


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (NaN kept quiet)."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    out = rounded.astype(np.uint16)
    nan = np.isnan(f)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def trits(g: np.random.Generator, N: int, K: int, p_zero: float = 0.4) -> np.ndarray:
    u = g.random((N, K), dtype=np.float32)
    p_neg = (1.0 - p_zero) / 2.0
    t = np.zeros((N, K), dtype=np.int8)
    t[u < p_neg] = -1
    t[u >= p_neg + p_zero] = 1
    return t


def scales_f16_bits(g: np.random.Generator, N: int, K: int) -> np.ndarray:
    s = np.abs(g.standard_normal((N, K // GROUP))) * 0.02
    return s.astype(np.float16).view(np.uint16)


def sign1024(seed: int = SIGN_SEED) -> np.ndarray:
    g = rng(seed)
    return np.where(g.random(BLOCK) < 0.5, -1, 1).astype(np.int8)


def activations_bf16_bits(g: np.random.Generator, M: int, K: int, outliers: bool) -> np.ndarray:
    x = g.standard_normal((M, K))
    if outliers and M * K > 0:
        n_out = math.ceil(0.001 * M * K)
        pos = g.choice(M * K, size=n_out, replace=False)
        x.reshape(-1)[pos] *= 20.0
    return round_to_bf16_bits(x.astype(np.float32))


def layer_inputs(config: str, layer: Layer, M: int | None = None, index: int = 0,
                 with_x: bool = True) -> dict:
    """Seeded arrays for one matrix of a config.

    `index` separates matrices of one config (layer position in the triple,
    stack number in the sweep): the generator is seeded with
    (config seed, index) so every matrix is reproducible on its own.
    """
    cfg = CONFIGS[config]
    if M is None:
        M = cfg["M"] if isinstance(cfg["M"], int) else cfg["M"][0]
    g = rng(cfg["seed"] * 1_000_003 + index)
    out = {
        "K": layer.K, "N": layer.N, "M": M,
        "trits": trits(g, layer.N, layer.K),
        "scales": scales_f16_bits(g, layer.N, layer.K),
        "sign": sign1024(),
    }
    if with_x:
        out["x"] = activations_bf16_bits(g, M, layer.K, cfg["outliers"])
    return out


def random_case(seed: int, M: int, N: int, K: int, p_zero: float = 0.4,
                outliers: bool = True) -> dict:
    """Arbitrary-shape case for parity tests (ragged N, several tiles)."""
    g = rng(seed)
    return {
        "K": K, "N": N, "M": M,
        "trits": trits(g, N, K, p_zero),
        "scales": scales_f16_bits(g, N, K),
        "sign": sign1024(),
        "x": activations_bf16_bits(g, M, K, outliers),
    }


def fwht_input(seed: int, M: int, K: int, outliers: bool = True) -> np.ndarray:
    return activations_bf16_bits(rng(seed), M, K, outliers)
