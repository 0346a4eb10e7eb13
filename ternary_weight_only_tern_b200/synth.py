"""Seeded synthetic inputs for the ternary linear layer.

This module only draws random numbers; it holds none of the method's arithmetic
(no packing, no dequantisation, no product). Tests hand the same arrays to the
CPU oracle and to the CUDA library, and the bench draws its workloads here.

Recipe (numpy ``Generator(PCG64(seed))``; per tensor the draws come in the order
x, T1, s1, residual rows, T2, s2):

* x ~ N(0, 1), rounded to fp16 (activations stay 16-bit).
* trits iid; either P(-1) = P(0) = P(+1) = 1/3, or P(0) = 0.4, P(+1) = P(-1) = 0.3.
* s1 ~ U[0.005, 0.02] and s2 ~ U[0.001, 0.005], rounded to fp16, one per
  (row, 128-wide K group).
* residual rows: r = round-half-up(pct% of N) rows drawn uniformly without
  replacement, then sorted.
* a stack of layers draws layer l from PCG64(SeedSequence([seed, l])).

The projection shapes are those of Qwen3-4B (hidden 2560, intermediate 9728)
and Qwen3-8B (hidden 4096, intermediate 12288), 36 decoder layers each with the
q, k, v, o, gate, up and down projections (the 252 targeted linear tensors of
the 4B paper, section 3.1, and of the 8B paper's model description).
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

GROUP = 128

# (N, K) = (output features, input features) of each projection
QWEN3_4B = {
    "q": (4096, 2560), "k": (1024, 2560), "v": (1024, 2560), "o": (2560, 4096),
    "gate": (9728, 2560), "up": (9728, 2560), "down": (2560, 9728),
}
QWEN3_8B = {
    "q": (4096, 4096), "k": (1024, 4096), "v": (1024, 4096), "o": (4096, 4096),
    "gate": (12288, 4096), "up": (12288, 4096), "down": (4096, 12288),
}
N_LAYERS = 36


@dataclass
class TernTensor:
    """One ternarized weight and a batch of activations for it (host numpy arrays)."""
    name: str
    N: int
    K: int
    x: np.ndarray         # float16 [M, K]
    T1: np.ndarray        # int8 [N, K]
    s1: np.ndarray        # float16 [N, K/128]
    res_rows: np.ndarray  # int32 [r], strictly increasing
    T2: np.ndarray        # int8 [r, K]
    s2: np.ndarray        # float16 [r, K/128]

    @property
    def r(self) -> int:
        return int(len(self.res_rows))


@dataclass
class Workload:
    """A named set of projections, the batch sizes to run them at, and the draw parameters."""
    name: str
    shapes: list            # [(name, N, K)]
    Ms: list
    p_zero: float           # P(t = 0); P(+1) = P(-1) = (1 - p_zero) / 2
    res_pct: int            # percent of rows carrying a second plane
    seed: int
    layers: int = 1
    s1_range: tuple = (0.005, 0.02)
    s2_range: tuple = (0.001, 0.005)
    notes: str = field(default="")


def residual_count(N: int, pct: int) -> int:
    """round-half-up(pct% of N), in integers: 10% of 4096 -> 410, 15% of 12288 -> 1843."""
    return (N * pct + 50) // 100


def draw_trits(rng: np.random.Generator, shape, p_zero: float) -> np.ndarray:
    if abs(p_zero - 1.0 / 3.0) < 1e-12:
        return (rng.integers(0, 3, size=shape, dtype=np.int8) - 1).astype(np.int8)
    if abs(p_zero - 0.4) < 1e-12:
        u = rng.integers(0, 10, size=shape, dtype=np.uint8)    # 0-2 -> -1, 3-6 -> 0, 7-9 -> +1
        return ((u >= 7).astype(np.int8) - (u < 3).astype(np.int8)).astype(np.int8)
    raise ValueError("unsupported trit distribution")


def draw_x(rng: np.random.Generator, M: int, K: int) -> np.ndarray:
    return rng.standard_normal((M, K), dtype=np.float32).astype(np.float16)


def draw_scales(rng: np.random.Generator, rows: int, K: int, lo: float, hi: float) -> np.ndarray:
    return rng.uniform(lo, hi, size=(rows, K // GROUP)).astype(np.float16)


def draw_offsets(rng: np.random.Generator, rows: int, K: int, bound: float = 0.01) -> np.ndarray:
    """Per-group offsets, uniform in [-bound, bound] (fp16): of the order of the scales, as an
    asymmetric group's centre would be."""
    return rng.uniform(-bound, bound, size=(rows, K // GROUP)).astype(np.float16)


def draw_exact_offsets(rng: np.random.Generator, rows: int, K: int) -> np.ndarray:
    """Offsets for the exact inputs: 0 or +-2^-k, k in 4..6, so mu + s*t stays exact in fp16."""
    mag = np.ldexp(1.0, -rng.integers(4, 7, size=(rows, K // GROUP)))
    sign = rng.integers(-1, 2, size=(rows, K // GROUP))
    return (mag * sign).astype(np.float16)


def draw_elem_plane(rng: np.random.Generator, N: int, K: int, masked_frac: float = 0.036, p_zero: float = 0.4,
                    s_range=(0.001, 0.005)):
    """An element-level second plane: each weight is masked with probability masked_frac (the
    pages' two most salient masks cover 3.6 % of a recorded projection), a masked weight draws a
    trit like the main plane, an unmasked one is 0; one fp16 scale per (row, group).
    Returns (T2e int8 [N, K], s2e fp16 [N, K/128], number of masked weights)."""
    mask = rng.random((N, K), dtype=np.float32) < masked_frac
    T2e = np.where(mask, draw_trits(rng, (N, K), p_zero), 0).astype(np.int8)
    return T2e, draw_scales(rng, N, K, *s_range), int(mask.sum())


def draw_tensor(rng: np.random.Generator, name: str, N: int, K: int, M: int, *, p_zero: float,
                res_pct: int, s1_range=(0.005, 0.02), s2_range=(0.001, 0.005)) -> TernTensor:
    x = draw_x(rng, M, K)
    T1 = draw_trits(rng, (N, K), p_zero)
    s1 = draw_scales(rng, N, K, *s1_range)
    r = residual_count(N, res_pct)
    res_rows = np.sort(rng.choice(N, size=r, replace=False)).astype(np.int32)
    T2 = draw_trits(rng, (r, K), p_zero)
    s2 = draw_scales(rng, r, K, *s2_range)
    return TernTensor(name, N, K, x, T1, s1, res_rows, T2, s2)


def draw_exact_tensor(rng: np.random.Generator, N: int, K: int, M: int, r: int) -> TernTensor:
    """Inputs on which fp32 accumulation is exact: integer x in [-4, 4], power-of-two scales
    in [2^-6, 2^-4]. Every product and partial sum is then a multiple of 2^-6 of magnitude
    well below 2^24 * 2^-6 (for K <= 12288), so fp32 accumulation is exact in any order, and
    s1*t1 + s2*t2 is exact in fp16; both sides then round the same exact value once to fp16."""
    x = rng.integers(-4, 5, size=(M, K)).astype(np.float16)
    T1 = draw_trits(rng, (N, K), 1.0 / 3.0)
    s1 = np.ldexp(1.0, -rng.integers(4, 7, size=(N, K // GROUP))).astype(np.float16)
    res_rows = np.sort(rng.choice(N, size=r, replace=False)).astype(np.int32)
    T2 = draw_trits(rng, (r, K), 1.0 / 3.0)
    s2 = np.ldexp(1.0, -rng.integers(4, 7, size=(r, K // GROUP))).astype(np.float16)
    return TernTensor("exact", N, K, x, T1, s1, res_rows, T2, s2)


# The five benchmark workloads. Seeds are the workload number minus one.
WORKLOADS = {
    1: Workload("single-gemv-4096x2560", [("single", 4096, 2560)], [1], 1.0 / 3.0, 0, seed=0),
    2: Workload("qwen3-4b-layer-decode", [(k, *v) for k, v in QWEN3_4B.items()], [1], 0.4, 10, seed=1),
    3: Workload("qwen3-4b-stack-decode", [(k, *v) for k, v in QWEN3_4B.items()], [1, 4, 16], 0.4, 10, seed=2,
                layers=N_LAYERS),
    4: Workload("qwen3-8b-projections-decode", [(k, *v) for k, v in QWEN3_8B.items()], [1, 4, 8, 16], 0.4, 15,
                seed=3),
    5: Workload("qwen3-8b-prefill-gemm", [(k, *QWEN3_8B[k]) for k in ("gate", "up", "down")], [2048], 0.4, 10,
                seed=4),
}


def layer_rng(w: Workload, layer: int) -> np.random.Generator:
    """PCG64(seed) for a one-layer workload; PCG64(SeedSequence([seed, layer])) per layer of a stack,
    so that any layer can be drawn on its own."""
    if w.layers == 1:
        return np.random.Generator(np.random.PCG64(w.seed))
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([w.seed, layer])))


def draw_workload(w: Workload, layers=None, only=None):
    """Yield TernTensor for every (layer, projection) of a workload, x drawn at max(Ms) rows.

    ``layers`` is a count (the first n layers) or a list of layer indices; ``only`` restricts
    to projection names (the skipped projections are still drawn, so a projection's arrays do
    not depend on it).
    """
    if layers is None or isinstance(layers, int):
        layer_ids = range(w.layers if layers is None else min(layers, w.layers))
    else:
        layer_ids = list(layers)
    M = max(w.Ms)
    for layer in layer_ids:
        rng = layer_rng(w, layer)
        for (name, N, K) in w.shapes:
            t = draw_tensor(rng, name, N, K, M, p_zero=w.p_zero, res_pct=w.res_pct,
                            s1_range=w.s1_range, s2_range=w.s2_range)
            if only is None or name in only:
                t.name = f"L{layer}.{name}" if w.layers > 1 else name
                yield t
