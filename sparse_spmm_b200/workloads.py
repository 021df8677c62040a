"""Seeded synthetic inputs shaped like the pages' workloads.

This module only draws inputs: weight positions and values, activations and upstream
gradients.  It holds none of the layer's arithmetic and is the one module that both the
CUDA path (tests, benchmark) and the CPU oracle consume.

Shapes follow the workloads the pages name: FC layers and 1x1 convolutions ("SparseRT:
Accelerating Unstructured Sparsity on GPUs for Deep Learning Inference", Abstract), and
transformer MLPs trained and served at small batch ("Beyond Masked Sparsity: SNACK ...",
Abstract).  No dataset is read; every array comes from numpy's PCG64 seeded through
``SeedSequence(seed).spawn(4)`` (streams: positions, values, X, dY).

Value arrays are float32, or uint16 holding bfloat16 bits (round-to-nearest-even of the
float32 draw, done by torch on the CPU).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

DTYPES = ("f32", "bf16")


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def cast(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "bf16":
        return to_bf16_bits(x)
    raise ValueError(dtype)


def nnz_for(M: int, K: int, sparsity: float) -> int:
    """nnz = round((1 - s) * M * K), halves rounded up."""
    return int(math.floor((1.0 - sparsity) * M * K + 0.5))


@dataclass
class Layer:
    """One sparse weight W (M x K) as unsorted COO triples."""

    name: str
    M: int
    K: int
    row: np.ndarray  # int32 [nnz]
    col: np.ndarray  # int32 [nnz]
    values: np.ndarray  # float32 or uint16 (bf16 bits) [nnz]
    dtype: str
    seed: int
    structure: str
    meta: dict = field(default_factory=dict)

    @property
    def nnz(self) -> int:
        return int(self.row.size)


def _streams(seed: int):
    ss = np.random.SeedSequence(seed).spawn(4)
    return [np.random.Generator(np.random.PCG64(s)) for s in ss]


def uniform_layer(M: int, K: int, sparsity: float, dtype: str, seed: int = 0,
                  name: str = "uniform", nnz: int | None = None) -> Layer:
    """Positions uniform over the M*K grid without replacement; values ~ N(0, 0.02)."""
    g_pos, g_val, _, _ = _streams(seed)
    n = nnz_for(M, K, sparsity) if nnz is None else nnz
    lin = g_pos.choice(M * K, size=n, replace=False).astype(np.int64)
    vals = g_val.normal(0.0, 0.02, size=n).astype(np.float32)
    return Layer(name, M, K, (lin // K).astype(np.int32), (lin % K).astype(np.int32),
                 cast(vals, dtype), dtype, seed, "uniform")


def magnitude_pruned_layer(M: int, K: int, sparsity: float, seed: int = 0,
                           name: str = "pruned", dtype: str = "f32") -> Layer:
    """Keep the nnz largest |w| of a dense N(0, 0.02) draw (ties: lower linear index).

    The kept values are the drawn weights; entries are handed over in a shuffled order.
    """
    g_pos, g_val, _, _ = _streams(seed)
    n = nnz_for(M, K, sparsity)
    dense = g_val.normal(0.0, 0.02, size=M * K).astype(np.float32)
    lin_all = np.arange(M * K, dtype=np.int64)
    order = np.lexsort((lin_all, -np.abs(dense)))[:n]
    order = order[g_pos.permutation(n)]
    return Layer(name, M, K, (order // K).astype(np.int32), (order % K).astype(np.int32),
                 cast(dense[order], dtype), dtype, seed, "magnitude-pruned")


def zipf_row_counts(M: int, K: int, nnz: int, s: float, rng: np.random.Generator) -> np.ndarray:
    """Per-row nnz counts ~ rank^-s over a random row order, capped at K by water-filling.

    Rows whose share exceeds K are capped and the excess is redistributed in proportion
    to the weights of the uncapped rows, repeatedly.  Integer counts come from floors
    plus largest remainders (ties to the lower rank).
    """
    if nnz > M * K:
        raise ValueError("nnz exceeds M*K")
    perm = rng.permutation(M)
    w = np.arange(1, M + 1, dtype=np.float64) ** (-s)
    capped = np.zeros(M, bool)
    target = nnz * w / w.sum()
    while True:
        over = (target > K) & ~capped
        if not over.any():
            break
        capped |= over
        rest = nnz - K * int(capped.sum())
        free = ~capped
        target = np.where(capped, float(K), rest * w / w[free].sum())
    base = np.floor(target).astype(np.int64)
    base = np.minimum(base, K)
    deficit = nnz - int(base.sum())
    rem = target - base
    rem[base >= K] = -1.0
    ranks = np.arange(M)
    order = np.lexsort((ranks, -rem))
    base[order[:deficit]] += 1
    counts = np.empty(M, np.int64)
    counts[perm] = base
    return counts


def zipf_layer(M: int, K: int, sparsity: float, dtype: str, s: float = 1.2, seed: int = 0,
               name: str = "zipf") -> Layer:
    """Row-skewed positions: per-row counts from zipf_row_counts, columns uniform per row."""
    g_pos, g_val, _, _ = _streams(seed)
    n = nnz_for(M, K, sparsity)
    counts = zipf_row_counts(M, K, n, s, g_pos)
    rows, cols = [], []
    for r in range(M):
        c = int(counts[r])
        if c == 0:
            continue
        cols.append(g_pos.choice(K, size=c, replace=False).astype(np.int32))
        rows.append(np.full(c, r, np.int32))
    row = np.concatenate(rows)
    col = np.concatenate(cols)
    shuf = g_pos.permutation(n)
    vals = g_val.normal(0.0, 0.02, size=n).astype(np.float32)
    return Layer(name, M, K, row[shuf], col[shuf], cast(vals, dtype), dtype, seed,
                 "zipf-rows", {"s": s, "dense_rows": int((counts == K).sum()),
                               "median_row_nnz": float(np.median(counts))})


def activations(rows: int, N: int, dtype: str, seed: int = 0, stream: int = 2,
                relu: bool = False) -> np.ndarray:
    """A rows x N row-major matrix ~ N(0, 1) (ReLU'd for the conv sweep).  stream 2 = X, 3 = dY."""
    g = _streams(seed)[stream]
    x = g.normal(0.0, 1.0, size=(rows, N)).astype(np.float32)
    if relu:
        x = np.maximum(x, 0.0)
    return cast(x, dtype)


# ----------------------------------------------------------------------------- configs

@dataclass
class Workload:
    name: str
    layers: list  # callables -> Layer
    dtype: str
    batches: tuple
    ops: tuple
    relu_x: bool = False
    note: str = ""


def tiny_fc(seed: int = 0) -> Workload:
    """W 512x512 at 90% (26,214 nnz, uniform), fp32, N = 8; forward, dX, dW."""
    return Workload("tiny-fc-512x512-s90-f32", [lambda: uniform_layer(512, 512, 0.90, "f32", seed, "W")],
                    "f32", (8,), ("forward", "backward_input", "backward_weight"))


def fc_4096(seed: int = 0) -> Workload:
    """W 4096x4096 at 95% (838,861 nnz, uniform), bf16 with fp32 accumulation, N in {1, 8, 32}."""
    return Workload("fc-4096x4096-s95-bf16", [lambda: uniform_layer(4096, 4096, 0.95, "bf16", seed, "W")],
                    "bf16", (1, 8, 32), ("forward", "backward_input", "backward_weight"))


def gpt2_mlp(seed: int = 0) -> Workload:
    """GPT-2 small MLP: W1 3072x768 and W2 768x3072 at 90% (magnitude-pruned), fp32, N = 1024."""
    return Workload("gpt2-mlp-3072x768-s90-f32",
                    [lambda: magnitude_pruned_layer(3072, 768, 0.90, seed, "W1"),
                     lambda: magnitude_pruned_layer(768, 3072, 0.90, seed + 1, "W2")],
                    "f32", (1024,), ("forward", "backward_input", "backward_weight", "restructure"))


def llama_mlp(seed: int = 0) -> Workload:
    """LLaMA-7B MLP projections 11008x4096 and 4096x11008 at 99%, Zipf(1.2) rows, bf16, N in {1, 4, 16}."""
    return Workload("llama-mlp-11008x4096-s99-zipf-bf16",
                    [lambda: zipf_layer(11008, 4096, 0.99, "bf16", 1.2, seed, "W_up"),
                     lambda: zipf_layer(4096, 11008, 0.99, "bf16", 1.2, seed + 1, "W_down")],
                    "bf16", (1, 4, 16), ("forward", "backward_input", "backward_weight"))


CONV_SHAPES = ((256, 1024), (1024, 256), (512, 2048))
CONV_SPARSITIES = (0.80, 0.90, 0.95, 0.98, 0.99)


def conv1x1(M: int, K: int, sparsity: float, seed: int = 0) -> Workload:
    """1x1 convolution as SpMM at a ResNet-50 shape: X is K x 6272 (= 32*14*14), ReLU(N(0,1)), fp32."""
    return Workload(f"conv1x1-{M}x{K}-s{int(round(sparsity * 100))}-f32",
                    [lambda: uniform_layer(M, K, sparsity, "f32", seed, "W")],
                    "f32", (6272,), ("forward",), relu_x=True)
