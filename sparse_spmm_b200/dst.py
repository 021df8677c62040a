"""Dynamic sparse training with the truly-sparse layer.

"Beyond Masked Sparsity: SNACK Enables Truly Sparse Neural Networks on GPU" (Abstract) pairs
the sparse forward/backward with an API that restructures a layer's connections during
training.  This module is that loop's glue: a layer module whose trainable tensor is the
layout's value array, a momentum-SGD optimizer, and the periodic prune-and-regrow step that
carries the optimizer state through the restructure with the library's old-to-new map.

The products, the restructure and the state remap run in the library's kernels; the
optimizer's elementwise update uses torch tensor arithmetic (it is not part of the sparse
path).
"""

from __future__ import annotations

import torch

from . import snk


class SparseLinear(torch.nn.Module):
    """Y = W X for W (M x K) stored only as its nonzeros; X is K x N (feature-major)."""

    def __init__(self, M: int, K: int, row: torch.Tensor, col: torch.Tensor, values: torch.Tensor, num_parts: int = 0):
        super().__init__()
        self.layout = snk.Layout(M, K, row, col, values, num_parts=num_parts)
        # the parameter shares storage with the layout's (sorted) value array
        self.weight = torch.nn.Parameter(self.layout.values, requires_grad=True)

    @property
    def nnz(self) -> int:
        return self.layout.nnz

    def forward(self, X: torch.Tensor) -> torch.Tensor:
        return snk.SparseLinearFunction.apply(self.weight, X, self.layout)


class MomentumSGD:
    """v = mu v + g; w -= lr v, with one state tensor per parameter (per nonzero for sparse layers)."""

    def __init__(self, params, lr: float, momentum: float = 0.9):
        self.params = list(params)
        self.lr = lr
        self.momentum = momentum
        self.state = {id(p): torch.zeros_like(p) for p in self.params}

    @torch.no_grad()
    def step(self):
        for p in self.params:
            if p.grad is None:
                continue
            v = self.state[id(p)]
            v.mul_(self.momentum).add_(p.grad)
            p.add_(v, alpha=-self.lr)

    def zero_grad(self):
        for p in self.params:
            p.grad = None

    def remap(self, p: torch.Tensor, old_to_new: torch.Tensor):
        """Carry p's state through a restructure: survivors keep it, regrown entries start at 0."""
        old = self.state[id(p)]
        self.state[id(p)] = snk.snk_remap_entries(old_to_new, old, torch.empty_like(old))


def prune_and_regrow(layer: SparseLinear, fraction: float, seed: int, optimizer: MomentumSGD | None = None,
                     regrow_value: float = 0.0) -> torch.Tensor:
    """Drop the round(fraction * nnz) smallest-magnitude connections of `layer`, regrow as many
    at positions drawn from the seeded SplitMix64 stream (library rule), remap the optimizer
    state, and return the old-to-new map.  The layer's function changes only by the dropped
    terms when regrow_value is 0."""
    k = int(round(fraction * layer.nnz))
    old_to_new = layer.layout.restructure(k, seed=seed, regrow_value=regrow_value)
    layer.weight.grad = None
    if optimizer is not None:
        optimizer.remap(layer.weight, old_to_new)
    return old_to_new
