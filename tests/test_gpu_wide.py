"""Wide operands (N >= 256): the TMA-staged row-block x column-slice kernels.

The dense operand's chunks reach shared memory through 2-D tensor copies, which need a
16-byte aligned base and row stride; other operands take the 64-column small kernels.
Cases: several column slices with a ragged last slice, padded leading dimensions, rows
longer than one 32-entry batch (and one dense row), a dense operand whose row count is no
multiple of the staged chunk, both rows-per-warp variants, and leading dimensions that
rule the tensor copies out.  Every result is compared with the oracle; afterwards the
layout's status word must show no abandoned wait.
"""

import numpy as np
import pytest
import torch

from helpers import check_build, check_products, explicit_layer, gpu_layout
from sparse_spmm_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from sparse_spmm_b200 import build
    build.build()
    yield


def _layer(dtype, seed, M=150, K=700, nnz=9000):
    rng = np.random.default_rng(seed)
    lin = set(rng.choice(M * K, size=nnz, replace=False).tolist()) | {33 * K + c for c in range(K)}
    lin = np.array(sorted(lin))
    lin = lin[rng.permutation(lin.size)]
    return explicit_layer(M, K, lin // K, lin % K, rng.normal(0, 0.02, size=lin.size).astype(np.float32), dtype)


# (dtype, N, pad): N*elem and (N+pad)*elem multiples of 16 take the tensor copies;
# 257 fp32 (1028 B rows) and 260 bf16 (520 B rows) do not
@pytest.mark.parametrize("dtype,N,pad", [("f32", 256, 0), ("f32", 300, 0), ("f32", 1000, 4), ("bf16", 264, 0),
                                         ("bf16", 520, 8), ("bf16", 1030, 2), ("f32", 257, 0), ("bf16", 260, 0)])
def test_wide_operands(dtype, N, pad):
    layer = _layer(dtype, N)
    L = gpu_layout(layer)
    ref = check_build(L, layer)
    check_products(layer, ref, L, N, seed=3, ops=("forward", "backward_input"), pad=pad)
    L.sync_status()


# shapes whose grids make the launcher pick 8 (4096 x 3000, N = 512: one round of 64-row
# blocks) and 6 (2500 x 600, N = 2048) rows per consumer warp on a 148-SM GPU
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("M,K,N", [(4096, 3000, 512), (2500, 600, 2048)])
def test_wide_rows_per_warp_variants(dtype, M, K, N):
    layer = wl.uniform_layer(M, K, 0.95, dtype, 5, "W")
    L = gpu_layout(layer)
    ref = check_build(L, layer)
    rows = np.unique(np.concatenate([np.arange(0, M, 37), [M - 1, K - 1]]))
    check_products(layer, ref, L, N, seed=4, ops=("forward", "backward_input"), sample_rows=rows)
    L.sync_status()
