"""Checkpoint and resume of a layout: save its sorted COO, rebuild, compare byte for byte.

The derived arrays (row/column pointers, CSC permutation, partitions) are a function of the
sorted COO and the part count, so a rebuilt layout must hold identical bytes and give
bit-identical products; this holds after a restructure too (the checkpoint is the
restructured COO).
"""

import numpy as np
import pytest
import torch

from helpers import bits, gpu_layout, to_dev
from sparse_spmm_b200 import snk
from sparse_spmm_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from sparse_spmm_b200 import build
    build.build()
    yield


def _same(L1, L2, layer, N):
    a1, a2 = L1.arrays(), L2.arrays()
    for k in a1:
        if isinstance(a1[k], torch.Tensor):
            assert bits(a1[k]).tobytes() == bits(a2[k]).tobytes(), k
        else:
            assert a1[k] == a2[k], k
    X = to_dev(wl.activations(layer.K, N, layer.dtype, 1, 2))
    dY = to_dev(wl.activations(layer.M, N, layer.dtype, 1, 3))
    assert bits(L1.forward(X)).tobytes() == bits(L2.forward(X)).tobytes()
    assert bits(L1.backward_input(dY)).tobytes() == bits(L2.backward_input(dY)).tobytes()
    assert bits(L1.backward_weight(dY, X)).tobytes() == bits(L2.backward_weight(dY, X)).tobytes()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_save_load_and_after_restructure(dtype, tmp_path):
    layer = wl.uniform_layer(900, 700, 0.95, dtype, 6, "W")
    L = gpu_layout(layer, num_parts=37)
    snk.save_layout(L, tmp_path / "a.npz")
    R = snk.load_layout(tmp_path / "a.npz")
    assert R.num_parts == 37
    _same(L, R, layer, 8)
    L.restructure(layer.nnz // 10, seed=3)
    snk.save_layout(L, tmp_path / "b.npz")
    R2 = snk.load_layout(tmp_path / "b.npz")
    _same(L, R2, layer, 33)
