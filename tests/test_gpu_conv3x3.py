"""Sparse 3x3 convolution: the GPU patch matrix and the convolution through the SpMM.

snk_im2col3x3 is pure data movement, so it must equal the oracle's patch matrix bit for
bit (fp32 and bf16, ragged image sizes).  The convolution (patch matrix, then the forward
SpMM with K = 9 C) is compared with the oracle's direct 3x3 convolution within the parity
tolerance: on small layers, and on sampled output channels of a ResNet-50 3x3 layer
(256 -> 256 channels, 14 x 14, batch 32) at 95% sparsity.
"""

import numpy as np
import pytest
import torch

import oracle
from helpers import bits, explicit_layer, f64, gpu_layout, to_dev
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


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(5, 2, 7, 9), (64, 4, 14, 14), (3, 1, 1, 1), (2, 3, 1, 6)])
def test_patch_matrix_bit_exact(dtype, shape):
    C, Nb, H, W = shape
    rng = np.random.default_rng(C * 100 + H)
    x = wl.cast(rng.normal(size=(C, Nb, H, W)).astype(np.float32), dtype)
    got = snk.snk_im2col3x3(to_dev(x.reshape(C, -1)).contiguous(), C, Nb, H, W)
    torch.cuda.synchronize()
    assert bits(got).tobytes() == oracle.im2col3x3(C, Nb, H, W, x).tobytes()


def _conv_layer(Co, C, density, dtype, seed):
    rng = np.random.default_rng(seed)
    K = 9 * C
    lin = rng.choice(Co * K, size=int(round(density * Co * K)), replace=False)
    return explicit_layer(Co, K, lin // K, lin % K, rng.normal(0, 0.05, size=lin.size).astype(np.float32), dtype)


@pytest.mark.parametrize("dtype,N_img", [("f32", (2, 9, 11)), ("bf16", (3, 8, 8)), ("f32", (32, 14, 14))])
def test_conv_matches_oracle(dtype, N_img):
    Nb, H, W = N_img
    Co, C = 24, 16
    layer = _conv_layer(Co, C, 0.2, dtype, 1)
    L = gpu_layout(layer)
    rng = np.random.default_rng(2)
    x = wl.cast(np.maximum(rng.normal(size=(C, Nb, H, W)), 0).astype(np.float32), dtype)
    Y = snk.sparse_conv3x3(L, to_dev(x.reshape(C, -1)).contiguous(), Nb, H, W)
    L.sync_status()
    arr = L.arrays()
    Yr, A = oracle.conv3x3(Co, C, Nb, H, W, arr["row"].cpu().numpy(), arr["col"].cpu().numpy(), f64(L.values),
                           oracle.widen(x.reshape(-1)).reshape(C, Nb, H, W))
    err = oracle.normalized_error(f64(Y), Yr, A)
    assert err <= oracle.tolerance(dtype), err


def test_resnet50_layer_sampled():
    Co, C, Nb, H, W = 256, 256, 32, 14, 14
    layer = _conv_layer(Co, C, 0.05, "f32", 4)
    L = gpu_layout(layer)
    rng = np.random.default_rng(5)
    x = np.maximum(rng.normal(size=(C, Nb, H, W)), 0).astype(np.float32)
    Y = snk.sparse_conv3x3(L, to_dev(x.reshape(C, -1)).contiguous(), Nb, H, W)
    L.sync_status()
    arr = L.arrays()
    row, col = arr["row"].cpu().numpy(), arr["col"].cpu().numpy()
    rows = np.array([0, 1, 77, 128, 200, 255])
    m = np.isin(row, rows)
    Yr, A = oracle.conv3x3(Co, C, Nb, H, W, row[m], col[m], f64(L.values)[m], x.astype(np.float64))
    err = oracle.normalized_error(f64(Y)[rows], Yr[rows], A[rows])
    assert err <= oracle.tolerance("f32"), err
