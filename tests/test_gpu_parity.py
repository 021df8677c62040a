"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Index work (sort, row pointers, CSC permutation, partitions, restructure) must be
byte-equal; fp outputs must satisfy max |g - r| / sum|terms| <= 1e-5 (fp32) or 2e-2 (bf16).
Workloads are the seeded synthetic layers of sparse_spmm_b200.workloads at full size
(where the oracle is fast enough) plus small edge cases.
"""

import numpy as np
import pytest
import torch

import oracle
from helpers import (bits, check_build, check_products, explicit_layer, f64, gpu_layout, to_dev)
from sparse_spmm_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from sparse_spmm_b200 import build
    build.build()
    yield


# ----------------------------------------------------------------------------- full-size configs

def test_tiny_fc_full():
    layer = wl.uniform_layer(512, 512, 0.90, "f32", 0, "W")
    assert layer.nnz == 26214
    L = gpu_layout(layer)
    ref = check_build(L, layer)
    check_products(layer, ref, L, 8)


@pytest.mark.parametrize("N", [1, 8, 32])
def test_fc4096_bf16_full(N):
    layer = wl.uniform_layer(4096, 4096, 0.95, "bf16", 0, "W")
    assert layer.nnz == 838861
    L = gpu_layout(layer)
    ref = check_build(L, layer)
    check_products(layer, ref, L, N)


@pytest.mark.parametrize("which", [0, 1])
def test_llama_mlp_zipf_full(which):
    layer = (wl.zipf_layer(11008, 4096, 0.99, "bf16", 1.2, 0, "W_up") if which == 0
             else wl.zipf_layer(4096, 11008, 0.99, "bf16", 1.2, 1, "W_down"))
    L = gpu_layout(layer)
    ref = check_build(L, layer)
    for N in (1, 4, 16):
        check_products(layer, ref, L, N)


def test_gpt2_mlp_full_chain_and_restructure():
    W1 = wl.magnitude_pruned_layer(3072, 768, 0.90, 0, "W1")
    W2 = wl.magnitude_pruned_layer(768, 3072, 0.90, 1, "W2")
    L1, L2 = gpu_layout(W1), gpu_layout(W2)
    r1, r2 = check_build(L1, W1), check_build(L2, W2)
    N = 1024
    # forward chain H = W1 X, Y = W2 H and the backward chain, each step against the oracle
    X = wl.activations(768, N, "f32", 0, stream=2)
    dY = wl.activations(768, N, "f32", 0, stream=3)
    Xd, dYd = to_dev(X), to_dev(dY)
    H = L1.forward(Xd)
    Y = L2.forward(H)
    dW2 = L2.backward_weight(dYd, H)
    dH = L2.backward_input(dYd)
    dW1 = L1.backward_weight(dH, Xd)
    dX = L1.backward_input(dH)
    v1, v2 = oracle.widen(r1["values"]), oracle.widen(r2["values"])
    Hg, Yg, dHg = f64(H), f64(Y), f64(dH)
    Hr, A = oracle.forward(3072, 768, r1["row"], r1["col"], v1, X.astype(np.float64))
    assert oracle.normalized_error(Hg, Hr, A) <= 1e-5
    # downstream steps take the GPU's own fp32 inputs so that each op is checked alone
    Yr, A = oracle.forward(768, 3072, r2["row"], r2["col"], v2, Hg)
    assert oracle.normalized_error(Yg, Yr, A) <= 1e-5
    dW2r, A = oracle.backward_weight(r2["row"], r2["col"], dY.astype(np.float64), Hg)
    assert oracle.normalized_error(f64(dW2), dW2r, A) <= 1e-5
    dHr, A = oracle.backward_input(768, 3072, r2["row"], r2["col"], v2, dY.astype(np.float64))
    assert oracle.normalized_error(dHg, dHr, A) <= 1e-5
    dW1r, A = oracle.backward_weight(r1["row"], r1["col"], dHg, X.astype(np.float64))
    assert oracle.normalized_error(f64(dW1), dW1r, A) <= 1e-5
    dXr, A = oracle.backward_input(3072, 768, r1["row"], r1["col"], v1, dHg)
    assert oracle.normalized_error(f64(dX), dXr, A) <= 1e-5
    # one restructure pass per layer: drop 10% and regrow as many, bit-exact
    for L, ref, layer in ((L1, r1, W1), (L2, r2, W2)):
        k = 23593
        o2n = L.restructure(k, seed=0)
        rs = oracle.restructure(layer.M, layer.K, ref["row"], ref["col"], ref["values"], k, 0)
        assert np.array_equal(L.row.cpu().numpy(), rs["row"])
        assert np.array_equal(L.col.cpu().numpy(), rs["col"])
        assert bits(L.values).tobytes() == rs["values"].tobytes()
        assert np.array_equal(o2n.cpu().numpy(), rs["old_to_new"])
        rebuilt = oracle.build(layer.M, layer.K, rs["row"], rs["col"], rs["values"], L.num_parts)
        arr = L.arrays()
        for key in ("row_ptr", "col_ptr", "csc_row", "perm", "part_nnz", "part_row", "part_nnz_t", "part_col"):
            assert np.array_equal(arr[key].cpu().numpy(), rebuilt[key]), key


@pytest.mark.parametrize("shape", wl.CONV_SHAPES)
@pytest.mark.parametrize("sparsity", wl.CONV_SPARSITIES)
def test_conv1x1_sweep_sampled(shape, sparsity):
    M, K = shape
    layer = wl.uniform_layer(M, K, sparsity, "f32", 0, "W")
    L = gpu_layout(layer)
    ref = check_build(L, layer)
    rng = np.random.default_rng(1)
    rows = np.sort(rng.choice(M, size=min(M, 48), replace=False))
    check_products(layer, ref, L, 6272, relu_x=True, ops=("forward",), sample_rows=rows)


# ----------------------------------------------------------------------------- edge cases

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [1, 2, 3, 5, 31, 33, 64, 65, 72, 130, 264])
def test_ragged_batches(dtype, N):
    layer = wl.uniform_layer(300, 211, 0.93, dtype, 3, "W")
    L = gpu_layout(layer)
    ref = check_build(L, layer)
    check_products(layer, ref, L, N, seed=N)


@pytest.mark.parametrize("pad", [1, 3, 8])
def test_padded_leading_dimension(pad):
    for dtype in ("f32", "bf16"):
        layer = wl.uniform_layer(257, 190, 0.9, dtype, 5, "W")
        L = gpu_layout(layer)
        ref = check_build(L, layer)
        for N in (1, 8, 17, 32, 96):
            check_products(layer, ref, L, N, seed=7, pad=pad)


@pytest.mark.parametrize("P", [1, 2, 7, 64, 1000, 5000])
def test_partition_counts(P):
    # one fully dense row among sparse ones: with many parts it spans a long chain of CTAs
    rng = np.random.default_rng(P)
    M, K = 40, 3000
    lin = set(rng.choice(M * K, size=2500, replace=False).tolist())
    lin |= {17 * K + c for c in range(K)}
    lin = np.array(sorted(lin))
    lin = lin[rng.permutation(lin.size)]
    vals = rng.normal(0, 0.02, size=lin.size).astype(np.float32)
    for dtype in ("f32", "bf16"):
        layer = explicit_layer(M, K, lin // K, lin % K, vals, dtype)
        L = gpu_layout(layer, num_parts=P)
        assert L.num_parts == min(P, layer.nnz)
        ref = check_build(L, layer)
        for N in (1, 8, 40, 136):
            check_products(layer, ref, L, N, seed=N)


def test_empty_and_degenerate_shapes():
    # nnz = 0: outputs are zero, dW is empty
    layer = explicit_layer(6, 9, [], [], [], "f32")
    L = gpu_layout(layer)
    assert L.nnz == 0 and L.num_parts == 1
    X = torch.randn(9, 5, device="cuda")
    dY = torch.randn(6, 5, device="cuda")
    assert torch.count_nonzero(L.forward(X)) == 0
    assert torch.count_nonzero(L.backward_input(dY)) == 0
    assert L.backward_weight(dY, X).numel() == 0
    # M = 1, K = 1 and a 1 x K / M x 1 matrix
    for (M, K) in ((1, 1), (1, 50), (50, 1)):
        lin = np.arange(M * K)[:: 2 if M * K > 1 else 1]
        vals = np.linspace(-1, 1, lin.size).astype(np.float32)
        layer = explicit_layer(M, K, lin // K, lin % K, vals)
        L = gpu_layout(layer)
        ref = check_build(L, layer)
        check_products(layer, ref, L, 3)
    # empty rows and columns everywhere (very sparse)
    layer = wl.uniform_layer(2000, 1500, 0.9995, "f32", 9, "W")
    L = gpu_layout(layer)
    ref = check_build(L, layer)
    check_products(layer, ref, L, 4)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [2048, 2056])
def test_wide_batches(dtype, N):
    # the row-block x column-slice kernel: several slices, a ragged last slice, long rows
    rng = np.random.default_rng(N)
    M, K = 150, 700
    lin = set(rng.choice(M * K, size=9000, replace=False).tolist()) | {33 * K + c for c in range(K)}
    lin = np.array(sorted(lin))
    lin = lin[rng.permutation(lin.size)]
    layer = explicit_layer(M, K, lin // K, lin % K, rng.normal(0, 0.02, size=lin.size).astype(np.float32), dtype)
    L = gpu_layout(layer)
    ref = check_build(L, layer)
    check_products(layer, ref, L, N, seed=3, ops=("forward", "backward_input"))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_identity_and_permutation_are_bit_exact(dtype):
    n, N = 1000, 24
    rng = np.random.default_rng(4)
    p = rng.permutation(n)
    X = wl.activations(n, N, dtype, 2)
    for cols in (np.arange(n), p):
        layer = explicit_layer(n, n, np.arange(n), cols, np.ones(n, np.float32), dtype)
        L = gpu_layout(layer)
        Y = L.forward(to_dev(X))
        assert bits(Y).tobytes() == X[cols].tobytes()  # Y[r] = X[p[r]] exactly
        dX = L.backward_input(to_dev(X))
        expect = np.empty_like(X)
        expect[cols] = X
        assert bits(dX).tobytes() == expect.tobytes()


def test_zipf_small_with_many_parts():
    layer = wl.zipf_layer(700, 300, 0.95, "bf16", 1.2, 3, "Z")
    for P in (3, 50, 400):
        L = gpu_layout(layer, num_parts=P)
        ref = check_build(L, layer)
        for N in (1, 16):
            check_products(layer, ref, L, N)


def test_autograd_function_matches_ops():
    from sparse_spmm_b200.snk import SparseLinearFunction
    layer = wl.uniform_layer(64, 48, 0.8, "f32", 2, "W")
    L = gpu_layout(layer)
    vals = L.values.clone().requires_grad_(True)
    X = torch.randn(48, 5, device="cuda", requires_grad=True)
    Y = SparseLinearFunction.apply(vals, X, L)
    dY = torch.randn_like(Y)
    Y.backward(dY)
    assert torch.equal(Y.detach(), L.forward(X.detach()))
    assert torch.equal(X.grad, L.backward_input(dY))
    assert torch.equal(vals.grad, L.backward_weight(dY, X.detach()))


# ----------------------------------------------------------------------------- restructure

@pytest.mark.parametrize("seed", range(8))
def test_restructure_random_small(seed):
    rng = np.random.default_rng(500 + seed)
    M, K = (int(x) for x in rng.integers(2, 60, size=2))
    nnz = int(rng.integers(1, M * K * 0.6 + 2))
    nnz = min(nnz, M * K - 1)
    dtype = "bf16" if seed % 2 else "f32"
    layer = wl.uniform_layer(M, K, 0.0, dtype, seed, "W", nnz=nnz)
    L = gpu_layout(layer, num_parts=int(rng.integers(1, 40)))
    ref = check_build(L, layer)
    k = int(min(rng.integers(0, nnz + 1), M * K - nnz))
    o2n = L.restructure(k, seed=seed * 1000003 + 17, regrow_value=0.1 * seed)
    rs = oracle.restructure(M, K, ref["row"], ref["col"], ref["values"], k, seed * 1000003 + 17, 0.1 * seed)
    assert np.array_equal(L.row.cpu().numpy(), rs["row"])
    assert np.array_equal(L.col.cpu().numpy(), rs["col"])
    assert bits(L.values).tobytes() == rs["values"].tobytes()
    assert np.array_equal(o2n.cpu().numpy(), rs["old_to_new"])
    new_layer = wl.Layer("W2", M, K, rs["row"], rs["col"], rs["values"], dtype, 0, "restructured")
    check_build(L, new_layer)
    # products after the rebuild still match
    check_products(new_layer, oracle.build(M, K, rs["row"], rs["col"], rs["values"], L.num_parts), L, 3)


def test_restructure_dense_complement_and_ties():
    # k equals the number of free positions: every free position must be regrown
    M, K = 7, 9
    rng = np.random.default_rng(1)
    lin = rng.choice(M * K, size=40, replace=False)
    vals = np.round(rng.normal(size=40), 1).astype(np.float32)  # many equal magnitudes
    vals[:3] = [0.0, -0.0, 0.0]
    layer = explicit_layer(M, K, lin // K, lin % K, vals)
    L = gpu_layout(layer, num_parts=5)
    ref = check_build(L, layer)
    k = M * K - 40
    o2n = L.restructure(k, seed=99)
    rs = oracle.restructure(M, K, ref["row"], ref["col"], ref["values"], k, 99)
    assert np.array_equal(L.row.cpu().numpy(), rs["row"]) and np.array_equal(L.col.cpu().numpy(), rs["col"])
    assert np.array_equal(o2n.cpu().numpy(), rs["old_to_new"])
    assert bits(L.values).tobytes() == rs["values"].tobytes()
