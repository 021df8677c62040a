"""Shared helpers of the GPU parity tests: moving seeded inputs to the device, reading
results back, and comparing the CUDA path with the oracle."""

from __future__ import annotations

import numpy as np
import torch

import oracle
from sparse_spmm_b200 import snk
from sparse_spmm_b200.workloads import Layer, activations, cast

BUILD_KEYS = ("row", "col", "row_ptr", "col_ptr", "csc_row", "perm", "part_nnz", "part_row",
              "part_nnz_t", "part_col")


def to_dev(a: np.ndarray) -> torch.Tensor:
    """numpy float32 / uint16 (bf16 bits) / int32 -> CUDA tensor of the matching type."""
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw bit patterns of a device tensor (uint16 for bf16)."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def gpu_layout(layer: Layer, num_parts: int = 0):
    row, col, vals = to_dev(layer.row), to_dev(layer.col), to_dev(layer.values)
    L = snk.Layout(layer.M, layer.K, row, col, vals, num_parts=num_parts)
    return L


def check_build(L: snk.Layout, layer: Layer) -> dict:
    """Every build array byte-equal to the oracle's (same P)."""
    arr = L.arrays()
    ref = oracle.build(layer.M, layer.K, layer.row, layer.col, layer.values, arr["num_parts"])
    assert ref["num_parts"] == arr["num_parts"]
    for k in BUILD_KEYS:
        got = arr[k].cpu().numpy()
        assert got.dtype == ref[k].dtype and got.shape == ref[k].shape, k
        assert np.array_equal(got, ref[k]), f"{k} differs"
    assert bits(arr["values"]).tobytes() == ref["values"].tobytes()
    return ref


def assert_close(got: np.ndarray, ref: np.ndarray, A: np.ndarray, dtype: str, what: str):
    err = oracle.normalized_error(got, ref, A)
    tol = oracle.tolerance(dtype)
    assert err <= tol, f"{what}: normalized error {err:.3e} > {tol:.1e}"
    return err


def dense_pair(layer: Layer, N: int, seed: int = 0, relu_x: bool = False):
    X = activations(layer.K, N, layer.dtype, seed, stream=2, relu=relu_x)
    dY = activations(layer.M, N, layer.dtype, seed, stream=3)
    return X, dY


def padded(a: np.ndarray, pad: int) -> tuple[torch.Tensor, torch.Tensor]:
    """Device copy of a 2-D array inside a wider buffer (leading dimension N + pad);
    returns (view, backing buffer)."""
    rows, N = a.shape
    full = np.zeros((rows, N + pad), dtype=a.dtype)
    full[:, :N] = a
    buf = to_dev(full)
    return buf[:, :N], buf


def check_products(layer: Layer, ref_build: dict, L: snk.Layout, N: int, seed: int = 0, relu_x: bool = False,
                   ops=("forward", "backward_input", "backward_weight"), pad: int = 0,
                   sample_rows: np.ndarray | None = None) -> dict:
    """Run the requested ops on the GPU and compare with the oracle.  With sample_rows,
    only those output rows (forward), columns (transposed) and entries (SDDMM) are
    computed by the oracle and compared."""
    X, dY = dense_pair(layer, N, seed, relu_x)
    Xd, _xb = padded(X, pad) if pad else (to_dev(X), None)
    dYd, _yb = padded(dY, pad) if pad else (to_dev(dY), None)
    row, col = ref_build["row"], ref_build["col"]
    v64 = oracle.widen(ref_build["values"])
    X64, dY64 = oracle.widen(X.reshape(-1)).reshape(X.shape), oracle.widen(dY.reshape(-1)).reshape(dY.shape)
    errs = {}
    M, K = layer.M, layer.K
    if "forward" in ops:
        if pad:
            Yb = torch.full((M, N + pad), float("nan"), dtype=Xd.dtype, device="cuda")
            Y = L.forward(Xd, Y=Yb[:, :N])
            assert torch.isnan(Yb[:, N:].float()).all(), "forward wrote outside its columns"
        else:
            Y = L.forward(Xd)
        if sample_rows is None:
            Yr, A = oracle.forward(M, K, row, col, v64, X64)
            errs["forward"] = assert_close(f64(Y), Yr, A, layer.dtype, "forward")
        else:
            m = np.isin(row, sample_rows)
            Yr, A = oracle.forward(M, K, row[m], col[m], v64[m], X64)
            errs["forward"] = assert_close(f64(Y)[sample_rows], Yr[sample_rows], A[sample_rows], layer.dtype,
                                           "forward (sampled rows)")
    if "backward_input" in ops:
        dX = L.backward_input(dYd)
        if sample_rows is None:
            dXr, A = oracle.backward_input(M, K, row, col, v64, dY64)
            errs["backward_input"] = assert_close(f64(dX), dXr, A, layer.dtype, "backward_input")
        else:
            cols = sample_rows[sample_rows < K]
            m = np.isin(col, cols)
            dXr, A = oracle.backward_input(M, K, row[m], col[m], v64[m], dY64)
            errs["backward_input"] = assert_close(f64(dX)[cols], dXr[cols], A[cols], layer.dtype,
                                                  "backward_input (sampled cols)")
    if "backward_weight" in ops:
        dW = L.backward_weight(dYd, Xd)
        if sample_rows is None:
            dWr, A = oracle.backward_weight(row, col, dY64, X64)
            errs["backward_weight"] = assert_close(f64(dW), dWr, A, layer.dtype, "backward_weight")
        else:
            idx = np.nonzero(np.isin(row, sample_rows))[0]
            dWr, A = oracle.backward_weight(row[idx], col[idx], dY64, X64)
            errs["backward_weight"] = assert_close(f64(dW)[idx], dWr, A, layer.dtype,
                                                   "backward_weight (sampled entries)")
    return errs


def explicit_layer(M, K, row, col, values_f32, dtype="f32", name="explicit") -> Layer:
    return Layer(name, M, K, np.asarray(row, np.int32), np.asarray(col, np.int32),
                 cast(np.asarray(values_f32, np.float32), dtype), dtype, 0, "explicit")
