"""Error paths of the C ABI on the GPU: every failure is a returned status read on the
host; no kernel traps, asserts or waits.  Inputs that would be invalid for a kernel are
rejected by the host checks or flagged by the kernels' own range checks."""

import numpy as np
import pytest
import torch

from helpers import explicit_layer, gpu_layout, to_dev
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


def _raw_build(M, K, row, col, vals, P=0, ws_bytes=None):
    r, c, v = to_dev(np.asarray(row, np.int32)), to_dev(np.asarray(col, np.int32)), to_dev(vals)
    need = snk.snk_workspace_bytes(M, K, r.numel(), P)
    ws = torch.empty(ws_bytes if ws_bytes is not None else need, dtype=torch.uint8, device="cuda")
    return r, c, v, ws


@pytest.mark.parametrize("bad", ["row_high", "row_neg", "col_high", "dup"])
def test_build_rejects_bad_coo_and_leaves_arrays(bad):
    row = np.array([3, 0, 2, 1, 0], np.int32)
    col = np.array([1, 4, 0, 2, 3], np.int32)
    if bad == "row_high":
        row[2] = 4
    elif bad == "row_neg":
        row[0] = -1
    elif bad == "col_high":
        col[4] = 5
    else:
        row[4], col[4] = 3, 1
    vals = np.arange(5, dtype=np.float32)
    r, c, v, ws = _raw_build(4, 5, row, col, vals)
    with pytest.raises(snk.SnkError) as e:
        snk.snk_build(4, 5, r, c, v, 0, ws)
    assert e.value.status == ("SNK_ERR_DUPLICATE" if bad == "dup" else "SNK_ERR_OUT_OF_RANGE")
    assert np.array_equal(r.cpu().numpy(), row) and np.array_equal(c.cpu().numpy(), col)
    assert np.array_equal(v.cpu().numpy(), vals)


def test_build_argument_checks():
    row, col = np.array([0, 1], np.int32), np.array([1, 0], np.int32)
    vals = np.ones(2, np.float32)
    r, c, v, ws = _raw_build(2, 2, row, col, vals)
    with pytest.raises(snk.SnkError) as e:
        snk.snk_build(2, 2, r, c, v, 0, ws[:16])
    assert e.value.status == "SNK_ERR_WORKSPACE_TOO_SMALL"
    with pytest.raises(snk.SnkError) as e:
        snk.snk_build(2, 2, r, c, v, 0, ws[1:])  # not 256-byte aligned
    assert e.value.status in ("SNK_ERR_INVALID_ARG", "SNK_ERR_WORKSPACE_TOO_SMALL")
    with pytest.raises(snk.SnkError) as e:
        snk.snk_build(0, 2, r, c, v, 0, ws)
    assert e.value.status == "SNK_ERR_INVALID_ARG"
    with pytest.raises(snk.SnkError) as e:
        snk.snk_build(2, 2, r, c, v, -3, ws)
    assert e.value.status == "SNK_ERR_INVALID_ARG"


def test_product_argument_checks():
    layer = wl.uniform_layer(30, 20, 0.8, "f32", 0, "W")
    L = gpu_layout(layer)
    X = torch.randn(20, 4, device="cuda")
    Y = torch.empty(30, 4, device="cuda")
    with pytest.raises(snk.SnkError) as e:  # dtype mismatch
        snk.snk_forward(L.handle, L.values, X.bfloat16(), 4, 4, Y.bfloat16(), 4)
    assert e.value.status == "SNK_ERR_INVALID_ARG"
    with pytest.raises(snk.SnkError) as e:  # ld < N
        snk.snk_forward(L.handle, L.values, X, 4, 3, Y, 4)
    assert e.value.status == "SNK_ERR_INVALID_ARG"
    with pytest.raises(snk.SnkError) as e:
        snk.snk_backward_input(L.handle, L.values, Y, -1, 4, X, 4)
    assert e.value.status == "SNK_ERR_INVALID_ARG"
    with pytest.raises(snk.SnkError) as e:
        snk.snk_backward_weight(L.handle, Y, 4, X, 4, 4, None)
    assert e.value.status == "SNK_ERR_INVALID_ARG"
    snk.snk_forward(L.handle, L.values, X, 0, 4, Y, 4)  # N = 0 is a no-op
    torch.cuda.synchronize()


def test_restructure_statuses_leave_layout_unchanged():
    layer = wl.uniform_layer(10, 10, 0.2, "bf16", 1, "W")  # 80 entries, 20 free positions
    L = gpu_layout(layer)
    before = (L.row.clone(), L.col.clone(), L.values.clone())
    with pytest.raises(snk.SnkError) as e:
        L.restructure(21, seed=1)
    assert e.value.status == "SNK_ERR_NO_ROOM"
    with pytest.raises(snk.SnkError) as e:
        L.restructure(81, seed=1)
    assert e.value.status == "SNK_ERR_INVALID_ARG"
    L.values[5] = float("nan")
    with pytest.raises(snk.SnkError) as e:
        L.restructure(3, seed=1)
    assert e.value.status == "SNK_ERR_INVALID_VALUE"
    assert torch.equal(L.row, before[0]) and torch.equal(L.col, before[1])
    assert torch.equal(L.values[:5], before[2][:5]) and torch.equal(L.values[6:], before[2][6:])


def test_layout_survives_many_launches_and_counters_reset():
    # the cross-CTA arrival counters must return to zero after every launch
    layer = explicit_layer(3, 5000, np.full(5000, 1), np.arange(5000), np.full(5000, 0.5, np.float32))
    L = gpu_layout(layer, num_parts=97)
    X = torch.ones(5000, 3, device="cuda")
    for _ in range(20):
        Y = L.forward(X)
        assert torch.all(Y[1] == 2500.0) and torch.all(Y[0] == 0) and torch.all(Y[2] == 0)
        dX = L.backward_input(torch.ones(3, 2, device="cuda"))
        assert torch.all(dX == 0.5)
