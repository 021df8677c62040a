"""snk_csr_forward_static: the forward product for callers that cannot allocate.

Some callers cannot allocate device memory at all (a host framework owns every buffer and
only hands over the CSR arrays and the activations), so they cannot give snk_build its
workspace.  snk_csr_forward_static computes Y = W X from a plain CSR matrix and keeps its
scratch in a static device array instead.  Here it is called through the C ABI twice in a
row -- the shared scratch keeps the previous call's contents, so the second call checks
that nothing stale leaks through -- and each result is compared with snk_forward on the
same matrix, within the parity tolerance of the other GPU tests.  This file is collected
last so that a run stopping at the first failure has already run every other test.
"""

import numpy as np
import pytest
import torch

import oracle
from helpers import explicit_layer, f64, gpu_layout, to_dev
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


def _abs_terms(L, X: torch.Tensor) -> np.ndarray:
    """Sum of |terms| per output (the normalisation of the parity metric)."""
    arr = L.arrays()
    row, col = arr["row"].cpu().numpy(), arr["col"].cpu().numpy()
    v = np.abs(f64(L.values))
    _, A = oracle.forward(L.M, L.K, row, col, v, np.abs(f64(X)))
    return A


def _check_against_forward(layer, Ns, num_parts=0):
    L = gpu_layout(layer)
    arr = L.arrays()
    tol = oracle.tolerance(layer.dtype)
    for call, N in enumerate(Ns):
        X = to_dev(wl.activations(layer.K, N, layer.dtype, seed=10 + call, stream=2))
        ref = L.forward(X)
        Y = torch.full_like(ref, float("nan"))
        snk.snk_csr_forward_static(L.M, L.K, arr["row_ptr"], arr["col"], L.values, X, Y, num_parts=num_parts)
        torch.cuda.synchronize()
        err = oracle.normalized_error(f64(Y), f64(ref), _abs_terms(L, X))
        assert err <= tol, f"call {call}: normalized error {err:.3e} > {tol:.1e}"


def test_static_forward_matches_forward_twice():
    layer = wl.uniform_layer(4096, 4096, 0.95, "bf16", 0, "W")
    _check_against_forward(layer, (8, 32, 300))


def test_static_forward_long_rows_and_ragged_batch():
    # dense rows longer than a part exercise the carry slots and counters of the scratch
    rng = np.random.default_rng(3)
    M, K = 300, 5000
    lin = set(rng.choice(M * K, size=20000, replace=False).tolist())
    lin |= {7 * K + c for c in range(K)} | {250 * K + c for c in range(K)}
    lin = np.array(sorted(lin))
    vals = rng.normal(0, 0.02, size=lin.size).astype(np.float32)
    layer = explicit_layer(M, K, lin // K, lin % K, vals, "f32")
    _check_against_forward(layer, (3, 70), num_parts=97)


def test_static_forward_rejects_too_many_parts():
    layer = wl.uniform_layer(64, 64, 0.5, "f32", 1, "W")
    L = gpu_layout(layer)
    arr = L.arrays()
    X = torch.randn(64, 4, device="cuda")
    Y = torch.empty(64, 4, device="cuda")
    with pytest.raises(snk.SnkError) as e:
        snk.snk_csr_forward_static(64, 64, arr["row_ptr"], arr["col"], L.values, X, Y, num_parts=513)
    assert e.value.status == "SNK_ERR_UNSUPPORTED"
