"""16-bit indices (snk_set_index_bits): the products must give bit-identical results.

When M and K fit 16 bits the layout also keeps 16-bit copies of col and csc_row, and the
kernels can read those instead of the int32 arrays.  Only the width of the index loads
changes, so every output must equal the 32-bit run's bit for bit: checked for the small-N
kernels, the TMA wide-N kernel and the SDDMM, for fp32 and bf16, after a restructure (the
copies are refreshed), and the switch is refused when a dimension exceeds 65536.
"""

import numpy as np
import pytest
import torch

from helpers import bits, explicit_layer, gpu_layout, to_dev
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


def _all_products(L, layer, N, seed=0):
    X = to_dev(wl.activations(layer.K, N, layer.dtype, seed, 2))
    dY = to_dev(wl.activations(layer.M, N, layer.dtype, seed, 3))
    return [bits(L.forward(X)), bits(L.backward_input(dY)), bits(L.backward_weight(dY, X))]


def _same_both_widths(L, layer, Ns):
    for N in Ns:
        L.set_index_bits(32)
        ref = _all_products(L, layer, N)
        L.set_index_bits(16)
        got = _all_products(L, layer, N)
        for name, a, b in zip(("forward", "backward_input", "backward_weight"), ref, got):
            assert a.tobytes() == b.tobytes(), f"{name} at N={N} differs between 32- and 16-bit indices"
    L.set_index_bits(32)


@pytest.mark.parametrize("N", [1, 8, 32])
def test_fc4096_bf16(N):
    layer = wl.uniform_layer(4096, 4096, 0.95, "bf16", 0, "W")
    _same_both_widths(gpu_layout(layer), layer, [N])


def test_tiny_fc_and_wide_f32():
    layer = wl.uniform_layer(512, 512, 0.90, "f32", 0, "W")
    _same_both_widths(gpu_layout(layer), layer, [8, 300])


def test_llama_up_zipf_bf16():
    layer = wl.zipf_layer(11008, 4096, 0.99, "bf16", 1.2, 0, "W_up")
    _same_both_widths(gpu_layout(layer), layer, [1, 16, 264])


def test_after_restructure():
    layer = wl.uniform_layer(700, 900, 0.9, "f32", 3, "W")
    L = gpu_layout(layer)
    L.restructure(layer.nnz // 10, seed=5)
    arr = L.arrays()
    new_layer = explicit_layer(700, 900, arr["row"].cpu().numpy(), arr["col"].cpu().numpy(),
                               L.values.cpu().numpy(), "f32")
    _same_both_widths(L, new_layer, [8, 256])


def test_refused_for_wide_dimensions():
    rng = np.random.default_rng(1)
    M, K = 8, 70000
    lin = np.sort(rng.choice(M * K, size=500, replace=False))
    layer = explicit_layer(M, K, lin // K, lin % K, rng.normal(size=lin.size).astype(np.float32), "f32")
    L = gpu_layout(layer)
    with pytest.raises(snk.SnkError) as e:
        L.set_index_bits(16)
    assert e.value.status == "SNK_ERR_UNSUPPORTED"
    with pytest.raises(snk.SnkError) as e:
        L.set_index_bits(8)
    assert e.value.status == "SNK_ERR_INVALID_ARG"
