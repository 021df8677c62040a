"""The TMA kernel's bounded waits: a wait that runs out is reported, and the GPU stays usable.

SNK_TEST_TMA_EXTRA_TX makes every staged chunk expect a few bytes more than its tensor copy
delivers, so no chunk barrier completes: every wait of the kernel runs out after about a
second, the kernel sets the timeout bit and returns (its copies have all landed; nothing
faults).  snk_sync_status must then report SNK_ERR_TIMEOUT, clear the bit, and the next
launch without the hook must give the right result.  The smallest launch that takes the
TMA path is used (one row block, two column slices).
"""

import os

import numpy as np
import pytest
import torch

import oracle
from helpers import f64, gpu_layout, to_dev
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


def test_wait_runs_out_and_is_reported():
    layer = wl.uniform_layer(16, 200, 0.8, "f32", 4, "W")
    L = gpu_layout(layer)
    X = to_dev(wl.activations(200, 256, "f32", 0, 2))
    os.environ["SNK_TEST_TMA_EXTRA_TX"] = "16"
    try:
        L.forward(X)
        with pytest.raises(snk.SnkError) as e:
            L.sync_status()
        assert e.value.status == "SNK_ERR_TIMEOUT"
    finally:
        del os.environ["SNK_TEST_TMA_EXTRA_TX"]
    L.sync_status()  # the bit was cleared
    Y = L.forward(X)
    L.sync_status()
    arr = L.arrays()
    Yr, A = oracle.forward(16, 200, arr["row"].cpu().numpy(), arr["col"].cpu().numpy(), f64(L.values), f64(X))
    err = oracle.normalized_error(f64(Y), Yr, A)
    assert err <= oracle.tolerance("f32")
