"""Concurrency and capture: the products on several streams at once, and inside CUDA graphs.

The header allows snk_forward, snk_backward_input and snk_backward_weight on one layout to
overlap in time (each product direction has its own carry slots; the SDDMM uses none), and
every product is capturable (no host synchronisation, no allocation).  Results must equal
the serial, eager run bit for bit, small-N and wide-N.
"""

import pytest
import torch

from helpers import bits, gpu_layout, to_dev
from sparse_spmm_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from sparse_spmm_b200 import build
    build.build()
    yield


@pytest.mark.parametrize("N", [8, 300])
def test_three_streams_match_serial(N):
    layer = wl.uniform_layer(2000, 1500, 0.95, "bf16", 8, "W")
    L = gpu_layout(layer)
    X = to_dev(wl.activations(layer.K, N, "bf16", 1, 2))
    dY = to_dev(wl.activations(layer.M, N, "bf16", 1, 3))
    ref = [bits(L.forward(X)), bits(L.backward_input(dY)), bits(L.backward_weight(dY, X))]
    streams = [torch.cuda.Stream() for _ in range(3)]
    outs = [torch.empty(layer.M, N, dtype=torch.bfloat16, device="cuda"),
            torch.empty(layer.K, N, dtype=torch.bfloat16, device="cuda"),
            torch.empty(layer.nnz, dtype=torch.bfloat16, device="cuda")]
    torch.cuda.synchronize()
    for _ in range(5):
        L.forward(X, Y=outs[0], stream=streams[0])
        L.backward_input(dY, dX=outs[1], stream=streams[1])
        L.backward_weight(dY, X, dW=outs[2], stream=streams[2])
    torch.cuda.synchronize()
    for r, o in zip(ref, outs):
        assert r.tobytes() == bits(o).tobytes()
    L.sync_status()


@pytest.mark.parametrize("N", [32, 256])
def test_graph_capture_matches_eager(N):
    layer = wl.uniform_layer(1200, 900, 0.9, "f32", 9, "W")
    L = gpu_layout(layer)
    X = to_dev(wl.activations(layer.K, N, "f32", 1, 2))
    dY = to_dev(wl.activations(layer.M, N, "f32", 1, 3))
    ref = [bits(L.forward(X)), bits(L.backward_input(dY)), bits(L.backward_weight(dY, X))]
    Y = torch.empty(layer.M, N, device="cuda")
    dX = torch.empty(layer.K, N, device="cuda")
    dW = torch.empty(layer.nnz, device="cuda")
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=s):
        L.forward(X, Y=Y, stream=s)
        L.backward_input(dY, dX=dX, stream=s)
        L.backward_weight(dY, X, dW=dW, stream=s)
    for _ in range(3):
        with torch.cuda.stream(s):
            g.replay()
    s.synchronize()
    for r, o in zip(ref, (Y, dX, dW)):
        assert r.tobytes() == bits(o).tobytes()
    L.sync_status()
