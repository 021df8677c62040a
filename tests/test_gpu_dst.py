"""Dynamic sparse training: state remap across a restructure, and a short training run.

snk_remap_entries must move every surviving entry's state to its new index and zero the
regrown ones (checked bit for bit against the definition, written out with numpy from the
map).  A two-layer sparse chain trained with momentum SGD on a teacher target, with a
prune-and-regrow every 20 steps, must keep nnz, keep its layouts sorted and unique, carry
the momentum of survivors unchanged, and still reduce the loss.
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


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_remap_entries_definition(dtype):
    layer = wl.uniform_layer(300, 200, 0.9, dtype, 2, "W")
    L = gpu_layout(layer)
    o2n = L.restructure(layer.nnz // 7, seed=11)
    rng = np.random.default_rng(0)
    src = to_dev(wl.cast(rng.normal(size=layer.nnz).astype(np.float32), dtype))
    dst = snk.snk_remap_entries(o2n, src, torch.full_like(src, 7.0))
    torch.cuda.synchronize()
    m = o2n.cpu().numpy()
    s_bits = bits(src)
    expect = np.zeros_like(s_bits)
    keep = m >= 0
    expect[m[keep]] = s_bits[keep]
    assert bits(dst).tobytes() == expect.tobytes()
    assert keep.sum() == layer.nnz - layer.nnz // 7


def _check_layout(layer_mod):
    arr = layer_mod.layout.arrays()
    r, c = arr["row"].cpu().numpy().astype(np.int64), arr["col"].cpu().numpy().astype(np.int64)
    lin = r * layer_mod.layout.K + c
    assert np.all(np.diff(lin) > 0), "entries not sorted and unique"
    assert lin.size == layer_mod.nnz


def test_short_dst_run():
    from sparse_spmm_b200.dst import MomentumSGD, SparseLinear, prune_and_regrow
    torch.manual_seed(0)
    K0, H, K1, N = 64, 96, 64, 256  # N = 256 takes the TMA kernels for the products
    l1 = wl.uniform_layer(H, K0, 0.8, "f32", 1, "W1")
    l2 = wl.uniform_layer(K1, H, 0.8, "f32", 2, "W2")
    W1 = SparseLinear(H, K0, to_dev(l1.row), to_dev(l1.col), to_dev(l1.values * 10))
    W2 = SparseLinear(K1, H, to_dev(l2.row), to_dev(l2.col), to_dev(l2.values * 10))
    teacher = torch.randn(K1, K0, device="cuda") / K0 ** 0.5
    X = torch.randn(K0, N, device="cuda")
    T = teacher @ X
    opt = MomentumSGD([W1.weight, W2.weight], lr=0.1, momentum=0.9)
    nnz0 = (W1.nnz, W2.nnz)
    losses = []
    for step in range(60):
        if step > 0 and step % 20 == 0:
            for j, lay in enumerate((W1, W2)):
                before = opt.state[id(lay.weight)].clone()
                o2n = prune_and_regrow(lay, 0.1, seed=100 * step + j, optimizer=opt)
                m = o2n.cpu().numpy()
                keep = m >= 0
                after = opt.state[id(lay.weight)].cpu().numpy()
                assert np.array_equal(after[m[keep]], before.cpu().numpy()[keep])
                assert np.all(after[np.setdiff1d(np.arange(lay.nnz), m[keep])] == 0)
                _check_layout(lay)
        opt.zero_grad()
        Y = W2(W1(X))
        loss = ((Y - T) ** 2).mean()
        loss.backward()
        opt.step()
        losses.append(float(loss.detach()))
    assert (W1.nnz, W2.nnz) == nnz0
    assert np.all(np.isfinite(losses))
    assert losses[-1] < 0.75 * losses[0], losses[::10]
    W1.layout.sync_status()
    W2.layout.sync_status()
