"""Property tests: random small problems against the oracle (hypothesis drives the shapes).

Each example draws M, K, a density, a structure (uniform, one dense row, empty rows and
columns), a dtype, N (up to 300, so the wide-N TMA kernel is reached too), a leading-
dimension pad and a part count, builds the layout on the GPU, checks the index arrays
byte for byte, and compares all three products with the oracle within the tolerances.
"""

import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
from helpers import check_build, check_products, explicit_layer, gpu_layout

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from sparse_spmm_b200 import build
    build.build()
    yield


@st.composite
def problems(draw):
    M = draw(st.integers(1, 120))
    K = draw(st.integers(1, 120))
    density = draw(st.sampled_from([0.01, 0.05, 0.2, 0.5, 1.0]))
    structure = draw(st.sampled_from(["uniform", "dense_row", "holes"]))
    dtype = draw(st.sampled_from(["f32", "bf16"]))
    N = draw(st.sampled_from([1, 2, 3, 7, 16, 33, 64, 65, 130, 256, 300]))
    pad = draw(st.sampled_from([0, 0, 1, 4]))
    parts = draw(st.sampled_from([0, 1, 3, 17, 500]))
    seed = draw(st.integers(0, 2**31 - 1))
    return M, K, density, structure, dtype, N, pad, parts, seed


@settings(max_examples=40, deadline=None, suppress_health_check=[HealthCheck.function_scoped_fixture])
@given(problems())
def test_random_problems_match_the_oracle(p):
    M, K, density, structure, dtype, N, pad, parts, seed = p
    rng = np.random.default_rng(seed)
    nnz = int(round(density * M * K))
    lin = set(rng.choice(M * K, size=nnz, replace=False).tolist()) if nnz else set()
    if structure == "dense_row":
        r = int(rng.integers(M))
        lin |= {r * K + c for c in range(K)}
    elif structure == "holes":  # drop every entry of a few rows and columns
        dead_r = set(rng.choice(M, size=max(1, M // 4), replace=False).tolist())
        dead_c = set(rng.choice(K, size=max(1, K // 4), replace=False).tolist())
        lin = {e for e in lin if e // K not in dead_r and e % K not in dead_c}
    lin = np.array(sorted(lin), dtype=np.int64)
    lin = lin[rng.permutation(lin.size)]
    vals = rng.normal(0, 0.02, size=lin.size).astype(np.float32)
    layer = explicit_layer(M, K, lin // K, lin % K, vals, dtype)
    P = 0 if parts == 0 else min(parts, max(lin.size, 1))
    L = gpu_layout(layer, num_parts=P)
    ref = check_build(L, layer)
    check_products(layer, ref, L, N, seed=seed % 1000, pad=pad)
    L.sync_status()
