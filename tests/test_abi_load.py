"""CPU-side checks of the C-ABI library: it loads without a GPU, exports every symbol the
header declares, and its pure host helpers behave as documented."""

import os
import re

import pytest

from sparse_spmm_b200 import build as snk_build_mod
from sparse_spmm_b200 import snk

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "snk.h")


@pytest.fixture(scope="module")
def lib():
    snk_build_mod.build()
    return snk.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(snk_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("snk_build", "snk_forward", "snk_backward_input", "snk_backward_weight",
                     "snk_restructure", "snk_workspace_bytes", "snk_layout_info", "snk_destroy"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(snk.EXPORTED) <= set(declared_functions())


def test_status_strings(lib):
    assert snk.snk_status_string(0) == "SNK_OK"
    assert snk.snk_status_string(3) == "SNK_ERR_DUPLICATE"
    assert snk.snk_status_string(9) == "SNK_ERR_CUDA"
    assert snk.snk_status_string(77) == "SNK_ERR_UNKNOWN"


def test_default_num_parts(lib):
    assert snk.snk_default_num_parts(0, 148) == 1
    assert snk.snk_default_num_parts(256, 148) == 1
    assert snk.snk_default_num_parts(257, 148) == 2
    assert snk.snk_default_num_parts(838861, 148) == 444
    assert snk.snk_default_num_parts(10**9, 148) == 444


def test_workspace_bytes_rejects_bad_sizes(lib):
    assert snk.snk_workspace_bytes(0, 5, 0, 4) == 0
    assert snk.snk_workspace_bytes(5, 5, 26, 4) == 0  # nnz > M*K
    assert snk.snk_workspace_bytes(5, 5, 3, -1) == 0
    assert snk.snk_workspace_bytes(4096, 4096, 838861, 592) > 0
