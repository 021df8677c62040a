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


def test_argument_checks_need_no_gpu(lib):
    """Calls reject bad arguments on the host, before touching the device."""
    import ctypes
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    INVALID = 1
    lib.snk_im2col3x3.restype = ctypes.c_int
    lib.snk_im2col3x3.argtypes = [vp, i64, i64, i64, i64, vp, i64, ctypes.c_int, vp]
    dummy = vp(256)
    assert lib.snk_im2col3x3(dummy, 0, 1, 2, 2, dummy, 4, 0, None) == INVALID       # C = 0
    assert lib.snk_im2col3x3(dummy, 2, 1, 2, 2, dummy, 3, 0, None) == INVALID       # ld < Nb*H*W
    assert lib.snk_im2col3x3(dummy, 7282, 1, 2, 2, dummy, 4, 0, None) == INVALID    # 9C > 65535
    assert lib.snk_im2col3x3(None, 2, 1, 2, 2, dummy, 4, 0, None) == INVALID        # null input
    assert lib.snk_im2col3x3(dummy, 2, 1, 2, 2, dummy, 4, 5, None) == INVALID       # no such dtype
    lib.snk_remap_entries.restype = ctypes.c_int
    lib.snk_remap_entries.argtypes = [vp, i64, vp, vp, i32, vp]
    assert lib.snk_remap_entries(dummy, 10, dummy, vp(512), 3, None) == INVALID     # element size
    assert lib.snk_remap_entries(dummy, 10, dummy, dummy, 4, None) == INVALID       # aliased
    assert lib.snk_remap_entries(None, 10, dummy, vp(512), 4, None) == INVALID      # null map
    assert lib.snk_remap_entries(None, 0, None, None, 4, None) == 0                 # nothing to do
    lib.snk_probe_fp32_fma.restype = ctypes.c_int
    lib.snk_probe_fp32_fma.argtypes = [i32, i32, vp, vp]
    assert lib.snk_probe_fp32_fma(0, 10, dummy, None) == INVALID
    assert lib.snk_probe_fp32_fma(4, 10, None, None) == INVALID
    lib.snk_probe_fp32_fma_flops.restype = i64
    lib.snk_probe_fp32_fma_flops.argtypes = [i32, i32]
    assert lib.snk_probe_fp32_fma_flops(2, 3) == 2 * 512 * 3 * 8 * 2 * 2
    lib.snk_set_index_bits.restype = ctypes.c_int
    lib.snk_set_index_bits.argtypes = [vp, i32]
    assert lib.snk_set_index_bits(None, 16) == INVALID
    lib.snk_sync_status.restype = ctypes.c_int
    lib.snk_sync_status.argtypes = [vp, vp]
    assert lib.snk_sync_status(None, None) == INVALID
