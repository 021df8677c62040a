"""B200-native truly-sparse layer: SpMM, transposed SpMM and SDDMM over a COO weight.

The compute lives in the CUDA library ``libsnk.so`` (C ABI in ``include/snk.h``, built by
``python -m sparse_spmm_b200.build``); ``sparse_spmm_b200.snk`` is its ctypes binding and
``sparse_spmm_b200.workloads`` draws the seeded synthetic inputs.
"""

__all__ = ["snk", "workloads"]
