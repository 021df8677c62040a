"""CPU oracle for the truly-sparse layer (plain C loops, fp64 accumulation).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this package.  The
product path (``sparse_spmm_b200``) never imports it and shares no code with it.

The arithmetic lives in ``oracle.c`` (compiled here with gcc into ``_build/liboracle.so``);
this module only marshals numpy arrays.  Value arrays arrive as raw bit patterns: float32
arrays, or uint16 arrays holding bfloat16 bits.  ``widen`` turns either into float64
exactly (a bfloat16 is the upper half of a float32).

Definitions follow "Beyond Masked Sparsity: SNACK Enables Truly Sparse Neural Networks on
GPU" (arXiv 2610.04093), Abstract; the readings taken where that page is silent are stated
in ``oracle.c``.  Parity pins for every function are in ``tests/test_oracle_pins.py``.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "liboracle.so")

STATUS = {
    0: "OK",
    1: "INVALID_ARG",
    2: "OUT_OF_RANGE",
    3: "DUPLICATE",
    6: "INVALID_VALUE",
    7: "NO_ROOM",
}

_lib = None


def compile_oracle(force: bool = False) -> str:
    """Compile oracle.c into _build/liboracle.so (plain -O2, no vectorisation flags)."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=gnu11", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(compile_oracle())
        i64, i32, vp, dbl, u64 = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p, ctypes.c_double, ctypes.c_uint64
        lib.orc_build.restype = ctypes.c_int
        lib.orc_build.argtypes = [i64, i64, i64, vp, vp, vp, ctypes.c_int, i32] + [vp] * 7 + [vp] + [vp] * 4
        lib.orc_effective_parts.restype = i32
        lib.orc_effective_parts.argtypes = [i64, i32]
        lib.orc_forward.restype = None
        lib.orc_forward.argtypes = [i64, i64, i64, vp, vp, vp, vp, i64, vp, vp]
        lib.orc_backward_input.restype = None
        lib.orc_backward_input.argtypes = [i64, i64, i64, vp, vp, vp, vp, i64, vp, vp]
        lib.orc_backward_weight.restype = None
        lib.orc_backward_weight.argtypes = [i64, vp, vp, vp, vp, i64, vp, vp]
        lib.orc_splitmix64.restype = None
        lib.orc_splitmix64.argtypes = [u64, i64, vp]
        lib.orc_conv3x3.restype = None
        lib.orc_conv3x3.argtypes = [i64, i64, i64, i64, i64, i64, vp, vp, vp, vp, vp, vp]
        lib.orc_im2col3x3.restype = None
        lib.orc_im2col3x3.argtypes = [i64, i64, i64, i64, ctypes.c_int, vp, vp, i64]
        lib.orc_restructure.restype = ctypes.c_int
        lib.orc_restructure.argtypes = [i64, i64, i64, vp, vp, vp, vp, ctypes.c_int, i64, u64, dbl,
                                        vp, vp, vp, vp, vp]
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def widen(values: np.ndarray) -> np.ndarray:
    """Exact float64 copy of float32 values or of bfloat16 bits held in uint16."""
    if values.dtype == np.float32:
        return values.astype(np.float64)
    if values.dtype == np.uint16:
        return (values.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    raise TypeError("values must be float32 or uint16 (bfloat16 bits)")


class OracleError(RuntimeError):
    def __init__(self, code: int):
        super().__init__(STATUS.get(code, str(code)))
        self.code = code
        self.status = STATUS.get(code, str(code))


def effective_parts(nnz: int, P: int) -> int:
    return int(_load().orc_effective_parts(nnz, P))


def build(M: int, K: int, row, col, values: np.ndarray, P: int) -> dict:
    """O1-O4.  Returns the sorted COO (values moved bit-exactly) and the derived arrays."""
    lib = _load()
    row = _c(row, np.int32)
    col = _c(col, np.int32)
    values = np.ascontiguousarray(values)
    nnz = row.size
    vb = values.dtype.itemsize
    out = {
        "row": np.empty(nnz, np.int32), "col": np.empty(nnz, np.int32),
        "values": np.empty(nnz, values.dtype),
        "row_ptr": np.empty(M + 1, np.int32), "perm": np.empty(nnz, np.int32),
        "col_ptr": np.empty(K + 1, np.int32), "csc_row": np.empty(nnz, np.int32),
    }
    Pe = effective_parts(nnz, P) if P >= 1 else 1
    for name in ("part_nnz", "part_row", "part_nnz_t", "part_col"):
        out[name] = np.empty(Pe + 1, np.int32)
    peff = np.zeros(1, np.int32)
    rc = lib.orc_build(M, K, nnz, _p(row), _p(col), _p(values), vb, P,
                       _p(out["row"]), _p(out["col"]), _p(out["values"]), _p(out["row_ptr"]),
                       _p(out["perm"]), _p(out["col_ptr"]), _p(out["csc_row"]), _p(peff),
                       _p(out["part_nnz"]), _p(out["part_row"]), _p(out["part_nnz_t"]),
                       _p(out["part_col"]))
    if rc != 0:
        raise OracleError(rc)
    out["num_parts"] = int(peff[0])
    return out


def conv3x3(Co: int, C: int, Nb: int, H: int, W: int, row, col, vals64, X64) -> tuple[np.ndarray, np.ndarray]:
    """3x3 convolution, stride 1, zero padding 1, of X (C x Nb x H x W) by the sparse kernel
    given as entries (co, ci*9 + kh*3 + kw); returns (Y, A), Co x (Nb*H*W) float64."""
    row, col = _c(row, np.int32), _c(col, np.int32)
    v, X = _c(vals64, np.float64), _c(np.asarray(X64).reshape(C, Nb * H * W), np.float64)
    Y = np.empty((Co, Nb * H * W)); A = np.empty((Co, Nb * H * W))
    _load().orc_conv3x3(Co, C, Nb, H, W, row.size, _p(row), _p(col), _p(v), _p(X), _p(Y), _p(A))
    return Y, A


def im2col3x3(C: int, Nb: int, H: int, W: int, X: np.ndarray) -> np.ndarray:
    """Patch matrix (9C) x (Nb*H*W) of X (C x Nb x H x W; float32 or bf16 bits), bit for bit."""
    X = np.ascontiguousarray(X)
    out = np.empty((9 * C, Nb * H * W), dtype=X.dtype)
    _load().orc_im2col3x3(C, Nb, H, W, X.itemsize, _p(X), _p(out), Nb * H * W)
    return out


def forward(M: int, K: int, row, col, vals64, X64) -> tuple[np.ndarray, np.ndarray]:
    """O5: (Y, A) with Y = W X and A = sum of |terms| per output, both M x N float64."""
    row, col = _c(row, np.int32), _c(col, np.int32)
    v, X = _c(vals64, np.float64), _c(X64, np.float64)
    N = X.shape[1]
    assert X.shape[0] == K
    Y = np.empty((M, N)); A = np.empty((M, N))
    _load().orc_forward(M, K, row.size, _p(row), _p(col), _p(v), _p(X), N, _p(Y), _p(A))
    return Y, A


def backward_input(M: int, K: int, row, col, vals64, dY64) -> tuple[np.ndarray, np.ndarray]:
    """O6: (dX, A) with dX = W^T dY, K x N float64."""
    row, col = _c(row, np.int32), _c(col, np.int32)
    v, dY = _c(vals64, np.float64), _c(dY64, np.float64)
    N = dY.shape[1]
    assert dY.shape[0] == M
    dX = np.empty((K, N)); A = np.empty((K, N))
    _load().orc_backward_input(M, K, row.size, _p(row), _p(col), _p(v), _p(dY), N, _p(dX), _p(A))
    return dX, A


def backward_weight(row, col, dY64, X64) -> tuple[np.ndarray, np.ndarray]:
    """O7: (dW, A) with dW[e] = sum_n dY[row_e, n] X[col_e, n], float64 per entry."""
    row, col = _c(row, np.int32), _c(col, np.int32)
    dY, X = _c(dY64, np.float64), _c(X64, np.float64)
    N = X.shape[1]
    assert dY.shape[1] == N
    dW = np.empty(row.size); A = np.empty(row.size)
    _load().orc_backward_weight(row.size, _p(row), _p(col), _p(dY), _p(X), N, _p(dW), _p(A))
    return dW, A


def splitmix64(seed: int, n: int) -> np.ndarray:
    """The first n outputs of SplitMix64 seeded with `seed`."""
    out = np.empty(n, np.uint64)
    _load().orc_splitmix64(seed, n, _p(out))
    return out


def restructure(M: int, K: int, row, col, values: np.ndarray, k: int, seed: int,
                regrow_value: float = 0.0) -> dict:
    """O8 on a sorted COO.  Returns new row/col/values (bit patterns), old_to_new, draws."""
    row, col = _c(row, np.int32), _c(col, np.int32)
    values = np.ascontiguousarray(values)
    v64 = widen(values)
    nnz = row.size
    out = {"row": np.empty(nnz, np.int32), "col": np.empty(nnz, np.int32),
           "values": np.empty(nnz, values.dtype), "old_to_new": np.empty(nnz, np.int32)}
    draws = np.zeros(1, np.int64)
    rc = _load().orc_restructure(M, K, nnz, _p(row), _p(col), _p(values), _p(v64),
                                 values.dtype.itemsize, k, seed, float(regrow_value),
                                 _p(out["row"]), _p(out["col"]), _p(out["values"]),
                                 _p(out["old_to_new"]), _p(draws))
    if rc != 0:
        raise OracleError(rc)
    out["draws"] = int(draws[0])
    return out


def tolerance(dtype: str) -> float:
    """Parity bound on max |g - r| / A: 1e-5 for fp32 inputs, 2e-2 for bf16 inputs."""
    return 1e-5 if dtype == "f32" else 2e-2


def normalized_error(got: np.ndarray, ref: np.ndarray, A: np.ndarray) -> float:
    """max |g - r| / A over all outputs; where A == 0 the output must be exactly 0."""
    got = np.asarray(got, np.float64)
    zero = A == 0
    if np.any(got[zero] != 0):
        return float("inf")
    nz = ~zero
    if not np.any(nz):
        return 0.0
    return float(np.max(np.abs(got[nz] - ref[nz]) / A[nz]))
