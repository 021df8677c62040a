"""Thin ctypes binding of libsnk.so (the C ABI declared in include/snk.h).

Argument marshalling only: torch tensors supply device memory and the current CUDA stream,
and every step of the layer runs in the library's kernels.  There is no fallback: if the
library is missing or a call fails, an exception is raised.

Low-level functions carry the C names (``snk_build``, ``snk_forward``, ...).  ``Layout``
bundles a built layout with its workspace tensor for convenience.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsnk.so")

SNK_F32, SNK_BF16 = 0, 1
_STATUS = ["SNK_OK", "SNK_ERR_INVALID_ARG", "SNK_ERR_OUT_OF_RANGE", "SNK_ERR_DUPLICATE",
           "SNK_ERR_WORKSPACE_TOO_SMALL", "SNK_ERR_UNSUPPORTED", "SNK_ERR_INVALID_VALUE",
           "SNK_ERR_NO_ROOM", "SNK_ERR_TIMEOUT", "SNK_ERR_CUDA"]

EXPORTED = ("snk_status_string", "snk_default_num_parts", "snk_workspace_bytes", "snk_build",
            "snk_forward", "snk_backward_input", "snk_backward_weight", "snk_restructure",
            "snk_layout_info", "snk_destroy")


class SnkError(RuntimeError):
    def __init__(self, code: int, where: str = ""):
        name = _STATUS[code] if 0 <= code < len(_STATUS) else str(code)
        super().__init__(f"{where}: {name}" if where else name)
        self.code = code
        self.status = name


class _View(ctypes.Structure):
    _fields_ = [("M", ctypes.c_int64), ("K", ctypes.c_int64), ("nnz", ctypes.c_int64),
                ("num_parts", ctypes.c_int32), ("dtype", ctypes.c_int32), ("device", ctypes.c_int32)] + \
               [(n, ctypes.c_void_p) for n in ("row", "col", "row_ptr", "col_ptr", "csc_row", "perm",
                                               "part_nnz", "part_row", "part_nnz_t", "part_col")]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libsnk.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m sparse_spmm_b200.build`")
    lib = ctypes.CDLL(path)
    i64, i32, vp, u64 = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p, ctypes.c_uint64
    st = ctypes.c_int
    lib.snk_status_string.restype = ctypes.c_char_p
    lib.snk_status_string.argtypes = [st]
    lib.snk_default_num_parts.restype = i32
    lib.snk_default_num_parts.argtypes = [i64, i32]
    lib.snk_workspace_bytes.restype = ctypes.c_size_t
    lib.snk_workspace_bytes.argtypes = [i64, i64, i64, i32]
    lib.snk_build.restype = st
    lib.snk_build.argtypes = [i64, i64, i64, vp, vp, vp, st, i32, vp, ctypes.c_size_t, vp,
                              ctypes.POINTER(vp)]
    lib.snk_forward.restype = st
    lib.snk_forward.argtypes = [vp, vp, vp, i64, i64, vp, i64, st, vp]
    lib.snk_backward_input.restype = st
    lib.snk_backward_input.argtypes = [vp, vp, vp, i64, i64, vp, i64, st, vp]
    lib.snk_backward_weight.restype = st
    lib.snk_backward_weight.argtypes = [vp, vp, i64, vp, i64, i64, vp, st, vp]
    lib.snk_restructure.restype = st
    lib.snk_restructure.argtypes = [vp, vp, i64, u64, ctypes.c_float, vp, vp]
    lib.snk_layout_info.restype = st
    lib.snk_layout_info.argtypes = [vp, ctypes.POINTER(_View)]
    lib.snk_destroy.restype = None
    lib.snk_destroy.argtypes = [vp]
    _lib = lib
    return lib


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return SNK_F32
    if t == torch.bfloat16:
        return SNK_BF16
    raise TypeError(f"unsupported dtype {t}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(code: int, where: str):
    if code != 0:
        raise SnkError(code, where)


def _ld(t: torch.Tensor) -> int:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("dense operands must be 2-D with unit column stride")
    return t.stride(0)


# ----------------------------------------------------------------------------- C-named calls

def snk_status_string(code: int) -> str:
    return load_library().snk_status_string(code).decode()


def snk_default_num_parts(nnz: int, sm_count: int) -> int:
    return int(load_library().snk_default_num_parts(nnz, sm_count))


def snk_workspace_bytes(M: int, K: int, nnz: int, num_parts: int = 0) -> int:
    return int(load_library().snk_workspace_bytes(M, K, nnz, num_parts))


def snk_build(M, K, row, col, values, num_parts, workspace, stream=None):
    """Sorts row/col/values in place and returns an opaque layout handle (c_void_p)."""
    out = ctypes.c_void_p()
    nnz = row.numel()
    code = load_library().snk_build(M, K, nnz, _ptr(row), _ptr(col), _ptr(values), _dtype_code(values.dtype),
                                    num_parts, _ptr(workspace), workspace.numel(), _stream(stream),
                                    ctypes.byref(out))
    _check(code, "snk_build")
    return out


def snk_forward(handle, values, X, N, ldx, Y, ldy, stream=None):
    _check(load_library().snk_forward(handle, _ptr(values), _ptr(X), N, ldx, _ptr(Y), ldy,
                                      _dtype_code(X.dtype), _stream(stream)), "snk_forward")


def snk_backward_input(handle, values, dY, N, lddy, dX, lddx, stream=None):
    _check(load_library().snk_backward_input(handle, _ptr(values), _ptr(dY), N, lddy, _ptr(dX), lddx,
                                             _dtype_code(dY.dtype), _stream(stream)), "snk_backward_input")


def snk_backward_weight(handle, dY, lddy, X, ldx, N, dW, stream=None):
    _check(load_library().snk_backward_weight(handle, _ptr(dY), lddy, _ptr(X), ldx, N, _ptr(dW),
                                              _dtype_code(X.dtype), _stream(stream)), "snk_backward_weight")


def snk_restructure(handle, values, drop_count, seed, regrow_value=0.0, old_to_new=None, stream=None):
    _check(load_library().snk_restructure(handle, _ptr(values), drop_count, seed, regrow_value,
                                          _ptr(old_to_new), _stream(stream)), "snk_restructure")


def snk_layout_info(handle) -> _View:
    v = _View()
    _check(load_library().snk_layout_info(handle, ctypes.byref(v)), "snk_layout_info")
    return v


def snk_destroy(handle):
    if handle:
        load_library().snk_destroy(handle)


def snk_csr_forward_static(M, K, row_ptr, col, values, X, Y, num_parts=0, stream=None):
    """Y = W X from a plain CSR matrix; the library allocates nothing (static scratch)."""
    lib = load_library()
    fn = lib.snk_csr_forward_static
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                   ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p]
    N = X.shape[1]
    _check(fn(M, K, col.numel(), _ptr(row_ptr), _ptr(col), _ptr(values), _dtype_code(X.dtype), _ptr(X), N,
              _ld(X), _ptr(Y), _ld(Y), num_parts, _stream(stream)), "snk_csr_forward_static")


def snk_im2col3x3(x, C, Nb, H, W, out=None, stream=None):
    """Patch matrix (9C) x (Nb*H*W) of a channel-major x (C x Nb x H x W) for a 3x3 convolution."""
    lib = load_library()
    lib.snk_im2col3x3.restype = ctypes.c_int
    lib.snk_im2col3x3.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                  ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p]
    if not x.is_contiguous():
        raise ValueError("x must be contiguous (C x Nb x H x W)")
    if out is None:
        out = torch.empty((9 * C, Nb * H * W), dtype=x.dtype, device=x.device)
    _check(lib.snk_im2col3x3(_ptr(x), C, Nb, H, W, _ptr(out), _ld(out), _dtype_code(x.dtype), _stream(stream)),
           "snk_im2col3x3")
    return out


def sparse_conv3x3(L, x, Nb, H, W, patch=None, Y=None, stream=None):
    """A sparse 3x3 convolution (stride 1, padding 1): Y (Co x Nb*H*W) = W * x with W held by
    layout L (Co x 9C, column ci*9 + kh*3 + kw) and x channel-major (C x Nb x H x W)."""
    C = L.K // 9
    patch = snk_im2col3x3(x, C, Nb, H, W, out=patch, stream=stream)
    return L.forward(patch, Y=Y, stream=stream)


def snk_remap_entries(old_to_new, src, dst, stream=None):
    """dst[old_to_new[e]] = src[e] for surviving entries, 0 elsewhere (state across a restructure)."""
    lib = load_library()
    lib.snk_remap_entries.restype = ctypes.c_int
    lib.snk_remap_entries.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                      ctypes.c_int32, ctypes.c_void_p]
    _check(lib.snk_remap_entries(_ptr(old_to_new), src.numel(), _ptr(src), _ptr(dst), src.element_size(),
                                 _stream(stream)), "snk_remap_entries")
    return dst


def snk_set_index_bits(handle, bits):
    """Read 16- or 32-bit indices in the products (16 needs M, K <= 65536)."""
    lib = load_library()
    lib.snk_set_index_bits.restype = ctypes.c_int
    lib.snk_set_index_bits.argtypes = [ctypes.c_void_p, ctypes.c_int32]
    _check(lib.snk_set_index_bits(handle, bits), "snk_set_index_bits")


def snk_sync_status(handle, stream=None):
    """Synchronise and raise SnkError(SNK_ERR_TIMEOUT) if a product launch gave up a wait."""
    lib = load_library()
    lib.snk_sync_status.restype = ctypes.c_int
    lib.snk_sync_status.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    _check(lib.snk_sync_status(handle, _stream(stream)), "snk_sync_status")


def snk_probe_fp32_fma(blocks, iters, sink, stream=None):
    """Launch the fp32 FMA-rate probe (a measurement aid); returns its floating-point operations."""
    lib = load_library()
    lib.snk_probe_fp32_fma.restype = ctypes.c_int
    lib.snk_probe_fp32_fma.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]
    lib.snk_probe_fp32_fma_flops.restype = ctypes.c_int64
    lib.snk_probe_fp32_fma_flops.argtypes = [ctypes.c_int32, ctypes.c_int32]
    _check(lib.snk_probe_fp32_fma(blocks, iters, _ptr(sink), _stream(stream)), "snk_probe_fp32_fma")
    return int(lib.snk_probe_fp32_fma_flops(blocks, iters))


# ----------------------------------------------------------------------------- convenience

class Layout:
    """A built layout plus the workspace tensor that backs it.

    ``row``, ``col`` (int32) and ``values`` (float32 or bfloat16) are CUDA tensors; they are
    sorted in place by the build and must stay alive with the layout.
    """

    def __init__(self, M: int, K: int, row: torch.Tensor, col: torch.Tensor, values: torch.Tensor,
                 num_parts: int = 0, stream=None, workspace: torch.Tensor | None = None):
        if row.dtype != torch.int32 or col.dtype != torch.int32:
            raise TypeError("row/col must be int32")
        if not (row.is_cuda and col.is_cuda and values.is_cuda):
            raise ValueError("row, col and values must be CUDA tensors")
        if not (row.is_contiguous() and col.is_contiguous() and values.is_contiguous()):
            raise ValueError("row, col and values must be contiguous")
        self.M, self.K = int(M), int(K)
        self.row, self.col, self.values = row, col, values
        self.dtype = values.dtype
        nbytes = snk_workspace_bytes(self.M, self.K, row.numel(), num_parts)
        if nbytes == 0:
            raise SnkError(1, "snk_workspace_bytes")
        if workspace is None:
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=row.device)
        elif workspace.dtype != torch.uint8 or workspace.numel() < nbytes or not workspace.is_contiguous():
            raise ValueError(f"workspace must be a contiguous uint8 tensor of >= {nbytes} bytes")
        self.workspace = workspace
        self.handle = snk_build(self.M, self.K, row, col, values, num_parts, self.workspace, stream)
        info = snk_layout_info(self.handle)
        self.nnz = int(info.nnz)
        self.num_parts = int(info.num_parts)

    def __del__(self):
        h = getattr(self, "handle", None)
        if h and _lib is not None:
            try:
                _lib.snk_destroy(h)
            except Exception:  # interpreter shutdown: the library may already be gone
                pass
        self.handle = None

    def close(self):
        self.__del__()

    # -- products
    def forward(self, X: torch.Tensor, Y: torch.Tensor | None = None, values=None, stream=None):
        values = self.values if values is None else values
        N = X.shape[1]
        if Y is None:
            Y = torch.empty((self.M, N), dtype=X.dtype, device=X.device)
        snk_forward(self.handle, values, X, N, _ld(X), Y, _ld(Y), stream)
        return Y

    def backward_input(self, dY: torch.Tensor, dX: torch.Tensor | None = None, values=None, stream=None):
        values = self.values if values is None else values
        N = dY.shape[1]
        if dX is None:
            dX = torch.empty((self.K, N), dtype=dY.dtype, device=dY.device)
        snk_backward_input(self.handle, values, dY, N, _ld(dY), dX, _ld(dX), stream)
        return dX

    def backward_weight(self, dY: torch.Tensor, X: torch.Tensor, dW: torch.Tensor | None = None, stream=None):
        N = X.shape[1]
        if dW is None:
            dW = torch.empty(self.nnz, dtype=X.dtype, device=X.device)
        snk_backward_weight(self.handle, dY, _ld(dY), X, _ld(X), N, dW, stream)
        return dW

    def restructure(self, drop_count: int, seed: int, regrow_value: float = 0.0, want_map: bool = True,
                    stream=None):
        o2n = torch.empty(self.nnz, dtype=torch.int32, device=self.row.device) if want_map else None
        snk_restructure(self.handle, self.values, drop_count, seed, regrow_value, o2n, stream)
        return o2n

    def set_index_bits(self, bits: int):
        """Make the products read 16- or 32-bit indices (results are bit-identical)."""
        snk_set_index_bits(self.handle, bits)

    def sync_status(self, stream=None):
        """Synchronise; raise if a product launch on this layout gave up a bounded wait."""
        snk_sync_status(self.handle, stream)

    # -- inspection
    def arrays(self) -> dict:
        """Device arrays of the layout as int32 tensors (views of the workspace)."""
        v = snk_layout_info(self.handle)
        base = self.workspace.data_ptr()
        ws32 = self.workspace[: self.workspace.numel() // 4 * 4].view(torch.int32)

        def sl(ptr, n):
            off = ptr - base
            assert off % 4 == 0
            return ws32[off // 4: off // 4 + n]

        P = int(v.num_parts)
        return {
            "row": self.row, "col": self.col, "values": self.values,
            "row_ptr": sl(v.row_ptr, self.M + 1), "col_ptr": sl(v.col_ptr, self.K + 1),
            "csc_row": sl(v.csc_row, self.nnz), "perm": sl(v.perm, self.nnz),
            "part_nnz": sl(v.part_nnz, P + 1), "part_row": sl(v.part_row, P + 1),
            "part_nnz_t": sl(v.part_nnz_t, P + 1), "part_col": sl(v.part_col, P + 1),
            "num_parts": P,
        }


def save_layout(L: Layout, path) -> None:
    """Checkpoint a layout: its sizes, part count and sorted COO (row, col, value bits).  The
    derived arrays are state of the build, so a load rebuilds them (byte-identical)."""
    import numpy as np
    torch.cuda.synchronize(L.row.device)
    vbits = L.values.view(torch.int16) if L.values.dtype == torch.bfloat16 else L.values.view(torch.int32)
    np.savez(path, M=L.M, K=L.K, num_parts=L.num_parts,
             dtype="bf16" if L.values.dtype == torch.bfloat16 else "f32",
             row=L.row.cpu().numpy(), col=L.col.cpu().numpy(), value_bits=vbits.cpu().numpy())


def load_layout(path, device="cuda") -> Layout:
    """Rebuild a layout saved by save_layout on `device`."""
    import numpy as np
    z = np.load(path)
    bits_t = torch.from_numpy(z["value_bits"]).to(device)
    values = bits_t.view(torch.bfloat16) if str(z["dtype"]) == "bf16" else bits_t.view(torch.float32)
    return Layout(int(z["M"]), int(z["K"]), torch.from_numpy(z["row"]).to(device),
                  torch.from_numpy(z["col"]).to(device), values.contiguous(), num_parts=int(z["num_parts"]))


class SparseLinearFunction(torch.autograd.Function):
    """Y = W X with W held by a Layout; backward returns dX = W^T dY and dW (per entry).

    Inputs: values (the layout's value tensor, the trainable parameter), X (K x N).
    """

    @staticmethod
    def forward(ctx, values, X, layout):
        ctx.layout = layout
        ctx.save_for_backward(values, X)
        return layout.forward(X.contiguous(), values=values)

    @staticmethod
    def backward(ctx, dY):
        values, X = ctx.saved_tensors
        L = ctx.layout
        dY = dY.contiguous()
        dX = L.backward_input(dY, values=values) if ctx.needs_input_grad[1] else None
        dW = L.backward_weight(dY, X) if ctx.needs_input_grad[0] else None
        return dW, dX, None
