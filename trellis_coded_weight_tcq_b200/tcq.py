"""Python binding of the C ABI in ``include/tcq.h`` (argument marshalling only).

The functions named like the C entry points (``tcq_encode`` ...) take raw device
pointers and sizes exactly as the C ABI does.  ``encode``/``decode`` accept
torch CUDA tensors, allocate outputs and workspace with torch, and launch on the
current torch stream; ``encode_host`` additionally stages host arrays through
pinned memory (the end-to-end path).  Every step of the search and the decode
runs in the CUDA library: when it is missing this module raises instead of
computing anything itself.
"""
from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass

_PKG = os.path.dirname(os.path.abspath(__file__))
# TCQ_LIBRARY=debug selects the bounds-checked build (libtcq_debug.so, see
# build.py); load only one of the two builds in a process.
LIB_PATH = os.path.join(_PKG, "libtcq_debug.so" if os.environ.get("TCQ_LIBRARY") == "debug"
                        else "libtcq.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "tcq.h")

TCQ_OK = 0
TCQ_ERR_INVALID_ARG = 1
TCQ_ERR_UNSUPPORTED = 2
TCQ_ERR_WORKSPACE = 3
TCQ_ERR_CUDA = 4
TCQ_ERR_INTERNAL = 5
TCQ_F32 = 0
TCQ_F16 = 1
TCQ_MAD = 2


class _ComputedCode:
    """Stands for the computed (lookup-free) code wherever a codebook tensor goes."""

    def __repr__(self):
        return "MAD"


MAD = _ComputedCode()  # pass as ``codebook`` to select TCQ_MAD
TCQ_MAX_L = 16
TCQ_MAX_K = 4
TCQ_MAX_T = 1 << 20

_lib = None


class TCQError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {tcq_status_string(status)}")


def load_library() -> ctypes.CDLL:
    """Load ``libtcq.so``; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m trellis_coded_weight_tcq_b200.build` "
            "(there is no CPU fallback)"
        )
    lib = ctypes.CDLL(LIB_PATH)
    vp, sz, i64, ci = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int64, ctypes.c_int
    lib.tcq_words_per_block.argtypes = [ci, ci]
    lib.tcq_words_per_block.restype = ci
    lib.tcq_encode_workspace_bytes.argtypes = [ci, ci, ci, i64, ci]
    lib.tcq_encode_workspace_bytes.restype = sz
    lib.tcq_encode.argtypes = [vp, vp, vp, ci, ci, ci, ci, i64, vp, vp, vp, vp, sz, vp]
    lib.tcq_encode.restype = ci
    lib.tcq_encode_fixed_start.argtypes = [vp, vp, vp, ci, ci, ci, ci, i64, vp, vp, vp, vp, vp,
                                           sz, vp]
    lib.tcq_encode_fixed_start.restype = ci
    lib.tcq_encode_vec_workspace_bytes.argtypes = [ci, ci, ci, ci, i64, ci]
    lib.tcq_encode_vec_workspace_bytes.restype = sz
    lib.tcq_encode_vec.argtypes = [vp, vp, vp, ci, ci, ci, ci, ci, i64, vp, vp, vp, vp, sz, vp]
    lib.tcq_encode_vec.restype = ci
    lib.tcq_decode_vec.argtypes = [vp, vp, vp, ci, ci, ci, ci, ci, i64, vp, vp]
    lib.tcq_decode_vec.restype = ci
    lib.tcq_decode.argtypes = [vp, vp, vp, ci, ci, ci, ci, i64, vp, vp]
    lib.tcq_decode.restype = ci
    lib.tcq_status_string.argtypes = [ci]
    lib.tcq_status_string.restype = ctypes.c_char_p
    lib.tcq_encode_path.argtypes = [ci, ci, ci]
    lib.tcq_encode_path.restype = ctypes.c_char_p
    lib.tcq_gemv.argtypes = [vp, vp, vp, vp, ci, ci, ci, ci, i64, i64, vp, vp, vp]
    lib.tcq_gemv.restype = ci
    lib.tcq_gemv_vec.argtypes = [vp, vp, vp, vp, ci, ci, ci, ci, ci, i64, i64, vp, vp, vp]
    lib.tcq_gemv_vec.restype = ci
    lib.tcq_ldlq_workspace_bytes.argtypes = [ci, ci, ci, i64, i64, ci]
    lib.tcq_ldlq_workspace_bytes.restype = sz
    lib.tcq_ldlq.argtypes = [vp, vp, vp, vp, ci, ci, ci, ci, i64, i64, vp, vp, vp, vp, vp, vp,
                             sz, vp]
    lib.tcq_ldlq.restype = ci
    lib.tcq_bcjr_workspace_bytes.argtypes = [ci, ci, ci, i64, ci]
    lib.tcq_bcjr_workspace_bytes.restype = sz
    lib.tcq_bcjr.argtypes = [vp, vp, vp, ci, ci, ci, ci, i64, ctypes.c_float, vp, vp, vp, sz, vp]
    lib.tcq_bcjr.restype = ci
    lib.tcq_ub8_words_per_block.argtypes = [ci, ci, ci]
    lib.tcq_ub8_words_per_block.restype = ci
    lib.tcq_ub8_encode.argtypes = [vp, vp, vp, ci, ci, ci, ci, i64, vp, vp, vp, vp, vp]
    lib.tcq_ub8_encode.restype = ci
    lib.tcq_ub8_decode.argtypes = [vp, vp, vp, ci, ci, ci, ci, i64, vp, vp]
    lib.tcq_ub8_decode.restype = ci
    lib.tcq_device_errors.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
    lib.tcq_device_errors.restype = ci
    _lib = lib
    return lib


def header_functions() -> list[str]:
    """Names of the functions ``include/tcq.h`` declares."""
    with open(HEADER_PATH) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    return sorted(set(re.findall(r"\b(tcq_[a-z0-9_]+)\s*\(", text)))


# ---------------------------------------------------------------------------
# the C entry points, one to one
# ---------------------------------------------------------------------------
def tcq_words_per_block(k: int, T: int) -> int:
    return int(load_library().tcq_words_per_block(k, T))


def tcq_encode_workspace_bytes(L: int, k: int, T: int, n_blocks: int, cb_dtype: int) -> int:
    return int(load_library().tcq_encode_workspace_bytes(L, k, T, n_blocks, cb_dtype))


def tcq_encode(x, d, codebook, cb_dtype, L, k, T, n_blocks, start_state, bits, path_cost,
               workspace, workspace_bytes, stream) -> int:
    return int(load_library().tcq_encode(x, d, codebook, cb_dtype, L, k, T, n_blocks, start_state,
                                          bits, path_cost, workspace, workspace_bytes, stream))


def tcq_encode_fixed_start(x, d, codebook, cb_dtype, L, k, T, n_blocks, fixed_start, start_state,
                           bits, path_cost, workspace, workspace_bytes, stream) -> int:
    return int(load_library().tcq_encode_fixed_start(x, d, codebook, cb_dtype, L, k, T, n_blocks,
                                                     fixed_start, start_state, bits, path_cost,
                                                     workspace, workspace_bytes, stream))


def tcq_encode_vec_workspace_bytes(L, k, V, T, n_blocks, cb_dtype) -> int:
    return int(load_library().tcq_encode_vec_workspace_bytes(L, k, V, T, n_blocks, cb_dtype))


def tcq_encode_vec(x, d, codebook, cb_dtype, L, k, V, T, n_blocks, start_state, bits, path_cost,
                   workspace, workspace_bytes, stream) -> int:
    return int(load_library().tcq_encode_vec(x, d, codebook, cb_dtype, L, k, V, T, n_blocks,
                                             start_state, bits, path_cost, workspace,
                                             workspace_bytes, stream))


def tcq_decode_vec(bits, start_state, codebook, cb_dtype, L, k, V, T, n_blocks, y, stream) -> int:
    return int(load_library().tcq_decode_vec(bits, start_state, codebook, cb_dtype, L, k, V, T,
                                             n_blocks, y, stream))


def tcq_decode(bits, start_state, codebook, cb_dtype, L, k, T, n_blocks, y, stream) -> int:
    return int(load_library().tcq_decode(bits, start_state, codebook, cb_dtype, L, k, T, n_blocks,
                                          y, stream))


def tcq_gemv(bits, start_state, scale, codebook, cb_dtype, L, k, T, rows, cols, x, y, stream) -> int:
    return int(load_library().tcq_gemv(bits, start_state, scale, codebook, cb_dtype, L, k, T, rows,
                                        cols, x, y, stream))


def tcq_gemv_vec(bits, start_state, scale, codebook, cb_dtype, L, k, V, T, rows, cols, x, y,
                 stream) -> int:
    return int(load_library().tcq_gemv_vec(bits, start_state, scale, codebook, cb_dtype, L, k, V, T,
                                            rows, cols, x, y, stream))


def tcq_ldlq_workspace_bytes(L: int, k: int, T: int, rows: int, cols: int, cb_dtype: int) -> int:
    return int(load_library().tcq_ldlq_workspace_bytes(L, k, T, rows, cols, cb_dtype))


def tcq_ldlq(w, u, d, codebook, cb_dtype, L, k, T, rows, cols, q, x, start_state, bits, path_cost,
             workspace, workspace_bytes, stream) -> int:
    return int(load_library().tcq_ldlq(w, u, d, codebook, cb_dtype, L, k, T, rows, cols, q, x,
                                       start_state, bits, path_cost, workspace, workspace_bytes,
                                       stream))


def tcq_bcjr_workspace_bytes(L: int, k: int, T: int, n_blocks: int, cb_dtype: int) -> int:
    return int(load_library().tcq_bcjr_workspace_bytes(L, k, T, n_blocks, cb_dtype))


def tcq_bcjr(x, d, codebook, cb_dtype, L, k, T, n_blocks, tau, y_soft, free_energy, workspace,
             workspace_bytes, stream) -> int:
    return int(load_library().tcq_bcjr(x, d, codebook, cb_dtype, L, k, T, n_blocks, tau, y_soft,
                                       free_energy, workspace, workspace_bytes, stream))


def tcq_ub8_words_per_block(V: int, m: int, T: int) -> int:
    return int(load_library().tcq_ub8_words_per_block(V, m, T))


def tcq_ub8_encode(x, d, codebook, cb_dtype, V, m, T, n_blocks, fixed_start, start_state, bits,
                   path_cost, stream) -> int:
    return int(load_library().tcq_ub8_encode(x, d, codebook, cb_dtype, V, m, T, n_blocks,
                                             fixed_start, start_state, bits, path_cost, stream))


def tcq_ub8_decode(bits, start_state, codebook, cb_dtype, V, m, T, n_blocks, y, stream) -> int:
    return int(load_library().tcq_ub8_decode(bits, start_state, codebook, cb_dtype, V, m, T,
                                             n_blocks, y, stream))


TCQ_DEVERR_WAIT_TIMEOUT = 0x1
TCQ_DEVERR_BOUNDS = 0x2


def tcq_device_errors(stream, flags) -> int:
    return int(load_library().tcq_device_errors(stream, flags))


def device_errors(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error flags."""
    flags = ctypes.c_uint32(0)
    st = tcq_device_errors(_stream_handle(stream), ctypes.byref(flags))
    if st not in (TCQ_OK, TCQ_ERR_INTERNAL):
        raise TCQError(st, "tcq_device_errors")
    return int(flags.value)


def tcq_status_string(status: int) -> str:
    return load_library().tcq_status_string(status).decode()


def tcq_encode_path(L: int, k: int, cb_dtype: int) -> str:
    return load_library().tcq_encode_path(L, k, cb_dtype).decode()


# ---------------------------------------------------------------------------
# torch conveniences (device memory and streams only)
# ---------------------------------------------------------------------------
def _torch():
    import torch

    return torch


def cb_dtype_of(codebook) -> int:
    if codebook is MAD:
        return TCQ_MAD
    torch = _torch()
    if codebook.dtype == torch.float16:
        return TCQ_F16
    if codebook.dtype == torch.float32:
        return TCQ_F32
    raise TypeError(f"codebook must be float16 or float32, got {codebook.dtype}")


def _ptr(t):
    return None if t is None or t is MAD else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream=None):
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, what: str) -> None:
    if status != TCQ_OK:
        raise TCQError(status, what)


@dataclass
class Encoded:
    start_state: "object"  # uint32 [n] as torch.int32 storage
    bits: "object"         # uint32 [n, W] as torch.int32 storage
    path_cost: "object"    # float32 [n]


class Workspace:
    """A reusable device workspace for ``encode`` (torch-allocated)."""

    def __init__(self, L: int, k: int, T: int, n_blocks: int, cb_dtype: int, device=None):
        torch = _torch()
        self.nbytes = max(tcq_encode_workspace_bytes(L, k, T, n_blocks, cb_dtype), 256)
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device or "cuda")


def encode(x, d, codebook, L: int, k: int, workspace: Workspace | None = None, out=None,
           stream=None, fixed_start=None) -> Encoded:
    """Viterbi TCQ of every row of ``x`` (fp32 CUDA tensor [n_blocks, T]); a free
    start state per block, or the int32 tensor ``fixed_start`` of start states."""
    torch = _torch()
    if x.dim() != 2 or x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous float32 CUDA tensor [n_blocks, T]")
    n, T = x.shape
    if d is not None and (d.shape != x.shape or d.dtype != torch.float32 or not d.is_contiguous()):
        raise ValueError("d must be None or a contiguous float32 tensor shaped like x")
    W = tcq_words_per_block(k, T)
    if W < 0:
        raise TCQError(TCQ_ERR_UNSUPPORTED, "tcq_words_per_block")
    if out is None:
        out = Encoded(
            torch.empty(n, dtype=torch.int32, device=x.device),
            torch.empty((n, W), dtype=torch.int32, device=x.device),
            torch.empty(n, dtype=torch.float32, device=x.device),
        )
    ws = workspace or Workspace(L, k, T, n, cb_dtype_of(codebook), x.device)
    if fixed_start is None:
        _check(tcq_encode(_ptr(x), _ptr(d), _ptr(codebook), cb_dtype_of(codebook), L, k, T, n,
                          _ptr(out.start_state), _ptr(out.bits), _ptr(out.path_cost),
                          ctypes.c_void_p(ws.buf.data_ptr()), ws.nbytes, _stream_handle(stream)),
               "tcq_encode")
    else:
        if fixed_start.numel() < n or fixed_start.dtype != torch.int32 or not fixed_start.is_cuda:
            raise ValueError("fixed_start must be an int32 CUDA tensor of n_blocks start states")
        _check(tcq_encode_fixed_start(_ptr(x), _ptr(d), _ptr(codebook), cb_dtype_of(codebook), L,
                                      k, T, n, _ptr(fixed_start), _ptr(out.start_state),
                                      _ptr(out.bits), _ptr(out.path_cost),
                                      ctypes.c_void_p(ws.buf.data_ptr()), ws.nbytes,
                                      _stream_handle(stream)), "tcq_encode_fixed_start")
    return out


def decode(bits, start_state, codebook, L: int, k: int, T: int, out=None, stream=None):
    """Values [n_blocks, T] (fp32) of packed ``bits`` from ``start_state``."""
    torch = _torch()
    n = start_state.shape[0]
    W = tcq_words_per_block(k, T)
    if bits.numel() < n * max(W, 0):
        raise ValueError("decode: bits holds fewer than n_blocks * W words")
    if out is None:
        out = torch.empty((n, T), dtype=torch.float32, device=bits.device)
    if out.numel() < n * T:
        raise ValueError("decode: out holds fewer than n_blocks * T values")
    _check(tcq_decode(_ptr(bits), _ptr(start_state), _ptr(codebook), cb_dtype_of(codebook), L, k,
                      T, n, _ptr(out), _stream_handle(stream)), "tcq_decode")
    return out


def gemv(bits, start_state, scale, codebook, L: int, k: int, T: int, rows: int, cols: int, x,
         out=None, stream=None):
    """y = (trellis-coded matrix) @ x, decoding on the fly; blocks row-major [rows, cols/T]."""
    torch = _torch()
    nb = rows * (cols // T) if T > 0 else 0
    W = tcq_words_per_block(k, T)
    if bits.numel() < nb * max(W, 0) or start_state.numel() < nb or x.numel() < cols or (
            scale is not None and scale.numel() < nb):
        raise ValueError(f"gemv: tensors too small for a {rows} x {cols} matrix of T={T} blocks")
    if out is None:
        out = torch.empty(rows, dtype=torch.float32, device=x.device)
    if out.numel() < rows:
        raise ValueError("gemv: out holds fewer than rows values")
    _check(tcq_gemv(_ptr(bits), _ptr(start_state), _ptr(scale), _ptr(codebook),
                    cb_dtype_of(codebook), L, k, T, rows, cols, _ptr(x), _ptr(out),
                    _stream_handle(stream)), "tcq_gemv")
    return out


def gemv_vec(bits, start_state, scale, codebook, L: int, k: int, V: int, T: int, rows: int,
             cols: int, x, out=None, stream=None):
    """gemv for the vector trellis (V weights per step, codebook [2^L, V])."""
    torch = _torch()
    nb = rows * (cols // T) if T > 0 else 0
    W = tcq_words_per_block(k, T)
    if bits.numel() < nb * max(W, 0) or start_state.numel() < nb or x.numel() < cols or (
            scale is not None and scale.numel() < nb):
        raise ValueError(f"gemv_vec: tensors too small for a {rows} x {cols} matrix of T={T} blocks")
    if out is None:
        out = torch.empty(rows, dtype=torch.float32, device=x.device)
    if out.numel() < rows:
        raise ValueError("gemv_vec: out holds fewer than rows values")
    _check(tcq_gemv_vec(_ptr(bits), _ptr(start_state), _ptr(scale), _ptr(codebook),
                        cb_dtype_of(codebook), L, k, V, T, rows, cols, _ptr(x), _ptr(out),
                        _stream_handle(stream)), "tcq_gemv_vec")
    return out


@dataclass
class LdlqResult:
    q: "object"            # float32 [rows, cols], the reconstruction
    x: "object"            # float32 [rows, cols], the targets, or None
    coded: Encoded         # blocks (r, j) at r * (cols / T) + j


def ldlq(w, u, d, codebook, L: int, k: int, T: int, keep_targets: bool = True, workspace=None,
         stream=None) -> LdlqResult:
    """Error-feedback TCQ of the matrix ``w`` (fp32 CUDA [rows, cols]) by column
    blocks of T, with H = U diag(d) U^T (``u`` fp32 [cols, cols], ``d`` fp32 [cols]
    or None)."""
    torch = _torch()
    if w.dim() != 2 or w.dtype != torch.float32 or not w.is_cuda or not w.is_contiguous():
        raise ValueError("w must be a contiguous float32 CUDA tensor [rows, cols]")
    rows, cols = w.shape
    if u.shape != (cols, cols) or u.dtype != torch.float32 or not u.is_contiguous():
        raise ValueError("u must be a contiguous float32 tensor [cols, cols]")
    if d is not None and (d.shape != (cols,) or d.dtype != torch.float32 or not d.is_contiguous()):
        raise ValueError("d must be None or a contiguous float32 tensor [cols]")
    W = tcq_words_per_block(k, T)
    if W < 0:
        raise TCQError(TCQ_ERR_UNSUPPORTED, "tcq_words_per_block")
    nb = cols // T if T > 0 else 0
    dev = w.device
    q = torch.empty((rows, cols), dtype=torch.float32, device=dev)
    x = torch.empty((rows, cols), dtype=torch.float32, device=dev) if keep_targets else None
    coded = Encoded(
        torch.empty(rows * nb, dtype=torch.int32, device=dev),
        torch.empty((rows * nb, W), dtype=torch.int32, device=dev),
        torch.empty(rows * nb, dtype=torch.float32, device=dev),
    )
    if workspace is None:
        nbytes = max(tcq_ldlq_workspace_bytes(L, k, T, rows, cols, cb_dtype_of(codebook)), 256)
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    _check(tcq_ldlq(_ptr(w), _ptr(u), _ptr(d), _ptr(codebook), cb_dtype_of(codebook), L, k, T,
                    rows, cols, _ptr(q), _ptr(x), _ptr(coded.start_state), _ptr(coded.bits),
                    _ptr(coded.path_cost), ctypes.c_void_p(workspace.data_ptr()),
                    workspace.numel(), _stream_handle(stream)), "tcq_ldlq")
    return LdlqResult(q, x, coded)


def bcjr(x, d, codebook, L: int, k: int, tau: float, workspace=None, out=None, stream=None):
    """Soft codewords [n_blocks, T] and free energies -tau ln Z [n_blocks] of the
    rows of ``x`` (fp32 CUDA [n_blocks, T]) at temperature ``tau``."""
    torch = _torch()
    if x.dim() != 2 or x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous float32 CUDA tensor [n_blocks, T]")
    n, T = x.shape
    if d is not None and (d.shape != x.shape or d.dtype != torch.float32 or not d.is_contiguous()):
        raise ValueError("d must be None or a contiguous float32 tensor shaped like x")
    if out is None:
        out = (torch.empty((n, T), dtype=torch.float32, device=x.device),
               torch.empty(n, dtype=torch.float32, device=x.device))
    y, F = out
    if y.numel() < n * T or (F is not None and F.numel() < n):
        raise ValueError("bcjr: output tensors too small")
    if workspace is None:
        nbytes = max(tcq_bcjr_workspace_bytes(L, k, T, n, cb_dtype_of(codebook)), 256)
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=x.device)
    _check(tcq_bcjr(_ptr(x), _ptr(d), _ptr(codebook), cb_dtype_of(codebook), L, k, T, n,
                    float(tau), _ptr(y), _ptr(F), ctypes.c_void_p(workspace.data_ptr()),
                    workspace.numel(), _stream_handle(stream)), "tcq_bcjr")
    return y, F


def encode_vec(x, d, codebook, L: int, k: int, V: int, workspace=None, out=None,
               stream=None) -> Encoded:
    """Viterbi TCQ over the vector trellis: V weights per step, codebook [2^L, V].

    ``workspace`` (a uint8 CUDA tensor of at least tcq_encode_vec_workspace_bytes
    for one block; more lets more blocks run at once) and ``out`` (an Encoded of
    int32 start [n], int32 bits [n, W] and float32 cost [n]) are allocated when
    not given."""
    torch = _torch()
    if x.dim() != 2 or x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous float32 CUDA tensor [n_blocks, T]")
    n, T = x.shape
    if d is not None and (d.shape != x.shape or d.dtype != torch.float32 or not d.is_contiguous()):
        raise ValueError("d must be None or a contiguous float32 tensor shaped like x")
    if codebook is not MAD and codebook.numel() != (1 << L) * V:
        raise ValueError("codebook must hold 2^L rows of V entries")
    W = max(tcq_words_per_block(k, T), 1)
    if out is None:
        out = Encoded(torch.empty(n, dtype=torch.int32, device=x.device),
                      torch.empty((n, W), dtype=torch.int32, device=x.device),
                      torch.empty(n, dtype=torch.float32, device=x.device))
    elif (out.start_state.numel() < n or out.bits.numel() < n * W or out.path_cost.numel() < n):
        raise ValueError("encode_vec: out is smaller than the blocks need")
    if workspace is None:
        nbytes = max(tcq_encode_vec_workspace_bytes(L, k, V, T, n, cb_dtype_of(codebook)), 256)
        ws = torch.empty(nbytes, dtype=torch.uint8, device=x.device)
    else:
        ws = workspace
    _check(tcq_encode_vec(_ptr(x), _ptr(d), _ptr(codebook), cb_dtype_of(codebook), L, k, V, T, n,
                          _ptr(out.start_state), _ptr(out.bits), _ptr(out.path_cost),
                          ctypes.c_void_p(ws.data_ptr()), ws.numel(), _stream_handle(stream)),
           "tcq_encode_vec")
    return out


def decode_vec(bits, start_state, codebook, L: int, k: int, V: int, T: int, out=None, stream=None):
    """Values [n_blocks, T] of the vector trellis (into ``out`` when given)."""
    torch = _torch()
    n = start_state.shape[0]
    W = tcq_words_per_block(k, T)
    if bits.numel() < n * max(W, 0):
        raise ValueError("decode_vec: bits holds fewer than n_blocks * W words")
    if out is None:
        out = torch.empty((n, T), dtype=torch.float32, device=bits.device)
    elif out.numel() < n * T or out.dtype != torch.float32 or not out.is_contiguous():
        raise ValueError("decode_vec: out must be a contiguous float32 tensor of n_blocks * T")
    _check(tcq_decode_vec(_ptr(bits), _ptr(start_state), _ptr(codebook), cb_dtype_of(codebook), L,
                          k, V, T, n, _ptr(out), _stream_handle(stream)), "tcq_decode_vec")
    return out


def ub8_encode(x, d, codebook, V: int, m: int, fixed_start=None, out=None,
               stream=None) -> Encoded:
    """TCQ over the 8-state set-partitioned trellis of every row of ``x`` (fp32
    CUDA [n_blocks, T], T / V steps of V weights); ``codebook`` holds 4 * 2^m rows
    of V values (row r in subset r mod 4).  A free start state per block, or the
    int32 tensor ``fixed_start``."""
    torch = _torch()
    if x.dim() != 2 or x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous float32 CUDA tensor [n_blocks, T]")
    n, T = x.shape
    if d is not None and (d.shape != x.shape or d.dtype != torch.float32 or not d.is_contiguous()):
        raise ValueError("d must be None or a contiguous float32 tensor shaped like x")
    if codebook is MAD or codebook.numel() != (4 << m) * V:
        raise ValueError("codebook must be a table of 4 * 2^m rows of V entries")
    W = tcq_ub8_words_per_block(V, m, T)
    if W < 0:
        raise TCQError(TCQ_ERR_UNSUPPORTED, "tcq_ub8_words_per_block")
    if out is None:
        out = Encoded(torch.empty(n, dtype=torch.int32, device=x.device),
                      torch.empty((n, W), dtype=torch.int32, device=x.device),
                      torch.empty(n, dtype=torch.float32, device=x.device))
    elif out.start_state.numel() < n or out.bits.numel() < n * W or out.path_cost.numel() < n:
        raise ValueError("ub8_encode: out is smaller than the blocks need")
    if fixed_start is not None and (fixed_start.numel() < n or fixed_start.dtype != torch.int32
                                    or not fixed_start.is_cuda):
        raise ValueError("fixed_start must be an int32 CUDA tensor of n_blocks start states")
    _check(tcq_ub8_encode(_ptr(x), _ptr(d), _ptr(codebook), cb_dtype_of(codebook), V, m, T, n,
                          _ptr(fixed_start), _ptr(out.start_state), _ptr(out.bits),
                          _ptr(out.path_cost), _stream_handle(stream)), "tcq_ub8_encode")
    return out


def ub8_decode(bits, start_state, codebook, V: int, m: int, T: int, out=None, stream=None):
    """Values [n_blocks, T] of 8-state set-partitioned trellis streams."""
    torch = _torch()
    n = start_state.shape[0]
    W = tcq_ub8_words_per_block(V, m, T)
    if W < 0:
        raise TCQError(TCQ_ERR_UNSUPPORTED, "tcq_ub8_words_per_block")
    if bits.numel() < n * W:
        raise ValueError("ub8_decode: bits holds fewer than n_blocks * W words")
    if codebook is MAD or codebook.numel() != (4 << m) * V:
        raise ValueError("codebook must be a table of 4 * 2^m rows of V entries")
    if out is None:
        out = torch.empty((n, T), dtype=torch.float32, device=bits.device)
    elif out.numel() < n * T or out.dtype != torch.float32 or not out.is_contiguous():
        raise ValueError("ub8_decode: out must be a contiguous float32 tensor of n_blocks * T")
    _check(tcq_ub8_decode(_ptr(bits), _ptr(start_state), _ptr(codebook), cb_dtype_of(codebook), V,
                          m, T, n, _ptr(out), _stream_handle(stream)), "tcq_ub8_decode")
    return out


def host_pipeline_parts(n_blocks: int, chunks: int, sm_count: int):
    """Block ranges [lo, hi) of HostPipeline: a short lead part (1 / (8 chunks)
    of the blocks) and ``chunks`` equal parts, one part when ``chunks`` is 1.
    For large inputs the sizes are whole waves of the encoder (8 blocks per SM:
    every grouped configuration runs 1, 2, 4 or 8 blocks per SM at a time), so
    that only the last part ends on a partly filled round."""
    chunks = max(1, chunks)
    wave = 8 * max(1, sm_count)
    lead = min(n_blocks, -(-n_blocks // (8 * chunks))) if chunks > 1 else 0
    per = max(1, -(-(n_blocks - lead) // chunks))
    if n_blocks >= 8 * chunks * wave:
        lead = -(-lead // wave) * wave
        per = -(-per // wave) * wave
    return ([(0, lead)] if lead else []) + [(lo, min(n_blocks, lo + per)) for lo in range(lead, n_blocks, per)]


class HostPipeline:
    """End-to-end encode of host arrays: pinned host -> device -> encode -> host.

    Buffers are allocated once.  ``run`` splits the blocks into a short lead
    part (1 / (8 chunks) of them) and ``chunks`` equal parts (one part when
    ``chunks`` is 1): a copy stream
    brings part i + 1's inputs in while the compute stream encodes and decodes
    part i, and takes part i's start states, bits and costs back while part i + 1
    is encoded, so only the lead part's input copy (short, so that the encoder
    starts early; the next part's copy hides behind its encode) and the last
    part's output copy are not hidden behind the encoder.
    """

    def __init__(self, n_blocks: int, T: int, L: int, k: int, weighted: bool, codebook_host,
                 device=None, with_decode: bool = True, chunks: int = 8):
        torch = _torch()
        dev = torch.device(device or "cuda")
        self.L, self.k, self.T, self.n = L, k, T, n_blocks
        W = tcq_words_per_block(k, T)
        self.x_dev = torch.empty((n_blocks, T), dtype=torch.float32, device=dev)
        self.d_dev = torch.empty((n_blocks, T), dtype=torch.float32, device=dev) if weighted else None
        self.cb_dev = codebook_host.to(dev)
        self.parts = host_pipeline_parts(n_blocks, chunks,
                                         torch.cuda.get_device_properties(dev).multi_processor_count)
        self.ws = Workspace(L, k, T, max(hi - lo for lo, hi in self.parts), cb_dtype_of(self.cb_dev), dev)
        self.enc = Encoded(torch.empty(n_blocks, dtype=torch.int32, device=dev),
                           torch.empty((n_blocks, W), dtype=torch.int32, device=dev),
                           torch.empty(n_blocks, dtype=torch.float32, device=dev))
        self.y_dev = torch.empty((n_blocks, T), dtype=torch.float32, device=dev) if with_decode else None
        self.start_h = torch.empty(n_blocks, dtype=torch.int32, pin_memory=True)
        self.bits_h = torch.empty((n_blocks, W), dtype=torch.int32, pin_memory=True)
        self.cost_h = torch.empty(n_blocks, dtype=torch.float32, pin_memory=True)
        self.copy_stream = torch.cuda.Stream(device=dev)
        self.ev_in = [torch.cuda.Event() for _ in self.parts]
        self.ev_done = [torch.cuda.Event() for _ in self.parts]

    def h2d_bytes(self) -> int:
        return self.x_dev.numel() * 4 + (self.d_dev.numel() * 4 if self.d_dev is not None else 0)

    def d2h_bytes(self) -> int:
        return (self.start_h.numel() + self.bits_h.numel() + self.cost_h.numel()) * 4

    def run(self, x_pinned, d_pinned=None, stream=None):
        torch = _torch()
        cs = self.copy_stream
        ms = stream or torch.cuda.current_stream()
        cs.wait_stream(ms)  # the previous run's readers of these buffers are done

        def copy_in(i):
            lo, hi = self.parts[i]
            with torch.cuda.stream(cs):
                self.x_dev[lo:hi].copy_(x_pinned[lo:hi], non_blocking=True)
                if self.d_dev is not None:
                    self.d_dev[lo:hi].copy_(d_pinned[lo:hi], non_blocking=True)
                self.ev_in[i].record(cs)

        copy_in(0)
        for i, (lo, hi) in enumerate(self.parts):
            if i + 1 < len(self.parts):
                copy_in(i + 1)
            ms.wait_event(self.ev_in[i])
            part = Encoded(self.enc.start_state[lo:hi], self.enc.bits[lo:hi], self.enc.path_cost[lo:hi])
            encode(self.x_dev[lo:hi], None if self.d_dev is None else self.d_dev[lo:hi], self.cb_dev,
                   self.L, self.k, self.ws, part, ms)
            if self.y_dev is not None:
                decode(part.bits, part.start_state, self.cb_dev, self.L, self.k, self.T,
                       self.y_dev[lo:hi], ms)
            self.ev_done[i].record(ms)
            with torch.cuda.stream(cs):
                cs.wait_event(self.ev_done[i])
                self.start_h[lo:hi].copy_(part.start_state, non_blocking=True)
                self.bits_h[lo:hi].copy_(part.bits, non_blocking=True)
                self.cost_h[lo:hi].copy_(part.path_cost, non_blocking=True)
        ms.wait_stream(cs)
        return self.start_h, self.bits_h, self.cost_h


def tcq_encode_static_scratch(x, d, codebook, cb_dtype, L, k, T, n_blocks, start_state, bits,
                              path_cost, stream) -> int:
    """The allocation-free encoder (scratch in a static device array of the library)."""
    fn = _static_scratch_fn()
    return int(fn(x, d, codebook, cb_dtype, L, k, T, n_blocks, start_state, bits, path_cost,
                  stream))


def _static_scratch_fn():
    lib = load_library()
    fn = lib.tcq_encode_static_scratch
    if fn.argtypes is None:
        vp, i64, ci = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        fn.argtypes = [vp, vp, vp, ci, ci, ci, ci, i64, vp, vp, vp, vp]
        fn.restype = ci
    return fn
