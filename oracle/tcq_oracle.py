"""ctypes wrapper of the plain C oracle (``tcq_oracle.c``).  Test infrastructure only.

Everything is converted to fp64 before the call: the codebook is the exact
widening of the caller's fp32 or fp16 entries, and x, d are the exact widening
of their fp32 values.  See ``tcq_oracle.c`` for the definition it computes and
the passages it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tcq_oracle.c")
_LIB = os.path.join(_HERE, "libtcq_oracle.so")
_lib = None


def build_oracle(force: bool = False) -> str:
    """Compile the oracle with plain gcc -O2 (IEEE arithmetic, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build_oracle())
        dp = ctypes.POINTER(ctypes.c_double)
        up = ctypes.POINTER(ctypes.c_uint32)
        i64 = ctypes.c_int64
        ci = ctypes.c_int
        lib.oracle_words_per_block.argtypes = [ci, ci]
        lib.oracle_words_per_block.restype = ci
        lib.oracle_encode.argtypes = [dp, dp, dp, ci, ci, ci, i64, i64, up, up, dp]
        lib.oracle_encode.restype = ci
        lib.oracle_decode.argtypes = [up, up, dp, ci, ci, ci, i64, dp]
        lib.oracle_decode.restype = ci
        lib.oracle_path_cost.argtypes = [dp, dp, dp, ci, i64, dp]
        lib.oracle_path_cost.restype = ci
        lib.oracle_greedy.argtypes = [dp, dp, dp, ci, ci, ci, i64, up, up, dp]
        lib.oracle_greedy.restype = ci
        lib.oracle_gemv.argtypes = [up, up, dp, dp, ci, ci, ci, i64, i64, dp, dp]
        lib.oracle_gemv.restype = ci
        lib.oracle_ldlq.argtypes = [dp, dp, dp, dp, ci, ci, ci, i64, i64, dp, dp, up, up, dp]
        lib.oracle_ldlq.restype = ci
        lib.oracle_feedback.argtypes = [dp, dp, dp, ci, i64, i64, i64, dp]
        lib.oracle_feedback.restype = ci
        lib.oracle_bcjr.argtypes = [dp, dp, dp, ci, ci, ci, i64, ctypes.c_double, dp, dp]
        lib.oracle_bcjr.restype = ci
        lib.oracle_mad_codebook.argtypes = [ci, dp]
        lib.oracle_mad_codebook.restype = ci
        lib.oracle_encode_vec.argtypes = [dp, dp, dp, ci, ci, ci, ci, i64, i64, up, up, dp]
        lib.oracle_encode_vec.restype = ci
        lib.oracle_decode_vec.argtypes = [up, up, dp, ci, ci, ci, ci, i64, dp]
        lib.oracle_decode_vec.restype = ci
        lib.oracle_ub8_encode.argtypes = [dp, dp, dp, ci, ci, ci, i64, i64, up, up, dp]
        lib.oracle_ub8_encode.restype = ci
        lib.oracle_ub8_decode.argtypes = [up, up, dp, ci, ci, ci, i64, dp]
        lib.oracle_ub8_decode.restype = ci
        _lib = lib
    return _lib


def _f64(a):
    return None if a is None else np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _u32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.uint32))


def _ptr(a, ctype):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def oracle_words_per_block(k: int, T: int) -> int:
    return int(_load().oracle_words_per_block(k, T))


def oracle_encode(x, d, codebook, L: int, k: int, fixed_start: int | None = None):
    """Viterbi-optimal TCQ of every row of ``x`` ([n_blocks, T]).

    Returns ``(start_state uint32[n], bits uint32[n, W], cost float64[n])``.
    ``d`` may be None (d_t = 1).  ``fixed_start`` None means a free start state.
    """
    x = _f64(x)
    if x.ndim == 1:
        x = x[None, :]
    n, T = x.shape
    d = _f64(d)
    if d is not None:
        d = np.ascontiguousarray(np.broadcast_to(d.reshape(-1, T) if d.ndim > 1 else d, (n, T)))
    cb = _f64(codebook).reshape(-1)
    if cb.size != (1 << L):
        raise ValueError(f"codebook must hold 2^L = {1 << L} entries, got {cb.size}")
    W = oracle_words_per_block(k, T)
    start = np.zeros(n, dtype=np.uint32)
    bits = np.zeros((n, W), dtype=np.uint32)
    cost = np.zeros(n, dtype=np.float64)
    rc = _load().oracle_encode(
        _ptr(x, ctypes.c_double), _ptr(d, ctypes.c_double), _ptr(cb, ctypes.c_double),
        L, k, T, n, -1 if fixed_start is None else int(fixed_start),
        _ptr(start, ctypes.c_uint32), _ptr(bits, ctypes.c_uint32), _ptr(cost, ctypes.c_double),
    )
    if rc != 0:
        raise ValueError(f"oracle_encode failed with code {rc}")
    return start, bits, cost


def oracle_decode(bits, start_state, codebook, L: int, k: int, T: int):
    """Decode ``bits`` ([n, W]) from ``start_state`` ([n]) to fp64 values [n, T]."""
    bits = _u32(bits)
    if bits.ndim == 1:
        bits = bits[None, :]
    start = _u32(start_state).reshape(-1)
    n = start.size
    cb = _f64(codebook).reshape(-1)
    y = np.zeros((n, T), dtype=np.float64)
    rc = _load().oracle_decode(
        _ptr(bits, ctypes.c_uint32), _ptr(start, ctypes.c_uint32), _ptr(cb, ctypes.c_double),
        L, k, T, n, _ptr(y, ctypes.c_double),
    )
    if rc != 0:
        raise ValueError(f"oracle_decode failed with code {rc}")
    return y


def oracle_path_cost(x, d, y):
    """sum_t d_t (x_t - y_t)^2 per row, in fp64."""
    x = _f64(x)
    if x.ndim == 1:
        x = x[None, :]
    n, T = x.shape
    y = _f64(y).reshape(n, T)
    d = _f64(d)
    if d is not None:
        d = np.ascontiguousarray(np.broadcast_to(d.reshape(-1, T) if d.ndim > 1 else d, (n, T)))
    cost = np.zeros(n, dtype=np.float64)
    rc = _load().oracle_path_cost(
        _ptr(x, ctypes.c_double), _ptr(d, ctypes.c_double), _ptr(y, ctypes.c_double),
        T, n, _ptr(cost, ctypes.c_double),
    )
    if rc != 0:
        raise ValueError(f"oracle_path_cost failed with code {rc}")
    return cost


def oracle_greedy(x, d, codebook, L: int, k: int, start_state):
    """Greedy trellis rounding from the given start states; returns (bits, cost)."""
    x = _f64(x)
    if x.ndim == 1:
        x = x[None, :]
    n, T = x.shape
    d = _f64(d)
    if d is not None:
        d = np.ascontiguousarray(np.broadcast_to(d.reshape(-1, T) if d.ndim > 1 else d, (n, T)))
    cb = _f64(codebook).reshape(-1)
    start = np.ascontiguousarray(np.broadcast_to(_u32(start_state).reshape(-1), (n,)))
    W = oracle_words_per_block(k, T)
    bits = np.zeros((n, W), dtype=np.uint32)
    cost = np.zeros(n, dtype=np.float64)
    rc = _load().oracle_greedy(
        _ptr(x, ctypes.c_double), _ptr(d, ctypes.c_double), _ptr(cb, ctypes.c_double),
        L, k, T, n, _ptr(start, ctypes.c_uint32), _ptr(bits, ctypes.c_uint32),
        _ptr(cost, ctypes.c_double),
    )
    if rc != 0:
        raise ValueError(f"oracle_greedy failed with code {rc}")
    return bits, cost


def oracle_gemv(bits, start_state, scale, codebook, L: int, k: int, T: int, rows: int, cols: int, x):
    """y = (decoded, block-scaled matrix) @ x in fp64; blocks row-major [rows, cols/T]."""
    bits = _u32(bits).reshape(-1)
    start = _u32(start_state).reshape(-1)
    sc = None if scale is None else _f64(scale).reshape(-1)
    cb = _f64(codebook).reshape(-1)
    xv = _f64(x).reshape(-1)
    y = np.zeros(rows, dtype=np.float64)
    rc = _load().oracle_gemv(
        _ptr(bits, ctypes.c_uint32), _ptr(start, ctypes.c_uint32), _ptr(sc, ctypes.c_double),
        _ptr(cb, ctypes.c_double), L, k, T, rows, cols, _ptr(xv, ctypes.c_double),
        _ptr(y, ctypes.c_double),
    )
    if rc != 0:
        raise ValueError(f"oracle_gemv failed with code {rc}")
    return y


def oracle_ldlq(w, u, d, codebook, L: int, k: int, T: int):
    """Error-feedback TCQ of the matrix ``w`` ([rows, cols]) by column blocks of T.

    ``u`` is the unit upper factor and ``d`` the diagonal of H = U diag(d) U^T.
    Returns (q [rows, cols], x targets [rows, cols], start [rows*nb],
    bits [rows*nb, W], cost [rows*nb]), blocks indexed r * (cols/T) + j.
    """
    w = _f64(w)
    rows, cols = w.shape
    u = _f64(u).reshape(cols, cols)
    d = _f64(d).reshape(cols)
    cb = _f64(codebook).reshape(-1)
    nb = cols // T
    W = oracle_words_per_block(k, T)
    q = np.zeros((rows, cols))
    xt = np.zeros((rows, cols))
    start = np.zeros(rows * nb, dtype=np.uint32)
    bits = np.zeros((rows * nb, W), dtype=np.uint32)
    cost = np.zeros(rows * nb)
    rc = _load().oracle_ldlq(
        _ptr(w, ctypes.c_double), _ptr(u, ctypes.c_double), _ptr(d, ctypes.c_double),
        _ptr(cb, ctypes.c_double), L, k, T, rows, cols, _ptr(q, ctypes.c_double),
        _ptr(xt, ctypes.c_double), _ptr(start, ctypes.c_uint32), _ptr(bits, ctypes.c_uint32),
        _ptr(cost, ctypes.c_double),
    )
    if rc != 0:
        raise ValueError(f"oracle_ldlq failed with code {rc}")
    return q, xt, start, bits, cost


def oracle_feedback_targets(w, u, q, T: int):
    """Targets of every column block given the reconstruction ``q`` ([rows, cols]):
    block j's targets use only q's columns before jT."""
    w = _f64(w)
    q = _f64(q)
    rows, cols = w.shape
    u = _f64(u).reshape(cols, cols)
    xt = np.zeros((rows, cols))
    lib = _load()
    for j in range(cols // T):
        rc = lib.oracle_feedback(_ptr(w, ctypes.c_double), _ptr(u, ctypes.c_double),
                                 _ptr(q, ctypes.c_double), T, rows, cols, j,
                                 _ptr(xt, ctypes.c_double))
        if rc != 0:
            raise ValueError(f"oracle_feedback failed with code {rc}")
    return xt


def oracle_bcjr(x, d, codebook, L: int, k: int, tau: float):
    """Soft codewords y [n, T] (expectation of c[s_t] under exp(-J/tau)/Z over
    trellis paths) and free energies F = -tau log Z [n] for the blocks of ``x``."""
    x = _f64(x)
    if x.ndim == 1:
        x = x[None, :]
    n, T = x.shape
    dd = None if d is None else _f64(d).reshape(n, T)
    cb = _f64(codebook).reshape(-1)
    y = np.zeros((n, T))
    F = np.zeros(n)
    rc = _load().oracle_bcjr(
        _ptr(x, ctypes.c_double), None if dd is None else _ptr(dd, ctypes.c_double),
        _ptr(cb, ctypes.c_double), L, k, T, n, float(tau), _ptr(y, ctypes.c_double),
        _ptr(F, ctypes.c_double),
    )
    if rc != 0:
        raise ValueError(f"oracle_bcjr failed with code {rc}")
    return y, F


def oracle_mad_codebook(L: int):
    """The 2^L codewords of the computed multiply-add code (fp64)."""
    cb = np.zeros(1 << L)
    rc = _load().oracle_mad_codebook(L, _ptr(cb, ctypes.c_double))
    if rc != 0:
        raise ValueError(f"oracle_mad_codebook failed with code {rc}")
    return cb


def oracle_encode_vec(x, d, codebook, L: int, k: int, V: int, fixed_start: int | None = None):
    """Viterbi TCQ over the vector trellis (V weights per step, kV bits shifted in,
    codebook [2^L, V]).  Returns (start, bits, cost) like oracle_encode."""
    x = _f64(x)
    if x.ndim == 1:
        x = x[None, :]
    n, T = x.shape
    dd = None if d is None else _f64(d).reshape(n, T)
    cb = _f64(codebook).reshape(-1)
    W = oracle_words_per_block(k, T)
    start = np.zeros(n, dtype=np.uint32)
    bits = np.zeros((n, W), dtype=np.uint32)
    cost = np.zeros(n)
    rc = _load().oracle_encode_vec(
        _ptr(x, ctypes.c_double), None if dd is None else _ptr(dd, ctypes.c_double),
        _ptr(cb, ctypes.c_double), L, k, V, T, n, -1 if fixed_start is None else int(fixed_start),
        _ptr(start, ctypes.c_uint32), _ptr(bits, ctypes.c_uint32), _ptr(cost, ctypes.c_double))
    if rc != 0:
        raise ValueError(f"oracle_encode_vec failed with code {rc}")
    return start, bits, cost


def oracle_decode_vec(bits, start_state, codebook, L: int, k: int, V: int, T: int):
    """Values [n, T] of the vector trellis from packed bits and start states."""
    bits = np.ascontiguousarray(bits, dtype=np.uint32)
    start = np.ascontiguousarray(start_state, dtype=np.uint32).reshape(-1)
    n = start.shape[0]
    cb = _f64(codebook).reshape(-1)
    y = np.zeros((n, T))
    rc = _load().oracle_decode_vec(_ptr(bits, ctypes.c_uint32), _ptr(start, ctypes.c_uint32),
                                   _ptr(cb, ctypes.c_double), L, k, V, T, n,
                                   _ptr(y, ctypes.c_double))
    if rc != 0:
        raise ValueError(f"oracle_decode_vec failed with code {rc}")
    return y


def oracle_ub8_encode(x, d, codebook, V: int, m: int, fixed_start: int | None = None):
    """TCQ over Ungerboeck's 8-state set-partitioned trellis (see tcq_oracle.c).

    ``x`` is [n_blocks, T] with V | T (steps of V weights); ``codebook`` holds
    4 * 2^m rows of V values, row r in subset r mod 4.  Returns
    ``(start_state uint32[n] in [0, 8), bits uint32[n, W], cost float64[n])``
    with W = ceil((T / V) (1 + m) / 32).
    """
    x = _f64(x)
    if x.ndim == 1:
        x = x[None, :]
    n, T = x.shape
    if T % V:
        raise ValueError("V must divide T")
    d = _f64(d)
    if d is not None:
        d = np.ascontiguousarray(np.broadcast_to(d.reshape(-1, T) if d.ndim > 1 else d, (n, T)))
    cb = _f64(codebook).reshape(-1)
    if cb.size != 4 * (1 << m) * V:
        raise ValueError(f"codebook must hold 4 * 2^m rows of V values, got {cb.size}")
    W = oracle_words_per_block(1 + m, T // V)
    start = np.zeros(n, dtype=np.uint32)
    bits = np.zeros((n, W), dtype=np.uint32)
    cost = np.zeros(n, dtype=np.float64)
    rc = _load().oracle_ub8_encode(
        _ptr(x, ctypes.c_double), _ptr(d, ctypes.c_double), _ptr(cb, ctypes.c_double),
        V, m, T, n, -1 if fixed_start is None else int(fixed_start),
        _ptr(start, ctypes.c_uint32), _ptr(bits, ctypes.c_uint32), _ptr(cost, ctypes.c_double),
    )
    if rc != 0:
        raise ValueError(f"oracle_ub8_encode failed with code {rc}")
    return start, bits, cost


def oracle_ub8_decode(bits, start_state, codebook, V: int, m: int, T: int):
    """Decode 8-state set-partitioned trellis streams ([n, W]) to fp64 values [n, T]."""
    bits = _u32(bits)
    if bits.ndim == 1:
        bits = bits[None, :]
    n = bits.shape[0]
    start = _u32(start_state).reshape(n)
    cb = _f64(codebook).reshape(-1)
    if cb.size != 4 * (1 << m) * V:
        raise ValueError("codebook must hold 4 * 2^m rows of V values")
    if bits.shape[1] != oracle_words_per_block(1 + m, T // V):
        raise ValueError("bits has the wrong number of words per block")
    y = np.zeros((n, T), dtype=np.float64)
    rc = _load().oracle_ub8_decode(_ptr(bits, ctypes.c_uint32), _ptr(start, ctypes.c_uint32),
                                   _ptr(cb, ctypes.c_double), V, m, T, n, _ptr(y, ctypes.c_double))
    if rc != 0:
        raise ValueError(f"oracle_ub8_decode failed with code {rc}")
    return y
