"""GPU parity of the decode-in-matvec kernel (tcq_gemv) against the fp64 oracle.

Tolerance: each product scale * c * x reaches y through at most
13 + ceil(cols / 256) fp32 roundings: at most 5 in the FMA chains of its quad or
8-weight item, at most 4 into a lane's per-fetch sum, one addition per fetch
(512 or 256 columns, depending on the kernel) into the lane's row sum, and a
5-level warp reduction.  So
|y_gpu - y_exact| <= (13 + ceil(cols / 256)) * 2^-24 * sum |scale * c * x|.
"""
import ctypes

import numpy as np
import pytest

from trellis_coded_weight_tcq_b200 import tcq, workloads

pytestmark = pytest.mark.gpu


def _rand_stream(rng, n, k, T):
    W = tcq.tcq_words_per_block(k, T)
    bits = rng.integers(0, 2**32, size=(n, W), dtype=np.uint64).astype(np.uint32)
    used = T * k - 32 * (W - 1)
    if used < 32:
        bits[:, -1] &= np.uint32(((1 << used) - 1) << (32 - used))
    start = rng.integers(0, 2**32, size=n, dtype=np.uint64).astype(np.uint32)
    return bits, start


def _gpu_gemv(bits, start, scale, cb, L, k, T, rows, cols, x):
    import torch

    dev = torch.device("cuda", 0)
    b = torch.from_numpy(np.ascontiguousarray(bits).view(np.int32)).to(dev)
    s = torch.from_numpy(np.ascontiguousarray(start).view(np.int32)).to(dev)
    sc = None if scale is None else torch.from_numpy(scale.astype(np.float32)).to(dev)
    c = torch.from_numpy(cb).to(dev)
    xv = torch.from_numpy(x.astype(np.float32)).to(dev)
    y = tcq.gemv(b, s, sc, c, L, k, T, rows, cols, xv)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def _check(bits, start, scale, cb, L, k, T, rows, cols, x, y):
    from oracle import oracle_decode, oracle_gemv

    y_o = oracle_gemv(bits, start, scale, cb, L, k, T, rows, cols, x.astype(np.float32))
    vals = oracle_decode(bits, start, cb, L, k, T).reshape(rows, cols)
    sc = np.ones(rows * (cols // T)) if scale is None else scale.astype(np.float32).astype(np.float64)
    terms = np.abs(vals * np.repeat(sc.reshape(rows, -1), T, axis=1) * x.astype(np.float32))
    bound = (13 + -(-cols // 256)) * 2.0**-24 * terms.sum(axis=1)
    assert np.all(np.abs(y.astype(np.float64) - y_o) <= bound + 1e-30), float(
        np.max(np.abs(y - y_o) / np.maximum(bound, 1e-30)))


@pytest.mark.parametrize("L,k,T,rows,nb,cb", [
    (16, 2, 256, 300, 16, "f16"),   # the MLP shape's blocks, fp16 table
    (16, 3, 256, 100, 16, "f16"),
    (12, 2, 256, 257, 8, "f32"),    # ragged row count
    (8, 2, 64, 33, 5, "f32"),
    (14, 4, 12, 40, 7, "f16"),      # fp16 input held as fp32, k=4
    (5, 3, 4, 9, 3, "f32"),         # tiny blocks: every quad reads the start state
    (16, 1, 512, 20, 40, "f16"),    # cols 20480: x from L1 instead of shared memory
    (16, 2, 256, 20, 80, "f16"),    # specialised kernel with x from L1
    (16, 2, 24, 33, 5, "f16"),      # specialised kernel, blocks of 3 items (not a power of 2)
    (8, 2, 64, 70, 3, "f16"),       # specialised fp32-table kernel from a binary16 input
])
@pytest.mark.parametrize("scaled", [False, True])
def test_gemv_random_bitstreams(L, k, T, rows, nb, cb, scaled, cuda_device):
    rng = np.random.default_rng(L * 101 + k * 7 + T + rows)
    cols = nb * T
    bits, start = _rand_stream(rng, rows * nb, k, T)
    codebook = rng.standard_normal(1 << L).astype(np.float16 if cb == "f16" else np.float32)
    scale = rng.lognormal(0.0, 0.5, rows * nb).astype(np.float32) if scaled else None
    x = rng.standard_normal(cols).astype(np.float32)
    y = _gpu_gemv(bits, start, scale, codebook, L, k, T, rows, cols, x)
    _check(bits, start, scale, codebook, L, k, T, rows, cols, x, y)


def test_gemv_of_encoded_matrix(cuda_device):
    """Encode the first 512 rows of the MLP-shape matrix, then multiply: the
    result matches the oracle's decode-then-product of the same bits."""
    from tests.parity import gpu_encode

    wl = workloads.mlp(0)
    rows, cols, T = 512, 4096, 256
    nb = cols // T
    wl.x = np.ascontiguousarray(wl.x[: rows * nb])
    wl.d = np.ascontiguousarray(wl.d[: rows * nb])
    start, bits, _ = gpu_encode(wl)
    x = np.random.default_rng(5).standard_normal(cols).astype(np.float32)
    scale = np.random.default_rng(6).lognormal(-4.0, 0.1, rows * nb).astype(np.float32)
    y = _gpu_gemv(bits, start, scale, wl.codebook, 16, 2, T, rows, cols, x)
    _check(bits, start, scale, wl.codebook, 16, 2, T, rows, cols, x, y)


def test_gemv_rejections(cuda_device):
    fake = ctypes.c_void_p(0x10000)
    args = dict(bits=fake, st=fake, sc=None, cb=fake, dt=tcq.TCQ_F16, L=16, k=2, T=256, rows=4,
                cols=512, x=fake, y=fake)

    def call(**o):
        v = dict(args, **o)
        return tcq.tcq_gemv(v["bits"], v["st"], v["sc"], v["cb"], v["dt"], v["L"], v["k"], v["T"],
                            v["rows"], v["cols"], v["x"], v["y"], None)

    assert call(rows=0) == tcq.TCQ_OK
    assert call(T=6, cols=12) == tcq.TCQ_ERR_UNSUPPORTED
    assert call(dt=tcq.TCQ_F32) == tcq.TCQ_ERR_UNSUPPORTED
    assert call(cols=500) == tcq.TCQ_ERR_INVALID_ARG
    assert call(x=ctypes.c_void_p(0x10004)) == tcq.TCQ_ERR_INVALID_ARG
    assert call(y=None) == tcq.TCQ_ERR_INVALID_ARG
    assert call(L=17) == tcq.TCQ_ERR_UNSUPPORTED
