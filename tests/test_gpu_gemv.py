"""GPU parity of the decode-in-matvec kernel (tcq_gemv) against the fp64 oracle.

Tolerance: each product scale * c * x reaches y through at most
13 + ceil(cols / 256) fp32 roundings: at most 5 in the FMA chains of its quad or
8-weight item, at most 4 into a lane's per-fetch sum, one addition per fetch
(512 or 256 columns, depending on the kernel) into the lane's row sum, and a
5-level warp reduction.  The kernel for L = 16, k = 2, T = 256 and 4096-column
chunks (lanes on half blocks, two rows per item) has at most 23 + cols / 4096:
8 in a stream word's FMA chain, 8 into a block sum, 1 for the two block sums,
1 for the scale, one per 4096-column chunk and 5 in the warp reduction (the
rows it leaves for a last partial round are summed in the same order).  So
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


# 148 CTAs x 16 warps = 2368 warps; three rows per item from 3 x 2368 = 7104 rows
# on, one row per item below
@pytest.mark.parametrize("rows,nb,code", [
    (7204, 16, "f16"),    # three-row items: one whole round, then 100 rows, one per CTA
    (7204, 16, "mad"),
    (9473, 16, "mad"),    # three-row items: a whole round, a partial round of 789 groups, then 2 rows
    (14336, 16, "f16"),   # the MLP matrix's rows: two whole rounds, then 128 rows one per CTA
    (5000, 16, "f16"),    # one-row items: two whole rounds, a partial round of 264 rows
    (4737, 32, "f16"),    # two 4096-column chunks per row; two whole rounds, 1 row one per CTA
    (4801, 32, "mad"),    # two whole rounds, 65 rows one per CTA
    (37, 16, "f16"),      # fewer rows than CTAs: only the per-CTA rows
])
@pytest.mark.parametrize("scaled", [False, True])
def test_gemv_half_block_kernel(rows, nb, code, scaled, cuda_device):
    """L = 16, k = 2, T = 256 with cols a multiple of 4096: the kernel that takes
    half a coding block per lane and three rows per item, in both of its phases
    (every warp's share of row groups of three rows or one, with the last
    partial round either kept there or, when it is at most one row per CTA,
    spread one row per CTA)."""
    import torch
    from oracle import oracle_mad_codebook

    L, k, T = 16, 2, 256
    rng = np.random.default_rng(rows + nb + (1 if code == "mad" else 0) + (2 if scaled else 0))
    cols = nb * T
    bits, start = _rand_stream(rng, rows * nb, k, T)
    scale = rng.lognormal(0.0, 0.5, rows * nb).astype(np.float32) if scaled else None
    x = rng.standard_normal(cols).astype(np.float32)
    if code == "mad":
        dev = torch.device("cuda", 0)
        b = torch.from_numpy(np.ascontiguousarray(bits).view(np.int32)).to(dev)
        s = torch.from_numpy(np.ascontiguousarray(start).view(np.int32)).to(dev)
        sc = None if scale is None else torch.from_numpy(scale).to(dev)
        y = tcq.gemv(b, s, sc, tcq.MAD, L, k, T, rows, cols, torch.from_numpy(x).to(dev))
        torch.cuda.synchronize()
        y = y.cpu().numpy()
        cb = oracle_mad_codebook(L).astype(np.float16)
    else:
        cb = rng.standard_normal(1 << L).astype(np.float16)
        y = _gpu_gemv(bits, start, scale, cb, L, k, T, rows, cols, x)
    _check(bits, start, scale, cb, L, k, T, rows, cols, x, y)


def test_gemv_misaligned_bits_take_the_general_kernel(cuda_device):
    """Bits that are 4-byte but not 16-byte aligned are legal: the call takes a
    kernel without 16-byte loads and gives the same product within the bound."""
    import torch

    L, k, T, rows, nb = 16, 2, 256, 40, 16
    rng = np.random.default_rng(77)
    cols = nb * T
    bits, start = _rand_stream(rng, rows * nb, k, T)
    cb = rng.standard_normal(1 << L).astype(np.float16)
    x = rng.standard_normal(cols).astype(np.float32)
    dev = torch.device("cuda", 0)
    padded = torch.zeros(bits.size + 1, dtype=torch.int32, device=dev)
    padded[1:] = torch.from_numpy(np.ascontiguousarray(bits).view(np.int32).reshape(-1)).to(dev)
    b = padded[1:]
    assert b.data_ptr() % 16 == 4
    s = torch.from_numpy(np.ascontiguousarray(start).view(np.int32)).to(dev)
    y = tcq.gemv(b, s, None, torch.from_numpy(cb).to(dev), L, k, T, rows, cols,
                 torch.from_numpy(x).to(dev))
    torch.cuda.synchronize()
    _check(bits, start, None, cb, L, k, T, rows, cols, x, y.cpu().numpy())


@pytest.mark.parametrize("rows", [7104 + 37,   # three-row items: one whole round, then 37 rows one per CTA
                                  2368 + 37])  # one-row items: one whole round, then 37 rows one per CTA
def test_gemv_half_block_kernel_rows_bit_identical_across_phases(rows, cuda_device):
    """Rows with the same blocks give the same bits whether the row falls in the
    warps' row groups or among the rows spread one per CTA."""
    import torch

    L, k, T, nb = 16, 2, 256, 16
    rng = np.random.default_rng(404)
    bits1, start1 = _rand_stream(rng, nb, k, T)
    bits = np.tile(bits1, (rows, 1))
    start = np.tile(start1, rows)
    cb = rng.standard_normal(1 << L).astype(np.float16)
    x = rng.standard_normal(nb * T).astype(np.float32)
    for code in ("f16", "mad"):
        dev = torch.device("cuda", 0)
        b = torch.from_numpy(np.ascontiguousarray(bits).view(np.int32)).to(dev)
        s = torch.from_numpy(np.ascontiguousarray(start).view(np.int32)).to(dev)
        c = tcq.MAD if code == "mad" else torch.from_numpy(cb).to(dev)
        y = tcq.gemv(b, s, None, c, L, k, T, rows, nb * T, torch.from_numpy(x).to(dev))
        torch.cuda.synchronize()
        y = y.cpu().numpy()
        assert np.all(y == y[0]), code


def test_gemv_half_block_kernel_rows_per_item_give_the_same_bits(cuda_device):
    """The same row through three-row items (7141 rows) and one-row items (2405
    rows): the same bits, since a row's arithmetic does not depend on the rows
    an item holds."""
    import torch

    L, k, T, nb = 16, 2, 256, 16
    rng = np.random.default_rng(405)
    bits1, start1 = _rand_stream(rng, nb, k, T)
    cb = rng.standard_normal(1 << L).astype(np.float16)
    x = rng.standard_normal(nb * T).astype(np.float32)
    dev = torch.device("cuda", 0)
    for code in ("f16", "mad"):
        c = tcq.MAD if code == "mad" else torch.from_numpy(cb).to(dev)
        first = []
        for rows in (7104 + 37, 2368 + 37):
            b = torch.from_numpy(np.ascontiguousarray(np.tile(bits1, (rows, 1))).view(np.int32)).to(dev)
            s = torch.from_numpy(np.ascontiguousarray(np.tile(start1, rows)).view(np.int32)).to(dev)
            y = tcq.gemv(b, s, None, c, L, k, T, rows, nb * T, torch.from_numpy(x).to(dev))
            torch.cuda.synchronize()
            first.append(y[0].item())
        assert first[0] == first[1], code
