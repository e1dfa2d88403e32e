"""GPU parity: the CUDA encoder and decoder, called through the C ABI, against
the fp64 CPU oracle on the same seeded inputs.

Encode parity is on cost (ties and fp32 rounding may pick a different but
equally good path); decode parity is bit-exact; on inputs whose fp32 search
is exact (dyadic grids) the encoder must match the oracle bit for bit.
"""
import ctypes

import numpy as np
import pytest

from tests.parity import check_encode, gpu_decode, gpu_encode, oracle_encode_parallel
from trellis_coded_weight_tcq_b200 import tcq, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device(cuda_device):
    tcq.load_library()
    return cuda_device


# --------------------------------------------------------------------------
# the named workloads
# --------------------------------------------------------------------------
@pytest.mark.parametrize("name", ["tiny", "l12"])
def test_named_workload_full(name):
    wl = workloads.NAMED[name]()
    start, bits, cost = gpu_encode(wl)
    check_encode(wl, start, bits, cost, pure=True)
    # decode of the GPU's own bits: bit-exact against the oracle's decode
    from oracle import oracle_decode

    y = gpu_decode(bits, start, wl.codebook, wl.L, wl.k, wl.T)
    y_o = oracle_decode(bits, start, wl.codebook, wl.L, wl.k, wl.T).astype(np.float32)
    np.testing.assert_array_equal(y, y_o)


def _sample_rows(n, count, seed):
    rng = np.random.default_rng(seed)
    rows = {0, n - 1} | set(rng.choice(n, size=min(n, count) - 2, replace=False).tolist())
    return np.array(sorted(rows))


@pytest.mark.parametrize("name", ["qtip", "heavy", "mlp"])
def test_named_workload_full_size_sampled(name):
    """Full-size encode in the bench's launch configuration; oracle on sampled
    blocks; the decode round trip checked on every block."""
    from oracle import oracle_decode

    wl = workloads.NAMED[name]()
    dt = tcq.TCQ_F16 if wl.codebook.dtype == np.float16 else tcq.TCQ_F32
    assert tcq.tcq_encode_path(wl.L, wl.k, dt).startswith("grouped")
    start, bits, cost = gpu_encode(wl)
    rows = _sample_rows(wl.n_blocks, 256, 7)  # first, last and 254 seeded
    check_encode(wl, start, bits, cost, rows=rows, pure=True)
    y = gpu_decode(bits, start, wl.codebook, wl.L, wl.k, wl.T)
    y_o = oracle_decode(bits[rows], start[rows], wl.codebook, wl.L, wl.k, wl.T).astype(np.float32)
    np.testing.assert_array_equal(y[rows], y_o)
    # every block: the decoded values reproduce the reported cost
    d = np.ones_like(wl.x) if wl.d is None else wl.d
    J = np.sum(d.astype(np.float64) * (wl.x.astype(np.float64) - y.astype(np.float64)) ** 2, axis=1)
    tol = 1e-5 * J + 1e-7 * d.astype(np.float64).sum(axis=1)
    assert np.all(np.abs(cost.astype(np.float64) - J) <= tol)
    assert np.all(start < (1 << (wl.L - wl.k)))


# --------------------------------------------------------------------------
# many shapes, both kernels, both codebook dtypes, ragged sizes
# --------------------------------------------------------------------------
SHAPES = [
    # (L, k, T, n_blocks, weighted, cb_dtype)
    (8, 2, 64, 300, False, "f32"),     # one warp per block, ragged last CTA
    (8, 2, 1, 33, True, "f32"),
    (8, 2, 257, 17, True, "f16"),
    (8, 2, 1024, 9, True, "f32"),      # the longest block the warp kernel holds
    (8, 2, 1025, 9, True, "f32"),      # one step more: the grouped kernel, sub-warp teams
    (12, 2, 256, 700, True, "f32"),    # grouped, several rounds per CTA
    (12, 2, 5, 9, False, "f16"),
    (16, 2, 256, 150, True, "f16"),    # grouped fp16-pair kernel
    (16, 2, 37, 40, False, "f16"),
    (16, 2, 600, 3, True, "f16"),      # T > staging chunk, odd
    (16, 3, 256, 150, True, "f16"),
    (16, 3, 11, 20, False, "f16"),
    (16, 2, 40, 6, True, "f32"),       # fp32 at L=16: generic kernel
    (1, 1, 50, 7, True, "f32"),        # generic from here on
    (2, 1, 3, 4, False, "f32"),
    (3, 2, 9, 11, True, "f16"),        # L < 2k
    (4, 4, 13, 5, True, "f32"),        # L = k: no memory
    (5, 3, 17, 8, False, "f32"),
    (6, 1, 64, 12, True, "f32"),
    (7, 4, 31, 6, True, "f16"),
    (10, 2, 129, 40, True, "f32"),
    (11, 3, 70, 12, True, "f16"),
    (13, 1, 20, 4, True, "f32"),
    (14, 2, 33, 5, False, "f16"),
    (15, 1, 9, 2, True, "f32"),        # metrics in global memory
    (16, 1, 7, 2, True, "f16"),
    (16, 4, 12, 3, True, "f16"),
]


@pytest.mark.parametrize("L,k,T,n,weighted,cb", SHAPES)
def test_random_shapes(L, k, T, n, weighted, cb):
    wl = workloads.small_random(L, k, T, n, weighted, cb, seed=L * 1000 + k * 100 + T + n)
    start, bits, cost = gpu_encode(wl)
    check_encode(wl, start, bits, cost)


@pytest.mark.parametrize("L,k,cb", [(16, 2, "f16"), (16, 3, "f16"), (12, 2, "f32"), (8, 2, "f32"),
                                    (10, 2, "f16"), (16, 2, "f32")])
@pytest.mark.parametrize("pattern", ["some_zero", "all_zero", "subnormal", "wide_range"])
def test_weight_edge_cases(L, k, cb, pattern):
    """d with zeros, all zero, subnormal entries, or spread over 32 decades:
    the weighted search still returns an optimal path (the fp16 kernels carry
    metrics divided by d and floor d relative to the block's largest weight)."""
    wl = workloads.small_random(L, k, 48, 12, True, cb, seed=["some_zero", "all_zero", "subnormal", "wide_range"].index(pattern) * 100 + L + k)
    rng = np.random.default_rng(L * 10 + k)
    d = wl.d.astype(np.float64)
    if pattern == "some_zero":
        d[:, ::3] = 0.0
    elif pattern == "all_zero":
        d[:] = 0.0
    elif pattern == "subnormal":
        d[:, ::2] = 1e-41
    else:
        d = 10.0 ** rng.uniform(-20, 12, d.shape)
    wl.d = d.astype(np.float32)
    start, bits, cost = gpu_encode(wl)
    check_encode(wl, start, bits, cost)


@pytest.mark.parametrize("L,k,cb", [(8, 2, "f32"), (12, 2, "f32"), (16, 2, "f16"), (16, 3, "f16"),
                                    (10, 2, "f32"), (6, 3, "f16"), (16, 2, "f32")])
@pytest.mark.parametrize("weighted", [False, True])
def test_exact_arithmetic_is_bit_exact(L, k, cb, weighted):
    """On dyadic inputs every fp32 operation of the search is exact, so the GPU
    takes the oracle's decisions, tie rules included: identical bits."""
    wl = workloads.dyadic_exact(L, k, 96 if L < 16 else 40, 24, weighted, cb, seed=L + 10 * k)
    start, bits, cost = gpu_encode(wl)
    s_o, b_o, c_o = oracle_encode_parallel(wl.x, wl.d, wl.codebook, L, k)
    np.testing.assert_array_equal(start, s_o)
    np.testing.assert_array_equal(bits, b_o)
    np.testing.assert_array_equal(cost.astype(np.float64), c_o)


# --------------------------------------------------------------------------
# decode
# --------------------------------------------------------------------------
@pytest.mark.parametrize("L,k,T,cb", [(16, 2, 256, "f16"), (16, 3, 256, "f16"), (12, 2, 256, "f32"),
                                      (8, 2, 64, "f32"), (16, 1, 7, "f16"), (16, 4, 255, "f32"),
                                      (5, 3, 10, "f16"), (3, 3, 1, "f32"), (15, 2, 130, "f32"),
                                      (14, 3, 3, "f16")])
def test_decode_random_bitstreams(L, k, T, cb):
    from oracle import oracle_decode

    rng = np.random.default_rng(L * 77 + k * 7 + T)
    n = 97
    W = tcq.tcq_words_per_block(k, T)
    bits = rng.integers(0, 2**32, size=(n, W), dtype=np.uint64).astype(np.uint32)
    used = T * k - 32 * (W - 1)
    if used < 32:
        bits[:, -1] &= np.uint32(((1 << used) - 1) << (32 - used))
    start = rng.integers(0, 2**32, size=n, dtype=np.uint64).astype(np.uint32)  # non-canonical
    codebook = rng.standard_normal(1 << L).astype(np.float16 if cb == "f16" else np.float32)
    y = gpu_decode(bits, start, codebook, L, k, T)
    y_o = oracle_decode(bits, start, codebook, L, k, T).astype(np.float32)
    np.testing.assert_array_equal(y, y_o)


def test_decode_unaligned_output():
    """An output pointer off 16-byte alignment takes the scalar-store path."""
    import torch

    from oracle import oracle_decode

    L, k, T, n = 12, 2, 64, 40
    rng = np.random.default_rng(3)
    W = tcq.tcq_words_per_block(k, T)
    bits = rng.integers(0, 2**32, size=(n, W), dtype=np.uint64).astype(np.uint32)
    start = rng.integers(0, 1 << (L - k), size=n).astype(np.uint32)
    codebook = rng.standard_normal(1 << L).astype(np.float32)
    buf = torch.zeros(n * T + 1, dtype=torch.float32, device="cuda")
    y = buf[1:].view(n, T)
    b = torch.from_numpy(bits.view(np.int32)).cuda()
    s = torch.from_numpy(start.view(np.int32)).cuda()
    tcq.decode(b, s, torch.from_numpy(codebook).cuda(), L, k, T, out=y)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(y.cpu().numpy(),
                                  oracle_decode(bits, start, codebook, L, k, T).astype(np.float32))
    assert buf[0].item() == 0.0


# --------------------------------------------------------------------------
# edge cases and the ABI's error behaviour
# --------------------------------------------------------------------------
def test_reduced_workspace_runs_one_cta():
    """The smallest workspace the encoder accepts runs one CTA: every block goes
    through it in turn, so each round's traceback overlaps the next round's
    forward pass and the last one runs after the loop."""
    for (L, k, cb) in [(16, 2, "f16"), (12, 2, "f32"), (8, 2, "f32"), (10, 2, "f32"), (16, 3, "f16")]:
        wl = workloads.small_random(L, k, 64, 23, True, cb, seed=5 + L)
        one = _min_workspace(L, k, 64, wl.codebook.dtype)
        start, bits, cost = gpu_encode(wl, workspace_bytes=one)
        check_encode(wl, start, bits, cost)


def _min_workspace(L, k, T, np_dtype):
    """Smallest workspace tcq_encode accepts for this shape (by bisection)."""
    import torch

    tdt = torch.float16 if np_dtype == np.float16 else torch.float32
    full = tcq.tcq_encode_workspace_bytes(L, k, T, 1, tcq.TCQ_F16 if tdt == torch.float16 else tcq.TCQ_F32)
    x = torch.zeros((1, T), device="cuda")
    cb = torch.zeros(1 << L, dtype=tdt, device="cuda")
    out = [torch.zeros(1, dtype=torch.int32, device="cuda"),
           torch.zeros((1, tcq.tcq_words_per_block(k, T)), dtype=torch.int32, device="cuda"),
           torch.zeros(1, device="cuda")]
    ws = torch.empty(full, dtype=torch.uint8, device="cuda")
    dt = tcq.TCQ_F16 if np_dtype == np.float16 else tcq.TCQ_F32
    lo, hi = 1, full
    while lo < hi:
        mid = (lo + hi) // 2
        st = tcq.tcq_encode(ctypes.c_void_p(x.data_ptr()), None, ctypes.c_void_p(cb.data_ptr()),
                            dt, L, k, T, 1, ctypes.c_void_p(out[0].data_ptr()),
                            ctypes.c_void_p(out[1].data_ptr()), ctypes.c_void_p(out[2].data_ptr()),
                            ctypes.c_void_p(ws.data_ptr()), mid, None)
        if st == tcq.TCQ_OK:
            hi = mid
        else:
            assert st == tcq.TCQ_ERR_WORKSPACE
            lo = mid + 1
    torch.cuda.synchronize()
    return lo


def test_empty_and_invalid_calls():
    import torch

    vp = ctypes.c_void_p
    x = torch.zeros((4, 8), device="cuda")
    cb = torch.zeros(256, device="cuda")
    st = torch.zeros(4, dtype=torch.int32, device="cuda")
    bits = torch.zeros((4, 1), dtype=torch.int32, device="cuda")
    cost = torch.zeros(4, device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    P = lambda t: vp(t.data_ptr())  # noqa: E731
    assert tcq.tcq_encode(None, None, None, 0, 8, 2, 8, 0, None, None, None, None, 0, None) == tcq.TCQ_OK
    assert tcq.tcq_decode(None, None, None, 0, 8, 2, 8, 0, None, None) == tcq.TCQ_OK
    args = (P(x), None, P(cb), tcq.TCQ_F32, 8, 2, 8, 4, P(st), P(bits), P(cost), P(ws), ws.numel(), None)
    assert tcq.tcq_encode(*args) == tcq.TCQ_OK
    bad = list(args); bad[0] = None
    assert tcq.tcq_encode(*bad) == tcq.TCQ_ERR_INVALID_ARG
    bad = list(args); bad[4] = 17
    assert tcq.tcq_encode(*bad) == tcq.TCQ_ERR_UNSUPPORTED
    bad = list(args); bad[5] = 9
    assert tcq.tcq_encode(*bad) == tcq.TCQ_ERR_UNSUPPORTED
    bad = list(args); bad[6] = 0
    assert tcq.tcq_encode(*bad) == tcq.TCQ_ERR_UNSUPPORTED
    bad = list(args); bad[3] = 7
    assert tcq.tcq_encode(*bad) == tcq.TCQ_ERR_INVALID_ARG
    bad = list(args); bad[12] = 16
    assert tcq.tcq_encode(*bad) == tcq.TCQ_ERR_WORKSPACE
    bad = list(args); bad[11] = vp(ws.data_ptr() + 4)
    assert tcq.tcq_encode(*bad) == tcq.TCQ_ERR_INVALID_ARG
    bad = list(args); bad[0] = vp(x.data_ptr() + 2)
    assert tcq.tcq_encode(*bad) == tcq.TCQ_ERR_INVALID_ARG
    torch.cuda.synchronize()
    # nothing launched by a rejected call, the stream is healthy
    assert torch.cuda.current_stream().query() in (True, False)


def test_maximum_block_length():
    """T = TCQ_MAX_T (2^20 weights in one block): staging chunks, backpointer
    records and the traceback over a million steps, with path metrics that
    would reach about 1e5 unless the kernel shifted them back towards 0."""
    wl = workloads.small_random(8, 2, tcq.TCQ_MAX_T, 2, True, "f32", seed=4242)
    start, bits, cost = gpu_encode(wl)
    check_encode(wl, start, bits, cost)


@pytest.mark.parametrize("L,k,T,cb", [
    (16, 2, 4096, "f16"),   # register-resident encoder, its long-block instantiation
    (16, 3, 2048, "f16"),
    (12, 2, 8192, "f32"),
    (16, 2, 1500, "f32"),   # runtime-(L,k) encoder
    (16, 2, 1025, "f16"),   # one step past the threshold
])
def test_long_blocks(L, k, T, cb):
    """Blocks longer than the renormalisation threshold (1024 steps) take the
    renormalising code; the cost stays within the short blocks' tolerance."""
    wl = workloads.small_random(L, k, T, 3, True, cb, seed=4300 + L + T)
    start, bits, cost = gpu_encode(wl)
    check_encode(wl, start, bits, cost)
