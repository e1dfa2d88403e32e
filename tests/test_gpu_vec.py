"""GPU parity of the vector trellis (tcq_encode_vec / tcq_decode_vec: V weights
per step, kV bits shifted in, V-dimensional codewords) against the oracle."""
import ctypes

import numpy as np
import pytest

from tests.parity import ABS_TOL_PER_D, REL_TOL
from trellis_coded_weight_tcq_b200 import tcq

pytestmark = pytest.mark.gpu

# L, k, V, T, blocks, codebook dtype, weighted
CASES = [
    (8, 1, 2, 32, 40, "f32", True),
    (8, 2, 2, 64, 30, "f32", False),
    (12, 2, 2, 128, 8, "f32", True),
    (6, 1, 4, 24, 50, "f16", True),
    (10, 2, 3, 48, 12, "f32", True),
    (16, 1, 2, 64, 3, "f16", True),    # metrics in the workspace
    (8, 4, 2, 16, 10, "f32", True),    # kV = L: no trellis memory
    (5, 1, 5, 35, 20, "f32", False),
    # the compile-time kernel (L=16, k=2, V=2, binary16 pairs)
    (16, 2, 2, 256, 3, "f16", True),
    (16, 2, 2, 2, 5, "f16", True),      # one step
    (16, 2, 2, 30, 4, "f16", False),    # 15 steps: a partial last word
    (16, 2, 2, 514, 2, "f16", True),    # 257 steps: three staging chunks
    (16, 2, 2, 2200, 1, "f16", True),   # 1100 steps: the renormalising instantiation
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "L{}k{}V{}T{}_B{}_{}{}".format(*c[:6], "_w" if c[6] else ""))
def test_encode_vec_parity(case, cuda_device):
    import torch
    from oracle import oracle_decode_vec, oracle_encode_vec

    L, k, V, T, n, cbt, weighted = case
    rng = np.random.default_rng(8000 + 31 * L + 7 * k + V + T)
    x = rng.standard_normal((n, T)).astype(np.float32)
    d = rng.lognormal(0.0, 1.0, (n, T)).astype(np.float32) if weighted else None
    cb = rng.standard_normal((1 << L, V))
    cb = cb.astype(np.float16) if cbt == "f16" else cb.astype(np.float32)
    out = tcq.encode_vec(torch.from_numpy(x).to(cuda_device),
                         None if d is None else torch.from_numpy(d).to(cuda_device),
                         torch.from_numpy(cb).to(cuda_device), L, k, V)
    torch.cuda.synchronize()
    start = out.start_state.cpu().numpy().view(np.uint32)
    bits = out.bits.cpu().numpy().view(np.uint32)
    cost = out.path_cost.cpu().numpy().astype(np.float64)
    assert np.all(start < (1 << (L - k * V)))
    _, _, J_o = oracle_encode_vec(x, d, cb, L, k, V)
    y = oracle_decode_vec(bits, start, cb, L, k, V, T)
    dd = np.ones((n, T)) if d is None else d.astype(np.float64)
    J_g = (dd * (x.astype(np.float64) - y) ** 2).sum(axis=1)
    tol = REL_TOL * J_o + ABS_TOL_PER_D * dd.sum(axis=1)
    assert np.all(np.abs(J_g - J_o) <= tol), float(np.max(np.abs(J_g - J_o) / J_o))
    assert np.all(np.abs(cost - J_g) <= tol)
    # the GPU's own decode of its bits
    yg = tcq.decode_vec(out.bits, out.start_state, torch.from_numpy(cb).to(cuda_device), L, k, V, T)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(yg.cpu().numpy(), y.astype(np.float32))


@pytest.mark.parametrize("L,k,V,T,cbt", [
    (8, 1, 2, 32, "f32"), (12, 2, 2, 256, "f32"), (16, 1, 4, 64, "f32"), (9, 3, 2, 30, "f32"),
    # the compile-time decoder (L=16, four bits per step, binary16 pairs, T % 8 == 0)
    (16, 2, 2, 256, "f16"), (16, 2, 2, 8, "f16"), (16, 2, 2, 264, "f16"), (16, 2, 2, 1024, "f16"),
    (16, 2, 2, 30, "f16"),    # T % 8 != 0: the runtime decoder
])
def test_decode_vec_bit_exact(L, k, V, T, cbt, cuda_device):
    import torch
    from oracle import oracle_decode_vec

    rng = np.random.default_rng(8100 + L + V + T)
    n = 33
    W = tcq.tcq_words_per_block(k, T)
    bits = rng.integers(0, 2**32, size=(n, W), dtype=np.uint64).astype(np.uint32)
    start = rng.integers(0, 2**32, size=n, dtype=np.uint64).astype(np.uint32)
    cb = rng.standard_normal((1 << L, V)).astype(np.float16 if cbt == "f16" else np.float32)
    y = tcq.decode_vec(torch.from_numpy(bits.view(np.int32)).to(cuda_device),
                       torch.from_numpy(start.view(np.int32)).to(cuda_device),
                       torch.from_numpy(cb).to(cuda_device), L, k, V, T)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(y.cpu().numpy(), oracle_decode_vec(bits, start, cb, L, k, V, T).astype(np.float32))


def test_v1_is_tcq_encode(cuda_device):
    import torch

    rng = np.random.default_rng(8200)
    x = torch.from_numpy(rng.standard_normal((20, 256)).astype(np.float32)).to(cuda_device)
    cb = torch.from_numpy(rng.standard_normal(1 << 12).astype(np.float32)).to(cuda_device)
    a = tcq.encode(x, None, cb, 12, 2)
    b = tcq.encode_vec(x, None, cb, 12, 2, 1)
    torch.cuda.synchronize()
    assert torch.equal(a.bits, b.bits) and torch.equal(a.start_state, b.start_state)
    assert torch.equal(a.path_cost, b.path_cost)


def test_vec_rejections(cuda_device):
    fake = ctypes.c_void_p(0x10000)
    enc = lambda **o: tcq.tcq_encode_vec(fake, None, o.get("cb", fake), o.get("dt", tcq.TCQ_F32),  # noqa: E731
                                         o.get("L", 8), o.get("k", 2), o.get("V", 2), o.get("T", 32),
                                         4, fake, fake, fake, fake, 1 << 30, None)
    assert enc(T=33) == tcq.TCQ_ERR_UNSUPPORTED            # V does not divide T
    assert enc(k=3, V=3, L=12) == tcq.TCQ_ERR_UNSUPPORTED  # kV = 9 > 8
    assert enc(k=2, V=3, L=5) == tcq.TCQ_ERR_UNSUPPORTED   # kV > L
    assert enc(V=9) == tcq.TCQ_ERR_UNSUPPORTED
    assert enc(dt=tcq.TCQ_MAD, cb=None) == tcq.TCQ_ERR_UNSUPPORTED
    assert enc(cb=None) == tcq.TCQ_ERR_INVALID_ARG


def _vec_case(L, k, V, T, n, seed, device, cb_offset=0):
    import torch

    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, T)).astype(np.float32)
    d = rng.lognormal(0.0, 1.0, (n, T)).astype(np.float32)
    cb = rng.standard_normal((1 << L, V)).astype(np.float16)
    cbt = torch.empty(cb.size + cb_offset, dtype=torch.float16, device=device)[cb_offset:]
    cbt.copy_(torch.from_numpy(cb.reshape(-1)))
    out = tcq.encode_vec(torch.from_numpy(x).to(device), torch.from_numpy(d).to(device), cbt, L, k, V)
    torch.cuda.synchronize()
    return x, d, cb, out


def _check_vec_rows(x, d, cb, L, k, V, out, rows):
    from oracle import oracle_decode_vec, oracle_encode_vec

    T = x.shape[1]
    start = out.start_state.cpu().numpy().view(np.uint32)
    bits = out.bits.cpu().numpy().view(np.uint32)
    cost = out.path_cost.cpu().numpy().astype(np.float64)
    # every block: the reported cost is its own path's
    y = oracle_decode_vec(bits, start, cb, L, k, V, T)
    J_g = (d.astype(np.float64) * (x.astype(np.float64) - y) ** 2).sum(axis=1)
    tol_all = REL_TOL * J_g + ABS_TOL_PER_D * d.astype(np.float64).sum(axis=1)
    assert np.all(np.abs(cost - J_g) <= tol_all)
    # sampled blocks: optimal
    _, _, J_o = oracle_encode_vec(x[rows], d[rows], cb, L, k, V)
    tol = REL_TOL * J_o + ABS_TOL_PER_D * d[rows].astype(np.float64).sum(axis=1)
    assert np.all(np.abs(J_g[rows] - J_o) <= tol), float(np.max(np.abs(J_g[rows] - J_o) / J_o))


def test_vec2_kernel_many_rounds(cuda_device):
    """More blocks than CTAs: each CTA encodes several blocks in turn, tracing
    one back while it searches the next (double-buffered backpointers)."""
    L, k, V, T, n = 16, 2, 2, 64, 400
    x, d, cb, out = _vec_case(L, k, V, T, n, 8300, cuda_device)
    _check_vec_rows(x, d, cb, L, k, V, out, [0, 1, 147, 148, 149, 296, 398, 399])


def test_vec2_unaligned_codebook_takes_the_runtime_kernel(cuda_device):
    """A binary16 codebook that is not 4-byte aligned cannot be read as pairs:
    the runtime kernel serves it, with the same optimum."""
    L, k, V, T, n = 16, 2, 2, 48, 3
    x, d, cb, out = _vec_case(L, k, V, T, n, 8400, cuda_device, cb_offset=1)
    _check_vec_rows(x, d, cb, L, k, V, out, [0, 1, 2])


@pytest.mark.parametrize("pattern", ["first_zero", "second_zero", "sparse", "all_zero"])
def test_vec2_zero_weights(pattern, cuda_device):
    """Weights of 0 in the first coordinate force the kernel's floor on the
    divisor of its metrics; in the second they zero the ratio; all zero makes
    every path cost 0.  The optimum is still the oracle's."""
    import torch

    L, k, V, T, n = 16, 2, 2, 40, 3
    rng = np.random.default_rng(8500 + len(pattern))
    x = rng.standard_normal((n, T)).astype(np.float32)
    d = rng.lognormal(0.0, 1.0, (n, T)).astype(np.float32)
    if pattern == "first_zero":
        d[:, 0::2] = 0.0
    elif pattern == "second_zero":
        d[:, 1::2] = 0.0
    elif pattern == "sparse":
        d[rng.random((n, T)) < 0.4] = 0.0
    else:
        d[:] = 0.0
    cb = rng.standard_normal((1 << L, V)).astype(np.float16)
    out = tcq.encode_vec(torch.from_numpy(x).to(cuda_device), torch.from_numpy(d).to(cuda_device),
                         torch.from_numpy(cb).to(cuda_device), L, k, V)
    torch.cuda.synchronize()
    _check_vec_rows(x, d, cb, L, k, V, out, list(range(n)))


def _gemv_vec_check(bits, start, scale, cb, L, k, V, T, rows, cols, x, y):
    """The oracle's decode of every block, scaled, times x in fp64; bound: each
    product passes through at most 8 ceil(NS/128) + V ceil(NS/32) fp32 roundings
    in its lane's block sum, one per block in the row sum and 5 in the warp
    reduction (NS = T / V steps per block)."""
    from oracle import oracle_decode_vec

    nb = cols // T
    vals = oracle_decode_vec(bits, start, cb, L, k, V, T).reshape(rows, cols)
    sc = np.ones(rows * nb) if scale is None else scale.astype(np.float64)
    m = vals * np.repeat(sc.reshape(rows, nb), T, axis=1)
    y_o = m @ x.astype(np.float64)
    NS = T // V
    n_round = 8 * -(-NS // 128) + V * -(-NS // 32) + nb + 8
    bound = n_round * 2.0**-24 * np.abs(m * x.astype(np.float64)).sum(axis=1)
    err = np.abs(y.astype(np.float64) - y_o)
    assert np.all(err <= bound + 1e-30), float(np.max(err / np.maximum(bound, 1e-30)))


@pytest.mark.parametrize("L,k,V,T,rows,nb,cbt,cb_offset", [
    (16, 2, 2, 256, 300, 16, "f16", 0),   # compile-time kernel, the MLP shape's blocks
    (16, 2, 2, 256, 4773, 16, "f16", 0),  # 4736 warps x one row, then 37 rows split over CTAs
    (16, 2, 2, 264, 37, 5, "f16", 0),     # 132 steps: a partial second chunk, rows split over CTAs
    (16, 2, 2, 256, 40, 4, "f16", 1),     # unaligned table: runtime kernel
    (16, 2, 2, 30, 20, 3, "f16", 0),      # T % 8 != 0: runtime kernel
    (12, 2, 2, 64, 50, 6, "f32", 0),
    (8, 1, 4, 32, 33, 7, "f16", 0),
])
@pytest.mark.parametrize("scaled", [False, True])
def test_gemv_vec(L, k, V, T, rows, nb, cbt, cb_offset, scaled, cuda_device):
    import torch
    from tests.test_gpu_gemv import _rand_stream

    rng = np.random.default_rng(8600 + L + T + rows + V)
    cols = nb * T
    bits, start = _rand_stream(rng, rows * nb, k * V, T // V)
    cb = rng.standard_normal((1 << L, V)).astype(np.float16 if cbt == "f16" else np.float32)
    scale = rng.lognormal(0.0, 0.5, rows * nb).astype(np.float32) if scaled else None
    x = rng.standard_normal(cols).astype(np.float32)
    cbt_dev = torch.empty(cb.size + cb_offset, dtype=torch.from_numpy(cb).dtype,
                          device=cuda_device)[cb_offset:]
    cbt_dev.copy_(torch.from_numpy(cb.reshape(-1)))
    y = tcq.gemv_vec(torch.from_numpy(bits.view(np.int32)).to(cuda_device),
                     torch.from_numpy(start.view(np.int32)).to(cuda_device),
                     None if scale is None else torch.from_numpy(scale).to(cuda_device),
                     cbt_dev, L, k, V, T, rows, cols, torch.from_numpy(x).to(cuda_device))
    torch.cuda.synchronize()
    _gemv_vec_check(bits, start, scale, cb, L, k, V, T, rows, cols, x, y.cpu().numpy())


def test_gemv_vec2_rows_bit_identical_across_phases(cuda_device):
    """Rows with the same blocks give the same bits whether a warp takes the
    row or the row's items are spread over a CTA's warps (the last round)."""
    import torch
    from tests.test_gpu_gemv import _rand_stream

    L, k, V, T, nb = 16, 2, 2, 256, 16
    rows = 4736 + 37  # 148 CTAs x 32 warps, then 37 rows, one per CTA
    rng = np.random.default_rng(8650)
    bits1, start1 = _rand_stream(rng, nb, k * V, T // V)
    bits = np.tile(bits1, (rows, 1))
    start = np.tile(start1, rows)
    cb = rng.standard_normal((1 << L, V)).astype(np.float16)
    x = rng.standard_normal(nb * T).astype(np.float32)
    y = tcq.gemv_vec(torch.from_numpy(np.ascontiguousarray(bits).view(np.int32)).to(cuda_device),
                     torch.from_numpy(np.ascontiguousarray(start).view(np.int32)).to(cuda_device),
                     None, torch.from_numpy(cb).to(cuda_device), L, k, V, T, rows, nb * T,
                     torch.from_numpy(x).to(cuda_device))
    torch.cuda.synchronize()
    y = y.cpu().numpy()
    assert np.all(y == y[0])


def test_gemv_vec_of_encoded_matrix(cuda_device):
    """Encode a matrix with the vector encoder and multiply through its bits: the
    product equals the decoded matrix times x within the bound."""
    import torch

    L, k, V, T, rows, nb = 16, 2, 2, 256, 24, 4
    cols = nb * T
    rng = np.random.default_rng(8700)
    w = rng.standard_normal((rows, cols)).astype(np.float32)
    cb = rng.standard_normal((1 << L, V)).astype(np.float16)
    cbd = torch.from_numpy(cb).to(cuda_device)
    enc = tcq.encode_vec(torch.from_numpy(w.reshape(rows * nb, T)).to(cuda_device), None, cbd, L, k, V)
    x = rng.standard_normal(cols).astype(np.float32)
    y = tcq.gemv_vec(enc.bits, enc.start_state, None, cbd, L, k, V, T, rows, cols,
                     torch.from_numpy(x).to(cuda_device))
    torch.cuda.synchronize()
    _gemv_vec_check(enc.bits.cpu().numpy().view(np.uint32), enc.start_state.cpu().numpy().view(np.uint32),
                    None, cb, L, k, V, T, rows, cols, x, y.cpu().numpy())


def test_gemv_vec_v1_and_rejections(cuda_device):
    import torch
    from tests.test_gpu_gemv import _rand_stream

    rng = np.random.default_rng(8800)
    L, k, T, rows, nb = 12, 2, 64, 10, 3
    bits, start = _rand_stream(rng, rows * nb, k, T)
    cb = torch.from_numpy(rng.standard_normal(1 << L).astype(np.float32)).to(cuda_device)
    x = torch.from_numpy(rng.standard_normal(nb * T).astype(np.float32)).to(cuda_device)
    b = torch.from_numpy(bits.view(np.int32)).to(cuda_device)
    s = torch.from_numpy(start.view(np.int32)).to(cuda_device)
    y1 = tcq.gemv(b, s, None, cb, L, k, T, rows, nb * T, x)
    yv = tcq.gemv_vec(b, s, None, cb, L, k, 1, T, rows, nb * T, x)
    torch.cuda.synchronize()
    assert torch.equal(y1, yv)
    fake = ctypes.c_void_p(0x10000)
    call = lambda **o: tcq.tcq_gemv_vec(fake, fake, None, o.get("cb", fake), o.get("dt", tcq.TCQ_F32),  # noqa: E731
                                        o.get("L", 8), o.get("k", 2), o.get("V", 2), o.get("T", 32),
                                        o.get("rows", 4), o.get("cols", 64), fake, fake, None)
    assert call(dt=tcq.TCQ_MAD, cb=None) == tcq.TCQ_ERR_UNSUPPORTED
    assert call(cols=48) == tcq.TCQ_ERR_INVALID_ARG        # cols % T != 0
    assert call(T=33) == tcq.TCQ_ERR_UNSUPPORTED           # V does not divide T
    assert call(V=9) == tcq.TCQ_ERR_UNSUPPORTED
    assert call(rows=0) == tcq.TCQ_OK
