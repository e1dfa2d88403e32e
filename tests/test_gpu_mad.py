"""GPU parity of every entry point with the computed (lookup-free) code, TCQ_MAD,
against the oracle run on the oracle's own table of that code.

The code is exact in binary16, so the encoders (which write it as a table to
their workspace) are checked by cost like any binary16 codebook, decode is
bit-exact, the matrix-vector product computes each codeword in registers and
keeps the table-based kernel's error bound, and the soft quantizer and the
error-feedback driver keep theirs.
"""
import ctypes

import numpy as np
import pytest

from tests.parity import ABS_TOL_PER_D, REL_TOL, oracle_encode_parallel
from trellis_coded_weight_tcq_b200 import tcq

pytestmark = pytest.mark.gpu


def _cb(L):
    from oracle import oracle_mad_codebook

    return oracle_mad_codebook(L)


@pytest.mark.parametrize("L,k,T,n,weighted", [
    (16, 2, 256, 24, True),    # register-resident L=16 encoder on the written table
    (16, 3, 256, 8, True),
    (12, 2, 256, 64, True),
    (10, 3, 40, 30, False),    # runtime-(L,k) encoder
    (8, 2, 64, 100, True),
])
def test_encode_with_computed_code(L, k, T, n, weighted, cuda_device):
    import torch
    from oracle import oracle_decode, oracle_path_cost

    rng = np.random.default_rng(7000 + L + 10 * k)
    x = rng.standard_normal((n, T)).astype(np.float32)
    d = rng.lognormal(0.0, 1.0, (n, T)).astype(np.float32) if weighted else None
    xt = torch.from_numpy(x).to(cuda_device)
    dt = None if d is None else torch.from_numpy(d).to(cuda_device)
    out = tcq.encode(xt, dt, tcq.MAD, L, k)
    torch.cuda.synchronize()
    start = out.start_state.cpu().numpy().view(np.uint32)
    bits = out.bits.cpu().numpy().view(np.uint32)
    cost = out.path_cost.cpu().numpy()
    cb = _cb(L)
    _, _, J_o = oracle_encode_parallel(x, d, cb, L, k)
    y = oracle_decode(bits, start, cb, L, k, T)
    J_g = oracle_path_cost(x, d, y)
    sd = np.full(n, float(T)) if d is None else d.astype(np.float64).sum(axis=1)
    tol = REL_TOL * J_o + ABS_TOL_PER_D * sd
    assert np.all(np.abs(J_g - J_o) <= tol)
    assert np.all(np.abs(cost.astype(np.float64) - J_g) <= tol)


@pytest.mark.parametrize("L,k,T", [(16, 2, 256), (16, 3, 96), (12, 2, 64), (5, 1, 7)])
def test_decode_computed_code_bit_exact(L, k, T, cuda_device):
    import torch
    from oracle import oracle_decode

    rng = np.random.default_rng(7100 + L + k)
    n = 50
    W = tcq.tcq_words_per_block(k, T)
    bits = rng.integers(0, 2**32, size=(n, W), dtype=np.uint64).astype(np.uint32)
    start = rng.integers(0, 2**32, size=n, dtype=np.uint64).astype(np.uint32)
    b = torch.from_numpy(bits.view(np.int32)).to(cuda_device)
    s = torch.from_numpy(start.view(np.int32)).to(cuda_device)
    y = tcq.decode(b, s, tcq.MAD, L, k, T)
    torch.cuda.synchronize()
    y_o = oracle_decode(bits, start, _cb(L), L, k, T).astype(np.float32)
    np.testing.assert_array_equal(y.cpu().numpy(), y_o)


@pytest.mark.parametrize("L,k,T,rows,nb", [
    (16, 2, 256, 300, 16),   # the MLP shape's blocks: compile-time kernel
    (16, 3, 256, 60, 16),
    (16, 2, 256, 40, 6),     # 6 blocks per row: the per-item compile-time kernel
    (12, 2, 256, 70, 8),     # runtime kernel
    (16, 2, 24, 33, 5),      # T not a multiple of 8: runtime kernel
])
@pytest.mark.parametrize("scaled", [False, True])
def test_gemv_computed_code(L, k, T, rows, nb, scaled, cuda_device):
    from tests.test_gpu_gemv import _check, _rand_stream

    rng = np.random.default_rng(7200 + L + T + rows)
    cols = nb * T
    bits, start = _rand_stream(rng, rows * nb, k, T)
    scale = rng.lognormal(0.0, 0.5, rows * nb) if scaled else None
    x = rng.standard_normal(cols)
    import torch

    b = torch.from_numpy(np.ascontiguousarray(bits).view(np.int32)).to(cuda_device)
    s = torch.from_numpy(np.ascontiguousarray(start).view(np.int32)).to(cuda_device)
    sc = None if scale is None else torch.from_numpy(scale.astype(np.float32)).to(cuda_device)
    xv = torch.from_numpy(x.astype(np.float32)).to(cuda_device)
    y = tcq.gemv(b, s, sc, tcq.MAD, L, k, T, rows, cols, xv)
    torch.cuda.synchronize()
    _check(bits, start, scale, _cb(L), L, k, T, rows, cols, x, y.cpu().numpy())


def test_bcjr_computed_code(cuda_device):
    import torch
    from oracle import oracle_bcjr
    from tests.test_gpu_bcjr import _tolerances

    L, k, T, n, tau = 16, 2, 48, 3, 0.3
    rng = np.random.default_rng(7300)
    x = rng.standard_normal((n, T)).astype(np.float32)
    d = rng.lognormal(0.0, 1.0, (n, T)).astype(np.float32)
    y, F = tcq.bcjr(torch.from_numpy(x).to(cuda_device), torch.from_numpy(d).to(cuda_device),
                    tcq.MAD, L, k, tau)
    torch.cuda.synchronize()
    cb = _cb(L)
    y_o, F_o = oracle_bcjr(x, d, cb, L, k, tau)
    y_tol, F_tol = _tolerances(T, cb, F_o, tau)
    assert np.abs(y.cpu().numpy() - y_o).max() <= y_tol
    assert np.all(np.abs(F.cpu().numpy().astype(np.float64) - F_o) <= F_tol)


def test_ldlq_computed_code(cuda_device):
    import torch
    from oracle import oracle_decode
    from tests.test_gpu_ldlq import _check_targets
    from trellis_coded_weight_tcq_b200.workloads import ldlq_random

    wl = ldlq_random(12, 2, 256, 20, 512, True, "f32", seed=7400)
    wl.codebook = _cb(12).astype(np.float32)  # the oracle side of the check
    res = tcq.ldlq(torch.from_numpy(wl.w).to(cuda_device), torch.from_numpy(wl.u).to(cuda_device),
                   torch.from_numpy(wl.d).to(cuda_device), tcq.MAD, wl.L, wl.k, wl.T)
    torch.cuda.synchronize()
    out = {"q": res.q.cpu().numpy(), "x": res.x.cpu().numpy()}
    start = res.coded.start_state.cpu().numpy().view(np.uint32)
    bits = res.coded.bits.cpu().numpy().view(np.uint32)
    y = oracle_decode(bits, start, wl.codebook, wl.L, wl.k, wl.T)
    np.testing.assert_array_equal(y.reshape(wl.rows, wl.cols), out["q"].astype(np.float64))
    _check_targets(wl, out, np.arange(wl.rows))


def test_workspace_holds_the_table_and_null_codebook(cuda_device):
    f16 = tcq.tcq_encode_workspace_bytes(16, 2, 256, 1, tcq.TCQ_F16)
    mad = tcq.tcq_encode_workspace_bytes(16, 2, 256, 1, tcq.TCQ_MAD)
    assert mad == f16 + (2 << 16)
    assert tcq.tcq_encode_path(16, 2, tcq.TCQ_MAD) == tcq.tcq_encode_path(16, 2, tcq.TCQ_F16)
    fake = ctypes.c_void_p(0x10000)
    # a NULL codebook is an error for a table and accepted for the computed code
    assert tcq.tcq_decode(fake, fake, None, tcq.TCQ_F16, 8, 2, 8, 4, fake, None) == tcq.TCQ_ERR_INVALID_ARG
    # a workspace too small for the table is refused before anything is launched
    assert tcq.tcq_encode(fake, None, None, tcq.TCQ_MAD, 16, 2, 256, 1, fake, fake, fake, fake,
                          100, None) == tcq.TCQ_ERR_WORKSPACE


def test_fixed_start_with_computed_code(cuda_device):
    import torch
    from oracle import oracle_decode, oracle_encode, oracle_path_cost

    L, k, T, n = 16, 2, 64, 6
    rng = np.random.default_rng(7500)
    x = rng.standard_normal((n, T)).astype(np.float32)
    starts = rng.integers(0, 1 << (L - k), size=n).astype(np.uint32)
    out = tcq.encode(torch.from_numpy(x).to(cuda_device), None, tcq.MAD, L, k,
                     fixed_start=torch.from_numpy(starts.view(np.int32)).to(cuda_device))
    torch.cuda.synchronize()
    cb = _cb(L)
    start = out.start_state.cpu().numpy().view(np.uint32)
    bits = out.bits.cpu().numpy().view(np.uint32)
    np.testing.assert_array_equal(start, starts)
    for b in range(n):
        _, _, J_o = oracle_encode(x[b:b + 1], None, cb, L, k, fixed_start=int(starts[b]))
        J_g = oracle_path_cost(x[b:b + 1], None, oracle_decode(bits[b:b + 1], start[b:b + 1], cb, L, k, T))
        assert abs(J_g[0] - J_o[0]) <= REL_TOL * J_o[0] + ABS_TOL_PER_D * T
