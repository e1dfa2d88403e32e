"""GPU parity of the 8-state set-partitioned trellis (tcq_ub8_encode,
tcq_ub8_decode) against the oracle, through the C ABI.

Encode parity is on cost, with the plain encoder's bound (the fp32 nearest
entry of a subset, or an fp32 path metric, may pick a different but equally
good path); decode is bit-exact; on dyadic inputs every fp32 operation of the
search is exact and the GPU must return the oracle's bits, tie rules included.
"""
import numpy as np
import pytest

from tests.parity import ABS_TOL_PER_D, REL_TOL
from trellis_coded_weight_tcq_b200 import tcq, workloads

pytestmark = pytest.mark.gpu


def _gpu_encode(x, d, cb, V, m, fixed=None, device="cuda"):
    import torch

    xt = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)
    dt = None if d is None else torch.from_numpy(np.ascontiguousarray(d, dtype=np.float32)).to(device)
    ct = torch.from_numpy(cb).to(device)
    ft = None if fixed is None else torch.from_numpy(fixed.astype(np.int32)).to(device)
    out = tcq.ub8_encode(xt, dt, ct, V, m, fixed_start=ft)
    torch.cuda.synchronize()
    return (out.start_state.cpu().numpy().view(np.uint32), out.bits.cpu().numpy().view(np.uint32),
            out.path_cost.cpu().numpy())


def _gpu_decode(bits, start, cb, V, m, T, device="cuda"):
    import torch

    b = torch.from_numpy(np.ascontiguousarray(bits).view(np.int32)).to(device)
    s = torch.from_numpy(np.ascontiguousarray(start).view(np.int32)).to(device)
    y = tcq.ub8_decode(b, s, torch.from_numpy(cb).to(device), V, m, T)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def _check(x, d, cb, V, m, got, fixed=None, pure=True):
    from oracle import oracle_ub8_decode, oracle_ub8_encode

    start, bits, cost = got
    T = x.shape[1]
    _, _, J_o = oracle_ub8_encode(x, d, cb, V, m, fixed_start=None)
    if fixed is not None:  # per block with its own start
        J_o = np.array([oracle_ub8_encode(x[i:i + 1], None if d is None else d[i:i + 1], cb, V, m,
                                          fixed_start=int(fixed[i]))[2][0] for i in range(x.shape[0])])
        np.testing.assert_array_equal(start, fixed.astype(np.uint32) & 7)
    assert np.all(start < 8)
    y = oracle_ub8_decode(bits, start, cb, V, m, T)
    dd = np.ones_like(x, dtype=np.float64) if d is None else d.astype(np.float64)
    J_g = (dd * (x.astype(np.float64) - y) ** 2).sum(axis=1)
    tol = REL_TOL * J_o + ABS_TOL_PER_D * dd.sum(axis=1)
    bad = np.abs(J_g - J_o) > tol
    assert not bad.any(), f"{int(bad.sum())} blocks off the optimum, worst rel " \
        f"{float(np.max(np.abs(J_g - J_o) / np.maximum(J_o, 1e-300))):.3e}"
    if pure:
        assert np.all(np.abs(J_g - J_o) <= REL_TOL * J_o)
    assert np.all(np.abs(cost.astype(np.float64) - J_g) <= tol), "path_cost is not its own path's"
    return J_o


# V, m, T, n_blocks, weighted, codebook dtype
SHAPES = [
    (4, 7, 256, 300, True, "f16"),    # Pingala-8's symbols: 4 weights, 8 bits per step
    (4, 7, 256, 37, False, "f32"),
    (1, 1, 64, 90, True, "f32"),      # scalar TCQ at 2 bits per weight
    (1, 2, 100, 41, False, "f16"),    # 3-bit symbols straddle words
    (2, 3, 130, 19, True, "f32"),     # 65 steps: a ragged lane tail
    (3, 4, 96, 8, True, "f16"),
    (8, 8, 512, 17, True, "f32"),     # the largest union (1024 rows of 8), 9-bit symbols
    (5, 0, 40, 33, False, "f32"),     # one entry per subset
    (6, 5, 6, 70, True, "f16"),       # one step per block
    (1, 8, 512, 5, True, "f32"),      # the longest block (512 steps)
    (7, 6, 3584, 3, True, "f16"),     # 512 steps of 7 weights
]


@pytest.mark.parametrize("V,m,T,n,weighted,cbt", SHAPES,
                         ids=lambda v: str(v))
def test_encode_parity(V, m, T, n, weighted, cbt, cuda_device):
    rng = np.random.default_rng(1000 * V + 10 * m + T + n)
    x = rng.standard_normal((n, T)).astype(np.float32)
    d = rng.lognormal(0.0, 1.0, (n, T)).astype(np.float32) if weighted else None
    cb = workloads.ub8_gaussian_codebook(V, m, cbt, seed=77 + V + m)
    got = _gpu_encode(x, d, cb, V, m, device=cuda_device)
    _check(x, d, cb, V, m, got)
    # decode of the GPU's own stream: bit-exact against the oracle's decode
    from oracle import oracle_ub8_decode

    y = _gpu_decode(got[1], got[0], cb, V, m, T, device=cuda_device)
    np.testing.assert_array_equal(y, oracle_ub8_decode(got[1], got[0], cb, V, m, T).astype(np.float32))


@pytest.mark.parametrize("V,m,T", [(4, 7, 256), (1, 1, 64), (2, 4, 34)])
def test_fixed_start(V, m, T, cuda_device):
    rng = np.random.default_rng(31 + V + m)
    n = 40
    x = rng.standard_normal((n, T)).astype(np.float32)
    d = rng.lognormal(0.0, 1.0, (n, T)).astype(np.float32)
    cb = workloads.ub8_gaussian_codebook(V, m, "f32")
    fixed = rng.integers(0, 2**31, n).astype(np.int64)  # only the low 3 bits matter
    got = _gpu_encode(x, d, cb, V, m, fixed=fixed, device=cuda_device)
    _check(x, d, cb, V, m, got, fixed=fixed)


@pytest.mark.parametrize("V,m,T,cbt", [(4, 7, 256, "f16"), (1, 2, 96, "f32"), (2, 3, 64, "f16")])
def test_dyadic_inputs_bit_exact(V, m, T, cbt, cuda_device):
    """Values on a coarse dyadic grid (multiples of 1/8 in [-2, 2], weights in
    {1/4, 1, 4}, so sqrt(d) is a power of two): every branch metric is a
    multiple of 1/256 below 64 V and every path metric of at most 64 steps fits
    the fp32 significand, so the GPU takes the oracle's decisions exactly."""
    from oracle import oracle_ub8_encode

    rng = np.random.default_rng(400 + V + m)
    n = 64
    x = (rng.integers(-16, 17, (n, T)) / 8.0).astype(np.float32)
    d = (4.0 ** rng.integers(-1, 2, (n, T))).astype(np.float32)
    cb = (rng.integers(-16, 17, (4 << m) * V) / 8.0)
    cb = cb.astype(np.float16) if cbt == "f16" else cb.astype(np.float32)
    start, bits, cost = _gpu_encode(x, d, cb, V, m, device=cuda_device)
    s_o, b_o, c_o = oracle_ub8_encode(x, d, cb, V, m)
    np.testing.assert_array_equal(start, s_o)
    np.testing.assert_array_equal(bits, b_o)
    np.testing.assert_array_equal(cost.astype(np.float64), c_o)


@pytest.mark.parametrize("V,m,T,n", [(4, 7, 256, 1000), (1, 0, 17, 65), (3, 8, 27, 31),
                                     (2, 2, 1024, 33), (8, 5, 4096, 9), (1, 3, 512, 100),
                                     (4, 7, 256, 14213),    # several groups of 32 blocks per CTA
                                     (4, 7, 256, 100000)])  # more groups than resident warps
def test_decode_random_streams_bit_exact(V, m, T, n, cuda_device):
    from oracle import oracle_ub8_decode

    rng = np.random.default_rng(V * 100 + m * 7 + T + n)
    S, K = T // V, 1 + m
    W = tcq.tcq_ub8_words_per_block(V, m, T)
    bits = rng.integers(0, 2**32, size=(n, W), dtype=np.uint64).astype(np.uint32)
    used = S * K - 32 * (W - 1)
    if used < 32:
        bits[:, -1] &= np.uint32(((1 << used) - 1) << (32 - used))
    start = rng.integers(0, 2**32, size=n, dtype=np.uint64).astype(np.uint32)  # high bits ignored
    cb = workloads.ub8_gaussian_codebook(V, m, "f32", seed=5 + V)
    y = _gpu_decode(bits, start, cb, V, m, T, device=cuda_device)
    np.testing.assert_array_equal(y, oracle_ub8_decode(bits, start, cb, V, m, T).astype(np.float32))


def test_mlp_matrix_full_size_sampled(cuda_device):
    """The bench's configuration: the 14336 x 4096 MLP matrix (229,376 blocks of
    256 weights, d per column), V = 4, m = 7 (2 bits per weight) with a Gaussian
    binary16 union codebook; the oracle on sampled blocks, the decode round trip
    on every block."""
    wl = workloads.mlp()
    V, m = 4, 7
    cb = workloads.ub8_gaussian_codebook(V, m, "f16")
    start, bits, cost = _gpu_encode(wl.x, wl.d, cb, V, m, device=cuda_device)
    rng = np.random.default_rng(9)
    rows = np.unique(np.concatenate([[0, wl.n_blocks - 1], rng.choice(wl.n_blocks, 1022, replace=False)]))
    _check(wl.x[rows], wl.d[rows], cb, V, m, (start[rows], bits[rows], cost[rows]))
    y = _gpu_decode(bits, start, cb, V, m, wl.T, device=cuda_device)
    J = (wl.d.astype(np.float64) * (wl.x.astype(np.float64) - y.astype(np.float64)) ** 2).sum(axis=1)
    tol = 1e-5 * J + 1e-7 * wl.d.astype(np.float64).sum(axis=1)
    assert np.all(np.abs(cost.astype(np.float64) - J) <= tol)


def test_empty_and_rejected_calls(cuda_device):
    import torch

    cb = torch.zeros(4 << 3, dtype=torch.float32, device=cuda_device)
    x0 = torch.zeros((0, 16), dtype=torch.float32, device=cuda_device)
    out = tcq.ub8_encode(x0, None, cb, 1, 3)
    assert out.bits.shape[0] == 0
    with pytest.raises(ValueError):  # codebook of the wrong size
        tcq.ub8_encode(torch.zeros((2, 16), device=cuda_device), None, cb[:-1], 1, 3)
    with pytest.raises(tcq.TCQError):  # more than 512 steps
        tcq.ub8_encode(torch.zeros((2, 1024), device=cuda_device), None, cb, 1, 3)


def test_decode_into_unaligned_output(cuda_device):
    """An output that is 4-byte but not 16-byte aligned takes the scalar stores:
    the same values as an aligned one (and as the oracle)."""
    import torch
    from oracle import oracle_ub8_decode

    V, m, T, n = 4, 7, 256, 70
    rng = np.random.default_rng(61)
    W = tcq.tcq_ub8_words_per_block(V, m, T)
    bits = rng.integers(0, 2**32, size=(n, W), dtype=np.uint64).astype(np.uint32)
    start = rng.integers(0, 8, size=n).astype(np.uint32)
    cb = workloads.ub8_gaussian_codebook(V, m, "f32")
    dev = cuda_device
    b = torch.from_numpy(bits.view(np.int32)).to(dev)
    s = torch.from_numpy(start.view(np.int32)).to(dev)
    c = torch.from_numpy(cb).to(dev)
    buf = torch.full((n * T + 1,), float("nan"), device=dev)
    y = buf[1:].view(n, T)
    assert y.data_ptr() % 16 == 4
    tcq.ub8_decode(b, s, c, V, m, T, out=y)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(y.cpu().numpy(), oracle_ub8_decode(bits, start, cb, V, m, T).astype(np.float32))
    assert np.isnan(buf[0].item())
