"""Seeded random shapes through the C ABI, each against the oracle: a sweep of
(L, k, T, n_blocks, weighting, codebook dtype) for the encoder (which kernel
runs depends on the shape: one warp per block, grouped, runtime), random
streams for the decoder, and (V, m, T) for the 8-state set-partitioned trellis.
Every case is small enough for the C oracle; the seeds fix the shapes, so a
failure names a reproducible case.
"""
import numpy as np
import pytest

from tests.parity import check_encode, gpu_encode
from trellis_coded_weight_tcq_b200 import tcq, workloads

pytestmark = pytest.mark.gpu


def _encode_cases(n, seed):
    rng = np.random.default_rng(seed)
    out = []
    while len(out) < n:
        L = int(rng.integers(2, 17))
        k = int(rng.integers(1, min(4, L) + 1))
        T = int(rng.choice([1, 2, 3, 7, 31, 64, 65, 128, 255, 256, 300, 513, 1024, 1025]))
        # keep the oracle's work (n T 2^L 2^k) to a few hundred million node updates
        budget = 3e8 / (T * (1 << L) * (1 << k))
        if budget < 1:
            continue
        nb = int(rng.integers(1, int(min(64, budget)) + 1))
        weighted = bool(rng.integers(0, 2))
        cbt = "f16" if rng.integers(0, 2) else "f32"
        out.append((L, k, T, nb, weighted, cbt, int(rng.integers(0, 2**31))))
    # and random blocks for each specialised kernel: one warp per block (L = 8,
    # k = 2, up to 1024 steps), the grouped kernels of L = 8 (longer blocks), 12, 16
    for (L, k, cbt) in [(8, 2, "f32"), (8, 2, "f16"), (8, 2, "f32"), (12, 2, "f32"), (16, 2, "f16"),
                        (16, 3, "f16")]:
        T = int(rng.choice([1, 2, 63, 64, 200, 256, 1000, 1024])) if L == 8 else int(rng.integers(1, 300))
        if (L, k, cbt) == (8, 2, "f32") and len(out) % 2 == 0:
            T = int(rng.integers(1025, 1500))
        nb = int(rng.integers(1, int(max(1, min(64, 3e8 / (T * (1 << L) * (1 << k))))) + 1))
        out.append((L, k, T, nb, bool(rng.integers(0, 2)), cbt, int(rng.integers(0, 2**31))))
    return out


@pytest.mark.parametrize("L,k,T,nb,weighted,cbt,seed", _encode_cases(40, 20261202),
                         ids=lambda v: str(v))
def test_encode_random_shape(L, k, T, nb, weighted, cbt, seed):
    wl = workloads.small_random(L, k, T, nb, weighted, cbt, seed=seed)
    start, bits, cost = gpu_encode(wl)
    check_encode(wl, start, bits, cost)


def _decode_cases(n, seed):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        L = int(rng.integers(1, 17))
        k = int(rng.integers(1, min(4, L) + 1))
        T = int(rng.choice([1, 5, 32, 64, 100, 256, 257, 1000]))
        out.append((L, k, T, int(rng.integers(1, 200)), "f16" if rng.integers(0, 2) else "f32",
                    int(rng.integers(0, 2**31))))
    return out


@pytest.mark.parametrize("L,k,T,nb,cbt,seed", _decode_cases(30, 77001), ids=lambda v: str(v))
def test_decode_random_shape(L, k, T, nb, cbt, seed, cuda_device):
    import torch
    from oracle import oracle_decode

    rng = np.random.default_rng(seed)
    W = tcq.tcq_words_per_block(k, T)
    bits = rng.integers(0, 2**32, size=(nb, W), dtype=np.uint64).astype(np.uint32)
    used = T * k - 32 * (W - 1)
    if used < 32:
        bits[:, -1] &= np.uint32(((1 << used) - 1) << (32 - used))
    start = rng.integers(0, 2**32, size=nb, dtype=np.uint64).astype(np.uint32)
    cb = rng.standard_normal(1 << L).astype(np.float16 if cbt == "f16" else np.float32)
    y = tcq.decode(torch.from_numpy(bits.view(np.int32)).to(cuda_device),
                   torch.from_numpy(start.view(np.int32)).to(cuda_device),
                   torch.from_numpy(cb).to(cuda_device), L, k, T)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(y.cpu().numpy(), oracle_decode(bits, start, cb, L, k, T).astype(np.float32))


def _ub8_cases(n, seed):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        V = int(rng.integers(1, 9))
        m = int(rng.integers(0, 9))
        S = int(rng.integers(1, 129))
        out.append((V, m, S * V, int(rng.integers(1, 48)), bool(rng.integers(0, 2)),
                    "f16" if rng.integers(0, 2) else "f32", int(rng.integers(0, 2**31))))
    return out


@pytest.mark.parametrize("V,m,T,nb,weighted,cbt,seed", _ub8_cases(20, 88002), ids=lambda v: str(v))
def test_ub8_random_shape(V, m, T, nb, weighted, cbt, seed, cuda_device):
    import torch
    from oracle import oracle_ub8_decode
    from tests.test_gpu_ub8 import _check

    rng = np.random.default_rng(seed)
    x = rng.standard_normal((nb, T)).astype(np.float32)
    d = rng.lognormal(0.0, 1.0, (nb, T)).astype(np.float32) if weighted else None
    cb = workloads.ub8_gaussian_codebook(V, m, cbt, seed=seed % 1000)
    xt = torch.from_numpy(x).to(cuda_device)
    dt = None if d is None else torch.from_numpy(d).to(cuda_device)
    ct = torch.from_numpy(cb).to(cuda_device)
    out = tcq.ub8_encode(xt, dt, ct, V, m)
    torch.cuda.synchronize()
    got = (out.start_state.cpu().numpy().view(np.uint32), out.bits.cpu().numpy().view(np.uint32),
           out.path_cost.cpu().numpy())
    _check(x, d, cb, V, m, got)
    y = tcq.ub8_decode(out.bits, out.start_state, ct, V, m, T)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(y.cpu().numpy(), oracle_ub8_decode(got[1], got[0], cb, V, m, T).astype(np.float32))


def _gemv_cases(n, seed):
    rng = np.random.default_rng(seed)
    out = []
    for q in range(n):
        if q % 3 == 0:  # the half-block kernel's shapes: L = 16, k = 2, T = 256, 4096-column chunks
            L, k, T, nb = 16, 2, 256, 16 * int(rng.integers(1, 3))
            rows = int(rng.choice([1, 37, 148, 2367, 2369, 4000, 7103, 7105, 9000]))
            rows = min(rows, 4000) if nb > 16 else rows  # keep the oracle's fp64 product small
        else:
            L = int(rng.integers(2, 17))
            k = int(rng.integers(1, min(4, L) + 1))
            T = int(rng.choice([4, 8, 24, 64, 100, 256, 512]))
            nb = int(rng.integers(1, 12))
            rows = int(rng.integers(1, 400))
        code = "mad" if (L == 16 and rng.integers(0, 3) == 0) else ("f16" if rng.integers(0, 2) else "f32")
        if code == "f32" and L >= 15:  # the header's rule: a binary16 table from L = 15 on
            code = "f16"
        out.append((L, k, T, rows, nb, code, bool(rng.integers(0, 2)), int(rng.integers(0, 2**31))))
    return out


@pytest.mark.parametrize("L,k,T,rows,nb,code,scaled,seed", _gemv_cases(24, 99003), ids=lambda v: str(v))
def test_gemv_random_shape(L, k, T, rows, nb, code, scaled, seed, cuda_device):
    import torch
    from oracle import oracle_mad_codebook
    from tests.test_gpu_gemv import _check, _rand_stream

    rng = np.random.default_rng(seed)
    cols = nb * T
    bits, start = _rand_stream(rng, rows * nb, k, T)
    scale = rng.lognormal(0.0, 0.5, rows * nb).astype(np.float32) if scaled else None
    x = rng.standard_normal(cols).astype(np.float32)
    if code == "mad":
        cb, cbt = oracle_mad_codebook(L).astype(np.float16), tcq.MAD
    else:
        cb = rng.standard_normal(1 << L).astype(np.float16 if code == "f16" else np.float32)
        cbt = torch.from_numpy(cb).to(cuda_device)
    y = tcq.gemv(torch.from_numpy(bits.view(np.int32)).to(cuda_device),
                 torch.from_numpy(start.view(np.int32)).to(cuda_device),
                 None if scale is None else torch.from_numpy(scale).to(cuda_device),
                 cbt, L, k, T, rows, cols, torch.from_numpy(x).to(cuda_device))
    torch.cuda.synchronize()
    _check(bits, start, scale, cb, L, k, T, rows, cols, x, y.cpu().numpy())
