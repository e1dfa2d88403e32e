"""Element counts past 2^31: encode, decode and the decode-in-matvec product
on inputs of more than 2^31 weights, so that every offset a kernel forms
(block x T, row x columns) needs 64 bits.

The inputs repeat a small seeded pattern of P blocks (or rows), so block b must
come out exactly like block b mod P: that checks every block of the launch, and
the oracle checks a sample, the last blocks among them.
"""
import numpy as np
import pytest

from tests.parity import ABS_TOL_PER_D, REL_TOL
from trellis_coded_weight_tcq_b200 import tcq

pytestmark = pytest.mark.gpu

BIG = (1 << 31) + 4096  # weights


def _tile_rows(pattern, n, device):
    """n rows on the device, row b = pattern[b mod P] (torch repeat and slice)."""
    import torch

    p = torch.from_numpy(np.ascontiguousarray(pattern)).to(device)
    reps = -(-n // p.shape[0])
    return p.repeat(reps, *([1] * (p.dim() - 1)))[:n].contiguous()


def _same_as_pattern(t, P):
    """Every row b of t equals row b mod P, compared in chunks of whole periods."""
    import torch

    n = t.shape[0]
    head = t[:P]
    row = max(1, t[0].numel())
    step = P * max(1, (1 << 26) // (row * P))  # about 2^26 elements per chunk
    for s in range(0, n, step):
        blk = t[s:min(n, s + step)]
        ref = head.repeat(-(-blk.shape[0] // P), *([1] * (t.dim() - 1)))[:blk.shape[0]]
        if not torch.equal(blk, ref):
            return False
    return True


def _sample(n, P, rng):
    picks = {0, 1, P - 1, P, (1 << 23) - 1, n - 3, n - 2, n - 1}
    picks.update(int(v) for v in rng.integers(0, n, 4))
    return np.array(sorted(b for b in picks if 0 <= b < n))


def test_encode_past_2_31_weights(cuda_device):
    import torch
    from oracle import oracle_decode, oracle_encode, oracle_path_cost

    L, k, T, P = 8, 2, 256, 1031
    n = -(-BIG // T)
    rng = np.random.default_rng(9300)
    pat = rng.standard_normal((P, T)).astype(np.float32)
    cb = rng.standard_normal(1 << L).astype(np.float32)
    x = _tile_rows(pat, n, cuda_device)
    assert x.numel() > (1 << 31)
    out = tcq.encode(x, None, torch.from_numpy(cb).to(cuda_device), L, k)
    torch.cuda.synchronize()
    del x
    assert _same_as_pattern(out.bits, P)
    assert _same_as_pattern(out.start_state, P)
    assert _same_as_pattern(out.path_cost, P)
    rows = _sample(n, P, rng)
    bits = out.bits[torch.from_numpy(rows).to(cuda_device)].cpu().numpy().view(np.uint32)
    start = out.start_state[torch.from_numpy(rows).to(cuda_device)].cpu().numpy().view(np.uint32)
    cost = out.path_cost[torch.from_numpy(rows).to(cuda_device)].cpu().numpy()
    xr = pat[rows % P]
    _, _, J_o = oracle_encode(xr, None, cb, L, k)
    J_g = oracle_path_cost(xr, None, oracle_decode(bits, start, cb, L, k, T))
    tol = REL_TOL * J_o + ABS_TOL_PER_D * T
    assert np.all(np.abs(J_g - J_o) <= tol)
    assert np.all(np.abs(cost.astype(np.float64) - J_g) <= tol)


@pytest.mark.parametrize("L,k,T,cbt", [
    (16, 2, 256, "f16"),   # whole-block fast decoder
    (12, 3, 100, "f32"),   # per-weight decoder, ragged words
])
def test_decode_past_2_31_weights(L, k, T, cbt, cuda_device):
    import torch
    from oracle import oracle_decode
    from tests.test_gpu_gemv import _rand_stream

    P = 4099
    n = -(-BIG // T)
    rng = np.random.default_rng(9400 + L)
    bits_p, start_p = _rand_stream(rng, P, k, T)
    cb = rng.standard_normal(1 << L).astype(np.float16 if cbt == "f16" else np.float32)
    bits = _tile_rows(bits_p.view(np.int32), n, cuda_device)
    start = _tile_rows(start_p.view(np.int32), n, cuda_device)
    y = tcq.decode(bits, start, torch.from_numpy(cb).to(cuda_device), L, k, T)
    torch.cuda.synchronize()
    assert y.numel() > (1 << 31)
    del bits, start
    assert _same_as_pattern(y, P)
    rows = _sample(n, P, rng)
    y_s = y[torch.from_numpy(rows).to(cuda_device)].cpu().numpy()
    y_o = oracle_decode(bits_p[rows % P], start_p[rows % P], cb, L, k, T).astype(np.float32)
    np.testing.assert_array_equal(y_s, y_o)


@pytest.mark.parametrize("code", ["f16", "mad"])
def test_gemv_past_2_31_weights(code, cuda_device):
    import torch
    from oracle import oracle_decode, oracle_gemv, oracle_mad_codebook
    from tests.test_gpu_gemv import _rand_stream

    L, k, T, nb, Pr = 16, 2, 256, 64, 257
    cols = nb * T
    rows = -(-BIG // cols) + 3  # ragged: not a multiple of the kernel's rows per CTA
    rng = np.random.default_rng(9500 + len(code))
    bits_p, start_p = _rand_stream(rng, Pr * nb, k, T)
    if code == "mad":
        cb_arg, cb = tcq.MAD, oracle_mad_codebook(L)
    else:
        cb = rng.standard_normal(1 << L).astype(np.float16)
        cb_arg = torch.from_numpy(cb).to(cuda_device)
    x = rng.standard_normal(cols).astype(np.float32)
    # row r's blocks are the pattern's row r mod Pr
    bits = _tile_rows(bits_p.view(np.int32).reshape(Pr, nb, -1), rows, cuda_device).reshape(rows * nb, -1)
    start = _tile_rows(start_p.view(np.int32).reshape(Pr, nb), rows, cuda_device).reshape(-1)
    assert rows * cols > (1 << 31)
    y = tcq.gemv(bits, start, None, cb_arg, L, k, T, rows, cols, torch.from_numpy(x).to(cuda_device))
    torch.cuda.synchronize()
    del bits, start
    assert _same_as_pattern(y.reshape(rows, 1), Pr)
    pick = _sample(rows, Pr, rng) % Pr
    bp = bits_p.reshape(Pr, nb, -1)[pick].reshape(len(pick) * nb, -1)
    sp = start_p.reshape(Pr, nb)[pick].reshape(-1)
    y_o = oracle_gemv(bp, sp, None, cb, L, k, T, len(pick), cols, x)
    vals = oracle_decode(bp, sp, cb, L, k, T).reshape(len(pick), cols)
    bound = (13 + cols // 256) * 2.0**-24 * np.abs(vals * x).sum(axis=1)
    y_s = y[:Pr].cpu().numpy()[pick]  # every row r equals row r mod Pr (checked above)
    assert np.all(np.abs(y_s.astype(np.float64) - y_o) <= bound)
