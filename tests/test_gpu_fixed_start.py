"""GPU parity of the fixed-start encode (tcq_encode_fixed_start) against the oracle,
including the 2-bit post's toy, which starts in state 0."""
import json
import os

import numpy as np
import pytest

from tests.parity import ABS_TOL_PER_D, REL_TOL

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _gpu(x, d, cb, L, k, starts, device):
    import torch
    from trellis_coded_weight_tcq_b200 import tcq

    xt = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)
    dt = None if d is None else torch.from_numpy(np.ascontiguousarray(d, dtype=np.float32)).to(device)
    ct = torch.from_numpy(cb).to(device)
    st = torch.from_numpy(np.asarray(starts, dtype=np.uint32).view(np.int32)).to(device)
    out = tcq.encode(xt, dt, ct, L, k, fixed_start=st)
    torch.cuda.synchronize()
    return (out.start_state.cpu().numpy().view(np.uint32), out.bits.cpu().numpy().view(np.uint32),
            out.path_cost.cpu().numpy())


def test_page_toy_from_state_zero(cuda_device):
    """Start 0, encode [-0.4, 0.1, 1.5]: the searched path, bits 011, costs 1.37
    (below the page's 1.42 for plain rounding)."""
    with open(os.path.join(GOLDEN, "page_toy_trellis.json")) as f:
        g = json.load(f)
    cb = np.array(g["codebook"], dtype=np.float32)
    start, bits, cost = _gpu(np.array([g["x"]]), None, cb, g["L"], g["k"], [g["start_state"]],
                             cuda_device)
    assert start[0] == 0
    assert bits[0, 0] >> 29 == 0b011
    assert cost[0] == pytest.approx(1.37, abs=1e-6)
    assert cost[0] < g["printed_plain_rounding_cost"]


# L, k, T, blocks, codebook dtype, weighted
CASES = [
    (16, 2, 256, 24, "f16", True),    # register-resident encoder
    (16, 3, 256, 12, "f16", True),
    (12, 2, 256, 40, "f32", True),
    (8, 2, 64, 64, "f32", False),     # one warp per block
    (8, 2, 1, 40, "f16", True),
    (8, 2, 1100, 3, "f32", True),     # longer than the warp kernel holds: grouped
    (10, 3, 33, 20, "f32", True),     # runtime-(L,k) encoder
    (16, 2, 1, 9, "f16", True),       # T = 1: only the successors of s_0
    (6, 1, 7, 16, "f32", True),
    (16, 2, 2048, 2, "f16", True),    # long blocks: the renormalising instantiation
    (12, 2, 3000, 2, "f32", False),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "L{}k{}T{}_B{}_{}{}".format(*c[:5], "_w" if c[5] else ""))
def test_fixed_start_parity(case, cuda_device):
    from oracle import oracle_decode, oracle_encode, oracle_path_cost

    L, k, T, n, cbt, weighted = case
    rng = np.random.default_rng(6000 + 13 * L + k + T)
    x = rng.standard_normal((n, T)).astype(np.float32)
    d = rng.lognormal(0.0, 1.0, (n, T)).astype(np.float32) if weighted else None
    cb = rng.standard_normal(1 << L)
    cb = cb.astype(np.float16) if cbt == "f16" else cb.astype(np.float32)
    # start states: random, with bits above L-k set on some (ignored)
    starts = rng.integers(0, 1 << 32, size=n, dtype=np.uint64).astype(np.uint32)
    start, bits, cost = _gpu(x, d, cb, L, k, starts, cuda_device)
    low = (1 << (L - k)) - 1
    np.testing.assert_array_equal(start, starts & low)
    for b in range(n):
        db = None if d is None else d[b:b + 1]
        _, _, J_o = oracle_encode(x[b:b + 1], db, cb, L, k, fixed_start=int(starts[b] & low))
        y = oracle_decode(bits[b:b + 1], start[b:b + 1], cb, L, k, T)
        J_g = oracle_path_cost(x[b:b + 1], db, y)
        tol = REL_TOL * J_o[0] + ABS_TOL_PER_D * (T if db is None else float(db.sum()))
        assert abs(J_g[0] - J_o[0]) <= tol, f"block {b}: {J_g[0]} vs {J_o[0]}"
        assert abs(float(cost[b]) - J_g[0]) <= tol
    # never better than the free start
    import torch
    from trellis_coded_weight_tcq_b200 import tcq

    xt = torch.from_numpy(x).to(cuda_device)
    dt = None if d is None else torch.from_numpy(d).to(cuda_device)
    free = tcq.encode(xt, dt, torch.from_numpy(cb).to(cuda_device), L, k)
    torch.cuda.synchronize()
    assert np.all(free.path_cost.cpu().numpy() <= cost * (1 + 1e-6) + 1e-6)


def test_fixed_start_rejects_null(cuda_device):
    import ctypes

    from trellis_coded_weight_tcq_b200 import tcq

    fake = ctypes.c_void_p(0x10000)
    assert tcq.tcq_encode_fixed_start(fake, None, fake, tcq.TCQ_F32, 8, 2, 16, 4, None, fake, fake,
                                      fake, fake, 1 << 20, None) == tcq.TCQ_ERR_INVALID_ARG
