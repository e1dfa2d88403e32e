"""Helpers shared by the GPU parity tests: run the CUDA path, run the oracle
(in a spawn-started process pool for the larger cases), and compare.

Tolerance for encode (floating point decides the path, so parity is on cost):
with J_o the oracle's exact optimum and J_g the fp64 cost of the GPU's path,
    |J_g - J_o| <= 1e-5 J_o + 1e-7 sum_t d_t     and the GPU path is valid,
and the GPU's own fp32 path_cost is within the same bound of J_g.  On the
named workloads the plain relative bound |J_g - J_o| <= 1e-5 J_o (no absolute
floor) is asserted as well (``pure=True``).
Decode is compared bit for bit.
"""
from __future__ import annotations

import multiprocessing as mp
import os

import numpy as np

REL_TOL = 1e-5
ABS_TOL_PER_D = 1e-7

_POOL = None


def _pool():
    global _POOL
    if _POOL is None:
        n = max(1, min(32, (os.cpu_count() or 2) - 1))
        _POOL = mp.get_context("spawn").Pool(n)
    return _POOL


def _oracle_chunk(args):
    from oracle import oracle_encode

    x, d, cb, L, k = args
    return oracle_encode(x, d, cb, L, k)


def oracle_encode_parallel(x, d, cb, L, k, chunk=None):
    """oracle_encode over row chunks in worker processes (same result as one call)."""
    from oracle import oracle_encode

    n = x.shape[0]
    work = n * x.shape[1] * (1 << L) * (1 << k)
    if work < 2e8 or n == 1:
        return oracle_encode(x, d, cb, L, k)
    if chunk is None:
        chunk = max(1, n // (4 * max(1, (os.cpu_count() or 2) - 1)))
    jobs = [(x[i:i + chunk], None if d is None else d[i:i + chunk], cb, L, k)
            for i in range(0, n, chunk)]
    parts = _pool().map(_oracle_chunk, jobs)
    return (np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts]),
            np.concatenate([p[2] for p in parts]))


def gpu_encode(wl, device="cuda", workspace_bytes=None):
    """Run the CUDA encoder on a workload; returns numpy (start uint32, bits uint32, cost f32)."""
    import torch

    from trellis_coded_weight_tcq_b200 import tcq

    x = torch.from_numpy(wl.x).to(device)
    d = None if wl.d is None else torch.from_numpy(wl.d).to(device)
    cb = torch.from_numpy(wl.codebook).to(device)
    ws = tcq.Workspace(wl.L, wl.k, wl.T, wl.n_blocks, tcq.cb_dtype_of(cb), device)
    if workspace_bytes is not None:
        ws.nbytes = workspace_bytes
    out = tcq.encode(x, d, cb, wl.L, wl.k, ws)
    torch.cuda.synchronize()
    return (out.start_state.cpu().numpy().view(np.uint32), out.bits.cpu().numpy().view(np.uint32),
            out.path_cost.cpu().numpy())


def gpu_decode(bits, start, codebook, L, k, T, device="cuda"):
    import torch

    from trellis_coded_weight_tcq_b200 import tcq

    b = torch.from_numpy(np.ascontiguousarray(bits).view(np.int32)).to(device)
    s = torch.from_numpy(np.ascontiguousarray(start).view(np.int32)).to(device)
    cb = torch.from_numpy(codebook).to(device)
    y = tcq.decode(b, s, cb, L, k, T)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def sum_d(wl, rows=None):
    if wl.d is None:
        n = wl.n_blocks if rows is None else len(rows)
        return np.full(n, float(wl.T))
    d = wl.d if rows is None else wl.d[rows]
    return d.astype(np.float64).sum(axis=1)


def check_encode(wl, start, bits, cost_gpu, rows=None, oracle_result=None, pure=False):
    """Compare GPU encode output on `rows` (all by default) with the oracle.

    ``pure``: also require the relative bound alone, |J_g - J_o| <= 1e-5 J_o."""
    from oracle import oracle_decode, oracle_path_cost

    rows = np.arange(wl.n_blocks) if rows is None else np.asarray(rows)
    x = wl.x[rows]
    d = None if wl.d is None else wl.d[rows]
    if oracle_result is None:
        oracle_result = oracle_encode_parallel(x, d, wl.codebook, wl.L, wl.k)
    _, _, J_o = oracle_result
    y_g = oracle_decode(bits[rows], start[rows], wl.codebook, wl.L, wl.k, wl.T)
    J_g = oracle_path_cost(x, d, y_g)
    tol = REL_TOL * J_o + ABS_TOL_PER_D * sum_d(wl, rows)
    assert np.all(start[rows] < (1 << (wl.L - wl.k))), "start state not canonical"
    bad = np.abs(J_g - J_o) > tol
    assert not bad.any(), (
        f"{wl.name}: {int(bad.sum())} blocks off the optimum, worst rel "
        f"{float(np.max(np.abs(J_g - J_o) / np.maximum(J_o, 1e-300))):.3e}")
    if pure:
        bad = np.abs(J_g - J_o) > REL_TOL * J_o
        assert not bad.any(), (
            f"{wl.name}: {int(bad.sum())} blocks outside the relative bound alone, worst rel "
            f"{float(np.max(np.abs(J_g - J_o) / np.maximum(J_o, 1e-300))):.3e}")
    bad = np.abs(cost_gpu[rows].astype(np.float64) - J_g) > tol
    assert not bad.any(), f"{wl.name}: path_cost disagrees with its own path on {int(bad.sum())} blocks"
    return J_o, J_g
