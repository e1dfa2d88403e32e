"""The allocation-free encoder (tcq_encode_static_scratch).

Some callers cannot allocate device memory (their own pool owns the GPU, or a
latency-critical path must not call cudaMalloc); for them the library offers an
encoder whose scratch is a static device array inside the library.  This test
calls it through the C ABI twice in a row, on different inputs, so the second
call runs on whatever the first left in the shared scratch, and checks each
result against the oracle's optimum (the parity tests' bound, check_encode)
and against tcq_encode's result on the same inputs.  The computed code, whose
table the entry point writes into the front of the static array, is covered
too, and so is the size limit: the longest block the array holds is encoded
and checked, one step longer is refused.  The file is collected last and
passes both alone in a fresh process and after the other tests (the first
call on a device does the set-up either way).
"""
import ctypes

import numpy as np
import pytest

from tests.parity import ABS_TOL_PER_D, REL_TOL, check_encode, gpu_encode, sum_d
from trellis_coded_weight_tcq_b200 import tcq, workloads

pytestmark = pytest.mark.gpu

STATIC_BYTES = 32 * 1024 * 1024  # TCQ_STATIC_SCRATCH_BYTES


def _mad_workload(wl):
    """The same inputs with the computed code (its table, exact in binary16, for the oracle)."""
    from oracle import oracle_mad_codebook

    return workloads.Workload(wl.name + "_mad", wl.L, wl.k, wl.T, wl.x, wl.d,
                              oracle_mad_codebook(wl.L).astype(np.float16))


def _static_scratch_encode(wl, dtype):
    import torch

    dev = torch.device("cuda", 0)
    x = torch.from_numpy(wl.x).to(dev)
    d = None if wl.d is None else torch.from_numpy(wl.d).to(dev)
    cb = None if dtype == tcq.TCQ_MAD else torch.from_numpy(wl.codebook).to(dev)
    W = tcq.tcq_words_per_block(wl.k, wl.T)
    start = torch.empty(wl.n_blocks, dtype=torch.int32, device=dev)
    bits = torch.empty((wl.n_blocks, W), dtype=torch.int32, device=dev)
    cost = torch.empty(wl.n_blocks, dtype=torch.float32, device=dev)
    P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = tcq.tcq_encode_static_scratch(P(x), P(d), P(cb), dtype, wl.L, wl.k, wl.T,
                                       wl.n_blocks, P(start), P(bits), P(cost),
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == tcq.TCQ_OK, tcq.tcq_status_string(st)
    torch.cuda.synchronize()
    return (start.cpu().numpy().view(np.uint32), bits.cpu().numpy().view(np.uint32),
            cost.cpu().numpy())


def _regular_encode(wl, dtype):
    """tcq_encode with a full workspace (the computed code through tcq.MAD)."""
    import torch

    if dtype != tcq.TCQ_MAD:
        return gpu_encode(wl)
    dev = torch.device("cuda", 0)
    x = torch.from_numpy(wl.x).to(dev)
    d = None if wl.d is None else torch.from_numpy(wl.d).to(dev)
    out = tcq.encode(x, d, tcq.MAD, wl.L, wl.k)
    torch.cuda.synchronize()
    return (out.start_state.cpu().numpy().view(np.uint32), out.bits.cpu().numpy().view(np.uint32),
            out.path_cost.cpu().numpy())


def _path_cost(wl, start, bits):
    from oracle import oracle_decode, oracle_path_cost

    y = oracle_decode(bits, start, wl.codebook, wl.L, wl.k, wl.T)
    return oracle_path_cost(wl.x, wl.d, y)


def _check_against_regular(wl, dtype, got):
    s_new, b_new, c_new = got
    s_ref, b_ref, c_ref = _regular_encode(wl, dtype)
    J_ref = _path_cost(wl, s_ref, b_ref)
    J_new = _path_cost(wl, s_new, b_new)
    tol = REL_TOL * J_ref + ABS_TOL_PER_D * sum_d(wl)
    assert np.all(np.abs(J_new - J_ref) <= tol)
    assert np.all(np.abs(c_new.astype(np.float64) - c_ref.astype(np.float64)) <= tol)


@pytest.mark.parametrize("dtype", [tcq.TCQ_F16, tcq.TCQ_MAD], ids=["f16_table", "computed_code"])
def test_static_scratch_encoder_on_two_calls_in_a_row(dtype, cuda_device):
    # more blocks than the static scratch holds CTAs at L=16, so each CTA runs
    # several rounds; the second call sees the first call's leftovers
    cases = [workloads.small_random(16, 2, 256, 64, True, "f16", seed=901),
             workloads.small_random(16, 2, 256, 64, False, "f16", seed=902)]
    for wl in cases:
        if dtype == tcq.TCQ_MAD:
            wl = _mad_workload(wl)
        got = _static_scratch_encode(wl, dtype)
        check_encode(wl, *got, pure=True)  # the oracle's optimum, the parity bound
        _check_against_regular(wl, dtype, got)


def _longest_block(dtype):
    """Largest T whose single-CTA share (the entry point's own test) fits the array."""
    lo, hi = 1, 1 << 20
    while lo < hi:
        mid = (lo + hi + 1) // 2
        if tcq.tcq_encode_workspace_bytes(16, 2, mid, 1, dtype) <= STATIC_BYTES:
            lo = mid
        else:
            hi = mid - 1
    return lo


@pytest.mark.parametrize("dtype,t_max", [(tcq.TCQ_F16, 4096), (tcq.TCQ_MAD, 4080)],
                         ids=["f16_table", "computed_code"])
def test_static_scratch_size_limit_is_exact(dtype, t_max, cuda_device):
    # the documented limit is the one the workspace query (and so run_encode's
    # own fit test) gives: 8 KiB of backpointers per step, plus the path and,
    # for the computed code, its 128 KiB table
    assert _longest_block(dtype) == t_max
    wl = workloads.small_random(16, 2, t_max, 2, True, "f16", seed=903)
    if dtype == tcq.TCQ_MAD:
        wl = _mad_workload(wl)
    got = _static_scratch_encode(wl, dtype)
    check_encode(wl, *got, pure=True)
    # one step longer is refused before anything is dereferenced
    fake = ctypes.c_void_p(256)
    st = tcq.tcq_encode_static_scratch(fake, None, None if dtype == tcq.TCQ_MAD else fake, dtype,
                                       16, 2, t_max + 1, 1, fake, fake, fake, None)
    assert st == tcq.TCQ_ERR_WORKSPACE


def test_static_scratch_rejects_shapes_beyond_its_size(cuda_device):
    # T = 8192 at L=16, k=2 needs 64 MiB of backpointers, above the 32 MiB
    # static array.  The pointers are never dereferenced: the size check comes first.
    fake = ctypes.c_void_p(256)
    st = tcq.tcq_encode_static_scratch(fake, None, fake, tcq.TCQ_F16, 16, 2, 8192, 1, fake, fake,
                                       fake, None)
    assert st == tcq.TCQ_ERR_WORKSPACE
