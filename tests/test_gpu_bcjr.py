"""GPU parity of the soft forward-backward quantizer (tcq_bcjr) against the oracle.

Tolerances (fp32 on the GPU against fp64): every step's log2 values carry the
ex2/lg2 approximation error (about 2^-22 each) and fp32 rounding of values kept
near 0 by the per-step normalisation, and these add up along the T steps of a
block, so a posterior weight is off by a relative (T + 16) * 2^-20 at most and
a soft codeword, a weighted mean of codewords, by that much of the codebook's
range; the free energy is tau ln 2 times a log2 Z off by the same T-fold sum,
plus fp32 rounding of F itself.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _tolerances(T, cb, F_o, tau):
    span = float(np.max(cb) - np.min(cb))
    y_tol = (T + 16) * 2.0 ** -20 * span
    F_tol = 2.0 ** -22 * np.abs(F_o) + tau * np.log(2.0) * (T + 16) * 2.0 ** -20
    return y_tol, F_tol


def _run(x, d, cb, L, k, tau, device, workspace=None):
    import torch
    from trellis_coded_weight_tcq_b200 import tcq

    xt = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)
    dt = None if d is None else torch.from_numpy(np.ascontiguousarray(d, dtype=np.float32)).to(device)
    ct = torch.from_numpy(cb).to(device)
    y, F = tcq.bcjr(xt, dt, ct, L, k, tau, workspace=workspace)
    torch.cuda.synchronize()
    return y.cpu().numpy(), F.cpu().numpy()


# L, k, T, blocks, codebook dtype, weighted, tau
CASES = [
    (8, 2, 64, 40, "f32", True, 0.5),
    (6, 1, 13, 30, "f32", False, 0.1),
    (12, 2, 256, 6, "f32", True, 0.2),
    (15, 3, 32, 3, "f16", True, 1.0),     # binary16 table of 64 KiB in shared memory
    (16, 2, 24, 2, "f16", True, 0.3),     # binary16 table of 128 KiB
    (16, 2, 12, 2, "f32", True, 0.3),     # binary32 table read through L1
    (4, 4, 20, 10, "f32", True, 0.5),     # no trellis memory
    (14, 4, 12, 4, "f16", True, 2.0),
    (2, 1, 7, 8, "f32", True, 0.05),      # the 2-bit post's toy trellis
    (3, 1, 1, 5, "f32", True, 0.7),       # T = 1
    (10, 2, 300, 3, "f32", True, 0.02),   # cold: close to the hard code
    # the register-resident kernel (L=16, k=2, binary16 codebook, T <= 1024)
    (16, 2, 256, 3, "f16", True, 0.1),
    (16, 2, 7, 5, "f16", False, 0.5),
    (16, 2, 1, 4, "f16", True, 0.3),
    (16, 2, 64, 2, "f16", True, 0.003),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "L{}k{}T{}_B{}_{}{}_tau{}".format(
    c[0], c[1], c[2], c[3], c[4], "_w" if c[5] else "", c[6]))
def test_bcjr_parity(case, cuda_device):
    from oracle import oracle_bcjr

    L, k, T, n, cbt, weighted, tau = case
    rng = np.random.default_rng(5000 + 31 * L + 7 * k + T)
    x = rng.standard_normal((n, T)).astype(np.float32)
    d = rng.lognormal(0.0, 1.0, (n, T)).astype(np.float32) if weighted else None
    cb = rng.standard_normal(1 << L)
    cb = cb.astype(np.float16) if cbt == "f16" else cb.astype(np.float32)
    y_g, F_g = _run(x, d, cb, L, k, tau, cuda_device)
    y_o, F_o = oracle_bcjr(x, d, cb, L, k, tau)
    y_tol, F_tol = _tolerances(T, cb.astype(np.float64), F_o, tau)
    err_y = np.abs(y_g - y_o)
    assert np.all(np.isfinite(y_g)) and np.all(np.isfinite(F_g))
    assert err_y.max() <= y_tol, f"soft codewords off by {err_y.max():.3e} (bound {y_tol:.3e})"
    err_F = np.abs(F_g.astype(np.float64) - F_o)
    assert np.all(err_F <= F_tol), f"free energy off by {err_F.max():.3e}"


def test_bcjr_cold_limit_matches_the_encoder(cuda_device):
    """At a temperature far below the cost gaps the soft code is the hard one:
    y equals the decoded Viterbi path and F the Viterbi cost."""
    import torch
    from trellis_coded_weight_tcq_b200 import tcq

    L, k, T, n = 8, 2, 32, 16
    rng = np.random.default_rng(77)
    x = rng.standard_normal((n, T)).astype(np.float32)
    cb = rng.standard_normal(1 << L).astype(np.float32)
    xt = torch.from_numpy(x).to(cuda_device)
    ct = torch.from_numpy(cb).to(cuda_device)
    enc = tcq.encode(xt, None, ct, L, k)
    yh = tcq.decode(enc.bits, enc.start_state, ct, L, k, T)
    tau = 1e-5
    y_s, F_s = tcq.bcjr(xt, None, ct, L, k, tau)
    torch.cuda.synchronize()
    cost = enc.path_cost.cpu().numpy().astype(np.float64)
    # J_min - tau ln N <= F <= J_min, N = 2^(L + k (T - 1)) paths
    log_n = (L + k * (T - 1)) * np.log(2.0)
    np.testing.assert_allclose(F_s.cpu().numpy(), cost, rtol=1e-5, atol=tau * log_n)
    # blocks whose optimum is clear by far more than tau give the hard code
    np.testing.assert_allclose(y_s.cpu().numpy(), yh.cpu().numpy(), atol=1e-4)


def test_bcjr_small_workspace_and_rejections(cuda_device):
    import torch
    from trellis_coded_weight_tcq_b200 import tcq

    L, k, T, n = 10, 2, 40, 20
    rng = np.random.default_rng(78)
    x = rng.standard_normal((n, T)).astype(np.float32)
    d = rng.lognormal(0.0, 1.0, (n, T)).astype(np.float32)
    cb = rng.standard_normal(1 << L).astype(np.float32)
    y_ref, F_ref = _run(x, d, cb, L, k, 0.4, cuda_device)
    one = tcq.tcq_bcjr_workspace_bytes(L, k, T, 1, tcq.TCQ_F32)
    ws = torch.empty(one, dtype=torch.uint8, device=cuda_device)
    y1, F1 = _run(x, d, cb, L, k, 0.4, cuda_device, workspace=ws)
    np.testing.assert_array_equal(y1, y_ref)
    np.testing.assert_array_equal(F1, F_ref)
    xt = torch.from_numpy(x).to(cuda_device)
    ct = torch.from_numpy(cb).to(cuda_device)
    for bad in (0.0, -1.0, float("inf"), float("nan")):
        with pytest.raises(tcq.TCQError):
            tcq.bcjr(xt, None, ct, L, k, bad)
    with pytest.raises(tcq.TCQError):
        tcq.bcjr(xt, None, ct, L, k, 0.5, workspace=torch.empty(one - 256, dtype=torch.uint8,
                                                                 device=cuda_device))
    y0, F0 = tcq.bcjr(torch.zeros((0, T), device=cuda_device), None, ct, L, k, 0.5)
    assert y0.shape == (0, T)


def test_bcjr_register_kernel_loops_over_blocks(cuda_device):
    """A workspace of one slot makes one CTA take every block in turn: the same
    results as one CTA per block, and the oracle's on a sample."""
    import torch
    from oracle import oracle_bcjr
    from trellis_coded_weight_tcq_b200 import tcq

    L, k, T, n = 16, 2, 48, 5
    rng = np.random.default_rng(79)
    x = rng.standard_normal((n, T)).astype(np.float32)
    d = rng.lognormal(0.0, 1.0, (n, T)).astype(np.float32)
    cb = rng.standard_normal(1 << L).astype(np.float16)
    y_ref, F_ref = _run(x, d, cb, L, k, 0.2, cuda_device)
    one = tcq.tcq_bcjr_workspace_bytes(L, k, T, 1, tcq.TCQ_F16)
    ws = torch.empty(one, dtype=torch.uint8, device=cuda_device)
    y1, F1 = _run(x, d, cb, L, k, 0.2, cuda_device, workspace=ws)
    np.testing.assert_array_equal(y1, y_ref)
    np.testing.assert_array_equal(F1, F_ref)
    y_o, F_o = oracle_bcjr(x[[0, 4]], d[[0, 4]], cb, L, k, 0.2)
    y_tol, F_tol = _tolerances(T, cb.astype(np.float64), F_o, 0.2)
    assert np.abs(y1[[0, 4]] - y_o).max() <= y_tol
    assert np.all(np.abs(F1[[0, 4]] - F_o) <= F_tol)


@pytest.mark.parametrize("L,k,T,cbt", [(16, 2, 64, "f16"), (10, 2, 40, "f32"), (8, 3, 30, "f32")])
def test_bcjr_zero_weights_uniform(L, k, T, cbt, cuda_device):
    """d = 0: uniform over paths, y_t = mean c, F = -tau (L + k (T - 1)) ln 2."""
    rng = np.random.default_rng(9000 + L)
    n, tau = 3, 0.4
    x = rng.standard_normal((n, T)).astype(np.float32)
    d = np.zeros((n, T), dtype=np.float32)
    cb = rng.standard_normal(1 << L)
    cb = cb.astype(np.float16) if cbt == "f16" else cb.astype(np.float32)
    y, F = _run(x, d, cb, L, k, tau, cuda_device)
    c64 = cb.astype(np.float64)
    y_tol, _ = _tolerances(T, c64, np.zeros(n), tau)
    assert np.abs(y - c64.mean()).max() <= y_tol
    F_exact = -tau * (L + k * (T - 1)) * np.log(2.0)
    np.testing.assert_allclose(F.astype(np.float64), F_exact, rtol=1e-6)


def test_bcjr_long_block_takes_the_runtime_kernel(cuda_device):
    """T beyond the register-resident kernel's staged steps (1024) at L=16, k=2:
    the runtime kernel, still against the oracle."""
    from oracle import oracle_bcjr

    L, k, T, n, tau = 16, 2, 1100, 1, 0.5
    rng = np.random.default_rng(9100)
    x = rng.standard_normal((n, T)).astype(np.float32)
    d = rng.lognormal(0.0, 1.0, (n, T)).astype(np.float32)
    cb = rng.standard_normal(1 << L).astype(np.float16)
    y_g, F_g = _run(x, d, cb, L, k, tau, cuda_device)
    y_o, F_o = oracle_bcjr(x, d, cb, L, k, tau)
    y_tol, F_tol = _tolerances(T, cb.astype(np.float64), F_o, tau)
    assert np.abs(y_g - y_o).max() <= y_tol
    assert np.all(np.abs(F_g.astype(np.float64) - F_o) <= F_tol)


def test_bcjr_maximum_block_length(cuda_device):
    """T = TCQ_MAX_T (2^20 weights in one block) through the runtime kernel: the
    per-step shifts and their fp64 sums keep a million steps finite and within
    the per-weight bound."""
    from oracle import oracle_bcjr
    from trellis_coded_weight_tcq_b200 import tcq

    L, k, T, n, tau = 4, 2, tcq.TCQ_MAX_T, 1, 0.5
    rng = np.random.default_rng(9200)
    x = rng.standard_normal((n, T)).astype(np.float32)
    d = rng.lognormal(0.0, 1.0, (n, T)).astype(np.float32)
    cb = rng.standard_normal(1 << L).astype(np.float32)
    y_g, F_g = _run(x, d, cb, L, k, tau, cuda_device)
    y_o, F_o = oracle_bcjr(x, d, cb, L, k, tau)
    assert np.all(np.isfinite(y_g)) and np.all(np.isfinite(F_g))
    # per weight: each step's posterior is renormalised to mass 1, so a soft
    # codeword carries the rounding of the forward and backward values near its
    # step rather than of all T steps: the 1024-step bound is used; the free
    # energy sums T fp64-accumulated shifts and stays within 1e-5 relative
    y_tol, _ = _tolerances(1024, cb.astype(np.float64), F_o, tau)
    assert np.abs(y_g - y_o).max() <= y_tol
    np.testing.assert_allclose(F_g.astype(np.float64), F_o, rtol=1e-5)
