"""GPU parity of the error-feedback (LDLQ) encode against the oracle.

The targets of a column block depend on the reconstruction of the blocks before
it, so the GPU and oracle runs can part ways once a block has two optimal
paths (or fp32 targets differ from fp64 ones in the last bits).  The checks
therefore compare what is unique given the GPU's own earlier decisions:

* the reconstruction q is the exact decode of the returned bits and starts;
* the targets x equal the oracle's feedback formula applied to the GPU's q,
  within the fp32 rounding of that sum;
* every block's path is optimal for its targets (oracle Viterbi, relative
  1e-5 as for the plain encode) and its reported cost is its own path's;
* with a U whose diagonal blocks are the identity, the proxy loss
  sum_r e_r H e_r^T (e = w - q) equals the sum of the block costs;
* U = I reduces the call to tcq_encode of w's blocks, bit for bit.
"""
import numpy as np
import pytest

from tests.parity import ABS_TOL_PER_D, REL_TOL, oracle_encode_parallel

pytestmark = pytest.mark.gpu

FP32_UNIT = 2.0 ** -24


def _torch_inputs(wl, device):
    import torch

    w = torch.from_numpy(wl.w).to(device)
    u = torch.from_numpy(wl.u).to(device)
    d = None if wl.d is None else torch.from_numpy(wl.d).to(device)
    cb = torch.from_numpy(wl.codebook).to(device)
    return w, u, d, cb


def _run(wl, device, keep_targets=True, workspace=None):
    import torch
    from trellis_coded_weight_tcq_b200 import tcq

    w, u, d, cb = _torch_inputs(wl, device)
    res = tcq.ldlq(w, u, d, cb, wl.L, wl.k, wl.T, keep_targets=keep_targets, workspace=workspace)
    torch.cuda.synchronize()
    out = {
        "q": res.q.cpu().numpy(),
        "x": None if res.x is None else res.x.cpu().numpy(),
        "start": res.coded.start_state.cpu().numpy().view(np.uint32),
        "bits": res.coded.bits.cpu().numpy().view(np.uint32),
        "cost": res.coded.path_cost.cpu().numpy(),
    }
    return out


def _check_targets(wl, out, rows):
    """x[rows] against the oracle's feedback sum on the GPU's own q."""
    from oracle import oracle_feedback_targets

    w = wl.w[rows].astype(np.float64)
    q = out["q"][rows].astype(np.float64)
    u = wl.u.astype(np.float64)
    xo = oracle_feedback_targets(w, u, q, wl.T)
    # |fp32 sum - exact| <= (terms + 3) u sum |terms|, terms = c0 per column
    absu = np.abs(np.triu(u, 1))
    mag = np.abs(w) + np.abs(w - q) @ absu
    c0 = (np.arange(wl.cols) // wl.T) * wl.T
    bound = (c0 + 3)[None, :] * FP32_UNIT * mag
    err = np.abs(out["x"][rows].astype(np.float64) - xo)
    assert np.all(err <= bound), f"{wl.name}: targets off by {float(np.max(err / np.maximum(bound, 1e-300))):.2f}x the bound"


def _block_index(wl, rows):
    nb = wl.cols // wl.T
    return (np.asarray(rows)[:, None] * nb + np.arange(nb)[None, :]).reshape(-1)


def _check_blocks(wl, out, rows):
    """Decode exactness, per-block optimality and self-consistent costs on `rows`."""
    from oracle import oracle_decode, oracle_path_cost

    T, nb = wl.T, wl.cols // wl.T
    blocks = _block_index(wl, rows)
    xb = out["x"][rows].reshape(-1, T).astype(np.float64)
    db = None if wl.d is None else np.tile(wl.d.reshape(nb, T), (len(rows), 1)).astype(np.float64)
    y = oracle_decode(out["bits"][blocks], out["start"][blocks], wl.codebook, wl.L, wl.k, T)
    assert np.array_equal(y, out["q"][rows].reshape(-1, T).astype(np.float64)), "q is not the decode of the bits"
    assert np.all(out["start"][blocks] < (1 << (wl.L - wl.k))), "start state not canonical"
    _, _, J_o = oracle_encode_parallel(xb, db, wl.codebook, wl.L, wl.k)
    J_g = oracle_path_cost(xb, db, y)
    sd = np.full(len(blocks), float(T)) if db is None else db.sum(axis=1)
    tol = REL_TOL * J_o + ABS_TOL_PER_D * sd
    bad = np.abs(J_g - J_o) > tol
    assert not bad.any(), f"{wl.name}: {int(bad.sum())} blocks off the optimum for their targets"
    bad = np.abs(out["cost"][blocks].astype(np.float64) - J_g) > tol
    assert not bad.any(), f"{wl.name}: path_cost disagrees with its own path on {int(bad.sum())} blocks"


# L, k, T, rows, cols, codebook dtype, weighted, block-free U
CASES = [
    (16, 2, 256, 37, 1024, "f16", True, False),
    (16, 3, 256, 9, 512, "f16", True, True),
    (12, 2, 256, 50, 768, "f32", True, False),
    (8, 2, 64, 130, 320, "f32", False, True),   # two row tiles of the feedback product, ragged
    (6, 1, 5, 33, 40, "f32", True, False),      # runtime-(L,k) encoder, T not a multiple of 4
    (10, 2, 96, 3, 288, "f32", True, True),
    (14, 4, 12, 20, 60, "f16", True, False),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "L{}k{}T{}_{}x{}_{}{}{}".format(
    c[0], c[1], c[2], c[3], c[4], c[5], "_w" if c[6] else "", "_bf" if c[7] else ""))
def test_ldlq_parity(case, cuda_device):
    from trellis_coded_weight_tcq_b200.workloads import ldlq_random

    L, k, T, rows, cols, cbt, weighted, block_free = case
    wl = ldlq_random(L, k, T, rows, cols, weighted, cbt, seed=4000 + 17 * L + T + rows,
                     block_free=block_free)
    out = _run(wl, cuda_device)
    all_rows = np.arange(rows)
    # block column 0 has no feedback: its targets are w exactly
    assert np.array_equal(out["x"][:, :T], wl.w[:, :T])
    _check_targets(wl, out, all_rows)
    sample = all_rows if L < 16 else np.unique(np.linspace(0, rows - 1, 6).astype(int))
    _check_blocks(wl, out, sample)
    if block_free:
        u = wl.u.astype(np.float64)
        dvec = np.ones(cols) if wl.d is None else wl.d.astype(np.float64)
        H = u @ np.diag(dvec) @ u.T
        e = wl.w.astype(np.float64) - out["q"].astype(np.float64)
        loss = float(np.einsum("ri,ij,rj->", e, H, e))
        total = float(out["cost"].astype(np.float64).sum())
        assert loss == pytest.approx(total, rel=1e-4)


def test_ldlq_identity_factor_is_blockwise_encode(cuda_device):
    """U = I: every block is coded from w alone, the same bits as tcq_encode."""
    import torch
    from trellis_coded_weight_tcq_b200 import tcq
    from trellis_coded_weight_tcq_b200.workloads import ldlq_random

    wl = ldlq_random(16, 2, 256, 20, 1024, True, "f16", seed=4242)
    wl.u = np.eye(wl.cols, dtype=np.float32)
    out = _run(wl, cuda_device)
    assert np.array_equal(out["x"], wl.w)
    nb = wl.cols // wl.T
    x = torch.from_numpy(wl.w.reshape(-1, wl.T)).to(cuda_device)
    d = torch.from_numpy(np.tile(wl.d.reshape(nb, wl.T), (wl.rows, 1))).to(cuda_device)
    cb = torch.from_numpy(wl.codebook).to(cuda_device)
    enc = tcq.encode(x, d, cb, wl.L, wl.k)
    torch.cuda.synchronize()
    assert np.array_equal(enc.bits.cpu().numpy().view(np.uint32), out["bits"])
    assert np.array_equal(enc.start_state.cpu().numpy().view(np.uint32), out["start"])
    assert np.array_equal(enc.path_cost.cpu().numpy(), out["cost"])


def test_ldlq_without_targets_and_with_small_workspace(cuda_device):
    """No target output (targets staged in the workspace), and a workspace that
    holds one CTA's encode share: the same results as the default call."""
    import torch
    from trellis_coded_weight_tcq_b200 import tcq
    from trellis_coded_weight_tcq_b200.workloads import ldlq_random

    wl = ldlq_random(12, 2, 256, 40, 512, True, "f32", seed=4343)
    ref = _run(wl, cuda_device)
    out = _run(wl, cuda_device, keep_targets=False)
    assert out["x"] is None
    for key in ("q", "start", "bits", "cost"):
        assert np.array_equal(out[key], ref[key]), key
    targets = ((wl.rows * wl.T * 4 + 255) // 256) * 256
    one_cta = tcq.tcq_encode_workspace_bytes(wl.L, wl.k, wl.T, 1, tcq.TCQ_F32)
    ws = torch.empty(targets + one_cta, dtype=torch.uint8, device=cuda_device)
    small = _run(wl, cuda_device, keep_targets=False, workspace=ws)
    for key in ("q", "start", "bits", "cost"):
        assert np.array_equal(small[key], ref[key]), key


def test_ldlq_rejections(cuda_device):
    import torch
    from trellis_coded_weight_tcq_b200 import tcq

    dev = cuda_device
    w = torch.zeros((4, 100), device=dev)
    u = torch.eye(100, device=dev)
    cb = torch.zeros(256, device=dev)
    with pytest.raises(tcq.TCQError):  # cols % T != 0
        tcq.ldlq(w, u, None, cb, 8, 2, 64)
    targets = ((4 * 50 * 4 + 255) // 256) * 256
    ws = torch.empty(targets, dtype=torch.uint8, device=dev)
    with pytest.raises(tcq.TCQError):  # no room for the encoder
        tcq.ldlq(w, u, None, cb, 8, 2, 50, workspace=ws)
    empty = tcq.ldlq(torch.zeros((0, 100), device=dev), u, None, cb, 8, 2, 50)
    assert empty.q.shape == (0, 100)


def test_ldlq_mlp_sampled(cuda_device):
    """The 14336 x 4096 MLP matrix at L=16, k=2, T=256: sampled rows checked in
    full (targets, optimality of every block of those rows, decode)."""
    from trellis_coded_weight_tcq_b200.workloads import ldlq_mlp

    wl = ldlq_mlp()
    out = _run(wl, cuda_device)
    assert np.all(np.isfinite(out["q"])) and np.all(np.isfinite(out["cost"]))
    rows = np.array([0, 1, 4097, 9000, 14335])
    _check_targets(wl, out, rows)
    _check_blocks(wl, out, rows[[0, 2, 4]])


# L, k, T, rows, cols, codebook dtype, weighted
DYADIC = [
    (8, 2, 64, 40, 256, "f32", True),     # fp32-pipe feedback product, grouped L=8 encoder
    (12, 2, 256, 130, 768, "f32", False),  # tensor-core feedback (two 128-row tiles), L=12 encoder
    (16, 2, 256, 6, 768, "f16", False),    # tensor-core feedback, register-resident L=16 encoder
]


@pytest.mark.parametrize("case", DYADIC, ids=lambda c: "L{}k{}T{}_{}x{}_{}{}".format(
    c[0], c[1], c[2], c[3], c[4], c[5], "_w" if c[6] else ""))
def test_ldlq_whole_matrix_bit_exact_on_dyadic_inputs(case, cuda_device):
    """With every fp32 operation exact (the workload's docstring says why), the
    GPU takes exactly the oracle's decisions in every block, its tie rules
    included: the whole reconstruction Q, the targets, the bits, the start
    states and the costs equal the fp64 driver's."""
    from oracle import oracle_ldlq
    from trellis_coded_weight_tcq_b200.workloads import ldlq_dyadic_exact

    L, k, T, rows, cols, cbt, weighted = case
    wl = ldlq_dyadic_exact(L, k, T, rows, cols, weighted, cbt, seed=5000 + L + T + rows)
    out = _run(wl, cuda_device)
    d_o = np.ones(cols) if wl.d is None else wl.d
    q_o, x_o, s_o, b_o, c_o = oracle_ldlq(wl.w, wl.u, d_o, wl.codebook, L, k, T)
    np.testing.assert_array_equal(out["x"].astype(np.float64), x_o)
    np.testing.assert_array_equal(out["q"].astype(np.float64), q_o)
    np.testing.assert_array_equal(out["start"], s_o)
    np.testing.assert_array_equal(out["bits"], b_o)
    np.testing.assert_array_equal(out["cost"].astype(np.float64), c_o)
    # the feedback did something: some targets differ from w
    assert not np.array_equal(out["x"], wl.w)
