"""Small parity shapes through the bounds-checked build (libtcq_debug.so).

Run in a process of its own with TCQ_LIBRARY=debug (tests/test_gpu_debug_build.py
does), so that only the debug build is loaded.  Every global-memory index of
the encode, decode, matrix-vector and set-partitioned-trellis kernels is
checked against its buffer there; a failed check sets TCQ_DEVERR_BOUNDS in the
device error word and skips the access.  Each case is checked against the
oracle like the regular parity tests, and the error word must stay clear.
Prints "DEBUG BUILD OK" at the end.
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from oracle import (oracle_decode, oracle_encode, oracle_gemv, oracle_ldlq,  # noqa: E402
                    oracle_mad_codebook, oracle_ub8_decode)
from tests.parity import check_encode, gpu_encode  # noqa: E402
from trellis_coded_weight_tcq_b200 import tcq, workloads  # noqa: E402


def main():
    assert os.environ.get("TCQ_LIBRARY") == "debug" and tcq.LIB_PATH.endswith("libtcq_debug.so")
    tcq.load_library()
    dev = torch.device("cuda", 0)

    def clean(what):
        flags = tcq.device_errors()
        assert flags == 0, f"{what}: device error flags {flags:#x}"
        print(f"ok {what}", flush=True)

    # encoders: register-resident kernels, several teams per CTA, sub-warp teams,
    # the runtime-(L, k) kernel, a fixed start, the computed code
    for (L, k, T, n, w, cb) in [(16, 2, 256, 24, True, "f16"), (16, 3, 256, 8, True, "f16"),
                                (12, 2, 256, 40, True, "f32"), (8, 2, 64, 50, False, "f32"),
                                (10, 3, 40, 9, True, "f32"), (16, 2, 1500, 2, True, "f16")]:
        wl = workloads.small_random(L, k, T, n, w, cb, seed=31 + L + T)
        # the oracle in this process (no worker pool: the shapes are small)
        check_encode(wl, *gpu_encode(wl, dev), oracle_result=oracle_encode(wl.x, wl.d, wl.codebook, L, k))
        clean(f"encode L{L} k{k} T{T}")
    wl = workloads.small_random(8, 2, 64, 20, True, "f32", seed=5)
    x = torch.from_numpy(wl.x).to(dev)
    d = torch.from_numpy(wl.d).to(dev)
    fs = torch.randint(0, 64, (wl.n_blocks,), dtype=torch.int32, device=dev)
    out = tcq.encode(x, d, torch.from_numpy(wl.codebook).to(dev), 8, 2, fixed_start=fs)
    torch.cuda.synchronize()
    assert torch.equal(out.start_state, fs)
    clean("encode fixed start")
    out = tcq.encode(torch.randn(12, 256, device=dev), None, tcq.MAD, 16, 2)
    torch.cuda.synchronize()
    clean("encode computed code")

    # decoders: the compile-time kernel and the runtime one
    rng = np.random.default_rng(3)
    for (L, k, T, cbt) in [(16, 2, 256, "f16"), (12, 2, 256, "f32"), (5, 3, 10, "f16"), (16, 4, 255, "f32")]:
        n = 37
        W = tcq.tcq_words_per_block(k, T)
        bits = rng.integers(0, 2**32, size=(n, W), dtype=np.uint64).astype(np.uint32)
        used = T * k - 32 * (W - 1)
        if used < 32:
            bits[:, -1] &= np.uint32(((1 << used) - 1) << (32 - used))
        start = rng.integers(0, 2**32, size=n, dtype=np.uint64).astype(np.uint32)
        cb = rng.standard_normal(1 << L).astype(np.float16 if cbt == "f16" else np.float32)
        y = tcq.decode(torch.from_numpy(bits.view(np.int32)).to(dev), torch.from_numpy(start.view(np.int32)).to(dev),
                       torch.from_numpy(cb).to(dev), L, k, T)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(y.cpu().numpy(), oracle_decode(bits, start, cb, L, k, T).astype(np.float32))
        clean(f"decode L{L} k{k} T{T}")

    # matrix-vector products: half-block lanes (both phases), whole-row warps, the runtime kernel
    for (L, k, T, rows, nb, code) in [(16, 2, 256, 4801, 16, "f16"), (16, 2, 256, 300, 16, "mad"),
                                      (16, 3, 256, 40, 16, "f16"), (8, 2, 64, 33, 5, "f32")]:
        W = tcq.tcq_words_per_block(k, T)
        bits = rng.integers(0, 2**32, size=(rows * nb, W), dtype=np.uint64).astype(np.uint32)
        used = T * k - 32 * (W - 1)
        if used < 32:
            bits[:, -1] &= np.uint32(((1 << used) - 1) << (32 - used))
        start = rng.integers(0, 2**32, size=rows * nb, dtype=np.uint64).astype(np.uint32)
        cols = nb * T
        xv = rng.standard_normal(cols).astype(np.float32)
        if code == "mad":
            cb, cbt_ = oracle_mad_codebook(L).astype(np.float16), tcq.MAD
        else:
            cb = rng.standard_normal(1 << L).astype(np.float16 if code == "f16" else np.float32)
            cbt_ = torch.from_numpy(cb).to(dev)
        y = tcq.gemv(torch.from_numpy(bits.view(np.int32)).to(dev), torch.from_numpy(start.view(np.int32)).to(dev),
                     None, cbt_, L, k, T, rows, cols, torch.from_numpy(xv).to(dev))
        torch.cuda.synchronize()
        y_o = oracle_gemv(bits, start, None, cb, L, k, T, rows, cols, xv)
        vals = oracle_decode(bits, start, cb, L, k, T).reshape(rows, cols)
        bound = (13 + -(-cols // 256)) * 2.0**-24 * np.abs(vals * xv).sum(axis=1)
        assert np.all(np.abs(y.cpu().numpy().astype(np.float64) - y_o) <= bound + 1e-30)
        clean(f"gemv L{L} k{k} rows{rows} {code}")

    # the 8-state set-partitioned trellis
    for (V, m, T, n) in [(4, 7, 256, 40), (1, 2, 100, 33), (3, 8, 27, 9)]:
        xx = rng.standard_normal((n, T)).astype(np.float32)
        cbu = workloads.ub8_gaussian_codebook(V, m, "f32")
        out = tcq.ub8_encode(torch.from_numpy(xx).to(dev), None, torch.from_numpy(cbu).to(dev), V, m)
        yv = tcq.ub8_decode(out.bits, out.start_state, torch.from_numpy(cbu).to(dev), V, m, T)
        torch.cuda.synchronize()
        s = out.start_state.cpu().numpy().view(np.uint32)
        b = out.bits.cpu().numpy().view(np.uint32)
        np.testing.assert_array_equal(yv.cpu().numpy(), oracle_ub8_decode(b, s, cbu, V, m, T).astype(np.float32))
        clean(f"ub8 V{V} m{m} T{T}")

    # error feedback: the tensor-core product (T = 256), its bounded waits must not give up
    lw = workloads.ldlq_dyadic_exact(12, 2, 256, 130, 768, False, "f32", seed=9)
    res = tcq.ldlq(torch.from_numpy(lw.w).to(dev), torch.from_numpy(lw.u).to(dev), None,
                   torch.from_numpy(lw.codebook).to(dev), 12, 2, 256)
    torch.cuda.synchronize()
    q_o = oracle_ldlq(lw.w, lw.u, np.ones(lw.cols), lw.codebook, 12, 2, 256)[0]
    np.testing.assert_array_equal(res.q.cpu().numpy().astype(np.float64), q_o)
    clean("ldlq tensor-core feedback")
    print("DEBUG BUILD OK", flush=True)


if __name__ == "__main__":
    main()
