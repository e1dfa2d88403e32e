"""Benchmark: Viterbi TCQ encode (+ decode round trip) of the 14336x4096 MLP-shape
matrix at L=16, k=2, T=256 on B200, one process per GPU.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...

A step is one pass of the whole hot path over the workload: the encode
(add-compare-select forward pass, backpointers, traceback, bit packing and the
path cost, all inside the encoder kernel) and the decode of the result.  Inputs
(x and d: 470 MB) are larger than the 126 MB L2, so no flush is needed between
steps.  Each rank encodes its own matrix of that shape (weak scaling); there is
no data-path collective.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import multiprocessing as mp
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Viterbi trellis nodes/sec (blocks·T·2^L) and weights encoded/sec at L=16,k=2"
ALGO_OPS_PER_NODE = 3  # error, square-accumulate, compare-select
VEC_OPS_PER_NODE = 5   # V = 2: two errors, two square-accumulates, one compare-select
SMS, LANES_PER_SM = 148, 128
SFU_PER_SM = 16  # ex2 / lg2 results per SM per clock (4 per sub-partition)
BCJR_TAU = 0.1
REJECT_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")
ROOFLINE_SRC = ["trellis_coded_weight_tcq_b200/csrc/acs_grouped.cuh",
                "trellis_coded_weight_tcq_b200/csrc/acs_grouped.cu",
                "trellis_coded_weight_tcq_b200/csrc/common.cuh"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "acs_grouped_L16k2_traffic.json")


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "sm_max_mhz": 1965.0}, "fallback"


def _kernel_hash() -> str:
    h = hashlib.sha256()
    for p in ROOFLINE_SRC:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _traffic_per_launch(n_blocks: int):
    """DRAM bytes per launch from the committed ncu capture, scaled by blocks;
    null when the kernel source changed since the capture."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
    except OSError:
        return None
    if rec.get("kernel_sha256_16") != _kernel_hash():
        return None
    return rec["dram_bytes_per_block"] * n_blocks


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=10)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        rows = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v == "Active"})
        load = [r[0] for r in rows]
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": max(r[1] for r in rows),
                "samples": len(rows), "reasons": reasons}


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline only)
# ---------------------------------------------------------------------------
def _oracle_job(args):
    from oracle import oracle_encode

    x, d, cb, L, k = args
    t0 = time.perf_counter()
    oracle_encode(x, d, cb, L, k)
    return time.perf_counter() - t0


def time_oracle(pool, cores, wl, blocks_per_core: int):
    """Wall time of the oracle on cores x blocks_per_core blocks spread over the pool."""
    n = min(wl.n_blocks, cores * blocks_per_core)
    jobs = [(wl.x[i:i + 1], None if wl.d is None else wl.d[i:i + 1], wl.codebook, wl.L, wl.k)
            for i in range(n)]
    t0 = time.perf_counter()
    per_job = pool.map(_oracle_job, jobs, chunksize=max(1, blocks_per_core))
    wall = time.perf_counter() - t0
    return n, wall, float(sum(per_job))


def peaks_hbm() -> float:
    peaks, _ = _peaks()
    return float(peaks.get("hbm_gbs", 6650.0))


def peaks_ops() -> float:
    peaks, _ = _peaks()
    return SMS * LANES_PER_SM * float(peaks.get("sm_max_mhz", 1965.0)) * 1e6


def _median_ms(pairs):
    return statistics.median(a.elapsed_time(b) for a, b in pairs)


def _hold_gpu(stream=None, ms=5.0):
    """Keep the GPU busy for about `ms` before a loop of short event-timed calls:
    the host enqueues every call and event while it waits, and the GPU then runs
    them back to back, so each event pair times its kernel rather than the
    host's time per call (longer than a 20 us kernel)."""
    import torch

    cycles = int(ms * 1e-3 * 2.0e9)
    if stream is None:
        torch.cuda._sleep(cycles)
    else:
        with torch.cuda.stream(stream):
            torch.cuda._sleep(cycles)


def time_workload(name, dev, tcq, workloads, peak_ops, warmup=3, steps=10):
    """Encode and decode timing of one named workload: `warmup` untimed
    encode + decode passes, then the median of `steps` event-timed passes."""
    import torch

    wl = workloads.NAMED[name](0)
    x = torch.from_numpy(wl.x).to(dev)
    d = None if wl.d is None else torch.from_numpy(wl.d).to(dev)
    cb = torch.from_numpy(wl.codebook).to(dev)
    ws = tcq.Workspace(wl.L, wl.k, wl.T, wl.n_blocks, tcq.cb_dtype_of(cb), dev)
    out = tcq.encode(x, d, cb, wl.L, wl.k, ws)
    y = tcq.decode(out.bits, out.start_state, cb, wl.L, wl.k, wl.T)
    for _ in range(warmup):
        tcq.encode(x, d, cb, wl.L, wl.k, ws, out)
        tcq.decode(out.bits, out.start_state, cb, wl.L, wl.k, wl.T, y)
    _hold_gpu()
    enc, dec = [], []
    for _ in range(steps):
        a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        a.record()
        tcq.encode(x, d, cb, wl.L, wl.k, ws, out)
        b.record()
        tcq.decode(out.bits, out.start_state, cb, wl.L, wl.k, wl.T, y)
        c.record()
        enc.append((a, b))
        dec.append((b, c))
    torch.cuda.synchronize()
    e_ms = _median_ms(enc)
    d_ms = _median_ms(dec)
    return {"workload": wl.name, "nodes_per_s": wl.nodes / (e_ms / 1e3),
            "weights_per_s": wl.weights / (e_ms / 1e3), "encode_ms": e_ms, "decode_ms": d_ms,
            "timing": f"median of {steps} after {warmup} warm-ups",
            "alu_frac": wl.nodes * ALGO_OPS_PER_NODE / (e_ms / 1e3) / peak_ops,
            "kernel": tcq.tcq_encode_path(wl.L, wl.k, tcq.cb_dtype_of(cb))}


def run_only(args):
    """One leg of the hot path on seeded inputs of the workload's shape, for
    profiling and quick timing (--warmup untimed calls, the median of --steps
    timed ones): the matrix-vector
    product (both codes), the decoder, the 8-state trellis encode, or the
    error-feedback encode of the first rows of the MLP matrix.  Prints one
    JSON line; not the benchmark's result line."""
    import numpy as np
    import torch

    from trellis_coded_weight_tcq_b200 import tcq, workloads

    tcq.load_library()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    g = torch.Generator(device=dev).manual_seed(5)
    L, k, T = 16, 2, 256

    def med(fn):
        for _ in range(args.warmup):
            fn()
        _hold_gpu()
        ev = []
        for _ in range(max(1, args.steps)):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            ev.append((a, b))
        torch.cuda.synchronize()
        return _median_ms(ev)

    out = {"only": args.only}
    if args.only in ("gemv", "decode"):
        rows, cols = 14336, 4096  # the MLP matrix; the kernels do not depend on the bit values
        n = rows * cols // T
        bits = torch.randint(-2**31, 2**31 - 1, (n, 16), dtype=torch.int32, device=dev, generator=g)
        start = torch.randint(0, 1 << 14, (n,), dtype=torch.int32, device=dev, generator=g)
        cb = torch.from_numpy(workloads.gaussian_sample_codebook_f16(1 << L)).to(dev)
        if args.only == "gemv":
            x = torch.randn(cols, device=dev, generator=g)
            y = torch.empty(rows, device=dev)
            out["table_ms"] = med(lambda: tcq.gemv(bits, start, None, cb, L, k, T, rows, cols, x, y))
            out["computed_ms"] = med(lambda: tcq.gemv(bits, start, None, tcq.MAD, L, k, T, rows, cols, x, y))
        else:
            y = torch.empty((n, T), device=dev)
            out["decode_ms"] = med(lambda: tcq.decode(bits, start, cb, L, k, T, y))
            out["hbm_frac"] = (n * T * 4 + n * 64 + n * 4) / (out["decode_ms"] / 1e3) / 1e9 / peaks_hbm()
    elif args.only == "ub8":
        wl = workloads.mlp(0)
        nb = args.blocks or wl.n_blocks
        x = torch.from_numpy(np.ascontiguousarray(wl.x[:nb])).to(dev)
        d = torch.from_numpy(np.ascontiguousarray(wl.d[:nb])).to(dev)
        cb = torch.from_numpy(workloads.ub8_gaussian_codebook(4, 7, "f16")).to(dev)
        o = tcq.ub8_encode(x, d, cb, 4, 7)
        y = tcq.ub8_decode(o.bits, o.start_state, cb, 4, 7, T)
        out["blocks"] = nb
        out["encode_ms"] = med(lambda: tcq.ub8_encode(x, d, cb, 4, 7, out=o))
        out["decode_ms"] = med(lambda: tcq.ub8_decode(o.bits, o.start_state, cb, 4, 7, T, out=y))
    elif args.only == "ldlq":
        lw = workloads.ldlq_mlp()
        r = args.blocks // (lw.cols // lw.T) if args.blocks else lw.rows
        a = [torch.from_numpy(np.ascontiguousarray(v)).to(dev) for v in (lw.w[:r], lw.u, lw.d, lw.codebook)]
        out["rows"] = r
        out["ms"] = med(lambda: tcq.ldlq(*a, lw.L, lw.k, lw.T, keep_targets=False))
    print(json.dumps(out), flush=True)


def run_reference(args, rank, world):
    if rank != 0:
        return
    from oracle import build_oracle
    from trellis_coded_weight_tcq_b200 import workloads

    build_oracle()
    cores = os.cpu_count() or 1
    pool = mp.get_context("spawn").Pool(cores)
    wl = workloads.mlp(0)
    per_block = wl.T * (1 << wl.L)
    for _ in range(args.warmup):
        time_oracle(pool, cores, wl, 1)
    times, blocks = [], 0
    for _ in range(args.steps):
        n, wall, _busy = time_oracle(pool, cores, wl, 1)
        times.append(wall)
        blocks = n
    pool.close()
    ms = 1e3 * sum(times) / len(times)
    value = blocks * per_block / (ms / 1e3)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "nodes/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "L": wl.L, "k": wl.k, "T": wl.T, "n_blocks": wl.n_blocks},
        "weights_per_s": blocks * wl.T / (ms / 1e3),
        "cpu_baseline": {"value": value, "unit": "nodes/s", "cores": cores, "kind": "oracle",
                         "sample": f"{blocks} blocks of the workload per step, one block per "
                                   f"process, {cores} spawn processes"},
        "e2e": {"value": value, "unit": "nodes/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------
def run_ours(args, rank, world, local_rank):
    cores = os.cpu_count() or 1
    pool = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import build_oracle

        build_oracle()
        pool = mp.get_context("spawn").Pool(cores)  # started before any CUDA work

    import numpy as np
    import torch
    import torch.distributed as dist

    from trellis_coded_weight_tcq_b200 import tcq, workloads

    tcq.load_library()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev,
                                timeout=__import__("datetime").timedelta(seconds=300))

    from trellis_coded_weight_tcq_b200.dist import max_over_ranks, workload_for_rank

    wl = workload_for_rank(args.workload, rank)
    if args.blocks and args.blocks < wl.n_blocks:
        wl.x = np.ascontiguousarray(wl.x[:args.blocks])
        wl.d = None if wl.d is None else np.ascontiguousarray(wl.d[:args.blocks])
        wl.name += f"_first{args.blocks}blocks"
    L, k, T, n = wl.L, wl.k, wl.T, wl.n_blocks
    weighted = wl.d is not None
    x = torch.from_numpy(wl.x).to(dev)
    d = None if wl.d is None else torch.from_numpy(wl.d).to(dev)
    cb = torch.from_numpy(wl.codebook).to(dev)
    ws = tcq.Workspace(L, k, T, n, tcq.cb_dtype_of(cb), dev)
    W = tcq.tcq_words_per_block(k, T)
    out = tcq.Encoded(torch.empty(n, dtype=torch.int32, device=dev),
                      torch.empty((n, W), dtype=torch.int32, device=dev),
                      torch.empty(n, dtype=torch.float32, device=dev))
    y = torch.empty((n, T), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    enc_ev = []

    dec_ev = []

    def step(record=False):
        if record:
            a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            a.record(stream)
        tcq.encode(x, d, cb, L, k, ws, out)
        if record:
            b.record(stream)
            enc_ev.append((a, b))
        tcq.decode(out.bits, out.start_state, cb, L, k, T, y)
        if record:
            c.record(stream)
            dec_ev.append((b, c))

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    def timed_region():
        enc_ev.clear()
        dec_ev.clear()
        with ClockSampler(local_rank) as clk:
            t_start.record(stream)
            for _ in range(args.steps):
                step(record=True)
            t_end.record(stream)
            torch.cuda.synchronize()
        barrier()
        return clk.summary()

    # a region that saw a hardware or thermal slowdown is measured once more;
    # every rank takes the same decision (the max of the flags)
    clock_record = timed_region()
    throttled = bool(clock_record) and any(r in REJECT_REASONS for r in clock_record["reasons"])
    remeasured = None
    if max_over_ranks([1.0 if throttled else 0.0], dev)[0] > 0:
        remeasured = {"first_clocks": clock_record}
        clock_record = timed_region()
    ms = t_start.elapsed_time(t_end) / args.steps
    acs_ms = sum(a.elapsed_time(b) for a, b in enc_ev) / len(enc_ev)
    dec_ms = sum(a.elapsed_time(b) for a, b in dec_ev) / len(dec_ev)
    ms, acs_ms, dec_ms = max_over_ranks([ms, acs_ms, dec_ms], dev)
    cost_last = out.path_cost.cpu().numpy()
    # per step: the encoder, the L2 discard of its dead backpointers, the decoder
    gpu_launches = 3 * args.steps

    # ---- decode-in-matvec on the encoded matrix (one row of the matrix per
    # block row: rows = blocks * T / cols)
    gemv = None
    mat = wl.meta.get("matrix")
    if mat and rank == 0 and (n * T) % int(mat[1]) == 0:
        # the rows the encoded blocks cover (all of the matrix unless --blocks cut it)
        cols_m = int(mat[1])
        rows_m = n * T // cols_m
        xv = torch.randn(cols_m, device=dev)
        scale = torch.ones(n, device=dev)
        ym = torch.empty(rows_m, device=dev)
        for _ in range(3):
            tcq.gemv(out.bits, out.start_state, scale, cb, L, k, T, rows_m, cols_m, xv, ym)
        _hold_gpu(stream)
        g_ev = []
        for _ in range(10):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            tcq.gemv(out.bits, out.start_state, scale, cb, L, k, T, rows_m, cols_m, xv, ym)
            b.record(stream)
            g_ev.append((a, b))
        torch.cuda.synchronize()
        g_ms = _median_ms(g_ev)
        g_bytes = n * W * 4 + n * 4 + n * 4 + cols_m * 4 + rows_m * 4
        peaks_g, _ = _peaks()
        # the table code is bound by shared memory, not HBM: one table lookup per
        # weight against one 32-lane wavefront per SM and clock (conflict-free);
        # 32 random 2-byte lookups over 32 banks cost about 3.5 wavefronts, so
        # about 1 / 3.5 of this peak is the floor of a random table
        smem_peak = SMS * 32 * float(peaks_g.get("sm_max_mhz", 1965.0)) * 1e6
        lookups_per_s = rows_m * cols_m / (g_ms / 1e3)
        gemv = {"rows": rows_m, "cols": cols_m, "ms": g_ms,
                "weights_per_s": rows_m * cols_m / (g_ms / 1e3),
                "hbm_gbs": g_bytes / (g_ms / 1e3) / 1e9,
                "hbm_frac": g_bytes / (g_ms / 1e3) / 1e9 / float(peaks_g.get("hbm_gbs", 6650.0)),
                "bytes": g_bytes,
                "bound": "smem", "lookups_per_s": lookups_per_s,
                "smem_frac": lookups_per_s / smem_peak,
                "smem_peak_basis": f"{SMS} SMs x 32 lookups per clock (one conflict-free wavefront) x "
                                   f"{peaks_g.get('sm_max_mhz', 1965.0)} MHz; random lookups cost about "
                                   "3.5 wavefronts, so the attainable fraction is about 0.29"}
        # the same bitstreams read as the computed (lookup-free) code: no table,
        # each codeword computed in registers
        for _ in range(3):
            tcq.gemv(out.bits, out.start_state, scale, tcq.MAD, L, k, T, rows_m, cols_m, xv, ym)
        _hold_gpu(stream)
        m_ev = []
        for _ in range(10):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            tcq.gemv(out.bits, out.start_state, scale, tcq.MAD, L, k, T, rows_m, cols_m, xv, ym)
            b.record(stream)
            m_ev.append((a, b))
        torch.cuda.synchronize()
        m_ms = _median_ms(m_ev)
        # issue-bound: about 6 instructions per weight at best (state, multiply,
        # byte sum, float, FMA) against 148 SMs x 128 lanes x the max clock
        issue_peak = SMS * LANES_PER_SM * float(peaks_g.get("sm_max_mhz", 1965.0)) * 1e6
        gemv["computed_code"] = {
            "ms": m_ms, "weights_per_s": rows_m * cols_m / (m_ms / 1e3),
            "hbm_gbs": g_bytes / (m_ms / 1e3) / 1e9,
            "bound": "alu", "ops_per_weight": 6,
            "frac": rows_m * cols_m * 6 / (m_ms / 1e3) / issue_peak}

    # ---- the same encode from fixed start states (one per block, seeded), the
    # separate fixed-start instantiation of the encoder
    fixed = None
    if rank == 0 and world == 1 and not args.no_fixed:
        starts = torch.randint(0, 1 << (L - k), (n,), dtype=torch.int32, device=dev,
                               generator=torch.Generator(device=dev).manual_seed(11))
        tcq.encode(x, d, cb, L, k, ws, out, fixed_start=starts)
        f_ev = []
        for _ in range(2):
            a, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            tcq.encode(x, d, cb, L, k, ws, out, fixed_start=starts)
            b2.record(stream)
            f_ev.append((a, b2))
        torch.cuda.synchronize()
        f_ms = sum(a.elapsed_time(b2) for a, b2 in f_ev) / len(f_ev)
        assert bool(torch.equal(out.start_state, starts))
        fixed = {"workload": wl.name + "_fixed_start", "ms": f_ms, "nodes_per_s": wl.nodes / (f_ms / 1e3),
                 "alu_frac": wl.nodes * ALGO_OPS_PER_NODE / (f_ms / 1e3) / peaks_ops(),
                 "cost_per_weight": float(out.path_cost.double().sum()) / wl.weights}
        del starts

    # ---- end to end through the C ABI from pinned host buffers
    e2e = None
    if not args.no_e2e:
        pipe = tcq.HostPipeline(n, T, L, k, d is not None, torch.from_numpy(wl.codebook), dev)
        x_h = torch.from_numpy(wl.x).pin_memory()
        d_h = None if wl.d is None else torch.from_numpy(wl.d).pin_memory()
        for _ in range(args.warmup):
            pipe.run(x_h, d_h)
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            pipe.run(x_h, d_h)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks([e0.elapsed_time(e1) / args.steps], dev)[0]
        e2e = {"value": world * wl.nodes / (e2e_ms / 1e3), "unit": "nodes/s",
               "ms_per_step": e2e_ms, "h2d_bytes_per_step": pipe.h2d_bytes(),
               "d2h_bytes_per_step": pipe.d2h_bytes()}
        del pipe

    # ---- the other named workloads: encode + decode throughput, short runs
    per_workload = []
    if rank == 0 and world == 1 and not args.no_per_workload:
        del x, d, y, ws, out
        torch.cuda.empty_cache()
        for name in [n for n in ("tiny", "l12", "qtip", "heavy", "mlp") if n != args.workload]:
            per_workload.append(time_workload(name, dev, tcq, workloads, peaks_ops()))
        per_workload.append({"workload": wl.name, "nodes_per_s": wl.nodes / (acs_ms / 1e3),
                             "weights_per_s": wl.weights / (acs_ms / 1e3), "encode_ms": acs_ms,
                             "decode_ms": dec_ms,
                             "alu_frac": wl.nodes * ALGO_OPS_PER_NODE / (acs_ms / 1e3) / peaks_ops(),
                             "kernel": tcq.tcq_encode_path(L, k, tcq.cb_dtype_of(cb))})

    # ---- error-feedback (LDLQ) encode of the MLP matrix: 16 column blocks, each
    # a feedback product, an encode of 14336 blocks and a decode
    ldlq = None
    if rank == 0 and world == 1 and not args.no_ldlq:
        torch.cuda.empty_cache()
        lw = workloads.ldlq_mlp()
        w_t = torch.from_numpy(lw.w).to(dev)
        u_t = torch.from_numpy(lw.u).to(dev)
        d_t = torch.from_numpy(lw.d).to(dev)
        cb_t = torch.from_numpy(lw.codebook).to(dev)
        lws = torch.empty(tcq.tcq_ldlq_workspace_bytes(lw.L, lw.k, lw.T, lw.rows, lw.cols,
                                                       tcq.cb_dtype_of(cb_t)),
                          dtype=torch.uint8, device=dev)
        tcq.ldlq(w_t, u_t, d_t, cb_t, lw.L, lw.k, lw.T, keep_targets=False, workspace=lws)
        l_ev = []
        for _ in range(2):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            res = tcq.ldlq(w_t, u_t, d_t, cb_t, lw.L, lw.k, lw.T, keep_targets=False, workspace=lws)
            b.record(stream)
            l_ev.append((a, b))
        torch.cuda.synchronize()
        l_ms = sum(a.elapsed_time(b) for a, b in l_ev) / len(l_ev)
        costs = res.coded.path_cost.cpu().numpy()
        assert np.all(np.isfinite(costs)) and np.all(costs >= 0)
        nbc = lw.cols // lw.T
        ldlq = {"workload": lw.name, "ms": l_ms, "nodes_per_s": lw.nodes / (l_ms / 1e3),
                "weights_per_s": lw.rows * lw.cols / (l_ms / 1e3),
                "feedback_flops": lw.rows * lw.T * lw.T * nbc * (nbc - 1),
                "launches_per_call": 3 * nbc,
                "alu_frac": lw.nodes * ALGO_OPS_PER_NODE / (l_ms / 1e3) / peaks_ops(),
                "proxy_loss_per_weight": float(costs.astype(np.float64).sum()) / (lw.rows * lw.cols)}
        del w_t, u_t, d_t, lws, res

    # ---- soft forward-backward quantization of the same blocks at tau = 0.1
    bcjr = None
    if rank == 0 and world == 1 and not args.no_bcjr:
        torch.cuda.empty_cache()
        xb_t = torch.from_numpy(wl.x).to(dev)
        db_t = None if wl.d is None else torch.from_numpy(wl.d).to(dev)
        bws = torch.empty(tcq.tcq_bcjr_workspace_bytes(L, k, T, n, tcq.cb_dtype_of(cb)),
                          dtype=torch.uint8, device=dev)
        yb = torch.empty((n, T), dtype=torch.float32, device=dev)
        fb = torch.empty(n, dtype=torch.float32, device=dev)
        tcq.bcjr(xb_t, db_t, cb, L, k, BCJR_TAU, workspace=bws, out=(yb, fb))
        a, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        tcq.bcjr(xb_t, db_t, cb, L, k, BCJR_TAU, workspace=bws, out=(yb, fb))
        b2.record(stream)
        torch.cuda.synchronize()
        b_ms = a.elapsed_time(b2)
        fe = fb.cpu().numpy()
        assert np.all(np.isfinite(fe)) and bool(torch.isfinite(yb).all())
        peaks_b, kind_b = _peaks()
        sfu_peak = SMS * SFU_PER_SM * float(peaks_b.get("sm_max_mhz", 1965.0)) * 1e6
        # ex2/lg2 per node: forward (H-1)/H ex2 + 1/H lg2 for the register-resident
        # kernel at k = 2 (the maximum's term is 1), H/H ex2 + 1/H lg2 otherwise;
        # backward 1 ex2 + 1/H lg2 + 1/H ex2 (the posterior weight)
        H = 1 << k
        fwd = 1.0 if (L == 16 and k == 2 and cb.dtype == torch.float16 and T <= 1024) else 1.0 + 1.0 / H
        sfu_per_node = fwd + 1.0 + 2.0 / H
        sfu_ops = wl.nodes * sfu_per_node
        bcjr = {"workload": wl.name, "tau": BCJR_TAU, "ms": b_ms,
                "nodes_per_s": wl.nodes / (b_ms / 1e3), "weights_per_s": wl.weights / (b_ms / 1e3),
                "bound": "sfu", "sfu_ops_per_node": sfu_per_node,
                "achieved": sfu_ops / (b_ms / 1e3) / 1e12, "peak": sfu_peak / 1e12, "unit": "TOP/s",
                "frac": sfu_ops / (b_ms / 1e3) / sfu_peak,
                "peak_basis": f"{SMS} SMs x {SFU_PER_SM} ex2/lg2 per clock x "
                              f"{peaks_b.get('sm_max_mhz', 1965.0)} MHz ({kind_b} max SM clock)",
                "free_energy_mean": float(fe.astype(np.float64).mean())}
        del xb_t, db_t, bws, yb, fb

    # ---- the vector trellis (V = 2 weights per step, 4 bits shifted in per step)
    # over the same blocks, with a binary16 codebook of 2^16 pairs
    vec = None
    if rank == 0 and world == 1 and not args.no_vec and L == 16 and k == 2:
        torch.cuda.empty_cache()
        V = 2
        xv_t = torch.from_numpy(wl.x).to(dev)
        dv_t = None if wl.d is None else torch.from_numpy(wl.d).to(dev)
        cbv = torch.from_numpy(workloads.gaussian_sample_codebook_f16((1 << L) * V)).to(dev)
        vws = torch.empty(tcq.tcq_encode_vec_workspace_bytes(L, k, V, T, n, tcq.TCQ_F16),
                          dtype=torch.uint8, device=dev)
        vout = tcq.Encoded(torch.empty(n, dtype=torch.int32, device=dev),
                           torch.empty((n, tcq.tcq_words_per_block(k, T)), dtype=torch.int32, device=dev),
                           torch.empty(n, dtype=torch.float32, device=dev))
        tcq.encode_vec(xv_t, dv_t, cbv, L, k, V, workspace=vws, out=vout)
        v_ev = []
        for _ in range(2):
            a, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            tcq.encode_vec(xv_t, dv_t, cbv, L, k, V, workspace=vws, out=vout)
            b2.record(stream)
            v_ev.append((a, b2))
        torch.cuda.synchronize()
        v_ms = sum(a.elapsed_time(b2) for a, b2 in v_ev) / len(v_ev)
        vcost = vout.path_cost.cpu().numpy()
        assert np.all(np.isfinite(vcost)) and np.all(vcost >= 0)
        v_nodes = n * (T // V) * (1 << L)
        # decode of the V = 2 stream: reads k/8 B and writes 4 B per weight
        yv = tcq.decode_vec(vout.bits, vout.start_state, cbv, L, k, V, T)
        _hold_gpu(stream)
        vd_ev = []
        for _ in range(3):
            a, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            tcq.decode_vec(vout.bits, vout.start_state, cbv, L, k, V, T, out=yv)
            b2.record(stream)
            vd_ev.append((a, b2))
        torch.cuda.synchronize()
        vd_ms = sum(a.elapsed_time(b2) for a, b2 in vd_ev) / len(vd_ev)
        vd_bytes = n * T * 4 + n * tcq.tcq_words_per_block(k, T) * 4 + n * 4
        del yv
        # decode-in-matvec over the matrix those blocks tile (rows x cols), timed
        # like the scalar product above (unit block scales, median of 10)
        vgemv = None
        vmat = wl.meta.get("matrix")
        if vmat and (n * T) % int(vmat[1]) == 0:
            g_cols = int(vmat[1])
            g_rows = n * T // g_cols
            xg = torch.randn(g_cols, device=dev)
            sg = torch.ones(n, device=dev)
            yg = torch.empty(g_rows, device=dev)
            for _ in range(3):
                tcq.gemv_vec(vout.bits, vout.start_state, sg, cbv, L, k, V, T, g_rows, g_cols, xg, out=yg)
            _hold_gpu(stream)
            vg_ev = []
            for _ in range(10):
                a, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                tcq.gemv_vec(vout.bits, vout.start_state, sg, cbv, L, k, V, T, g_rows, g_cols, xg, out=yg)
                b2.record(stream)
                vg_ev.append((a, b2))
            torch.cuda.synchronize()
            vg_ms = _median_ms(vg_ev)
            vg_bytes = n * tcq.tcq_words_per_block(k, T) * 4 + n * 8 + g_cols * 4 + g_rows * 4
            assert bool(torch.isfinite(yg).all())
            vgemv = {"rows": g_rows, "cols": g_cols, "ms": vg_ms,
                     "weights_per_s": g_rows * g_cols / (vg_ms / 1e3),
                     "hbm_gbs": vg_bytes / (vg_ms / 1e3) / 1e9,
                     "hbm_frac": vg_bytes / (vg_ms / 1e3) / 1e9 / peaks_hbm()}
            del xg, yg, sg
        vec = {"workload": wl.name + "_V2", "V": V, "ms": v_ms, "nodes_per_s": v_nodes / (v_ms / 1e3),
               "weights_per_s": n * T / (v_ms / 1e3), "ops_per_node": VEC_OPS_PER_NODE,
               "alu_frac": v_nodes * VEC_OPS_PER_NODE / (v_ms / 1e3) / peaks_ops(),
               "kernel": "vec2<16,2,f16x2,512>",
               "decode_ms": vd_ms, "decode_hbm_frac": vd_bytes / (vd_ms / 1e3) / 1e9 / peaks_hbm(),
               "gemv": vgemv,
               "cost_per_weight": float(vcost.astype(np.float64).sum()) / (n * T)}
        del xv_t, dv_t, vws, vout

    # ---- Ungerboeck's 8-state set-partitioned trellis over the same blocks:
    # symbols of V = 4 weights, 1 + m = 8 bits per step (2 bits per weight),
    # a Gaussian binary16 union codebook of 512 rows in four subsets
    ub8 = None
    if rank == 0 and world == 1 and not args.no_ub8:
        torch.cuda.empty_cache()
        V8, m8 = 4, 7
        xu = torch.from_numpy(wl.x).to(dev)
        du = None if wl.d is None else torch.from_numpy(wl.d).to(dev)
        cbu = torch.from_numpy(workloads.ub8_gaussian_codebook(V8, m8, "f16")).to(dev)
        uout = tcq.ub8_encode(xu, du, cbu, V8, m8)
        yu = tcq.ub8_decode(uout.bits, uout.start_state, cbu, V8, m8, T)
        for _ in range(3):
            tcq.ub8_encode(xu, du, cbu, V8, m8, out=uout)
            tcq.ub8_decode(uout.bits, uout.start_state, cbu, V8, m8, T, out=yu)
        ue, ud = [], []
        for _ in range(10):
            a, b2, c2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            a.record(stream)
            tcq.ub8_encode(xu, du, cbu, V8, m8, out=uout)
            b2.record(stream)
            tcq.ub8_decode(uout.bits, uout.start_state, cbu, V8, m8, T, out=yu)
            c2.record(stream)
            ue.append((a, b2))
            ud.append((b2, c2))
        torch.cuda.synchronize()
        u_ms, ud_ms = _median_ms(ue), _median_ms(ud)
        ucost = uout.path_cost.cpu().numpy()
        assert np.all(np.isfinite(ucost)) and np.all(ucost >= 0)
        steps = n * (T // V8)
        cands = steps * (4 << m8)  # every row of the union scored at every step
        u_ops = cands * (2 * V8 + 1)  # V errors, V square-accumulates, one compare-select
        Wu = tcq.tcq_ub8_words_per_block(V8, m8, T)
        ud_bytes = n * T * 4 + n * Wu * 4 + n * 4
        ub8 = {"workload": wl.name + "_ub8_V4_m7", "V": V8, "m": m8, "bits_per_weight": (1 + m8) / V8,
               "timing": "median of 10 after 3 warm-ups",
               "ms": u_ms, "weights_per_s": n * T / (u_ms / 1e3),
               "candidates_per_s": cands / (u_ms / 1e3), "ops_per_candidate": 2 * V8 + 1,
               "bound": "alu", "alu_frac": u_ops / (u_ms / 1e3) / peaks_ops(),
               "decode_ms": ud_ms, "decode_hbm_frac": ud_bytes / (ud_ms / 1e3) / 1e9 / peaks_hbm(),
               "cost_per_weight": float(ucost.astype(np.float64).sum()) / (n * T)}
        del xu, du, cbu, uout, yu

    # sanity: the last step's result is a valid encode of the workload (cheap host check)
    cost_h = cost_last
    assert np.all(np.isfinite(cost_h)) and np.all(cost_h >= 0)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks, peak_kind = _peaks()
    peak_ops = SMS * LANES_PER_SM * float(peaks.get("sm_max_mhz", 1965.0)) * 1e6
    achieved_ops = wl.nodes * ALGO_OPS_PER_NODE / (acs_ms / 1e3)
    roofline = {
        "bound": "alu", "kernel": tcq.tcq_encode_path(L, k, tcq.cb_dtype_of(cb)),
        "achieved": achieved_ops / 1e12, "peak": peak_ops / 1e12, "unit": "TOP/s",
        "frac": achieved_ops / peak_ops,
        "traffic": _traffic_per_launch(n),
        "peak_basis": f"{SMS} SMs x {LANES_PER_SM} lanes x {peaks.get('sm_max_mhz', 1965.0)} MHz "
                      f"({peak_kind} max SM clock); {ALGO_OPS_PER_NODE} ops per trellis node",
        "acs_ms_per_launch": acs_ms,
    }
    # the decoder, HBM bound: y written (4 B per weight), bits and start states read
    dec_bytes = wl.weights * 4 + n * W * 4 + n * 4
    decode_roofline = {
        "bound": "hbm", "kernel": "decode_kernel", "ms_per_launch": dec_ms,
        "achieved": dec_bytes / (dec_ms / 1e3) / 1e9, "peak": float(peaks.get("hbm_gbs", 6650.0)),
        "unit": "GB/s", "frac": dec_bytes / (dec_ms / 1e3) / 1e9 / float(peaks.get("hbm_gbs", 6650.0)),
        "bytes_per_launch": dec_bytes, "weights_per_s": wl.weights / (dec_ms / 1e3),
    }
    cpu_baseline = None
    if pool is not None:
        nb, wall, busy = time_oracle(pool, cores, wl, args.cpu_blocks_per_core)
        pool.close()
        v = nb * T * (1 << L) / wall
        cpu_baseline = {"value": v, "unit": "nodes/s", "cores": cores, "kind": "oracle",
                        "one_core_value": nb * T * (1 << L) / busy,
                        "sample": f"{nb} blocks of {wl.name}, {args.cpu_blocks_per_core} per "
                                  f"process on {cores} spawn processes, {wall:.1f} s wall, "
                                  f"{busy:.1f} s of single-threaded oracle time"}
    line = {
        "metric": METRIC, "value": world * wl.nodes / (ms / 1e3), "unit": "nodes/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": wl.name, "L": L, "k": k, "T": T, "n_blocks": n,
                   "codebook": str(wl.codebook.dtype), "weighted": weighted,
                   "l2": "inputs larger than L2 (x and d are 470 MB per GPU), no flush",
                   "parallelism": f"blocks sharded per GPU (dp{world})"},
        "weights_per_s": world * wl.weights / (ms / 1e3),
        "encode_ms_per_step": acs_ms, "decode_ms_per_step": dec_ms,
        "roofline": roofline, "decode_roofline": decode_roofline, "cpu_baseline": cpu_baseline, "e2e": e2e,
        "per_workload": per_workload, "gemv": gemv, "ldlq": ldlq, "bcjr": bcjr, "vec": vec, "fixed_start": fixed,
        "ub8": ub8,
        "clocks": clock_record, "remeasured": remeasured, "gpu_launches": gpu_launches,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["mlp", "qtip", "heavy", "l12", "tiny"], default="mlp")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="skip the short encode/decode timing of the other named workloads")
    ap.add_argument("--no-bcjr", action="store_true",
                    help="skip the soft forward-backward quantization of the workload")
    ap.add_argument("--no-fixed", action="store_true",
                    help="skip the fixed-start encode of the workload")
    ap.add_argument("--no-vec", action="store_true",
                    help="skip the vector-trellis (V = 2) encode of the workload")
    ap.add_argument("--no-ub8", action="store_true",
                    help="skip the 8-state set-partitioned trellis encode of the workload")
    ap.add_argument("--no-ldlq", action="store_true",
                    help="skip the error-feedback encode of the MLP matrix")
    ap.add_argument("--cpu-blocks-per-core", type=int, default=16)
    ap.add_argument("--only", choices=["gemv", "decode", "ub8", "ldlq"], default=None,
                    help="run one leg on seeded inputs of the workload's shape and print its "
                         "timing (profiling); not the benchmark line")
    ap.add_argument("--blocks", type=int, default=0,
                    help="encode only the first N blocks of the workload (a smaller profiling "
                         "case; reported in config.n_blocks)")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.only:
        run_only(args)
    elif args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
