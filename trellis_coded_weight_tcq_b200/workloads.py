"""Seeded synthetic inputs for the encoder: the five named workloads and small cases.

This module only draws and shapes inputs (random weights, curvature weights d,
codebooks); it holds none of the quantiser's arithmetic, and both the CUDA path
and the CPU oracle are fed from it.

Seeds: x = 1000, d = 1001, codebook = 1002, permutation = 1003 (plus an offset
per shard when several ranks each take their own matrix).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
from scipy.special import ndtri

SEED_X, SEED_D, SEED_CB, SEED_PERM = 1000, 1001, 1002, 1003


@dataclass
class Workload:
    name: str
    L: int
    k: int
    T: int
    x: np.ndarray                 # float32 [n_blocks, T]
    d: np.ndarray | None          # float32 [n_blocks, T] or None (d = 1)
    codebook: np.ndarray          # float32 or float16 [2^L]
    meta: dict = field(default_factory=dict)

    @property
    def n_blocks(self) -> int:
        return self.x.shape[0]

    @property
    def nodes(self) -> int:
        """Trellis nodes of one encode: n_blocks * T * 2^L."""
        return self.n_blocks * self.T * (1 << self.L)

    @property
    def weights(self) -> int:
        return self.n_blocks * self.T


def gaussian_quantile_codebook(n: int, seed_perm: int = SEED_PERM) -> np.ndarray:
    """c_i = Phi^-1((i + 1/2) / n) in float64, rounded to float32, seed-permuted."""
    q = ndtri((np.arange(n, dtype=np.float64) + 0.5) / n).astype(np.float32)
    perm = np.random.default_rng(seed_perm).permutation(n)
    return q[perm]


def gaussian_sample_codebook_f16(n: int, seed: int = SEED_CB) -> np.ndarray:
    """n draws of N(0, 1), rounded to binary16."""
    return np.random.default_rng(seed).standard_normal(n).astype(np.float16)


def _bf16_round(a: np.ndarray) -> np.ndarray:
    """Round float32 to the nearest bfloat16 (ties to even), returned as float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def _matrix_blocks(W: np.ndarray, T: int) -> np.ndarray:
    """Blocks of T consecutive columns along each row, each scaled to unit RMS."""
    blocks = W.reshape(-1, T).astype(np.float32)
    rms = np.sqrt(np.mean(blocks.astype(np.float64) ** 2, axis=1, keepdims=True))
    rms[rms == 0] = 1.0
    return (blocks / rms).astype(np.float32)


def tiny(shard: int = 0) -> Workload:
    """L=8, k=2, T=64, 256 blocks; x ~ N(0,1); d = 1; 256 fp32 Gaussian quantiles, permuted."""
    rng = np.random.default_rng(SEED_X + 7919 * shard)
    x = rng.standard_normal((256, 64)).astype(np.float32)
    return Workload("tiny_L8_k2_T64_B256", 8, 2, 64, x, None, gaussian_quantile_codebook(256),
                    {"shape": "256 blocks x 64"})


def l12(shard: int = 0) -> Workload:
    """L=12, k=2, T=256, 4096 blocks; x ~ N(0,1); d ~ LogNormal(0,1) per element."""
    x = np.random.default_rng(SEED_X + 7919 * shard).standard_normal((4096, 256)).astype(np.float32)
    d = np.random.default_rng(SEED_D + 7919 * shard).lognormal(0.0, 1.0, (4096, 256)).astype(np.float32)
    return Workload("L12_k2_T256_B4096_weighted", 12, 2, 256, x, d, gaussian_quantile_codebook(4096),
                    {"shape": "4096 blocks x 256"})


def _weight_matrix_gaussian(rows: int, cols: int, seed: int) -> np.ndarray:
    return _bf16_round(np.random.default_rng(seed).standard_normal((rows, cols)).astype(np.float32) * 0.02)


def qtip(shard: int = 0) -> Workload:
    """4096x4096 N(0, 0.02^2) bf16 matrix, unit-RMS blocks of 256; L=16, k=2; d = 1; fp16 codebook."""
    W = _weight_matrix_gaussian(4096, 4096, SEED_X + 7919 * shard)
    return Workload("qtip_4096x4096_L16_k2_T256", 16, 2, 256, _matrix_blocks(W, 256), None,
                    gaussian_sample_codebook_f16(1 << 16), {"matrix": [4096, 4096]})


def heavy(shard: int = 0) -> Workload:
    """4096x4096 Student-t(4) scaled to RMS 0.02, bf16; L=16, k=3; d per column ~ LogNormal(0,1.5)."""
    rng = np.random.default_rng(SEED_X + 7919 * shard)
    t = rng.standard_t(4.0, (4096, 4096)).astype(np.float32)
    W = _bf16_round(t * np.float32(0.02 / np.sqrt(2.0)))  # Var t_4 = 2
    d_col = np.random.default_rng(SEED_D + 7919 * shard).lognormal(0.0, 1.5, 4096).astype(np.float32)
    d = np.ascontiguousarray(np.broadcast_to(d_col[None, :], (4096, 4096))).reshape(-1, 256)
    return Workload("heavy_t4_4096x4096_L16_k3_T256_weighted", 16, 3, 256, _matrix_blocks(W, 256), d,
                    gaussian_sample_codebook_f16(1 << 16), {"matrix": [4096, 4096]})


def mlp(shard: int = 0) -> Workload:
    """14336x4096 N(0, 0.02^2) bf16, T=256 blocks (229,376); L=16, k=2; d per column ~ LogNormal(0,1)."""
    W = _weight_matrix_gaussian(14336, 4096, SEED_X + 7919 * shard)
    d_col = np.random.default_rng(SEED_D + 7919 * shard).lognormal(0.0, 1.0, 4096).astype(np.float32)
    d = np.ascontiguousarray(np.broadcast_to(d_col[None, :], (14336, 4096))).reshape(-1, 256)
    return Workload("mlp_14336x4096_L16_k2_T256_weighted", 16, 2, 256, _matrix_blocks(W, 256), d,
                    gaussian_sample_codebook_f16(1 << 16), {"matrix": [14336, 4096]})


NAMED = {"tiny": tiny, "l12": l12, "qtip": qtip, "heavy": heavy, "mlp": mlp}


def small_random(L: int, k: int, T: int, n_blocks: int, weighted: bool, cb_dtype: str,
                 seed: int) -> Workload:
    """A small seeded case: x ~ N(0,1), d ~ LogNormal(0,1), codebook N(0,1) in fp32 or fp16."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n_blocks, T)).astype(np.float32)
    d = rng.lognormal(0.0, 1.0, (n_blocks, T)).astype(np.float32) if weighted else None
    cb = rng.standard_normal(1 << L)
    cb = cb.astype(np.float16) if cb_dtype == "f16" else cb.astype(np.float32)
    return Workload(f"rand_L{L}_k{k}_T{T}_B{n_blocks}", L, k, T, x, d, cb)


def dyadic_exact(L: int, k: int, T: int, n_blocks: int, weighted: bool, cb_dtype: str,
                 seed: int) -> Workload:
    """Values on a coarse dyadic grid so that every fp32 operation of the search is exact.

    Codewords and x are multiples of 1/8 in [-2, 2] (exact in fp16 too), d is in
    {1/4, 1, 4} so that sqrt(d) is a power of two as well.  A branch metric is
    then a multiple of 1/256 below 64, and for T <= 1024 every partial path
    cost fits the 24-bit significand exactly.
    """
    assert T <= 1024
    rng = np.random.default_rng(seed)
    cb = (rng.integers(-16, 17, 1 << L) / 8.0)
    cb = cb.astype(np.float16) if cb_dtype == "f16" else cb.astype(np.float32)
    x = (rng.integers(-16, 17, (n_blocks, T)) / 8.0).astype(np.float32)
    d = (4.0 ** rng.integers(-1, 2, (n_blocks, T))).astype(np.float32) if weighted else None
    return Workload(f"dyadic_L{L}_k{k}_T{T}_B{n_blocks}", L, k, T, x, d, cb)


@dataclass
class LdlqWorkload:
    """A matrix for the error-feedback encode, with the factor of its Hessian.

    H = U diag(d) U^T is implied by (u, d): u is unit upper triangular, so H is
    symmetric positive definite whenever d > 0.
    """
    name: str
    L: int
    k: int
    T: int
    w: np.ndarray                 # float32 [rows, cols]
    u: np.ndarray                 # float32 [cols, cols], unit upper triangular
    d: np.ndarray | None          # float32 [cols] or None (d = 1)
    codebook: np.ndarray          # float32 or float16 [2^L]
    meta: dict = field(default_factory=dict)

    @property
    def rows(self) -> int:
        return self.w.shape[0]

    @property
    def cols(self) -> int:
        return self.w.shape[1]

    @property
    def n_blocks(self) -> int:
        return self.rows * (self.cols // self.T)

    @property
    def nodes(self) -> int:
        return self.n_blocks * self.T * (1 << self.L)


def unit_upper_factor(cols: int, T: int, rho: float, seed: int, block_free: bool = False) -> np.ndarray:
    """I plus strictly upper entries ~ N(0, rho^2 / cols); with ``block_free`` the
    entries inside the T x T diagonal blocks are zero as well."""
    rng = np.random.default_rng(seed)
    u = np.triu(rng.standard_normal((cols, cols)).astype(np.float32) * np.float32(rho / np.sqrt(cols)), 1)
    if block_free:
        for j in range(cols // T):
            u[j * T:(j + 1) * T, j * T:(j + 1) * T] = 0.0
    u[np.arange(cols), np.arange(cols)] = 1.0
    return u


def ldlq_random(L: int, k: int, T: int, rows: int, cols: int, weighted: bool, cb_dtype: str,
                seed: int, rho: float = 0.5, block_free: bool = False) -> LdlqWorkload:
    """A small seeded case: w ~ N(0,1); U as unit_upper_factor; d ~ LogNormal(0,1)
    per column; codebook N(0,1) in fp32 or fp16."""
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((rows, cols)).astype(np.float32)
    d = rng.lognormal(0.0, 1.0, cols).astype(np.float32) if weighted else None
    cb = rng.standard_normal(1 << L)
    cb = cb.astype(np.float16) if cb_dtype == "f16" else cb.astype(np.float32)
    u = unit_upper_factor(cols, T, rho, seed + 1, block_free)
    tag = "_blockfree" if block_free else ""
    return LdlqWorkload(f"ldlq_L{L}_k{k}_T{T}_{rows}x{cols}{tag}", L, k, T, w, u, d, cb)


def ldlq_mlp(shard: int = 0) -> LdlqWorkload:
    """The MLP matrix (14336x4096 N(0, 0.02^2), bf16) divided by 0.02, with
    U = I + N(0, 0.25/4096) strictly upper and d ~ LogNormal(0,1) per column;
    L=16, k=2, T=256; fp16 N(0,1) codebook."""
    W = _weight_matrix_gaussian(14336, 4096, SEED_X + 7919 * shard) / np.float32(0.02)
    d = np.random.default_rng(SEED_D + 7919 * shard).lognormal(0.0, 1.0, 4096).astype(np.float32)
    u = unit_upper_factor(4096, 256, 0.5, SEED_PERM + 1 + 7919 * shard)
    return LdlqWorkload("ldlq_mlp_14336x4096_L16_k2_T256_weighted", 16, 2, 256, W.astype(np.float32),
                        u, d, gaussian_sample_codebook_f16(1 << 16), {"matrix": [14336, 4096]})


def ldlq_dyadic_exact(L: int, k: int, T: int, rows: int, cols: int, weighted: bool,
                      cb_dtype: str, seed: int) -> LdlqWorkload:
    """An error-feedback case on which every fp32 operation is exact.

    w and the codewords are multiples of 1/8 in [-2, 2]; U is the identity plus,
    in each column past the first block, one entry of +1 or -1 in a random row of
    an earlier block (only those entries feed errors forward); d is in {1/4, 1, 4}
    or absent.  Each target is then w plus one weight error, a multiple of 1/8
    below 8 in magnitude, every product and partial sum of the feedback is an
    exact small dyadic (also after a split into TF32 halves), and every branch
    metric and path metric of a block of at most 64 weighted (or 256 unweighted)
    steps fits the fp32 significand, so the whole matrix Q, the bits and the
    targets have a single correct value.
    """
    assert cols % T == 0 and T <= (64 if weighted else 256)
    rng = np.random.default_rng(seed)
    w = (rng.integers(-16, 17, (rows, cols)) / 8.0).astype(np.float32)
    u = np.eye(cols, dtype=np.float32)
    for c in range(T, cols):
        c0 = (c // T) * T
        u[rng.integers(0, c0), c] = np.float32(rng.choice([-1.0, 1.0]))
    d = (4.0 ** rng.integers(-1, 2, cols)).astype(np.float32) if weighted else None
    cb = rng.integers(-16, 17, 1 << L) / 8.0
    cb = cb.astype(np.float16) if cb_dtype == "f16" else cb.astype(np.float32)
    return LdlqWorkload(f"ldlq_dyadic_L{L}_k{k}_T{T}_{rows}x{cols}", L, k, T, w, u, d, cb)


def ub8_gaussian_codebook(V: int, m: int, dtype: str = "f16", seed: int = SEED_CB + 8) -> np.ndarray:
    """Union codebook of 4 * 2^m rows of V values for the 8-state set-partitioned
    trellis (row r in subset r mod 4).  V = 1: the N(0,1) quantiles
    Phi^{-1}((i + 1/2) / N) in increasing order, so that the subsets interleave
    along the line as in Ungerboeck's partition; V > 1: seeded N(0,1) vectors."""
    n = 4 << m
    if V == 1:
        import torch

        u = (torch.arange(n, dtype=torch.float64) + 0.5) / n
        cb = torch.special.ndtri(u).numpy()
    else:
        cb = np.random.default_rng(seed).standard_normal((n, V))
    cb = cb.reshape(-1)
    return cb.astype(np.float16) if dtype == "f16" else cb.astype(np.float32)
