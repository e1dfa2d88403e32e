"""Exhaustive reference for tiny trellises, written independently of the oracle.

It shares nothing with ``oracle/``: no recurrence, no traceback.  Every start
state s_0 in [0, 2^L) and every bitstream b in [0, 2^k)^T is enumerated, and the
state at step t is read straight off the bit window: with the stream as one
integer n of T*k bits (b_1 in the most significant bits),

    s_t = ((s_0 << t*k) | (n >> (T - t)*k)) mod 2^L,

which is the "last L bits written" reading of the bitshift trellis.
"""
from __future__ import annotations

import numpy as np


def states_for(L: int, k: int, T: int, s0: np.ndarray, n: np.ndarray) -> np.ndarray:
    """s_t for every (s0, n) pair given as broadcastable int64 arrays; shape [..., T]."""
    mask = (1 << L) - 1
    out = []
    for t in range(1, T + 1):
        out.append(((s0 << (t * k)) | (n >> ((T - t) * k))) & mask)
    return np.stack(out, axis=-1)


def brute_force(x, d, codebook, L: int, k: int, fixed_start: int | None = None):
    """Minimum of J(s_0, b) over all start states and bitstreams for one block.

    Returns (J_min, s0_min, n_min) with the first minimiser in (s0, n) order.
    """
    x = np.asarray(x, dtype=np.float64).reshape(-1)
    T = x.size
    d = np.ones(T) if d is None else np.asarray(d, dtype=np.float64).reshape(-1)
    c = np.asarray(codebook, dtype=np.float64).reshape(-1)
    assert c.size == 1 << L
    assert T * k <= 16, "keep the enumeration small"
    s0 = np.arange(1 << L, dtype=np.int64) if fixed_start is None else np.array([fixed_start])
    n = np.arange(1 << (T * k), dtype=np.int64)
    st = states_for(L, k, T, s0[:, None], n[None, :])  # [S0, N, T]
    err = d * (x - c[st]) ** 2
    J = err.sum(axis=-1)
    flat = int(np.argmin(J))
    i0, i1 = np.unravel_index(flat, J.shape)
    return float(J[i0, i1]), int(s0[i0]), int(n[i1])


def unpack_symbols(words, k: int, T: int) -> np.ndarray:
    """Symbols b_1..b_T of one block from its packed words.

    Stream bit p is bit 31 - (p mod 32) of word p // 32, so the words written
    big-endian are the stream in order; numpy's unpackbits reads each byte
    most significant bit first.
    """
    w = np.asarray(words, dtype=np.uint32).reshape(-1)
    stream = np.unpackbits(w.astype(">u4").view(np.uint8))
    sym = np.zeros(T, dtype=np.int64)
    for i in range(k):
        sym = (sym << 1) | stream[np.arange(T) * k + i].astype(np.int64)
    return sym


def stream_value(symbols, k: int) -> int:
    n = 0
    for b in symbols:
        n = (n << k) | int(b)
    return n


def decode_window(words, start: int, codebook, L: int, k: int, T: int) -> np.ndarray:
    """Values y_t = c[s_t] of one block from its words and start, by the bit window."""
    sym = unpack_symbols(words, k, T)
    n = stream_value(sym, k)  # Python int: T*k may exceed 64 bits
    s0 = int(start) & 0xFFFFFFFF
    mask = (1 << L) - 1
    st = [((s0 << (t * k)) | (n >> ((T - t) * k))) & mask for t in range(1, T + 1)]
    return np.asarray(codebook, dtype=np.float64)[np.array(st, dtype=np.int64)]


def path_table(x, d, codebook, L: int, k: int):
    """Every distinct path of one block (first state free, counted once) with its
    states [P, T] and cost J [P].  A path is fixed by s_0 in [0, 2^(L-k)) and the
    bitstream, since the top k bits of s_0 never reach s_1."""
    x = np.asarray(x, dtype=np.float64).reshape(-1)
    T = x.size
    d = np.ones(T) if d is None else np.asarray(d, dtype=np.float64).reshape(-1)
    c = np.asarray(codebook, dtype=np.float64).reshape(-1)
    assert c.size == 1 << L
    assert (L - k) + T * k <= 20, "keep the enumeration small"
    s0 = np.arange(1 << (L - k), dtype=np.int64)
    n = np.arange(1 << (T * k), dtype=np.int64)
    st = states_for(L, k, T, s0[:, None], n[None, :]).reshape(-1, T)
    J = (d * (x - c[st]) ** 2).sum(axis=-1)
    return st, J


def boltzmann_brute_force(x, d, codebook, L: int, k: int, tau: float):
    """Soft codewords E[c[s_t]] and free energy -tau log Z under P ~ exp(-J/tau),
    summed over every path."""
    st, J = path_table(x, d, codebook, L, k)
    c = np.asarray(codebook, dtype=np.float64).reshape(-1)
    a = -J / tau
    m = a.max()
    logz = m + np.log(np.exp(a - m).sum())
    p = np.exp(a - logz)
    y = (p[:, None] * c[st]).sum(axis=0)
    return y, -tau * logz


def brute_force_vec(x, d, codebook, L: int, k: int, V: int):
    """Minimum over every start state and bitstream of the vector trellis (V
    weights per step, kV bits per step, codebook [2^L, V]); (J_min, s0, n)."""
    x = np.asarray(x, dtype=np.float64).reshape(-1)
    T = x.size
    d = np.ones(T) if d is None else np.asarray(d, dtype=np.float64).reshape(-1)
    c = np.asarray(codebook, dtype=np.float64).reshape(1 << L, V)
    steps, K = T // V, k * V
    assert steps * K <= 16, "keep the enumeration small"
    s0 = np.arange(1 << L, dtype=np.int64)
    n = np.arange(1 << (steps * K), dtype=np.int64)
    st = states_for(L, K, steps, s0[:, None], n[None, :])  # [S0, N, steps]
    vals = c[st]                                          # [S0, N, steps, V]
    err = (d.reshape(steps, V) * (x.reshape(steps, V) - vals) ** 2).sum(axis=(-1, -2))
    flat = int(np.argmin(err))
    i0, i1 = np.unravel_index(flat, err.shape)
    return float(err[i0, i1]), int(s0[i0]), int(n[i1])


def decode_window_vec(words, start: int, codebook, L: int, k: int, V: int, T: int) -> np.ndarray:
    """Values of one vector-trellis block by the bit window (symbols of kV bits)."""
    K, steps = k * V, T // V
    sym = unpack_symbols(words, K, steps)
    n = stream_value(sym, K)
    s0 = int(start) & 0xFFFFFFFF
    mask = (1 << L) - 1
    st = [((s0 << (t * K)) | (n >> ((steps - t) * K))) & mask for t in range(1, steps + 1)]
    c = np.asarray(codebook, dtype=np.float64).reshape(1 << L, V)
    return c[np.array(st, dtype=np.int64)].reshape(-1)


# ---------------------------------------------------------------------------
# Ungerboeck's 8-state set-partitioned trellis, read from its parity-check
# equation alone (no state machine): a label sequence (z1_t, z0_t) is a path
# of the code with h0 = D^3 + D + 1 and h1 = D^2 iff
#     z0_t = z0_{t-1} ^ z0_{t-3} ^ z1_{t-2}      for t >= 4,
# with z0_1, z0_2, z0_3 free (they carry the start state).  Step t emits row
# 4 i_t + 2 z1_t + z0_t of the union codebook.
# ---------------------------------------------------------------------------
def ub8_first_parities(start: int, z1_first: int):
    """z0_1, z0_2, z0_3 of a path from state start = 4p + 2q + r whose first
    branch bit is z1_first: the register contents read off the code's
    realisation (p, then p ^ q, then p ^ q ^ r ^ z1_1)."""
    p, q, r = (start >> 2) & 1, (start >> 1) & 1, start & 1
    return p, p ^ q, p ^ q ^ r ^ z1_first


def ub8_parities(z1, head):
    """Every z0_t of a path from its branch bits and its first three parities."""
    S = len(z1)
    z0 = list(head[:min(3, S)])
    for t in range(3, S):  # 0-based t is step t + 1
        z0.append(z0[t - 1] ^ z0[t - 3] ^ z1[t - 2])
    return z0


def ub8_brute_force(x, d, codebook, V: int, m: int, fixed_start: int | None = None):
    """Minimum of J over every code sequence of the trellis (every choice of the
    three free parities, of the branch bits and of the entries inside the
    subsets), enumerated without the state machine.  Returns (J_min, rows)."""
    import itertools

    x = np.asarray(x, dtype=np.float64).reshape(-1)
    T = x.size
    S = T // V
    d = np.ones(T) if d is None else np.asarray(d, dtype=np.float64).reshape(-1)
    c = np.asarray(codebook, dtype=np.float64).reshape(4 << m, V)
    assert 3 + S * (1 + m) <= 18, "keep the enumeration small"
    xs, ds = x.reshape(S, V), d.reshape(S, V)
    best, best_rows = np.inf, None
    for z1 in itertools.product((0, 1), repeat=S):
        if fixed_start is None:
            heads = list(itertools.product((0, 1), repeat=3))
        else:
            heads = [ub8_first_parities(fixed_start & 7, z1[0])]
        for head in heads:
            z0 = ub8_parities(z1, head)
            subs = [2 * z1[t] + z0[t] for t in range(S)]
            # every choice of entries: [2^(mS), S] row indices
            ii = np.array(list(itertools.product(range(1 << m), repeat=S)), dtype=np.int64)
            rows = 4 * ii + np.array(subs, dtype=np.int64)[None, :]
            J = (ds[None] * (xs[None] - c[rows]) ** 2).sum(axis=(1, 2))
            a = int(np.argmin(J))
            if J[a] < best:
                best, best_rows = float(J[a]), rows[a]
    return best, best_rows


def ub8_decode_parity(words, start: int, codebook, V: int, m: int, T: int) -> np.ndarray:
    """Values of one block from its words and start state, through the parity
    equation instead of the state machine."""
    S = T // V
    sym = unpack_symbols(words, 1 + m, S)
    z1 = [int(b) >> m for b in sym]
    ii = [int(b) & ((1 << m) - 1) for b in sym]
    z0 = ub8_parities(z1, ub8_first_parities(int(start) & 7, z1[0]))
    c = np.asarray(codebook, dtype=np.float64).reshape(4 << m, V)
    return np.concatenate([c[4 * ii[t] + 2 * z1[t] + z0[t]] for t in range(S)])
