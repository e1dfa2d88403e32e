/*
 * tcq_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, single-threaded CPU oracle for trellis-coded quantization
 * (TCQ) of weight blocks over the bitshift trellis, computed in fp64.  Only
 * the test suite, the smoke check and the CPU-baseline leg of the benchmark
 * may load this file's library; the CUDA library never does, and the two share
 * no code, header, table or helper.
 *
 * What it computes, and where the sources state it:
 *   - Trellis-coded quantization with a stateful decoder and a "bitshift"
 *     trellis: "QTIP: Quantization with Trellises and Incoherence Processing"
 *     (abstract).  The state is the last L bits written, k new bits are shifted
 *     in per weight, and the reconstruction is a codebook lookup by state.
 *   - The search is the Viterbi dynamic program that retains, per state, the
 *     lowest-cost path reaching it, with work linear in the block length: "How do you fit a 4B LLM in 1.24 GB:
 *     trellis-coded 2-bit" (section on trellis memory and the Viterbi search).
 *   - The branch metric is the per-coordinate weighted error d_j (x_j - c)^2,
 *     with d_j the diagonal of the Hessian's LDL factor, and a start state is
 *     stored per coding block: CurveTQ abstract (aggregator page, paper
 *     2610.09212).
 *
 * Notation (one block): T weights x_1..x_T, weights d_1..d_T (d == NULL means
 * d_t = 1), codebook c[0 .. 2^L).  With mask = 2^L - 1,
 *     s_t = ((s_{t-1} << k) | b_t) & mask,      y_t = c[s_t],
 *     J(s_0, b) = sum_t d_t (x_t - c[s_t])^2.
 * The oracle returns the minimiser of J over every start state s_0 and every
 * bitstream b (or over b alone for a fixed start), J_min, and the packed bits.
 *
 * The dynamic program is written per STATE on purpose (the plain textbook
 * form), in double precision:
 *   C_1[s]  = d_1 (x_1 - c[s])^2                 (every s_1 reachable: free start)
 *   C_t[s]  = min_h C_{t-1}[(h << (L-k)) | (s >> k)] + d_t (x_t - c[s])^2
 *   bp_t[s] = the smallest h reaching that minimum
 *   s_T     = the smallest s minimising C_T; trace back through bp.
 *   b_t = s_t & (2^k - 1); stored start = s_1 >> k (its low L-k bits are all
 *   the decoder can see).
 *
 * Bit packing (the pages are silent; this reading is fixed here): symbol t
 * (1-based) occupies stream bits [(t-1)k, tk), most significant bit first;
 * stream bit p is bit 31 - (p mod 32) of 32-bit word p / 32; unused bits of the
 * last word are zero.  Words per block W = ceil(T k / 32).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL (-1)
#define ORACLE_ENOMEM (-2)

static int valid_shape(int L, int k, int T)
{
    if (L < 1 || L > 20) return 0;
    if (k < 1 || k > L || k > 8) return 0;
    if (T < 1) return 0;
    return 1;
}

int oracle_words_per_block(int k, int T)
{
    if (k < 1 || T < 1) return -1;
    return (int)(((int64_t)T * k + 31) / 32);
}

/* Write the k-bit symbol b_t (1-based t) into a block's word array, one bit at
 * a time, most significant bit first. */
static void put_symbol(uint32_t* words, int k, int t, uint32_t sym)
{
    for (int i = 0; i < k; ++i) {
        uint32_t bit = (sym >> (k - 1 - i)) & 1u;
        int64_t p = (int64_t)(t - 1) * k + i;
        if (bit) words[p / 32] |= 1u << (31 - (int)(p % 32));
    }
}

/* Read the k-bit symbol b_t back, one bit at a time. */
static uint32_t get_symbol(const uint32_t* words, int k, int t)
{
    uint32_t sym = 0;
    for (int i = 0; i < k; ++i) {
        int64_t p = (int64_t)(t - 1) * k + i;
        uint32_t bit = (words[p / 32] >> (31 - (int)(p % 32))) & 1u;
        sym = (sym << 1) | bit;
    }
    return sym;
}

static double weight_at(const double* d, int64_t i)
{
    return d ? d[i] : 1.0;
}

/*
 * Viterbi encode of n_blocks independent blocks.
 *   x, d        : [n_blocks, T] row-major (d may be NULL: d_t = 1)
 *   cb          : codebook, 2^L values (the exact widening of the caller's
 *                 fp32 / fp16 entries)
 *   fixed_start : < 0 for a free start state; otherwise s_0 is fixed to it
 *   start_state : [n_blocks] canonical stored start, s_1 >> k
 *   bits        : [n_blocks, W] packed symbols
 *   cost        : [n_blocks] J_min
 */
int oracle_encode(const double* x, const double* d, const double* cb, int L, int k,
                  int T, int64_t n_blocks, int64_t fixed_start, uint32_t* start_state,
                  uint32_t* bits, double* cost)
{
    if (!valid_shape(L, k, T) || n_blocks < 0) return ORACLE_EINVAL;
    if (n_blocks == 0) return ORACLE_OK;
    if (!x || !cb || !start_state || !bits || !cost) return ORACLE_EINVAL;

    const int64_t S = (int64_t)1 << L;
    const uint32_t mask = (uint32_t)(S - 1);
    const uint32_t low_mask = (uint32_t)(((uint64_t)1 << (L - k)) - 1); /* low L-k bits */
    const int H = 1 << k;
    const int W = oracle_words_per_block(k, T);

    double* prev = (double*)malloc(sizeof(double) * S);
    double* cur = (double*)malloc(sizeof(double) * S);
    uint8_t* bp = (uint8_t*)malloc((size_t)T * (size_t)S); /* bp[t-1][s], t = 1..T */
    uint32_t* path = (uint32_t*)malloc(sizeof(uint32_t) * (size_t)T);
    if (!prev || !cur || !bp || !path) {
        free(prev); free(cur); free(bp); free(path);
        return ORACLE_ENOMEM;
    }

    for (int64_t blk = 0; blk < n_blocks; ++blk) {
        const double* xb = x + blk * T;
        const double* db = d ? d + blk * T : NULL;

        /* t = 1 */
        for (int64_t s = 0; s < S; ++s) {
            int reachable = 1;
            if (fixed_start >= 0)
                reachable = (((uint32_t)s >> k) == ((uint32_t)fixed_start & low_mask));
            double e = xb[0] - cb[s];
            prev[s] = reachable ? weight_at(db, 0) * e * e : INFINITY;
            bp[s] = 0;
        }

        /* t = 2 .. T */
        for (int t = 2; t <= T; ++t) {
            const double xt = xb[t - 1];
            const double dt = weight_at(db, t - 1);
            uint8_t* bpt = bp + (size_t)(t - 1) * (size_t)S;
            for (int64_t s = 0; s < S; ++s) {
                double best = INFINITY;
                int best_h = 0;
                for (int h = 0; h < H; ++h) {
                    uint32_t pred = (((uint32_t)h << (L - k)) | ((uint32_t)s >> k)) & mask;
                    if (prev[pred] < best) { /* strict: the smallest h wins a tie */
                        best = prev[pred];
                        best_h = h;
                    }
                }
                double e = xt - cb[s];
                cur[s] = best + dt * e * e;
                bpt[s] = (uint8_t)best_h;
            }
            double* tmp = prev; prev = cur; cur = tmp;
        }

        /* final state: the smallest s on ties */
        int64_t s_best = 0;
        for (int64_t s = 1; s < S; ++s)
            if (prev[s] < prev[s_best]) s_best = s;
        cost[blk] = prev[s_best];

        /* trace back */
        uint32_t s = (uint32_t)s_best;
        path[T - 1] = s;
        for (int t = T; t >= 2; --t) {
            uint32_t h = bp[(size_t)(t - 1) * (size_t)S + s];
            s = ((h << (L - k)) | (s >> k)) & mask;
            path[t - 2] = s;
        }

        uint32_t* wb = bits + blk * W;
        memset(wb, 0, sizeof(uint32_t) * (size_t)W);
        for (int t = 1; t <= T; ++t)
            put_symbol(wb, k, t, path[t - 1] & (uint32_t)(H - 1));
        start_state[blk] = path[0] >> k;
    }

    free(prev); free(cur); free(bp); free(path);
    return ORACLE_OK;
}

/*
 * Decode: s_t = ((s_{t-1} << k) | b_t) & mask starting from the stored start
 * state as given (its bits above L-k fall out of the mask), y_t = c[s_t].
 */
int oracle_decode(const uint32_t* bits, const uint32_t* start_state, const double* cb, int L,
                  int k, int T, int64_t n_blocks, double* y)
{
    if (!valid_shape(L, k, T) || n_blocks < 0) return ORACLE_EINVAL;
    if (n_blocks == 0) return ORACLE_OK;
    if (!bits || !start_state || !cb || !y) return ORACLE_EINVAL;
    const uint64_t mask = ((uint64_t)1 << L) - 1;
    const int W = oracle_words_per_block(k, T);
    for (int64_t blk = 0; blk < n_blocks; ++blk) {
        uint64_t s = start_state[blk];
        for (int t = 1; t <= T; ++t) {
            uint32_t b = get_symbol(bits + blk * W, k, t);
            s = ((s << k) | b) & mask;
            y[blk * T + t - 1] = cb[s];
        }
    }
    return ORACLE_OK;
}

/* J = sum_t d_t (x_t - y_t)^2 per block, in fp64. */
int oracle_path_cost(const double* x, const double* d, const double* y, int T, int64_t n_blocks,
                     double* cost)
{
    if (T < 1 || n_blocks < 0) return ORACLE_EINVAL;
    if (n_blocks == 0) return ORACLE_OK;
    if (!x || !y || !cost) return ORACLE_EINVAL;
    for (int64_t blk = 0; blk < n_blocks; ++blk) {
        double acc = 0.0;
        for (int t = 0; t < T; ++t) {
            double e = x[blk * T + t] - y[blk * T + t];
            acc += weight_at(d, blk * T + t) * e * e;
        }
        cost[blk] = acc;
    }
    return ORACLE_OK;
}

/*
 * Greedy trellis rounding, the baseline the Pingala-8 post shows losing to the
 * searched path: from the given start state, at each step take the symbol whose
 * codeword (within the current coset) is nearest, the smallest symbol on ties.
 */
int oracle_greedy(const double* x, const double* d, const double* cb, int L, int k, int T,
                  int64_t n_blocks, const uint32_t* start_in, uint32_t* bits, double* cost)
{
    if (!valid_shape(L, k, T) || n_blocks < 0) return ORACLE_EINVAL;
    if (n_blocks == 0) return ORACLE_OK;
    if (!x || !cb || !start_in || !bits || !cost) return ORACLE_EINVAL;
    const uint64_t mask = ((uint64_t)1 << L) - 1;
    const int H = 1 << k;
    const int W = oracle_words_per_block(k, T);
    for (int64_t blk = 0; blk < n_blocks; ++blk) {
        uint64_t s = start_in[blk];
        double acc = 0.0;
        uint32_t* wb = bits + blk * W;
        memset(wb, 0, sizeof(uint32_t) * (size_t)W);
        for (int t = 1; t <= T; ++t) {
            double xt = x[blk * T + t - 1];
            double dt = weight_at(d, blk * T + t - 1);
            double best = INFINITY;
            int best_b = 0;
            for (int b = 0; b < H; ++b) {
                uint64_t sn = ((s << k) | (uint64_t)b) & mask;
                double e = xt - cb[sn];
                double m = dt * e * e;
                if (m < best) { best = m; best_b = b; }
            }
            s = ((s << k) | (uint64_t)best_b) & mask;
            acc += best;
            put_symbol(wb, k, t, (uint32_t)best_b);
        }
        cost[blk] = acc;
    }
    return ORACLE_OK;
}

/*
 * Matrix-vector product with a trellis-coded matrix: rows x cols weights stored
 * as rows * (cols / T) coding blocks of T consecutive columns (block (r, j) =
 * index r * (cols/T) + j covers columns [jT, jT + T) of row r), each scaled by
 * scale[block] (NULL: 1).  y[r] = sum_j scale[r, j] * sum_t c[s_{r,j,t}] * x[jT + t],
 * i.e. decode every block, then the dense product, accumulated in fp64.
 */
int oracle_gemv(const uint32_t* bits, const uint32_t* start_state, const double* scale,
                const double* cb, int L, int k, int T, int64_t rows, int64_t cols,
                const double* x, double* y)
{
    if (!valid_shape(L, k, T) || rows < 0 || cols < 0 || cols % T != 0) return ORACLE_EINVAL;
    if (rows == 0) return ORACLE_OK;
    if (!bits || !start_state || !cb || !x || !y) return ORACLE_EINVAL;
    const int64_t nb = cols / T;
    const int W = oracle_words_per_block(k, T);
    double* vals = (double*)malloc(sizeof(double) * (size_t)T);
    if (!vals) return ORACLE_ENOMEM;
    for (int64_t r = 0; r < rows; ++r) {
        double acc = 0.0;
        for (int64_t j = 0; j < nb; ++j) {
            const int64_t b = r * nb + j;
            int rc = oracle_decode(bits + b * W, start_state + b, cb, L, k, T, 1, vals);
            if (rc != ORACLE_OK) { free(vals); return rc; }
            double part = 0.0;
            for (int t = 0; t < T; ++t) part += vals[t] * x[j * T + t];
            acc += (scale ? scale[b] : 1.0) * part;
        }
        y[r] = acc;
    }
    free(vals);
    return ORACLE_OK;
}

/*
 * The targets of column block j given the reconstruction of the blocks before
 * it (the feedback step of the error-feedback encode below):
 *   x[r][c] = w[r][c] + sum_{i < jT} (w[r][i] - q[r][i]) u[i][c],  c in [jT, jT + T).
 * Only x's columns of block j are written.
 */
int oracle_feedback(const double* w, const double* u, const double* q, int T, int64_t rows,
                    int64_t cols, int64_t j, double* xt)
{
    if (T < 1 || rows < 0 || cols < 0 || cols % T != 0 || j < 0 || j * T >= cols)
        return ORACLE_EINVAL;
    for (int64_t r = 0; r < rows; ++r) {
        const double* wr = w + r * cols;
        const double* qr = q + r * cols;
        for (int64_t c = j * T; c < (j + 1) * T; ++c) {
            double acc = wr[c];
            for (int64_t i = 0; i < j * T; ++i) acc += (wr[i] - qr[i]) * u[i * cols + c];
            xt[r * cols + c] = acc;
        }
    }
    return ORACLE_OK;
}

/*
 * Error-feedback (LDLQ) encode of a rows x cols matrix, column block by column
 * block.  "How do you fit a 4B LLM in 1.24 GB? Trellis-coded 2-bit", section on
 * error feedback and LDLQ: columns are quantised in order and each one's error
 * is pushed onto the columns not yet quantised, in proportions set by
 * H = E[x x^T]; CurveTQ abstract: the feedback runs between coding blocks and
 * the Viterbi metric inside a block is weighted by the diagonal of H's LDL
 * factorisation.
 *
 * With H = U diag(d) U^T, U unit upper triangular (cols x cols, row-major, only
 * the strictly upper part is read) and w_r the r-th row:
 *   for block B = [jT, jT + T):
 *     x_r[c] = w_r[c] + sum_{i < jT} (w_r[i] - q_r[i]) U[i][c],   c in B
 *     (q_r[B], bits, start) = Viterbi TCQ of x_r[B] with weights d[B]
 * Outputs: q [rows, cols], the targets x [rows, cols], and per coding block
 * (block (r, j) = r * cols/T + j) start state, bits and cost.
 */
int oracle_ldlq(const double* w, const double* u, const double* dd, const double* cb, int L,
                int k, int T, int64_t rows, int64_t cols, double* q, double* xt,
                uint32_t* start_state, uint32_t* bits, double* cost)
{
    if (!valid_shape(L, k, T) || rows < 0 || cols < 0 || cols % T != 0) return ORACLE_EINVAL;
    if (rows == 0 || cols == 0) return ORACLE_OK;
    if (!w || !u || !dd || !cb || !q || !xt || !start_state || !bits || !cost)
        return ORACLE_EINVAL;
    const int64_t nb = cols / T;
    const int W = oracle_words_per_block(k, T);
    for (int64_t r = 0; r < rows; ++r) {
        const double* wr = w + r * cols;
        double* qr = q + r * cols;
        double* xr = xt + r * cols;
        for (int64_t j = 0; j < nb; ++j) {
            oracle_feedback(wr, u, qr, T, 1, cols, j, xr);
            const int64_t b = r * nb + j;
            int rc = oracle_encode(xr + j * T, dd + j * T, cb, L, k, T, 1, -1, start_state + b,
                                   bits + b * W, cost + b);
            if (rc != ORACLE_OK) return rc;
            rc = oracle_decode(bits + b * W, start_state + b, cb, L, k, T, 1, qr + j * T);
            if (rc != ORACLE_OK) return rc;
        }
    }
    return ORACLE_OK;
}

/*
 * Soft trellis quantization by the forward-backward (BCJR) sum-product
 * recursion at temperature tau: "BCJR-QAT: A Differentiable Relaxation of
 * Trellis-Coded Weight Quantization" (abstract, aggregator page).  The Viterbi
 * minimum over paths is replaced by the Boltzmann distribution
 *     P(path) = exp(-J(path) / tau) / Z,
 * the soft codeword of position t is the expectation of c[s_t] under P, and it
 * returns to the hard Viterbi code as tau -> 0.  A path is a state sequence
 * s_1..s_T of the bitshift trellis with the first state free (each of the 2^L
 * first states counted once) and J the weighted cost above.
 *
 * Per block, in natural-log units and double precision, per STATE:
 *   la_1[s] = -d_1 (x_1 - c[s])^2 / tau
 *   la_t[s] = -d_t (x_t - c[s])^2 / tau + lse_h la_{t-1}[(h << (L-k)) | (s >> k)]
 *   lb_T[s] = 0
 *   lb_t[s] = lse_b ( -d_{t+1} (x_{t+1} - c[s'])^2 / tau + lb_{t+1}[s'] ),
 *             s' = ((s << k) | b) & mask
 *   log Z   = lse_s la_T[s]
 *   y_t     = sum_s exp(la_t[s] + lb_t[s] - log Z) c[s]
 *   F       = -tau log Z                      (the free energy; F -> J_min)
 * with lse the log-sum-exp.  Outputs y [n_blocks, T] and F [n_blocks].
 */
static double lse_add(double a, double b)
{
    if (a == -INFINITY) return b;
    if (b == -INFINITY) return a;
    const double m = a > b ? a : b;
    return m + log(exp(a - m) + exp(b - m));
}

int oracle_bcjr(const double* x, const double* d, const double* cb, int L, int k, int T,
                int64_t n_blocks, double tau, double* y, double* free_energy)
{
    if (!valid_shape(L, k, T) || n_blocks < 0 || !(tau > 0.0) || !isfinite(tau))
        return ORACLE_EINVAL;
    if (n_blocks == 0) return ORACLE_OK;
    if (!x || !cb || !y || !free_energy) return ORACLE_EINVAL;
    const int64_t S = (int64_t)1 << L;
    const uint32_t mask = (uint32_t)(S - 1);
    const int H = 1 << k;
    double* la = (double*)malloc(sizeof(double) * (size_t)T * (size_t)S);
    double* lb = (double*)malloc(sizeof(double) * (size_t)T * (size_t)S);
    if (!la || !lb) {
        free(la);
        free(lb);
        return ORACLE_EINVAL;
    }
    for (int64_t blk = 0; blk < n_blocks; ++blk) {
        const double* xb = x + blk * T;
        const int64_t base = blk * T;
        /* forward */
        for (int64_t s = 0; s < S; ++s) {
            const double e = xb[0] - cb[s];
            la[s] = -weight_at(d, base) * e * e / tau;
        }
        for (int t = 1; t < T; ++t) {
            const double w = weight_at(d, base + t);
            for (int64_t s = 0; s < S; ++s) {
                double acc = -INFINITY;
                for (int h = 0; h < H; ++h) {
                    const uint32_t prev = (((uint32_t)h << (L - k)) | ((uint32_t)s >> k)) & mask;
                    acc = lse_add(acc, la[(int64_t)(t - 1) * S + prev]);
                }
                const double e = xb[t] - cb[s];
                la[(int64_t)t * S + s] = -w * e * e / tau + acc;
            }
        }
        /* backward */
        for (int64_t s = 0; s < S; ++s) lb[(int64_t)(T - 1) * S + s] = 0.0;
        for (int t = T - 2; t >= 0; --t) {
            const double w = weight_at(d, base + t + 1);
            for (int64_t s = 0; s < S; ++s) {
                double acc = -INFINITY;
                for (int b = 0; b < H; ++b) {
                    const uint32_t next = (((uint32_t)s << k) | (uint32_t)b) & mask;
                    const double e = xb[t + 1] - cb[next];
                    acc = lse_add(acc, -w * e * e / tau + lb[(int64_t)(t + 1) * S + next]);
                }
                lb[(int64_t)t * S + s] = acc;
            }
        }
        double logz = -INFINITY;
        for (int64_t s = 0; s < S; ++s) logz = lse_add(logz, la[(int64_t)(T - 1) * S + s]);
        for (int t = 0; t < T; ++t) {
            double acc = 0.0;
            for (int64_t s = 0; s < S; ++s)
                acc += exp(la[(int64_t)t * S + s] + lb[(int64_t)t * S + s] - logz) * cb[s];
            y[base + t] = acc;
        }
        free_energy[blk] = -tau * logz;
    }
    free(la);
    free(lb);
    return ORACLE_OK;
}

/*
 * A computed ("lookup-free") code: the codeword of a state is computed from the
 * state's bits instead of read from a table.  "QTIP: Quantization with
 * Trellises and Incoherence Processing" (abstract) introduces codes from
 * lookup-only to computed lookup-free for the bitshift trellis and gives no
 * formula; the code here is this library's reading: a multiplicative hash of
 * the state (its high half is a well-mixed function of every state bit) and
 * the sum of that half's two bytes (a triangular, roughly bell-shaped value),
 * centred and scaled by a power of two so that every codeword is exact in
 * binary16:
 *     v    = (A s) mod 2^32,   A = 0x9E3779B1
 *     c[s] = (v_2 + v_3 - 255) / 128,   v_2, v_3 bits 16..23 and 24..31 of v.
 * Writes the 2^L codewords to cb.
 */
int oracle_mad_codebook(int L, double* cb)
{
    if (L < 1 || L > 20 || !cb) return ORACLE_EINVAL;
    const uint32_t A = 0x9E3779B1u;
    for (uint32_t s = 0; s < (1u << L); ++s) {
        const uint32_t v = A * s; /* unsigned arithmetic wraps mod 2^32 */
        const int sum = (int)((v >> 16) & 0xFFu) + (int)(v >> 24);
        cb[s] = (double)(sum - 255) / 128.0;
    }
    return ORACLE_OK;
}

/*
 * Vector trellis: V weights per trellis step ("QTIP: Quantization with
 * Trellises and Incoherence Processing", abstract: the bitshift trellis with a
 * stateful decoder that separates the codebook size from the bitrate and the
 * effective dimension).  Each step shifts kV bits into the state and the state
 * selects a V-dimensional codeword; V = 1 is oracle_encode.
 *
 * One block: T weights (V | T), steps tau = 1..T/V, codebook cb[2^L][V]
 * (row-major), with mask = 2^L - 1:
 *     s_tau = ((s_{tau-1} << kV) | b_tau) & mask,   b_tau in [0, 2^{kV})
 *     y_{(tau-1)V + v} = cb[s_tau][v]
 *     J = sum_tau sum_v d_{(tau-1)V+v} (x_{(tau-1)V+v} - cb[s_tau][v])^2
 * Same dynamic program per state as oracle_encode (smallest predecessor on
 * ties, smallest final state), same packing with symbols of kV bits, the
 * stored start s_1 >> kV.  Requires kV <= L and kV <= 8.
 */
int oracle_encode_vec(const double* x, const double* d, const double* cb, int L, int k, int V,
                      int T, int64_t n_blocks, int64_t fixed_start, uint32_t* start_state,
                      uint32_t* bits, double* cost)
{
    if (V < 1 || k < 1 || k * V > L || k * V > 8 || T < 1 || T % V != 0 || n_blocks < 0 ||
        !valid_shape(L, k, T))
        return ORACLE_EINVAL;
    if (n_blocks == 0) return ORACLE_OK;
    if (!x || !cb || !start_state || !bits || !cost) return ORACLE_EINVAL;
    const int K = k * V;          /* bits per step */
    const int NS = T / V;         /* steps */
    const int64_t S = (int64_t)1 << L;
    const uint32_t mask = (uint32_t)(S - 1);
    const uint32_t low_mask = (uint32_t)(((uint64_t)1 << (L - K)) - 1);
    const int H = 1 << K;
    const int W = oracle_words_per_block(k, T);
    double* prev = (double*)malloc(sizeof(double) * S);
    double* cur = (double*)malloc(sizeof(double) * S);
    uint8_t* bp = (uint8_t*)malloc((size_t)NS * (size_t)S);
    uint32_t* path = (uint32_t*)malloc(sizeof(uint32_t) * (size_t)NS);
    if (!prev || !cur || !bp || !path) {
        free(prev); free(cur); free(bp); free(path);
        return ORACLE_ENOMEM;
    }
    for (int64_t blk = 0; blk < n_blocks; ++blk) {
        const double* xb = x + blk * T;
        const double* db = d ? d + blk * T : NULL;
        for (int tau = 1; tau <= NS; ++tau) {
            uint8_t* bpt = bp + (size_t)(tau - 1) * (size_t)S;
            for (int64_t s = 0; s < S; ++s) {
                double bm = 0.0; /* the step's branch metric: V weighted squared errors */
                for (int v = 0; v < V; ++v) {
                    const int i = (tau - 1) * V + v;
                    const double e = xb[i] - cb[s * V + v];
                    bm += weight_at(db, i) * e * e;
                }
                double best;
                int best_h = 0;
                if (tau == 1) {
                    int reachable = 1;
                    if (fixed_start >= 0)
                        reachable = (((uint32_t)s >> K) == ((uint32_t)fixed_start & low_mask));
                    best = reachable ? 0.0 : INFINITY;
                } else {
                    best = INFINITY;
                    for (int h = 0; h < H; ++h) {
                        const uint32_t pred = (((uint32_t)h << (L - K)) | ((uint32_t)s >> K)) & mask;
                        if (prev[pred] < best) {
                            best = prev[pred];
                            best_h = h;
                        }
                    }
                }
                cur[s] = best + bm;
                bpt[s] = (uint8_t)best_h;
            }
            double* tmp = prev; prev = cur; cur = tmp;
        }
        int64_t s_best = 0;
        for (int64_t s = 1; s < S; ++s)
            if (prev[s] < prev[s_best]) s_best = s;
        cost[blk] = prev[s_best];
        uint32_t s = (uint32_t)s_best;
        path[NS - 1] = s;
        for (int tau = NS; tau >= 2; --tau) {
            const uint32_t h = bp[(size_t)(tau - 1) * (size_t)S + s];
            s = ((h << (L - K)) | (s >> K)) & mask;
            path[tau - 2] = s;
        }
        uint32_t* wb = bits + blk * W;
        memset(wb, 0, sizeof(uint32_t) * (size_t)W);
        for (int tau = 1; tau <= NS; ++tau) put_symbol(wb, K, tau, path[tau - 1] & (uint32_t)(H - 1));
        start_state[blk] = path[0] >> K;
    }
    free(prev); free(cur); free(bp); free(path);
    return ORACLE_OK;
}

/* Decode of the vector trellis: y_{(tau-1)V + v} = cb[s_tau][v]. */
int oracle_decode_vec(const uint32_t* bits, const uint32_t* start_state, const double* cb, int L,
                      int k, int V, int T, int64_t n_blocks, double* y)
{
    if (V < 1 || k < 1 || k * V > L || T < 1 || T % V != 0 || n_blocks < 0 ||
        !valid_shape(L, k, T))
        return ORACLE_EINVAL;
    if (n_blocks == 0) return ORACLE_OK;
    if (!bits || !start_state || !cb || !y) return ORACLE_EINVAL;
    const int K = k * V;
    const uint64_t mask = ((uint64_t)1 << L) - 1;
    const int W = oracle_words_per_block(k, T);
    for (int64_t blk = 0; blk < n_blocks; ++blk) {
        uint64_t s = start_state[blk];
        for (int tau = 1; tau <= T / V; ++tau) {
            s = ((s << K) | get_symbol(bits + blk * W, K, tau)) & mask;
            for (int v = 0; v < V; ++v) y[blk * T + (tau - 1) * V + v] = cb[s * V + v];
        }
    }
    return ORACLE_OK;
}

/*
 * Ungerboeck's 8-state set-partitioned trellis (the 2-bit post, Pingala-8
 * section: an 8-state set-partitioned trellis over symbols of several weights
 * at about 2 bits per weight, its labels Ungerboeck's; the post's section on
 * trellis-coded quantization: the state decides which subset the next group
 * may use, the written bits pick a value inside the subset and set the next
 * state, so the format holds twice as many values as its bits address; its
 * background reading: Marcellin and Fischer's trellis-coded quantization).
 * The pages give no labels and no codebook; the reading taken here is
 * Marcellin and Fischer's TCQ on Ungerboeck's 8-state code for one-dimensional
 * signals, generalised to V weights per symbol:
 *
 *   Union codebook: 4 * 2^m rows of V values; row r belongs to subset
 *   D_{r mod 4} and is entry r >> 2 of it (for V = 1 and rows sorted
 *   ascending this is Ungerboeck's partition of an amplitude alphabet).
 *
 *   Trellis: the rate-1/2 systematic feedback code with parity-check
 *   polynomials h0 = D^3 + D + 1 and h1 = D^2 (octal 13 and 04): a label
 *   sequence (z1_t, z0_t) is a code sequence iff
 *       z0_t ^ z0_{t-1} ^ z0_{t-3} ^ z1_{t-2} = 0.
 *   Realised with three memory bits, state sigma = 4p + 2q + r: a branch from
 *   sigma with branch bit z uses subset j = 2z + p (z0 = p, z1 = z) and leads to
 *       sigma' = 4 (p ^ q) + 2 (r ^ z) + p.
 *   Both branches leaving a state use the two subsets of one half {D_p, D_p+2};
 *   the two branches entering a state come from states with the same p.
 *
 *   A step codes V weights with 1 + m bits: symbol b_t = (z_t << m) | i_t, the
 *   branch bit and the entry i_t of subset j_t; y_t = row 4 i_t + j_t.
 *   Symbols are packed like every other stream here (MSB first, 1 + m bits
 *   per step); the stored start state is sigma_0 (3 bits).
 *
 * The search, in the textbook order: for every step and subset the nearest
 * entry (the branch metric of every branch carrying that subset, smallest i on
 * ties), then the Viterbi program over the 8 states:
 *   M_0[s] = 0 (free start; a fixed start leaves only that state at 0),
 *   M_t[s'] = min over the branches (s, z) into s' of M_{t-1}[s] + e_t[2z + p(s)]
 *   (predecessors taken in increasing s, strict <), final state the smallest
 *   s minimising M_S, and the traceback.
 */
static int ub8_p(int s) { return (s >> 2) & 1; }

static int ub8_next(int s, int z)
{
    const int p = (s >> 2) & 1, q = (s >> 1) & 1, r = s & 1;
    return 4 * (p ^ q) + 2 * (r ^ z) + p;
}

int oracle_ub8_encode(const double* x, const double* d, const double* cb, int V, int m, int T,
                      int64_t n_blocks, int64_t fixed_start, uint32_t* start_state,
                      uint32_t* bits, double* cost)
{
    if (V < 1 || m < 0 || m > 16 || T < 1 || T % V != 0 || n_blocks < 0) return ORACLE_EINVAL;
    if (n_blocks == 0) return ORACLE_OK;
    if (!x || !cb || !start_state || !bits || !cost) return ORACLE_EINVAL;
    const int NS = T / V;
    const int K = 1 + m;
    const int64_t per_subset = (int64_t)1 << m;
    const int W = oracle_words_per_block(K, NS);
    double* e = (double*)malloc(sizeof(double) * 4 * (size_t)NS);
    uint32_t* idx = (uint32_t*)malloc(sizeof(uint32_t) * 4 * (size_t)NS);
    uint8_t* bp_state = (uint8_t*)malloc(8 * (size_t)NS);
    uint8_t* bp_z = (uint8_t*)malloc(8 * (size_t)NS);
    if (!e || !idx || !bp_state || !bp_z) {
        free(e); free(idx); free(bp_state); free(bp_z);
        return ORACLE_ENOMEM;
    }
    for (int64_t blk = 0; blk < n_blocks; ++blk) {
        const double* xb = x + blk * T;
        const double* db = d ? d + blk * T : NULL;
        /* branch metrics: nearest entry of every subset at every step */
        for (int t = 0; t < NS; ++t) {
            for (int j = 0; j < 4; ++j) {
                double best = INFINITY;
                uint32_t best_i = 0;
                for (int64_t i = 0; i < per_subset; ++i) {
                    const double* row = cb + (4 * i + j) * V;
                    double dist = 0.0;
                    for (int v = 0; v < V; ++v) {
                        const double diff = xb[t * V + v] - row[v];
                        dist += weight_at(db, t * V + v) * diff * diff;
                    }
                    if (dist < best) {
                        best = dist;
                        best_i = (uint32_t)i;
                    }
                }
                e[4 * t + j] = best;
                idx[4 * t + j] = best_i;
            }
        }
        /* Viterbi over the 8 states */
        double M[8], Mn[8];
        for (int s = 0; s < 8; ++s)
            M[s] = (fixed_start < 0 || s == (int)(fixed_start & 7)) ? 0.0 : INFINITY;
        for (int t = 0; t < NS; ++t) {
            for (int s2 = 0; s2 < 8; ++s2) {
                double best = INFINITY;
                int bs = 0, bz = 0;
                for (int s = 0; s < 8; ++s)
                    for (int z = 0; z < 2; ++z) {
                        if (ub8_next(s, z) != s2) continue;
                        const double c = M[s] + e[4 * t + 2 * z + ub8_p(s)];
                        if (c < best) {
                            best = c;
                            bs = s;
                            bz = z;
                        }
                    }
                Mn[s2] = best;
                bp_state[8 * t + s2] = (uint8_t)bs;
                bp_z[8 * t + s2] = (uint8_t)bz;
            }
            for (int s = 0; s < 8; ++s) M[s] = Mn[s];
        }
        int s_end = 0;
        for (int s = 1; s < 8; ++s)
            if (M[s] < M[s_end]) s_end = s;
        cost[blk] = M[s_end];
        /* traceback: the state before step t and the branch bit taken */
        uint32_t* wb = bits + blk * W;
        memset(wb, 0, sizeof(uint32_t) * (size_t)W);
        int s = s_end;
        for (int t = NS - 1; t >= 0; --t) {
            const int prev = bp_state[8 * t + s];
            const int z = bp_z[8 * t + s];
            const uint32_t i = idx[4 * t + 2 * z + ub8_p(prev)];
            put_symbol(wb, K, t + 1, ((uint32_t)z << m) | i);
            s = prev;
        }
        start_state[blk] = (uint32_t)s;
    }
    free(e); free(idx); free(bp_state); free(bp_z);
    return ORACLE_OK;
}

/* Decode of the 8-state set-partitioned trellis: from sigma_0 = start & 7,
 * step t reads (z, i), emits row 4 i + 2 z + p(sigma_{t-1}), moves to
 * sigma_t = next(sigma_{t-1}, z). */
int oracle_ub8_decode(const uint32_t* bits, const uint32_t* start_state, const double* cb, int V,
                      int m, int T, int64_t n_blocks, double* y)
{
    if (V < 1 || m < 0 || m > 16 || T < 1 || T % V != 0 || n_blocks < 0) return ORACLE_EINVAL;
    if (n_blocks == 0) return ORACLE_OK;
    if (!bits || !start_state || !cb || !y) return ORACLE_EINVAL;
    const int NS = T / V;
    const int K = 1 + m;
    const int W = oracle_words_per_block(K, NS);
    for (int64_t blk = 0; blk < n_blocks; ++blk) {
        int s = (int)(start_state[blk] & 7u);
        for (int t = 1; t <= NS; ++t) {
            const uint32_t sym = get_symbol(bits + blk * W, K, t);
            const int z = (int)(sym >> m);
            const int64_t i = (int64_t)(sym & (((uint32_t)1 << m) - 1));
            const double* row = cb + (4 * i + 2 * z + ub8_p(s)) * V;
            for (int v = 0; v < V; ++v) y[blk * T + (t - 1) * V + v] = row[v];
            s = ub8_next(s, z);
        }
    }
    return ORACLE_OK;
}
