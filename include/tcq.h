/*
 * tcq.h -- C ABI of the B200 (sm_100a) trellis-coded quantization library.
 *
 * Trellis-coded quantization (TCQ) of weight blocks over the bitshift trellis
 * with a per-coordinate weighted branch metric, and the matching decoder.
 *
 * The operation, and where the sources define it:
 *   - "QTIP: Quantization with Trellises and Incoherence Processing" (abstract):
 *     TCQ with a stateful decoder over a hardware-efficient "bitshift" trellis,
 *     lookup codes (one codeword per state).
 *   - "How do you fit a 4B LLM in 1.24 GB? Trellis-coded 2-bit" (sections on
 *     trellis-coded quantization and the Viterbi search): the state picks the
 *     coset for the next weight, the written bits pick the value and set the
 *     next state; the encoder is the Viterbi dynamic program, linear in length;
 *     decoding walks the bits, advancing the state and fetching the codeword.
 *   - CurveTQ abstract (aggregator page for paper 2610.09212): the Viterbi
 *     branch metric weighted per coordinate by the diagonal d_j of the
 *     Hessian's LDL factor, and a start state stored per coding block.
 *
 * Notation for one block of T weights: state bits L, bits per weight k,
 * mask = 2^L - 1, codebook c[0 .. 2^L).
 *     s_t = ((s_{t-1} << k) | b_t) & mask,   y_t = c[s_t],   t = 1..T
 *     J   = sum_t d_t (x_t - y_t)^2
 * tcq_encode returns, per block, a start state and bitstream b_1..b_T that
 * minimise J over every start state and every bitstream (a free start).
 *
 * Storage format:
 *   - start_state: one uint32 per block, the canonical value s_1 >> k
 *     (< 2^(L-k)).  Decoders ignore its bits above L-k.
 *   - bits: W = ceil(T*k/32) uint32 words per block.  Symbol t occupies stream
 *     bits [(t-1)k, tk), most significant bit first; stream bit p is bit
 *     31 - (p mod 32) of word p/32; unused bits of the last word are zero.
 *     s_t is therefore the last L bits of (start_state || stream[0, tk)).
 *
 * Conventions for every entry point:
 *   - All array pointers are DEVICE pointers owned by the caller.  The library
 *     never allocates, never frees and keeps no global state (thread-safe),
 *     with two documented exceptions: tcq_encode_static_scratch's fixed device
 *     array and the device error word read by tcq_device_errors (see there).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream) and never synchronise.  Device-side failures surface on
 *     the stream like any kernel failure.
 *   - Arguments are validated on the host before anything is launched; a
 *     rejected call launches nothing and writes nothing.
 *   - No C++ exception crosses the ABI.
 *   - Preconditions the host cannot check (values in device memory): x, d and
 *     the codebook are finite and d_t >= 0.  Outside them the returned path
 *     and cost are unspecified, but every memory access stays in bounds.
 */
#ifndef TCQ_H_
#define TCQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* tcq_stream_t;

typedef enum {
    TCQ_OK = 0,
    TCQ_ERR_INVALID_ARG = 1, /* null pointer, misaligned pointer, bad size      */
    TCQ_ERR_UNSUPPORTED = 2, /* L, k or T outside the supported ranges          */
    TCQ_ERR_WORKSPACE = 3,   /* workspace smaller than one resident CTA needs   */
    TCQ_ERR_CUDA = 4,        /* a CUDA runtime call or a launch failed          */
    TCQ_ERR_INTERNAL = 5     /* a library invariant broke (report it)           */
} tcq_status;

typedef enum {
    TCQ_F32 = 0, /* codebook entries are IEEE binary32 */
    TCQ_F16 = 1, /* codebook entries are IEEE binary16 */
    TCQ_MAD = 2  /* no table: the computed code below; the codebook pointer is
                    ignored and may be NULL */
} tcq_dtype;

/*
 * The computed (lookup-free) code selected by TCQ_MAD.  QTIP (abstract)
 * introduces codes for the bitshift trellis from lookup-only tables to
 * codewords computed from the state, without a formula; this library's code is
 *     v = 0x9E3779B1 * s mod 2^32,   c[s] = (v_2 + v_3 - 255) / 128
 * with v_2, v_3 bits 16..23 and 24..31 of v: a multiplicative hash of the state
 * and the sum of its high two bytes, every codeword exact in binary16.  Decode
 * and the matrix-vector product compute it per weight; the encoders and the
 * soft quantizer write it as a binary16 table to the front of their workspace
 * (the workspace queries include it) and then run as for TCQ_F16.
 */
#define TCQ_MAD_MULTIPLIER 0x9E3779B1u

/* Supported ranges: 1 <= k <= TCQ_MAX_K, k <= L <= TCQ_MAX_L, 1 <= T <= TCQ_MAX_T. */
#define TCQ_MAX_L 16
#define TCQ_MAX_K 4
#define TCQ_MAX_T (1 << 20)

/* Words of packed bits per block, ceil(T*k/32); -1 if k or T is out of range. */
int tcq_words_per_block(int k, int T);

/*
 * Workspace bytes tcq_encode wants for this problem on the CURRENT device
 * (enough for every persistent CTA the encoder would keep resident; it holds
 * the Viterbi backpointers, k bits per group of 2^k states per step, double
 * buffered per CTA, and for TCQ_MAD the code's binary16 table in front).  Returns 0 for arguments tcq_encode would reject and for
 * n_blocks == 0.  A smaller workspace is accepted down to one CTA's share: the
 * encoder then runs fewer CTAs, and slower.
 */
size_t tcq_encode_workspace_bytes(int L, int k, int T, int64_t n_blocks, tcq_dtype cb_dtype);

/*
 * Viterbi TCQ encode of n_blocks independent blocks (the sources above: QTIP
 * abstract for the bitshift trellis, the Viterbi section of the 2-bit post,
 * the CurveTQ abstract for the weighted metric and the free start state).
 *
 *   x           fp32 [n_blocks, T] row-major, 4-byte aligned.
 *   d           fp32 [n_blocks, T] row-major, 4-byte aligned; NULL means d_t = 1
 *               (plain Euclidean search).
 *   codebook    2^L entries of cb_dtype, aligned to the entry size.
 *   start_state out: uint32 [n_blocks], canonical start s_1 >> k.
 *   bits        out: uint32 [n_blocks, W], W = tcq_words_per_block(k, T).
 *   path_cost   out: fp32 [n_blocks], J of the returned path (accumulated in
 *               fp64 along the path, rounded once to fp32).
 *   workspace   device scratch of workspace_bytes, 256-byte aligned; its
 *               contents on entry do not matter and are garbage on return
 *               (the call ends by discarding the used part from L2 without
 *               write-back, so nothing else may use it until the call's
 *               work on `stream` has finished).
 *
 * Every returned path is optimal up to fp32 rounding of the search: J of the
 * returned path exceeds the exact minimum by at most a few fp32 rounding
 * errors of the path metrics.  Ties may be broken either way.
 * n_blocks == 0 is a no-op (pointers may then be NULL).
 */
tcq_status tcq_encode(const float* x, const float* d, const void* codebook, tcq_dtype cb_dtype,
                      int L, int k, int T, int64_t n_blocks, uint32_t* start_state,
                      uint32_t* bits, float* path_cost, void* workspace, size_t workspace_bytes,
                      tcq_stream_t stream);

/*
 * Encode with the start state of every block fixed instead of free (the 2-bit
 * post's trellis toy starts in state 0; CurveTQ's free start per coding block
 * is tcq_encode).  Block b minimises J over bitstreams alone from
 * s_0 = fixed_start[b]; only the low L-k bits of fixed_start[b] matter, and the
 * returned start_state[b] equals them.
 *
 *   fixed_start  uint32 [n_blocks], device, 4-byte aligned, not NULL.
 * Everything else, including the workspace and the error codes, as tcq_encode.
 */
tcq_status tcq_encode_fixed_start(const float* x, const float* d, const void* codebook,
                                  tcq_dtype cb_dtype, int L, int k, int T, int64_t n_blocks,
                                  const uint32_t* fixed_start, uint32_t* start_state,
                                  uint32_t* bits, float* path_cost, void* workspace,
                                  size_t workspace_bytes, tcq_stream_t stream);

/*
 * Decode (the 2-bit post's state-tracking table-lookup decoder; QTIP's
 * stateful bitshift decoder): y[b, t-1] = c[s_t] with s_t the last L bits of
 * (start_state[b] || stream[0, tk)).  Bit-exact: y is the exact fp32 widening
 * of the codebook entry.
 *
 *   bits        uint32 [n_blocks, W], 4-byte aligned.
 *   start_state uint32 [n_blocks]; only its low L-k bits are read.
 *   codebook    2^L entries of cb_dtype, aligned to the entry size.
 *   y           out: fp32 [n_blocks, T] row-major, 4-byte aligned.
 * n_blocks == 0 is a no-op.
 */
tcq_status tcq_decode(const uint32_t* bits, const uint32_t* start_state, const void* codebook,
                      tcq_dtype cb_dtype, int L, int k, int T, int64_t n_blocks, float* y,
                      tcq_stream_t stream);

/*
 * Matrix-vector product with a trellis-coded matrix, decoding on the fly (the
 * 2-bit post's Pingala-8 section: the decoder, which advances the state from the
 * bits and fetches each codeword, runs inside the matrix-vector product, so the
 * weights are never materialised).
 *
 * The rows x cols matrix is stored as rows * (cols / T) coding blocks of T
 * consecutive columns, block (r, j) = r * (cols / T) + j covering columns
 * [jT, jT + T) of row r -- what tcq_encode returns for the row-major matrix
 * viewed as [rows * cols / T, T] -- each with optional fp32 scale:
 *     y[r] = sum_j scale[r, j] * sum_t c[s_{r,j,t}] * x[jT + t]
 * accumulated in fp32.
 *
 *   bits, start_state  as tcq_decode, for rows * (cols / T) blocks.
 *   scale              fp32 [rows * cols / T] or NULL (all 1).
 *   x                  fp32 [cols], 16-byte aligned.   y  out: fp32 [rows].
 * Requires T % 4 == 0 and cols % T == 0 (else TCQ_ERR_UNSUPPORTED /
 * TCQ_ERR_INVALID_ARG), and a binary16 codebook when L >= 15 (the table lives
 * in shared memory).  rows == 0 is a no-op.
 */
tcq_status tcq_gemv(const uint32_t* bits, const uint32_t* start_state, const float* scale,
                    const void* codebook, tcq_dtype cb_dtype, int L, int k, int T, int64_t rows,
                    int64_t cols, const float* x, float* y, tcq_stream_t stream);

/*
 * Error-feedback quantisation of a matrix, one column block at a time (the 2-bit
 * post's section on error feedback and LDLQ: each quantised column's error is
 * pushed onto the columns not yet quantised, in proportions set by
 * H = E[x x^T]; CurveTQ's abstract: the feedback runs between coding blocks and
 * the Viterbi metric of a block is weighted by the diagonal of H's LDL
 * factorisation).
 *
 * With H = U diag(d) U^T, U unit upper triangular, and W the rows x cols weight
 * matrix, for each column block B = [jT, jT + T) in order and every row r:
 *     X[r, c] = W[r, c] + sum_{i < jT} (W[r, i] - Q[r, i]) U[i, c]      c in B
 *     coding block (r, j) = tcq_encode of X[r, B] with weights d[B]
 *     Q[r, B] = tcq_decode of that block
 * Only U's entries above its T x T diagonal blocks are read: feedback inside a
 * block is not applied (the Viterbi search codes the block jointly).  The
 * factorisation H -> (U, d) is the caller's.
 *
 *   w           fp32 [rows, cols] row-major.
 *   u           fp32 [cols, cols] row-major.
 *   d           fp32 [cols], or NULL for d = 1.
 *   codebook    as tcq_encode.
 *   q           out: fp32 [rows, cols], the reconstruction Q.
 *   x           out: fp32 [rows, cols], the targets X, or NULL if not wanted.
 *   start_state out: uint32 [rows * cols / T]; bits out: uint32 [rows * cols / T, W];
 *   path_cost   out: fp32 [rows * cols / T]; block (r, j) at index r * (cols / T) + j,
 *               the layout tcq_gemv reads.
 *   workspace   device scratch, 256-byte aligned, at least
 *               tcq_ldlq_workspace_bytes(...) for full speed (it holds one column
 *               block's targets plus an encode workspace for `rows` blocks).
 * Every pointer except d and x must be non-NULL and 4-byte aligned (the codebook
 * to its entry size).  Requires cols % T == 0 and rows <= 65535 * 128, else
 * TCQ_ERR_INVALID_ARG; a workspace too small for the targets and one CTA's
 * encode share returns TCQ_ERR_WORKSPACE.  Launches 3 kernels per column block
 * on `stream`; rows == 0 or cols == 0 is a no-op.  Each block's path and cost
 * have tcq_encode's guarantees for that block's targets.
 */
size_t tcq_ldlq_workspace_bytes(int L, int k, int T, int64_t rows, int64_t cols,
                                tcq_dtype cb_dtype);

tcq_status tcq_ldlq(const float* w, const float* u, const float* d, const void* codebook,
                    tcq_dtype cb_dtype, int L, int k, int T, int64_t rows, int64_t cols, float* q,
                    float* x, uint32_t* start_state, uint32_t* bits, float* path_cost,
                    void* workspace, size_t workspace_bytes, tcq_stream_t stream);

/*
 * Soft trellis quantization (BCJR-QAT abstract: the Viterbi argmax replaced by
 * the BCJR forward-backward sum-product recursion at temperature tau, giving
 * the Boltzmann expectation of the codeword over trellis paths, which returns
 * to the hard code as tau -> 0).
 *
 * Over the paths s_1..s_T of the bitshift trellis (first state free, each of
 * the 2^L first states counted once) with cost J = sum_t d_t (x_t - c[s_t])^2:
 *     P(path)      = exp(-J / tau) / Z
 *     y_soft[b, t] = E_P[c[s_t]]            (the soft codeword)
 *     free_energy[b] = -tau ln Z            (F <= J_min, F -> J_min as tau -> 0)
 * computed in fp32 with the normalising constants summed in fp64.
 *
 *   x, d, codebook  as tcq_encode.
 *   tau             > 0 and finite, with d_t (x_t - c)^2 / tau finite in fp32
 *                   for every t and codeword (else TCQ_ERR_INVALID_ARG for tau
 *                   itself, undefined values otherwise).
 *   y_soft          out: fp32 [n_blocks, T], 4-byte aligned.
 *   free_energy     out: fp32 [n_blocks], or NULL.
 *   workspace       device scratch, 256-byte aligned, at least
 *                   tcq_bcjr_workspace_bytes(...) for full speed; it holds the
 *                   forward values of every step of a block (T * 2^(L-k) fp32)
 *                   per concurrently processed block.  Smaller workspaces run
 *                   fewer blocks at a time; one block's share is the minimum
 *                   (else TCQ_ERR_WORKSPACE).
 * n_blocks == 0 is a no-op.  One kernel launch on `stream`.
 */
size_t tcq_bcjr_workspace_bytes(int L, int k, int T, int64_t n_blocks, tcq_dtype cb_dtype);

tcq_status tcq_bcjr(const float* x, const float* d, const void* codebook, tcq_dtype cb_dtype,
                    int L, int k, int T, int64_t n_blocks, float tau, float* y_soft,
                    float* free_energy, void* workspace, size_t workspace_bytes,
                    tcq_stream_t stream);

/*
 * Vector trellis: V weights per trellis step (QTIP abstract: the bitshift
 * trellis with a stateful decoder separates the codebook size from the bitrate
 * and the effective dimension).  Each step shifts k V bits into the L-bit state
 * and the state selects a V-dimensional codeword:
 *     s_t = ((s_{t-1} << kV) | b_t) & (2^L - 1),   y_{(t-1)V + v} = c[s_t][v],
 * and the search minimises J = sum_i d_i (x_i - y_i)^2 over every start state and
 * bitstream.  Bits are packed as for tcq_encode with symbols of kV bits (still
 * k bits per weight, W = ceil(T k / 32)); start_state = s_1 >> kV.
 *
 *   codebook  2^L rows of V entries (row-major), binary32 or binary16; the
 *             computed code (TCQ_MAD) is scalar: TCQ_ERR_UNSUPPORTED for V > 1.
 * Supported: 1 <= V <= 8, V | T, k V <= min(L, 8) (else TCQ_ERR_UNSUPPORTED).
 * V == 1 is exactly tcq_encode / tcq_decode.  L = 16, k = 2, V = 2 with a
 * binary16 codebook runs compile-time kernels: the encoder when the codebook is
 * 4-byte aligned, the decoder when it is 16-byte aligned, T % 8 == 0 and y is
 * 16-byte aligned; every other V > 1 shape runs the runtime-(L, k) kernels.
 * Results do not depend on which kernel runs beyond fp32 rounding of the search
 * (costs within the tolerance of tcq_encode; decode is exact either way), and
 * the workspace query covers either encoder.  Other arguments, outputs and
 * errors as tcq_encode / tcq_decode.
 */
size_t tcq_encode_vec_workspace_bytes(int L, int k, int V, int T, int64_t n_blocks,
                                      tcq_dtype cb_dtype);

tcq_status tcq_encode_vec(const float* x, const float* d, const void* codebook, tcq_dtype cb_dtype,
                          int L, int k, int V, int T, int64_t n_blocks, uint32_t* start_state,
                          uint32_t* bits, float* path_cost, void* workspace,
                          size_t workspace_bytes, tcq_stream_t stream);

tcq_status tcq_decode_vec(const uint32_t* bits, const uint32_t* start_state, const void* codebook,
                          tcq_dtype cb_dtype, int L, int k, int V, int T, int64_t n_blocks,
                          float* y, tcq_stream_t stream);

/*
 * Decode-in-matvec for the vector trellis: tcq_gemv's product, with each
 * block's weights those of tcq_decode_vec (step t of block (r, j) holds columns
 * jT + (t-1)V .. jT + tV - 1):
 *     y[r] = sum_j scale[r, j] * sum_t sum_v c[s_{r,j,t}][v] * x[jT + (t-1)V + v]
 * accumulated in fp32.  Arguments as tcq_gemv plus V; shapes as tcq_encode_vec
 * (TCQ_MAD is TCQ_ERR_UNSUPPORTED for V > 1); cols % T == 0 (else
 * TCQ_ERR_INVALID_ARG); V == 1 is exactly tcq_gemv.  L = 16, k = 2, V = 2 with a
 * 16-byte aligned binary16 codebook and T % 8 == 0 runs a compile-time kernel
 * (seven eighths of the pair table in shared memory), every other shape a
 * runtime kernel.  rows == 0 is a no-op.
 */
tcq_status tcq_gemv_vec(const uint32_t* bits, const uint32_t* start_state, const float* scale,
                        const void* codebook, tcq_dtype cb_dtype, int L, int k, int V, int T,
                        int64_t rows, int64_t cols, const float* x, float* y, tcq_stream_t stream);

/*
 * Trellis-coded quantization over Ungerboeck's 8-state set-partitioned trellis
 * (the 2-bit post, Pingala-8 section: an 8-state set-partitioned trellis with
 * Ungerboeck's labels over symbols of several weights at about 2 bits per
 * weight; its section on trellis-coded quantization: the state decides which
 * subset the next symbol may use, the written bits pick a value inside the
 * subset and set the next state, so the format holds twice as many values as
 * its bits address; its background reading, Marcellin and Fischer's
 * trellis-coded quantization, fixes the labels used here).  The pages give
 * neither labels nor codebook; this library's reading:
 *
 *   - Union codebook: 4 * 2^m rows of V values (row-major); row r belongs to
 *     subset D_{r mod 4} and is entry r >> 2 of it.  For V = 1 and rows sorted
 *     ascending this is Ungerboeck's partition of an amplitude alphabet.
 *   - Trellis: Ungerboeck's 8-state code for one-dimensional signals (the
 *     rate-1/2 systematic feedback code with parity-check polynomials
 *     h0 = D^3 + D + 1, h1 = D^2, octal 13 and 04).  State sigma = 4p + 2q + r;
 *     the branch with bit z uses subset D_{2z+p} and leads to state
 *     4 (p ^ q) + 2 (r ^ z) + p.  Both branches out of a state use the two
 *     subsets of one half, {D_p, D_{p+2}}.
 *   - A step codes V consecutive weights with 1 + m bits, symbol (z << m) | i,
 *     and reconstructs them as row 4 i + 2 z + p.  Symbols are packed like
 *     tcq_encode's (MSB first, symbol t at stream bits [t(1+m), (t+1)(1+m)));
 *     W = tcq_ub8_words_per_block(V, m, T) words per block.  The stored start
 *     state is sigma_0 (0..7).  Pingala-8's symbols of 4 weights at 2 bits per
 *     weight are V = 4, m = 7 (512 rows, 8 bits per step).
 *
 * tcq_ub8_encode returns per block the start state, branch bits and entries
 * that minimise J = sum_i d_i (x_i - y_i)^2 over every path of the trellis (free
 * start, or fixed_start[b] & 7 when fixed_start is not NULL): per step the
 * nearest entry of each subset (fp32, ties to the smaller entry), then the
 * Viterbi recursion over the 8 states (fp32 path metrics, ties to the smaller
 * predecessor and the smaller final state).  path_cost is J of the returned
 * path summed in fp64 and rounded once.  Like tcq_encode, every returned path
 * is optimal up to fp32 rounding of the search.  No workspace: the search of a
 * block lives in shared memory.
 *
 *   x, d            fp32 [n_blocks, T] (d NULL: d = 1), 4-byte aligned.
 *   codebook        4 * 2^m * V entries of cb_dtype (TCQ_F32 or TCQ_F16; the
 *                   computed code is TCQ_ERR_UNSUPPORTED), aligned to the entry.
 *   fixed_start     uint32 [n_blocks] or NULL.
 *   start_state     out: uint32 [n_blocks].   bits: out uint32 [n_blocks, W].
 *   path_cost       out: fp32 [n_blocks].
 * tcq_ub8_decode writes y[b, (t-1)V + v] = row[v] of each step's row; it reads
 * only the low 3 bits of start_state.  Bit-exact (the exact fp32 widening).
 * Supported: 1 <= V <= TCQ_UB8_MAX_V, 0 <= m <= TCQ_UB8_MAX_M, V | T,
 * T / V <= TCQ_UB8_MAX_STEPS (else TCQ_ERR_UNSUPPORTED); pointers as for
 * tcq_encode / tcq_decode (else TCQ_ERR_INVALID_ARG).  n_blocks == 0 is a
 * no-op.  One kernel launch each.
 */
#define TCQ_UB8_MAX_V 8
#define TCQ_UB8_MAX_M 8
#define TCQ_UB8_MAX_STEPS 512

/* ceil((T / V) (1 + m) / 32); -1 for a shape tcq_ub8_encode rejects. */
int tcq_ub8_words_per_block(int V, int m, int T);

tcq_status tcq_ub8_encode(const float* x, const float* d, const void* codebook, tcq_dtype cb_dtype,
                          int V, int m, int T, int64_t n_blocks, const uint32_t* fixed_start,
                          uint32_t* start_state, uint32_t* bits, float* path_cost,
                          tcq_stream_t stream);

tcq_status tcq_ub8_decode(const uint32_t* bits, const uint32_t* start_state, const void* codebook,
                          tcq_dtype cb_dtype, int V, int m, int T, int64_t n_blocks, float* y,
                          tcq_stream_t stream);

/*
 * Device-side failures that do not fault the GPU.  (The sources have no
 * counterpart: this is an engineering part of this library.)  Kernels OR a
 * flag into one error word per device:
 *   TCQ_DEVERR_WAIT_TIMEOUT  a bounded wait gave up: the tensor-core feedback
 *                            product of tcq_ldlq stopped issuing work, waited
 *                            (bounded) for what it had issued, wrote NaN
 *                            targets for its rows and freed its tensor memory;
 *                            the affected blocks then carry non-finite costs.
 *   TCQ_DEVERR_BOUNDS        an index failed its bounds check and the access
 *                            was skipped (only the TCQ_DEBUG build,
 *                            libtcq_debug.so, checks indices).
 * tcq_device_errors synchronises `stream`, returns the current device's flags
 * in *flags (if not NULL) and clears them: TCQ_OK when none is set,
 * TCQ_ERR_INTERNAL when any is, TCQ_ERR_CUDA if the stream or the copy failed.
 * It allocates nothing.  The word is shared by every stream and host thread on
 * the device (the second piece of device state this library keeps, next to
 * tcq_encode_static_scratch's array): read it while no other call runs.
 */
#define TCQ_DEVERR_WAIT_TIMEOUT 0x1u
#define TCQ_DEVERR_BOUNDS 0x2u

tcq_status tcq_device_errors(tcq_stream_t stream, uint32_t* flags);

/* Static, human-readable name of a status code. */
const char* tcq_status_string(tcq_status status);

/*
 * Static name of the encoder kernel tcq_encode would launch for this shape with
 * blocks of at most 1024 steps ("warp<L,k>" for the one-warp-per-block kernel
 * of small trellises, "grouped<L,k,...>" for the specialised add-compare-select
 * kernels, "generic" for the runtime-(L,k) kernel), or "unsupported".  Longer
 * blocks at L = 8, k = 2 take "grouped<8,2,...>".
 */
const char* tcq_encode_path(int L, int k, tcq_dtype cb_dtype);

/*
 * Encoder for callers that cannot allocate device memory.  (The sources have no
 * counterpart: this is an engineering addition of this library.)
 *
 * Some callers cannot provide tcq_encode's workspace: a host program whose own
 * pool allocator owns the GPU's memory (a raw cudaMalloc would fail or fragment
 * that pool), code held to a fixed device-memory budget, or a latency-critical
 * path that must not call cudaMalloc because it may synchronise the device.
 * This entry point takes the same arguments as tcq_encode without the
 * workspace, and allocates nothing: it calls no cudaMalloc, cudaFree or other
 * allocating routine.  Its scratch is a single file-scope device array of
 * TCQ_STATIC_SCRATCH_BYTES that every GPU loading this library holds until the
 * process exits.
 *
 *   - Every call made outside stream capture looks up that array's device
 *     address on the current device (a host query, no allocation) and caches
 *     it; a call made while `stream` is capturing uses the cached address, so
 *     make at least one call on the device before any stream capture.  After a
 *     cudaDeviceReset in the caller's process the array may move: the next call
 *     outside capture picks up the new address, but a CUDA graph captured
 *     before the reset holds the old one and must not be replayed.  Calls are
 *     thread-safe on the host.
 *   - The scratch limits concurrency, not problem size: blocks are processed by
 *     as many persistent CTAs as the scratch holds (at L=16, k=2, T=256 each CTA
 *     needs about 2 MiB, so about 15 CTAs run and the call is roughly 10x slower
 *     than tcq_encode with a full workspace).  A shape whose single-CTA share,
 *     tcq_encode_workspace_bytes(L, k, T, 1, cb_dtype), exceeds
 *     TCQ_STATIC_SCRATCH_BYTES returns TCQ_ERR_WORKSPACE: at L = 16 with k = 2
 *     or 3 the longest block is T = 4096 for a binary16 table and T = 4080 for
 *     TCQ_MAD (whose table takes 128 KiB of the array).
 *   - Every call uses the same array.  Nothing in it needs to start at zero, and
 *     a call never depends on what an earlier call left there; but calls that
 *     overlap on the GPU (two streams, or two host threads on different
 *     streams) race on it and produce garbage.  Serialise them.
 * Other arguments, outputs and errors: as tcq_encode.
 */
#define TCQ_STATIC_SCRATCH_BYTES (32u * 1024u * 1024u)

tcq_status tcq_encode_static_scratch(const float* x, const float* d, const void* codebook,
                                     tcq_dtype cb_dtype, int L, int k, int T, int64_t n_blocks,
                                     uint32_t* start_state, uint32_t* bits, float* path_cost,
                                     tcq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* TCQ_H_ */
