// common.cuh -- device helpers and the internal launch interface shared by the
// encoder and decoder kernels of the TCQ library.  Nothing here is visible
// through the C ABI.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/tcq.h"

namespace tcq {

// Arguments of one encode launch (validated on the host before launch).
struct EncodeArgs {
    const float* x;        // block b at x + b * x_stride, T values
    const float* d;        // block b at d + b * d_stride (0: one row for all), or nullptr (d_t = 1)
    const void* cb;        // 2^L entries
    int cb_f16;            // 1: binary16 entries, 0: binary32
    int L, K, T, W;        // state bits, bits per weight, block length, words per block
    long long n_blocks;
    uint32_t* start_state; // block b at start_state[b * out_stride]
    uint32_t* bits;        // block b at bits + b * out_stride * W
    float* path_cost;      // block b at path_cost[b * out_stride]
    long long x_stride, d_stride, out_stride;
    const uint32_t* fixed_start;  // block b starts in fixed_start[b] (low L-k bits), or nullptr: free
    unsigned char* ws;     // workspace base: gridDim.x slots of slot_bytes
    size_t slot_bytes;
    int V = 1;             // weights per trellis step (kV bits shifted in; codebook [2^L][V])
};

// Device-side error flags (tcq_device_errors in tcq.h).
constexpr unsigned int kDevErrWaitTimeout = TCQ_DEVERR_WAIT_TIMEOUT;
constexpr unsigned int kDevErrBounds = TCQ_DEVERR_BOUNDS;

// Index checks of the TCQ_DEBUG build: TCQ_IN_BOUNDS(i, n) is true when
// 0 <= i < n and otherwise ORs kDevErrBounds into the device error word; the
// caller then skips the access.  In the regular build it is the constant true
// and its arguments are not evaluated, so the kernels compile unchanged.
#ifdef TCQ_DEBUG
extern __device__ unsigned int g_tcq_device_errors;
__device__ __forceinline__ bool dbg_in_bounds(long long i, long long n)
{
    if (i >= 0 && i < n) return true;
    atomicOr(&g_tcq_device_errors, kDevErrBounds);
    return false;
}
#define TCQ_IN_BOUNDS(i, n) ::tcq::dbg_in_bounds((long long)(i), (long long)(n))
#else
#define TCQ_IN_BOUNDS(i, n) true
#endif

// Host: device address of the current device's error word (looked up on every
// call made outside stream capture), or nullptr.
unsigned int* device_error_word(cudaStream_t stream);

// A value the compiler must treat as unknown at each use: a volatile move keeps
// a per-block product such as b * x_stride at its use instead of being hoisted
// out of a persistent loop, where the extra live registers slowed the 128-register
// L=16 encoder by 15% (measured, 181 vs 157 ms on 59,200 blocks).
__device__ __forceinline__ long long opaque(long long v)
{
    long long r;
    asm volatile("mov.b64 %0, %1;" : "=l"(r) : "l"(v));
    return r;
}

// Blocks longer than this many trellis steps have their path metrics shifted
// by a common constant every 64 steps (state 0's metric), so that they stay
// near 0, where fp32 still resolves the differences that decide each argmin;
// without it a block of 2^20 steps grows metrics near 1e5 and loses about
// 7e-5 of the optimal cost to mis-decided near-ties.  Costs are recomputed
// along the traced path, so the shift does not reach them.
constexpr int kRenormAfter = 1024;

struct DecodeArgs {
    const uint32_t* bits;         // block b at bits + b * in_stride * W
    const uint32_t* start_state;  // block b at start_state[b * in_stride]
    const void* cb;
    int cb_f16;
    int L, K, T, W;
    long long n_blocks;
    float* y;                     // block b at y + b * y_stride
    long long in_stride, y_stride;
};

// Error feedback into one column block: x[r * x_ld + c] = w[r, c0 + c] +
// sum_{i < c0} (w[r, i] - q[r, i]) u[i, c0 + c] for r < rows, c < n; w, q are
// [rows, cols] and u [cols, cols], row-major.
struct FeedbackArgs {
    const float* w;
    const float* q;
    const float* u;
    long long rows, cols, c0;
    int n;
    float* x;
    long long x_ld;
    unsigned int* err;  // device error word (a bounded wait that gave up), or nullptr
};

struct GemvArgs {
    const uint32_t* bits;         // [rows * cols / T, W]
    const uint32_t* start_state;  // [rows * cols / T]
    const float* scale;           // [rows * cols / T] or nullptr
    const void* cb;
    int cb_f16;
    int L, K, T, W;
    long long rows, cols;
    const float* x;               // [cols]
    float* y;                     // [rows]
};

// Soft (forward-backward) quantization of n_blocks blocks at temperature tau.
struct BcjrArgs {
    const float* x;        // [n_blocks, T]
    const float* d;        // [n_blocks, T] or nullptr (d_t = 1)
    const void* cb;
    int cb_f16;
    int L, K, T;
    long long n_blocks;
    float w_scale;         // log2(e) / tau: branch metrics in log2 units of exp(-J / tau)
    double tau_ln2;        // tau * ln 2: F = -tau_ln2 * log2 Z
    float* y;              // [n_blocks, T] soft codewords
    float* free_energy;    // [n_blocks] or nullptr
    unsigned char* ws;     // gridDim.x slots of slot_bytes
    size_t slot_bytes;
};

// Encode over the 8-state set-partitioned trellis (ub8.cu): n_blocks blocks of
// T weights, T / V steps of V weights and 1 + m bits each.
struct Ub8EncodeArgs {
    const float* x;               // [n_blocks, T]
    const float* d;               // [n_blocks, T] or nullptr (d = 1)
    const void* cb;               // union codebook [4 * 2^m, V]
    int cb_f16;
    int V, m, T, W;               // W = words per block
    long long n_blocks;
    const uint32_t* fixed_start;  // [n_blocks] (low 3 bits) or nullptr: free start
    uint32_t* start_state;        // [n_blocks]
    uint32_t* bits;               // [n_blocks, W]
    float* path_cost;             // [n_blocks]
};

struct Ub8DecodeArgs {
    const uint32_t* bits;         // [n_blocks, W]
    const uint32_t* start_state;  // [n_blocks], low 3 bits read
    const void* cb;
    int cb_f16;
    int V, m, T, W;
    long long n_blocks;
    float* y;                     // [n_blocks, T]
};

// One codebook entry, widened exactly to fp32.
__device__ __forceinline__ float load_codeword(const void* cb, int f16, uint32_t s)
{
    if (f16) return __half2float(reinterpret_cast<const __half*>(cb)[s]);
    return reinterpret_cast<const float*>(cb)[s];
}

// Named barrier over `count` threads (a multiple of 32).
__device__ __forceinline__ void named_barrier(int id, int count)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Writes one block's packed symbols from the last symbol back to the first.
// Stream bit p is bit 31 - (p mod 32) of word p / 32; symbol t (1-based)
// occupies stream bits [(t-1)k, tk), most significant bit first.  Every word
// from W-1 down to 0 is written exactly once, unused low bits of the last word
// stay zero.
struct BackwardBitWriter {
    uint32_t* words;
    int idx;      // word being filled
    uint32_t cur; // its bits so far

    __device__ __forceinline__ BackwardBitWriter(uint32_t* w, int W) : words(w), idx(W - 1), cur(0) {}

    __device__ __forceinline__ void put(int t, int k, uint32_t sym)
    {
        const int p1 = t * k - 1;  // stream position of the symbol's last bit
        const int w1 = p1 >> 5;
        if (w1 != idx) {           // the previous symbol closed word idx
            words[idx] = cur;
            idx = w1;
            cur = 0;
        }
        const int nlow = (p1 & 31) + 1;  // symbol bits that land in word w1
        if (nlow >= k) {
            cur |= sym << (32 - nlow);
        } else {                          // straddles words w1 - 1 and w1
            cur |= (sym & ((1u << nlow) - 1u)) << (32 - nlow);
            words[idx] = cur;
            idx = w1 - 1;
            cur = sym >> nlow;
        }
    }

    __device__ __forceinline__ void finish() { words[idx] = cur; }
};

// Lexicographic (value, state) minimum: the smallest state wins a tie.
__device__ __forceinline__ void keep_best(float v, uint32_t s, float& bv, uint32_t& bs)
{
    if (v < bv || (v == bv && s < bs)) {
        bv = v;
        bs = s;
    }
}

// ---------------------------------------------------------------------------
// host-side launch interface
// ---------------------------------------------------------------------------
struct EncodeKernelInfo {
    const char* name;
    int nteam;                              // blocks one CTA advances together
    int threads;                            // CTA size
    int max_ctas_per_sm;                    // cap on resident CTAs (0: occupancy decides)
    size_t (*slot_bytes)(int L, int K, int T);  // workspace per CTA
    size_t (*smem_bytes)(int L, int K, int T);  // dynamic shared memory per CTA
    const void* kernel;                     // for occupancy queries
    cudaError_t (*launch)(const EncodeArgs&, int grid, cudaStream_t);
};

// nullptr if no specialised grouped kernel exists for (L, k, codebook dtype).
const EncodeKernelInfo* find_grouped_kernel(int L, int K, int cb_f16);
// nullptr if no one-warp-per-block kernel exists for (L, k) and blocks of T steps.
const EncodeKernelInfo* find_warp_kernel(int L, int K, int T);
const EncodeKernelInfo* generic_kernel_info(int L, int K);
// nullptr if no compile-time vector-trellis kernel exists for (L, k, V, dtype);
// its size callbacks take (L, k V, steps per block) like the runtime kernel's.
const EncodeKernelInfo* find_vec_kernel(int L, int k, int V, int cb_f16);

cudaError_t launch_feedback(const FeedbackArgs& a, cudaStream_t stream);
size_t bcjr_slot_bytes(int L, int K, int T);
int bcjr_ctas_per_sm(int L, int K, int cb_f16);
cudaError_t launch_bcjr(const BcjrArgs& a, int grid, cudaStream_t stream);
cudaError_t launch_decode(const DecodeArgs& a, int num_sms, cudaStream_t stream);
// vector trellis: a.K = k V bits per step, a.T weights per block (V | T)
cudaError_t launch_decode_vec(const DecodeArgs& a, int V, int num_sms, cudaStream_t stream);
cudaError_t launch_gemv_vec(const GemvArgs& a, int V, int num_sms, cudaStream_t stream);
// Drops [base, base + bytes) from L2 without write-back (base 128-byte aligned).
cudaError_t launch_discard_l2(void* base, size_t bytes, int num_sms, cudaStream_t stream);
cudaError_t launch_gemv(const GemvArgs& a, int num_sms, cudaStream_t stream);
// 8-state set-partitioned trellis: shared memory per CTA, and the launches
size_t ub8_encode_smem_bytes(int V, int m, int T);
size_t ub8_decode_smem_bytes(int V, int m, int T);
cudaError_t launch_ub8_encode(const Ub8EncodeArgs& a, int num_sms, cudaStream_t stream);
cudaError_t launch_ub8_decode(const Ub8DecodeArgs& a, int num_sms, cudaStream_t stream);

}  // namespace tcq
