// ldlq.cu -- the error-feedback step between coding blocks.
//
// The 2-bit post's section on error feedback (LDLQ from QuIP): columns are
// quantised in order and each one's error moves onto the columns still to be
// quantised, in proportions taken from H = E[x x^T]; CurveTQ's abstract applies
// it between coding blocks.  With H = U diag(d) U^T (U unit upper triangular),
// the targets of column block B = [c0, c0 + n) are
//
//     X[r, c] = W[r, c0 + c] + sum_{i < c0} (W[r, i] - Q[r, i]) U[i, c0 + c]
//
// a rows x n x c0 product whose left operand, the error W - Q of the blocks
// already coded, is formed while its tile is staged.  Summed over the column
// blocks this is rows * cols^2 / 2 multiply-adds, a small fraction of the
// Viterbi work of the same matrix, so it runs on the fp32 FMA pipe: the targets
// decide the trellis path, and a TF32 tensor-core product would put a relative
// error near 1e-3 into them.
#include "common.cuh"

namespace tcq {

namespace {

constexpr int BM = 128;  // rows of W per CTA tile
constexpr int BN = 64;   // target columns per CTA tile
constexpr int BK = 16;   // reduction depth per stage
constexpr int TM = 8;    // rows per thread
constexpr int TN = 4;    // columns per thread
constexpr int kThreads = (BM / TM) * (BN / TN);  // 256
constexpr int A_PER_THREAD = BM * BK / kThreads;  // 8
constexpr int B_PER_THREAD = BK * BN / kThreads;  // 4

// Shared tiles: the error tile transposed (As[k][m]) so that a thread's TM rows
// are one contiguous run, each k row padded by 4 words so that the transposing
// stores of 16 consecutive k spread over the banks; the U tile as stored (Bs[k][n]).
constexpr int AP = BM + 4;
struct __align__(16) FeedbackSmem {
    float As[2][BK][AP];
    float Bs[2][BK][BN];
};

__global__ void __launch_bounds__(kThreads) feedback_kernel(FeedbackArgs a)
{
    __shared__ FeedbackSmem sm;
    const int tid = threadIdx.x;
    const int tm = tid / (BN / TN);  // 0..15
    const int tn = tid % (BN / TN);  // 0..15
    const long long m0 = (long long)blockIdx.y * BM;
    const int n0 = blockIdx.x * BN;
    const long long K = a.c0;

    float ra[A_PER_THREAD];
    float rb[B_PER_THREAD];
    // Stage k0..k0+BK of the error tile and the U tile into registers (zero
    // outside the matrix).
    auto fetch = [&](long long k0) {
#pragma unroll
        for (int i = 0; i < A_PER_THREAD; ++i) {
            const int idx = tid + i * kThreads;
            const int m = idx / BK, kk = idx % BK;
            const long long r = m0 + m, c = k0 + kk;
            float v = 0.f;
            if (r < a.rows && c < K) {
                const long long o = r * a.cols + c;
                v = __ldg(a.w + o) - __ldg(a.q + o);
            }
            ra[i] = v;
        }
#pragma unroll
        for (int i = 0; i < B_PER_THREAD; ++i) {
            const int idx = tid + i * kThreads;
            const int kk = idx / BN, n = idx % BN;
            const long long c = k0 + kk;
            float v = 0.f;
            if (c < K && n0 + n < a.n) v = __ldg(a.u + c * a.cols + a.c0 + n0 + n);
            rb[i] = v;
        }
    };
    auto stash = [&](int buf) {
#pragma unroll
        for (int i = 0; i < A_PER_THREAD; ++i) {
            const int idx = tid + i * kThreads;
            sm.As[buf][idx % BK][idx / BK] = ra[i];
        }
#pragma unroll
        for (int i = 0; i < B_PER_THREAD; ++i) {
            const int idx = tid + i * kThreads;
            sm.Bs[buf][idx / BN][idx % BN] = rb[i];
        }
    };

    float acc[TM][TN];
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;

    const long long n_stages = (K + BK - 1) / BK;
    if (n_stages > 0) {
        fetch(0);
        stash(0);
        __syncthreads();
        for (long long s = 0; s < n_stages; ++s) {
            const int buf = (int)(s & 1);
            if (s + 1 < n_stages) fetch((s + 1) * BK);
#pragma unroll
            for (int kk = 0; kk < BK; ++kk) {
                const float4 a0 = *reinterpret_cast<const float4*>(&sm.As[buf][kk][tm * TM]);
                const float4 a1 = *reinterpret_cast<const float4*>(&sm.As[buf][kk][tm * TM + 4]);
                const float4 b0 = *reinterpret_cast<const float4*>(&sm.Bs[buf][kk][tn * TN]);
                const float av[TM] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                const float bv[TN] = {b0.x, b0.y, b0.z, b0.w};
#pragma unroll
                for (int i = 0; i < TM; ++i)
#pragma unroll
                    for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
            }
            if (s + 1 < n_stages) stash(buf ^ 1);
            __syncthreads();
        }
    }

    // X = W[:, c0 + c] + accumulated feedback
#pragma unroll
    for (int i = 0; i < TM; ++i) {
        const long long r = m0 + tm * TM + i;
        if (r >= a.rows) break;
#pragma unroll
        for (int j = 0; j < TN; ++j) {
            const int c = n0 + tn * TN + j;
            if (c < a.n) a.x[r * a.x_ld + c] = __ldg(a.w + r * a.cols + a.c0 + c) + acc[i][j];
        }
    }
}

}  // namespace

cudaError_t launch_feedback(const FeedbackArgs& a, cudaStream_t stream)
{
    if (a.rows <= 0 || a.n <= 0) return cudaSuccess;
    const dim3 grid((unsigned)((a.n + BN - 1) / BN), (unsigned)((a.rows + BM - 1) / BM));
    feedback_kernel<<<grid, kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace tcq
