// acs_generic.cu -- Viterbi TCQ encoder for any supported (L, k) at run time.
//
// Same search and the same fp32 arithmetic as the grouped kernels (the
// u-formulation of the recurrence, e = fma(-sqrt(d), c, sqrt(d) x),
// cand = fma(e, e, M), strict compares so the smallest predecessor wins a tie),
// without their compile-time layout: one thread per u per step, codewords read
// through the L1 cache, one byte of backpointer per (step, u) in the workspace,
// and the traceback done by thread 0 after each block's forward pass.  It
// covers shapes the grouped kernels do not (L < 2k, odd sizes) and the vector
// trellis (V weights per step: kV bits shifted in, a V-dimensional codeword per
// state, the branch metric summed over the V weights), and serves as a second,
// independent GPU path in the tests; it is not tuned.
#include "common.cuh"

namespace tcq {

namespace {

constexpr int kGenericThreads = 256;
constexpr int kMaxV = 8;  // weights per step
// path metrics stay in shared memory up to this many bytes of ping-pong, else
// they go to the workspace slot (global memory, L2 resident)
constexpr size_t kGenericSmemMetricBytes = 96 * 1024;

__host__ __device__ inline size_t round256(size_t v) { return (v + 255) & ~(size_t)255; }

__host__ __device__ inline size_t generic_metric_bytes(int L, int K)
{
    return 2 * sizeof(float) * ((size_t)1 << (L - K));
}

__host__ __device__ inline bool generic_metrics_in_smem(int L, int K)
{
    return generic_metric_bytes(L, K) <= kGenericSmemMetricBytes;
}

__host__ __device__ inline size_t generic_bp_bytes(int L, int K, int T)
{
    return round256((size_t)(T - 1) * ((size_t)1 << (L - K)));
}

__global__ void __launch_bounds__(kGenericThreads) acs_generic_kernel(EncodeArgs a)
{
    extern __shared__ __align__(16) float gsm[];
    __shared__ float redv[kGenericThreads / 32];
    __shared__ uint32_t reds[kGenericThreads / 32];
    __shared__ uint32_t fin;

    // a step shifts in K = k V bits and covers V weights; NS steps per block
    const int L = a.L, V = a.V, K = a.K * a.V, NS = a.T / a.V;
    const int LK = L - K;
    const uint32_t NU = 1u << LK;
    const int H = 1 << K;
    unsigned char* slot = a.ws + (size_t)blockIdx.x * a.slot_bytes;
    uint8_t* bp = slot;
    float* Mbase = generic_metrics_in_smem(L, K)
                       ? gsm
                       : reinterpret_cast<float*>(slot + generic_bp_bytes(L, K, NS));
#ifdef TCQ_DEBUG
    const long long x_n = (a.n_blocks - 1) * a.x_stride + a.T, d_n = (a.n_blocks - 1) * a.d_stride + a.T;
    const long long o_n = (a.n_blocks - 1) * a.out_stride + 1;
    const long long ws_n = (long long)gridDim.x * (long long)a.slot_bytes;
    const long long cb_n = (1LL << L) * V;
#endif

    for (long long b = blockIdx.x; b < a.n_blocks; b += gridDim.x) {
        const float* xb = a.x + b * a.x_stride;
        const float* db = a.d ? a.d + b * a.d_stride : nullptr;
        float bestv = __int_as_float(0x7f800000);
        uint32_t bests = 0xffffffffu;
        // a fixed start s_0 leaves only its successors reachable at step 1
        const uint32_t s0 = a.fixed_start && TCQ_IN_BOUNDS(b, a.n_blocks) ? (a.fixed_start[b] & (NU - 1u)) : 0xffffffffu;
        for (int t = 1; t <= NS; ++t) {
            float ca[kMaxV], cx[kMaxV];
#pragma unroll
            for (int v = 0; v < kMaxV; ++v) {
                if (v < V) {
                    const int i = (t - 1) * V + v;
                    const bool ok = TCQ_IN_BOUNDS(xb + i - a.x, x_n) && (!db || TCQ_IN_BOUNDS(db + i - a.d, d_n));
                    const float sd = db && ok ? sqrtf(db[i]) : 1.f;
                    ca[v] = -sd;
                    cx[v] = ok ? sd * xb[i] : 0.f;
                }
            }
            const float* Mp = Mbase + ((t - 1) & 1) * NU;
            float* Mn = Mbase + (t & 1) * NU;
            for (uint32_t u = threadIdx.x; u < NU; u += blockDim.x) {
                float best = __int_as_float(0x7f800000);
                uint32_t bh = 0;
                for (int h = 0; h < H; ++h) {
                    const uint32_t s = ((uint32_t)h << LK) | u;
                    const float m0 = (s0 == 0xffffffffu || (s >> K) == s0) ? 0.f : __int_as_float(0x7f800000);
                    float v = t == 1 ? m0 : Mp[s >> K];
#pragma unroll
                    for (int w = 0; w < kMaxV; ++w) {
                        if (w < V) {
                            const float c = TCQ_IN_BOUNDS((long long)s * V + w, cb_n) ? load_codeword(a.cb, a.cb_f16, s * V + w) : 0.f;
                            const float e = fmaf(ca[w], c, cx[w]);
                            v = fmaf(e, e, v);
                        }
                    }
                    if (v < best) {
                        best = v;
                        bh = (uint32_t)h;
                    }
                }
                if (t < NS) {
                    Mn[u] = best;
                    if (TCQ_IN_BOUNDS(bp + (size_t)(t - 1) * NU + u - a.ws, ws_n)) bp[(size_t)(t - 1) * NU + u] = (uint8_t)bh;
                } else {
                    keep_best(best, (bh << LK) | u, bestv, bests);
                }
            }
            __syncthreads();
            // long blocks: shift the metrics by state 0's every 64 steps
            if (NS > kRenormAfter && (t & 63) == 0 && t < NS) {
                const float o = Mn[0];
                const float off = (o < __int_as_float(0x7f800000)) ? o : 0.f;
                __syncthreads();
                for (uint32_t u = threadIdx.x; u < NU; u += blockDim.x) Mn[u] -= off;
                __syncthreads();
            }
        }
        // final state: lexicographic (cost, state) minimum over the CTA
        for (int o = 16; o >= 1; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bestv, o);
            const uint32_t os = __shfl_xor_sync(0xffffffffu, bests, o);
            keep_best(ov, os, bestv, bests);
        }
        if ((threadIdx.x & 31) == 0) {
            redv[threadIdx.x >> 5] = bestv;
            reds[threadIdx.x >> 5] = bests;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            float bv = redv[0];
            uint32_t bs = reds[0];
            for (int w = 1; w < (int)(blockDim.x >> 5); ++w) keep_best(redv[w], reds[w], bv, bs);
            fin = bs;
            // traceback, bit packing and the fp64 cost along the path
            BackwardBitWriter bw(a.bits + b * a.out_stride * a.W, a.W);
            uint32_t s = fin;
            double cost = 0.0;
            for (int t = NS; t >= 1; --t) {
                for (int w = 0; w < V; ++w) {
                    const int i = (t - 1) * V + w;
                    if (!TCQ_IN_BOUNDS(xb + i - a.x, x_n) || (db && !TCQ_IN_BOUNDS(db + i - a.d, d_n)) ||
                        !TCQ_IN_BOUNDS((long long)s * V + w, cb_n))
                        continue;
                    const float dv = db ? db[i] : 1.f;
                    const double e = (double)xb[i] - (double)load_codeword(a.cb, a.cb_f16, s * V + w);
                    cost += (double)dv * e * e;
                }
                bw.put(t, K, s & (uint32_t)(H - 1));
                if (t > 1) {
                    const uint32_t u = s >> K;
                    const uint32_t h = TCQ_IN_BOUNDS(bp + (size_t)(t - 2) * NU + u - a.ws, ws_n) ? bp[(size_t)(t - 2) * NU + u] : 0u;
                    s = (h << LK) | u;
                }
            }
            bw.finish();
            if (TCQ_IN_BOUNDS(b * a.out_stride, o_n)) {
                a.start_state[b * a.out_stride] = s >> K;
                a.path_cost[b * a.out_stride] = (float)cost;
            }
        }
        __syncthreads();
    }
}

size_t generic_slot_bytes(int L, int K, int T)
{
    size_t v = generic_bp_bytes(L, K, T);
    if (!generic_metrics_in_smem(L, K)) v += round256(generic_metric_bytes(L, K));
    return v;
}

size_t generic_smem_bytes(int L, int K, int)
{
    return generic_metrics_in_smem(L, K) ? generic_metric_bytes(L, K) : 0;
}

cudaError_t launch_generic(const EncodeArgs& a, int grid, cudaStream_t stream)
{
    const size_t smem = generic_smem_bytes(a.L, a.K * a.V, a.T / a.V);  // per step: kV bits
    cudaError_t e = cudaFuncSetAttribute(acs_generic_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    acs_generic_kernel<<<grid, kGenericThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

// two CTAs per SM: enough to overlap one CTA's serial traceback; more would only
// multiply the workspace
const EncodeKernelInfo kGenericInfo = {"generic", 1, kGenericThreads, 2, &generic_slot_bytes,
                                       &generic_smem_bytes,
                                       reinterpret_cast<const void*>(&acs_generic_kernel),
                                       &launch_generic};

}  // namespace

// K: bits shifted in per step (k V for the vector trellis), at most 8 since a
// backpointer is one byte.  The info's size callbacks take (L, bits per step,
// steps per block).
const EncodeKernelInfo* generic_kernel_info(int L, int K)
{
    if (L < 1 || L > TCQ_MAX_L || K < 1 || K > 8 || K > L) return nullptr;
    return &kGenericInfo;
}

}  // namespace tcq
