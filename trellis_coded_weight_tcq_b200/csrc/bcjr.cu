// bcjr.cu -- soft trellis quantization by the forward-backward (BCJR)
// sum-product recursion at temperature tau.
//
// BCJR-QAT (abstract, aggregator page): the Viterbi minimum over paths becomes
// the Boltzmann distribution P(path) ~ exp(-J(path) / tau) over the same
// bitshift trellis; the soft codeword of position t is E_P[c[s_t]], and it
// returns to the hard Viterbi code as tau -> 0.  The first state is free, each
// of the 2^L first states weighted once.
//
// Arithmetic, in log2 units of exp(-J / tau) (w_t = d_t log2(e) / tau):
//   forward   A_t[u] = sum_h 2^{-w_t (x_t - c[s])^2} A_{t-1}[s >> k],
//             s = (h << (L-k)) | u,  A_0 = 1
//   backward  B_{t-1}[u'] = sum_b 2^{-w_t (x_t - c[s])^2} B_t[s & (2^(L-k) - 1)],
//             s = (u' << k) | b,  B_T = 1
//   posterior of state s = (u' << k) | b at step t:
//             A_{t-1}[u'] 2^{-w_t (x_t - c[s])^2} B_t[s & (2^(L-k) - 1)] / Z
// -- the same reformulation over u = s mod 2^(L-k) as the Viterbi kernels, with
// (min, +) replaced by (log-sum-exp, +).  Both recursions run in the log domain
// (a 2^k-way log-sum-exp per u: one ex2 per state and one lg2 per u), and each
// step subtracts the previous step's maximum so that stored values stay near 0
// where fp32 is precise; the subtracted constants are summed in fp64 and give
// log2 Z and the exact normalisation of every step's posterior.
//
// Layout: one block per CTA at a time (the CTA loops over blocks).  The forward
// pass writes log2 A_t for every step to the CTA's workspace slot; the backward
// pass reads it back, keeps log2 B in a ping-pong pair in the slot, and reduces
// each step's posterior mass and first moment over the CTA.  Only
// __syncthreads waits, and none depends on another CTA.
#include "common.cuh"

namespace tcq {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxH = 16;  // k <= 4

enum BcjrTable { kTabGlobal = 0, kTabF32 = 1, kTabF16 = 2 };

__device__ __forceinline__ float ex2(float v)
{
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

__device__ __forceinline__ float lg2(float v)
{
    float r;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

size_t round256(size_t v) { return (v + 255) & ~(size_t)255; }

__host__ __device__ inline size_t s_bytes(int L, int K, int T)
{
    return ((size_t)T * ((size_t)1 << (L - K)) * sizeof(float) + 255) & ~(size_t)255;
}
__host__ __device__ inline size_t r_bytes(int L, int K)
{
    return (2 * ((size_t)1 << (L - K)) * sizeof(float) + 255) & ~(size_t)255;
}

int table_mode(int L, int cb_f16)
{
    if (((size_t)4 << L) <= 64 * 1024) return kTabF32;
    if (cb_f16 && ((size_t)2 << L) <= 128 * 1024) return kTabF16;
    return kTabGlobal;
}

size_t table_bytes(int L, int mode)
{
    return mode == kTabF32 ? ((size_t)4 << L) : mode == kTabF16 ? ((size_t)2 << L) : 0;
}

// shared memory ahead of the codebook table: per-warp maxima [2][kWarps] and
// per-warp (mass, moment) partials [2][kWarps][2]
constexpr size_t kHeadBytes = 256;

template <int TAB>
__global__ void __launch_bounds__(kThreads) bcjr_kernel(BcjrArgs a)
{
    extern __shared__ __align__(16) unsigned char sm[];
    float* wmax = reinterpret_cast<float*>(sm);  // [2][kWarps]
    float* red = wmax + 2 * kWarps;              // [2][kWarps][2]
    unsigned char* tab = sm + kHeadBytes;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int L = a.L, K = a.K, T = a.T, H = 1 << K, LK = L - K;
    const int NU = 1 << LK;
    const uint32_t low = (uint32_t)NU - 1u;

    if constexpr (TAB == kTabF32) {
        float* t32 = reinterpret_cast<float*>(tab);
        for (int i = tid; i < (1 << L); i += kThreads) t32[i] = load_codeword(a.cb, a.cb_f16, i);
    } else if constexpr (TAB == kTabF16) {
        const uint4* s4 = reinterpret_cast<const uint4*>(a.cb);
        uint4* d4 = reinterpret_cast<uint4*>(tab);
        for (int i = tid; i < (1 << L) / 8; i += kThreads) d4[i] = s4[i];
    }
    __syncthreads();
    auto cw = [&](uint32_t s) -> float {
        if constexpr (TAB == kTabF32)
            return reinterpret_cast<const float*>(tab)[s];
        else if constexpr (TAB == kTabF16)
            return __half2float(reinterpret_cast<const __half*>(tab)[s]);
        else
            return load_codeword(a.cb, a.cb_f16, s);
    };

    unsigned char* slot = a.ws + (size_t)blockIdx.x * a.slot_bytes;
    float* S = reinterpret_cast<float*>(slot);                           // [T][NU]: log2 A_t - K_t
    float* R = reinterpret_cast<float*>(slot + s_bytes(L, K, T));         // [2][NU]: log2 B_t - G_t
    double* Kc = reinterpret_cast<double*>(slot + s_bytes(L, K, T) + r_bytes(L, K));  // [T]: K_t

    for (long long b = blockIdx.x; b < a.n_blocks; b += gridDim.x) {
        const float* xb = a.x + b * T;
        const float* db = a.d ? a.d + b * T : nullptr;

        // ---- forward: S_t = log2 A_t - K_t, K_t = K_{t-1} + c_{t-1}, c = step max
        double Kcum = 0.0;  // K_{t-1} at the top of step t
        for (int t = 1; t <= T; ++t) {
            const float xt = xb[t - 1];
            const float w = (db ? db[t - 1] : 1.f) * a.w_scale;
            float cp = 0.f;
            if (t >= 2) {
                cp = wmax[((t - 1) & 1) * kWarps];
                for (int i = 1; i < kWarps; ++i) cp = fmaxf(cp, wmax[((t - 1) & 1) * kWarps + i]);
            }
            if (tid == 0) Kc[t - 1] = Kcum;
            Kcum += (double)cp;
            const float* Sp = S + (size_t)(t >= 2 ? t - 2 : 0) * NU;
            float* So = S + (size_t)(t - 1) * NU;
            float lmax = -INFINITY;
            for (int u = tid; u < NU; u += kThreads) {
                float cand[kMaxH];
                float m = -INFINITY;
#pragma unroll
                for (int h = 0; h < kMaxH; ++h) {
                    if (h < H) {
                        const uint32_t s = ((uint32_t)h << LK) | (uint32_t)u;
                        const float prev = t >= 2 ? Sp[s >> K] - cp : 0.f;
                        const float e = cw(s) - xt;
                        cand[h] = fmaf(-w * e, e, prev);
                        m = fmaxf(m, cand[h]);
                    }
                }
                float sum = 0.f;
#pragma unroll
                for (int h = 0; h < kMaxH; ++h)
                    if (h < H) sum += ex2(cand[h] - m);
                const float out = m + lg2(sum);
                So[u] = out;
                lmax = fmaxf(lmax, out);
            }
            lmax = warp_max(lmax);
            if (lane == 0) wmax[(t & 1) * kWarps + warp] = lmax;
            __syncthreads();
        }
        // log2 Z = K_T + c_T + log2 sum_u 2^(S_T[u] - c_T)
        float cT = wmax[(T & 1) * kWarps];
        for (int i = 1; i < kWarps; ++i) cT = fmaxf(cT, wmax[(T & 1) * kWarps + i]);
        {
            const float* ST = S + (size_t)(T - 1) * NU;
            float part = 0.f;
            for (int u = tid; u < NU; u += kThreads) part += ex2(ST[u] - cT);
            part = warp_sum(part);
            if (lane == 0) red[warp] = part;
        }
        __syncthreads();
        double zsum = 0.0;
        for (int i = 0; i < kWarps; ++i) zsum += (double)red[i];
        const double log2z = Kcum + (double)cT + log2(zsum);
        if (tid == 0 && a.free_energy) a.free_energy[b] = (float)(-a.tau_ln2 * log2z);
        __syncthreads();  // red is reused below

        // ---- backward: R_t = log2 B_t - G_t, G_{t-1} = G_t + e_t, e = step max
        double G = 0.0;
        for (int t = T; t >= 1; --t) {
            const float xt = xb[t - 1];
            const float w = (db ? db[t - 1] : 1.f) * a.w_scale;
            float ep = 0.f;
            if (t < T) {
                ep = wmax[(t & 1) * kWarps];
                for (int i = 1; i < kWarps; ++i) ep = fmaxf(ep, wmax[(t & 1) * kWarps + i]);
            }
            // log2 of a state's posterior = S_{t-1}[u'] + cand + shift
            const float shift = (float)(Kc[t - 1] + G + (double)ep - log2z);
            const float* Ri = R + (size_t)(t & 1) * NU;
            float* Ro = R + (size_t)((t - 1) & 1) * NU;
            const float* Sp = S + (size_t)(t >= 2 ? t - 2 : 0) * NU;
            float num = 0.f, den = 0.f, lmax = -INFINITY;
            for (int u = tid; u < NU; u += kThreads) {
                float cand[kMaxH];
                float m = -INFINITY;
#pragma unroll
                for (int bb = 0; bb < kMaxH; ++bb) {
                    if (bb < H) {
                        const uint32_t s = ((uint32_t)u << K) | (uint32_t)bb;
                        const float rin = t < T ? Ri[s & low] - ep : 0.f;
                        const float e = cw(s) - xt;
                        cand[bb] = fmaf(-w * e, e, rin);
                        m = fmaxf(m, cand[bb]);
                    }
                }
                float sum = 0.f, mom = 0.f;
#pragma unroll
                for (int bb = 0; bb < kMaxH; ++bb) {
                    if (bb < H) {
                        const float E = ex2(cand[bb] - m);
                        sum += E;
                        mom = fmaf(E, cw(((uint32_t)u << K) | (uint32_t)bb), mom);
                    }
                }
                if (t > 1) {
                    const float out = m + lg2(sum);
                    Ro[u] = out;
                    lmax = fmaxf(lmax, out);
                }
                const float W = ex2((t >= 2 ? Sp[u] : 0.f) + m + shift);
                den = fmaf(W, sum, den);
                num = fmaf(W, mom, num);
            }
            num = warp_sum(num);
            den = warp_sum(den);
            lmax = warp_max(lmax);
            if (lane == 0) {
                red[((t & 1) * kWarps + warp) * 2 + 0] = num;
                red[((t & 1) * kWarps + warp) * 2 + 1] = den;
                wmax[((t - 1) & 1) * kWarps + warp] = lmax;
            }
            __syncthreads();
            if (tid == 0) {
                float n2 = 0.f, d2 = 0.f;
                for (int i = 0; i < kWarps; ++i) {
                    n2 += red[((t & 1) * kWarps + i) * 2 + 0];
                    d2 += red[((t & 1) * kWarps + i) * 2 + 1];
                }
                a.y[b * T + (t - 1)] = n2 / d2;
            }
            G += (double)ep;
        }
        __syncthreads();  // the next block's forward reuses wmax and the slot
    }
}

template <int TAB>
cudaError_t launch_tab(const BcjrArgs& a, int grid, cudaStream_t stream)
{
    const size_t smem = kHeadBytes + table_bytes(a.L, TAB);
    cudaError_t e = cudaFuncSetAttribute(bcjr_kernel<TAB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    bcjr_kernel<TAB><<<grid, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

// bcjr_grouped.cu: the register-resident kernel for the shapes it is compiled for
cudaError_t launch_bcjr_grouped(const BcjrArgs& a, int grid, cudaStream_t stream, bool* handled);

// A slot serves either kernel (the register-resident one needs only the
// forward values, the first part of this layout).
size_t bcjr_slot_bytes(int L, int K, int T)
{
    return s_bytes(L, K, T) + r_bytes(L, K) + round256((size_t)T * sizeof(double));
}

int bcjr_ctas_per_sm(int L, int, int cb_f16)
{
    const size_t t = table_bytes(L, table_mode(L, cb_f16));
    return t > 64 * 1024 ? 1 : t > 0 ? 2 : 4;
}

cudaError_t launch_bcjr(const BcjrArgs& a, int grid, cudaStream_t stream)
{
    bool handled = false;
    const cudaError_t eg = launch_bcjr_grouped(a, grid, stream, &handled);
    if (handled || eg != cudaSuccess) return eg;
    int mode = table_mode(a.L, a.cb_f16);
    if (mode == kTabF16 && (reinterpret_cast<uintptr_t>(a.cb) & 15) != 0) mode = kTabGlobal;
    switch (mode) {
    case kTabF32: return launch_tab<kTabF32>(a, grid, stream);
    case kTabF16: return launch_tab<kTabF16>(a, grid, stream);
    default: return launch_tab<kTabGlobal>(a, grid, stream);
    }
}

}  // namespace tcq
