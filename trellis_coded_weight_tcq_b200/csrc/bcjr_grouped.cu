// bcjr_grouped.cu -- the soft (forward-backward) quantizer for compile-time
// (L, k), with every codeword of a thread's states held in registers.
//
// Same arithmetic as bcjr.cu (BCJR-QAT abstract: the Viterbi argmax replaced by
// the sum-product recursion at temperature tau; log2 units of exp(-J / tau),
// per-step normalisation by the previous step's maximum, constants summed in
// fp64), arranged like the grouped Viterbi encoder: group g of a thread covers
// the 2^(2k) states s = (h << (L-k)) | (g << k) | j.  In the forward pass they
// read the 2^k values S_{t-1}[(h << (L-2k)) | g] and produce S_t[(g << k) | j];
// in the backward pass the same states read R_t[(g << k) | j] and produce
// R_{t-1}[(h << (L-2k)) | g], and the posterior of state (h, j) is
// 2^{S_{t-1}[(h << (L-2k)) | g] + cand(h, j) + shift_t}.  So one thread owns the
// same 2^(2k) codewords in both passes, and both passes keep their running
// values in a shared-memory ping-pong with one barrier per step.
//
// The forward values of every step go to the workspace (coalesced 16-byte
// stores); the backward pass brings each thread's own values for the next step
// into private shared-memory slots with cp.async while it works on the current
// step.  Per state: one ex2 per pass (three per four states in the forward
// pass, where the maximum's term is exactly 1), one lg2 per 2^k states, three
// FP32 operations for the branch metric and two for the log-sum-exp; the
// special-function unit bounds the kernel.
#include "acs_grouped.cuh"

namespace tcq {

namespace {

__device__ __forceinline__ float ex2g(float v)
{
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

__device__ __forceinline__ float lg2g(float v)
{
    float r;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

__device__ __forceinline__ float max3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

template <int H>
__device__ __forceinline__ float hmax(const float (&v)[H])
{
    if constexpr (H == 4) {
        return max3(fmaxf(v[0], v[1]), v[2], v[3]);
    } else {
        float m = v[0];
#pragma unroll
        for (int i = 1; i < H; ++i) m = fmaxf(m, v[i]);
        return m;
    }
}

// `after` is a value computed from the slot's previous contents: taking it as an
// operand keeps the copy from issuing before that read has returned.
__device__ __forceinline__ void cp_async4(float* dst, const float* src, float after)
{
    const uint32_t s = (uint32_t)__cvta_generic_to_shared(dst);
    asm volatile("{.reg .f32 dep;\n\tmov.f32 dep, %2;\n\tcp.async.ca.shared.global [%0], [%1], 4;}"
                 ::"r"(s), "l"(src), "f"(after) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

constexpr int kMaxT = 1024;  // steps staged in shared memory

template <class C>
struct BG {
    static constexpr int NT = C::NT, GPT = C::GPT, H = C::H, K = C::K, NU = C::NU;
    static constexpr int SH = C::L - 2 * C::K;  // bits of g
    static constexpr int NW = NT / 32;
    // shared memory: 3 value arrays (two ping-pong, one of backward slots),
    // (x, w) per step, K_t per step, per-warp maxima, partial sums
    static constexpr size_t smem_bytes()
    {
        return sizeof(float) * 3 * NU + sizeof(float2) * kMaxT + sizeof(double) * kMaxT +
               sizeof(float) * 2 * NW + sizeof(float2) * 2 * NW + sizeof(float) * NW +
               sizeof(float) * kMaxT;
    }
};

template <class C>
__global__ void __launch_bounds__(C::NT, 1) bcjr_grouped_kernel(BcjrArgs a)
{
    using B = BG<C>;
    constexpr int NT = B::NT, GPT = B::GPT, H = B::H, K = B::K, NU = B::NU, SH = B::SH, NW = B::NW;
    extern __shared__ __align__(16) unsigned char sm[];
    float* buf = reinterpret_cast<float*>(sm);                   // [2][NU] ping-pong
    float* slots = buf + 2 * NU;                                 // [NU] backward S_{t-1}
    float2* xw = reinterpret_cast<float2*>(slots + NU);          // [kMaxT] (x_t, w_t)
    double* Kc = reinterpret_cast<double*>(xw + kMaxT);          // [kMaxT] K_{t-1}
    float* wmax = reinterpret_cast<float*>(Kc + kMaxT);          // [2][NW]
    float2* red = reinterpret_cast<float2*>(wmax + 2 * NW);      // [2][NW] (moment, mass)
    float* zred = reinterpret_cast<float*>(red + 2 * NW);        // [NW]
    float* rwv = zred + NW;                                      // [kMaxT] 1 / w_t

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = a.T;
    Codewords<C, C::CB16> cw;
    cw.load(a.cb, a.cb_f16, tid);
    // c - x for state (h, j) of group i
    auto diff = [&](int i, int h, int j, float x) -> float {
        if constexpr (C::CB16)
            return cw.diff(i, h, j, -x);
        else
            return cw.get(i, h, j) - x;
    };
    float* S = reinterpret_cast<float*>(a.ws + (size_t)blockIdx.x * a.slot_bytes);  // [T][NU]

    for (long long b = blockIdx.x; b < a.n_blocks; b += gridDim.x) {
        const float* xb = a.x + b * T;
        const float* db = a.d ? a.d + b * T : nullptr;
        for (int t = tid; t < T; t += NT) {
            // w_t floored at 2^-100 (a zero weight): 1 / w_t stays finite and the
            // scaled values below stay inside fp32; the change to any exponent is
            // below 2^-100 e^2
            const float w = fmaxf((db ? db[t] : 1.f) * a.w_scale, 0x1p-100f);
            xw[t] = make_float2(xb[t], w);
            rwv[t] = 1.f / w;
        }
        __syncthreads();

        // ---- forward
        double Kcum = 0.0;
        for (int t = 1; t <= T; ++t) {
            const float2 st = xw[t - 1];
            const float rw = rwv[t - 1];
            float cp = 0.f;
            if (t >= 2) {
                cp = wmax[((t - 1) & 1) * NW];
#pragma unroll
                for (int i = 1; i < NW; ++i) cp = fmaxf(cp, wmax[((t - 1) & 1) * NW + i]);
            }
            const float pc = -cp * rw;
            if (tid == 0) Kc[t - 1] = Kcum;
            Kcum += (double)cp;
            const float* Sp = buf + ((t - 1) & 1) * NU;
            float* Sn = buf + (t & 1) * NU;
            float* Sg = S + (size_t)(t - 1) * NU;
            float lmax = -INFINITY;
#pragma unroll
            for (int i = 0; i < GPT; ++i) {
                const int g = tid + i * NT;
                float p[H];
#pragma unroll
                for (int h = 0; h < H; ++h) p[h] = t >= 2 ? fmaf(Sp[(h << SH) | g], rw, pc) : 0.f;
                float out[H];
#pragma unroll
                for (int j = 0; j < H; ++j) {
                    float c[H];
#pragma unroll
                    for (int h = 0; h < H; ++h) {
                        const float e = diff(i, h, j, st.x);
                        c[h] = fmaf(-e, e, p[h]);  // (value - w e^2) / w
                    }
                    float m, s;
                    if constexpr (H == 4) {
                        // the maximum's term is exactly 1: the other three by a
                        // min/max network, so three exponentials instead of four
                        const float lo01 = fminf(c[0], c[1]), hi01 = fmaxf(c[0], c[1]);
                        const float lo23 = fminf(c[2], c[3]), hi23 = fmaxf(c[2], c[3]);
                        m = fmaxf(hi01, hi23) * st.y;
                        s = 1.f + ex2g(fmaf(lo01, st.y, -m)) + ex2g(fmaf(lo23, st.y, -m)) +
                            ex2g(fmaf(fminf(hi01, hi23), st.y, -m));
                    } else {
                        m = hmax<H>(c) * st.y;
                        s = 0.f;
#pragma unroll
                        for (int h = 0; h < H; ++h) s += ex2g(fmaf(c[h], st.y, -m));
                    }
                    out[j] = m + lg2g(s);
                    lmax = fmaxf(lmax, out[j]);
                }
                store_metrics<H>(Sn + (g << K), out);
                if (t < T) store_metrics<H>(Sg + (g << K), out);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
            if (lane == 0) wmax[(t & 1) * NW + warp] = lmax;
            __syncthreads();
        }
        // log2 Z = K_T + c_T + log2 sum_u 2^(S_T[u] - c_T)
        float cT = wmax[(T & 1) * NW];
#pragma unroll
        for (int i = 1; i < NW; ++i) cT = fmaxf(cT, wmax[(T & 1) * NW + i]);
        {
            const float* ST = buf + (T & 1) * NU;
            float part = 0.f;
#pragma unroll
            for (int i = 0; i < GPT; ++i)
#pragma unroll
                for (int j = 0; j < H; ++j) part += ex2g(ST[((tid + i * NT) << K) | j] - cT);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
            if (lane == 0) zred[warp] = part;
        }
        // the backward pass's first values: S_{T-1} into each thread's slots
        if (T >= 2) {
            const float* src = S + (size_t)(T - 2) * NU;
#pragma unroll
            for (int i = 0; i < GPT; ++i)
#pragma unroll
                for (int h = 0; h < H; ++h) {
                    const int idx = (h << SH) | (tid + i * NT);
                    cp_async4(slots + idx, src + idx, 0.f);
                }
            cp_async_commit();
        }
        __syncthreads();
        double zsum = 0.0;
#pragma unroll
        for (int i = 0; i < NW; ++i) zsum += (double)zred[i];
        const double log2z = Kcum + (double)cT + log2(zsum);
        if (tid == 0 && a.free_energy) a.free_energy[b] = (float)(-a.tau_ln2 * log2z);

        // ---- backward
        double G = 0.0;
        for (int t = T; t >= 1; --t) {
            const float2 st = xw[t - 1];
            const float rw = rwv[t - 1];
            float ep = 0.f;
            if (t < T) {
                ep = wmax[(t & 1) * NW];
#pragma unroll
                for (int i = 1; i < NW; ++i) ep = fmaxf(ep, wmax[(t & 1) * NW + i]);
            }
            const float pe = -ep * rw;
            const float shift = (float)(Kc[t - 1] + G + (double)ep - log2z);
            const float* Ri = buf + (t & 1) * NU;
            float* Ro = buf + ((t - 1) & 1) * NU;
            cp_async_wait_all();
            const float* src = S + (size_t)(t >= 3 ? t - 3 : 0) * NU;  // S_{t-2}, for step t-1
            float num = 0.f, den = 0.f, lmax = -INFINITY;
#pragma unroll
            for (int i = 0; i < GPT; ++i) {
                const int g = tid + i * NT;
                float r[H];
                if (t < T) {
                    if constexpr (H == 4) {
                        const float4 v = *reinterpret_cast<const float4*>(Ri + (g << K));
                        r[0] = fmaf(v.x, rw, pe);
                        r[1] = fmaf(v.y, rw, pe);
                        r[2] = fmaf(v.z, rw, pe);
                        r[3] = fmaf(v.w, rw, pe);
                    } else {
#pragma unroll
                        for (int j = 0; j < H; ++j) r[j] = fmaf(Ri[(g << K) + j], rw, pe);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < H; ++j) r[j] = 0.f;
                }
#pragma unroll
                for (int h = 0; h < H; ++h) {
                    float e[H], c[H];
#pragma unroll
                    for (int j = 0; j < H; ++j) {
                        e[j] = diff(i, h, j, st.x);
                        c[j] = fmaf(-e[j], e[j], r[j]);  // (value - w e^2) / w
                    }
                    const float mq = hmax<H>(c);
                    const float m = mq * st.y;
                    float s = 0.f, se = 0.f;
#pragma unroll
                    for (int j = 0; j < H; ++j) {
                        const float E = ex2g(fmaf(c[j], st.y, -m));
                        s += E;
                        se = fmaf(E, e[j], se);
                    }
                    const int idx = (h << SH) | g;
                    if (t > 1) {
                        const float ro = m + lg2g(s);
                        Ro[idx] = ro;
                        lmax = fmaxf(lmax, ro);
                    }
                    const float W = ex2g((t >= 2 ? slots[idx] : 0.f) + m + shift);
                    den = fmaf(W, s, den);
                    num = fmaf(W, fmaf(st.x, s, se), num);  // sum E c = sum E e + x sum E
                    if (t >= 3) cp_async4(slots + idx, src + idx, W);  // slot consumed by W
                }
            }
            cp_async_commit();
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                num += __shfl_xor_sync(0xffffffffu, num, o);
                den += __shfl_xor_sync(0xffffffffu, den, o);
                lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
            }
            if (lane == 0) {
                red[(t & 1) * NW + warp] = make_float2(num, den);
                wmax[((t - 1) & 1) * NW + warp] = lmax;
            }
            __syncthreads();
            if (warp == 0) {
                float2 v = lane < NW ? red[(t & 1) * NW + lane] : make_float2(0.f, 0.f);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    v.x += __shfl_xor_sync(0xffffffffu, v.x, o);
                    v.y += __shfl_xor_sync(0xffffffffu, v.y, o);
                }
                if (lane == 0) a.y[b * T + (t - 1)] = v.x / v.y;
            }
            G += (double)ep;
        }
        __syncthreads();  // xw, Kc and the buffers are rewritten by the next block
    }
}

template <class C>
cudaError_t launch_g(const BcjrArgs& a, int grid, cudaStream_t stream)
{
    const size_t smem = BG<C>::smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(bcjr_grouped_kernel<C>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bcjr_grouped_kernel<C><<<grid, C::NT, smem, stream>>>(a);
    return cudaGetLastError();
}

using BcjrL16K2 = GCfg<16, 2, 512, 8, 1, true>;

}  // namespace

// Launches the register-resident kernel when one is compiled for (L, k, dtype)
// and the block fits the staged steps; *handled reports whether it did.
cudaError_t launch_bcjr_grouped(const BcjrArgs& a, int grid, cudaStream_t stream, bool* handled)
{
    *handled = false;
    if (a.T > kMaxT) return cudaSuccess;
    if (a.L == 16 && a.K == 2 && a.cb_f16) {
        *handled = true;
        return launch_g<BcjrL16K2>(a, grid, stream);
    }
    return cudaSuccess;
}

}  // namespace tcq
