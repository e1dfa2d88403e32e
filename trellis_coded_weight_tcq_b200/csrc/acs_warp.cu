// acs_warp.cu -- Viterbi encoder for small trellises: one warp per coding block.
//
// Method: the same search as the grouped encoder (Viterbi over the bitshift
// trellis, weighted branch metric d_t (x_t - c[s])^2, free or fixed start, the
// 2-bit post's Viterbi section, QTIP abstract, CurveTQ abstract), in the
// M-grouped form C_t[s] = M_{t-1}[s >> k] + d_t (x_t - c[s])^2,
// M_t[u] = min_h C_t[(h << (L-k)) | u], bp_t[u] = argmin_h.
//
// Layout for 2^(L-k) path metrics of a few dozen: lane l of the block's warp
// takes u = l, l + 32, ... (U values), i.e. 2^k candidates per u per step, so a
// step is a few instructions per lane and a warp synchronisation instead of a
// CTA barrier over sixteen-state groups.  The metrics ping-pong in the warp's
// shared memory; a step's k backpointer bits of each u are k ballots (one word
// per u slot and bit) stored in shared memory, so the traceback walks shared
// memory, not L2.  Blocks of at most kWarpEncMaxT steps (the backpointers of a
// whole block stay in shared memory); longer blocks take the grouped kernel.
// Branch metric in fp32 without cancellation, as in the grouped fp32 kernel:
// e = fma(-sqrt(d_t), c, sqrt(d_t) x_t), cand = fma(e, e, M).
#include "acs_grouped.cuh"

namespace tcq {

constexpr int kWarpEncWarps = 4;     // blocks (warps) per CTA
constexpr int kWarpEncMaxT = 1024;   // steps whose backpointers fit in shared memory

template <int L, int K>
struct WCfg {
    static constexpr int H = 1 << K, LK = L - K, NU = 1 << LK, U = NU / 32;
    static_assert(NU % 32 == 0 && U >= 1 && U <= 4, "one to four metrics per lane");
    static_assert(LK >= K, "predecessor index (h << (L - 2k)) | (u >> k)");
    // per warp: ping-pong metrics, staged (a, xs) per step, U K backpointer
    // words per step, the path s_1..s_T
    static __host__ __device__ size_t r16(size_t v) { return (v + 15) & ~(size_t)15; }
    static __host__ __device__ size_t m_bytes() { return r16((size_t)2 * NU * 4); }
    static __host__ __device__ size_t st_bytes(int T) { return r16((size_t)T * 8); }
    static __host__ __device__ size_t bp_bytes(int T) { return r16((size_t)T * U * K * 4); }
    static __host__ __device__ size_t warp_bytes(int T)
    {
        return m_bytes() + st_bytes(T) + bp_bytes(T) + r16((size_t)T * 2);
    }
    static size_t smem_bytes(int, int, int T) { return (size_t)kWarpEncWarps * warp_bytes(T); }
    static size_t slot_bytes(int, int, int) { return 256; }  // no workspace is read or written
};

template <int L, int K, bool FIXED>
__global__ void __launch_bounds__(kWarpEncWarps * 32) acs_warp_kernel(EncodeArgs a)
{
    using C = WCfg<L, K>;
    constexpr int H = C::H, LK = C::LK, NU = C::NU, U = C::U;
    extern __shared__ __align__(16) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = a.T;
    unsigned char* base = smem + (size_t)warp * C::warp_bytes(T);
    float* Mbuf = reinterpret_cast<float*>(base);
    float2* st = reinterpret_cast<float2*>(base + C::m_bytes());
    uint32_t* BP = reinterpret_cast<uint32_t*>(base + C::m_bytes() + C::st_bytes(T));
    uint16_t* P = reinterpret_cast<uint16_t*>(base + C::m_bytes() + C::st_bytes(T) + C::bp_bytes(T));
#ifdef TCQ_DEBUG
    const long long x_n = (a.n_blocks - 1) * a.x_stride + T, d_n = (a.n_blocks - 1) * a.d_stride + T;
    const long long o_n = (a.n_blocks - 1) * a.out_stride + 1;
#endif

    // the codewords of the lane's candidate states, fixed for every step and block
    float cw[U][H];
#pragma unroll
    for (int i = 0; i < U; ++i)
#pragma unroll
        for (int h = 0; h < H; ++h)
            cw[i][h] = load_codeword(a.cb, a.cb_f16, ((uint32_t)h << LK) | (uint32_t)(lane + 32 * i));
    // the predecessors' metrics of the lane's u values: (h << (L - 2k)) | (u >> k)
    int off[U][H];
#pragma unroll
    for (int i = 0; i < U; ++i)
#pragma unroll
        for (int h = 0; h < H; ++h) off[i][h] = (h << (LK - K)) | ((lane + 32 * i) >> K);

    for (long long b = (long long)blockIdx.x * kWarpEncWarps + warp; b < a.n_blocks;
         b += (long long)gridDim.x * kWarpEncWarps) {
        const float* xb = a.x + b * a.x_stride;
        const float* db = a.d ? a.d + b * a.d_stride : nullptr;
        for (int t = lane; t < T; t += 32) {
            if (!TCQ_IN_BOUNDS(xb + t - a.x, x_n) || (db && !TCQ_IN_BOUNDS(db + t - a.d, d_n))) continue;
            const float sd = sqrtf(db ? db[t] : 1.f);
            st[t] = make_float2(-sd, sd * xb[t]);
        }
        // M_0: 0 everywhere (free start) or only at the fixed start's low L - k bits
        uint32_t s0 = 0xffffffffu;
        if constexpr (FIXED)
            if (TCQ_IN_BOUNDS(b, a.n_blocks)) s0 = a.fixed_start[b] & (uint32_t)(NU - 1);
#pragma unroll
        for (int i = 0; i < U; ++i)
            Mbuf[lane + 32 * i] = (!FIXED || (uint32_t)(lane + 32 * i) == s0) ? 0.f : __int_as_float(0x7f800000);
        __syncwarp();

        float bestv = __int_as_float(0x7f800000);
        uint32_t bests = 0xffffffffu;
        // one trellis step (t + 1) from metrics Mp into Mn; LAST keeps the best
        // final state instead of storing metrics and backpointers.  Mp and Mn are
        // the two halves of Mbuf, fixed per call site (the loop is unrolled by
        // two), so every metric access is a register offset plus a constant.
        auto step = [&](const float* Mp, float* Mn, int t, auto last_tag) {
            constexpr bool LAST = decltype(last_tag)::value;
            const float2 ax = st[t];
            uint32_t w[U * K];
#pragma unroll
            for (int i = 0; i < U; ++i) {
                float cand[H];
#pragma unroll
                for (int h = 0; h < H; ++h) {
                    const float e = fmaf(ax.x, cw[i][h], ax.y);
                    cand[h] = fmaf(e, e, Mp[off[i][h]]);
                }
                uint32_t sb[K];
                const float v = SignTree<H, 0>::template run<H, K>(cand, sb);
                if constexpr (LAST) {
                    uint32_t idx = 0;
#pragma unroll
                    for (int l = 0; l < K; ++l) idx = (idx << 1) | (sb[l] >> 31);
                    keep_best(v, (idx << LK) | (uint32_t)(lane + 32 * i), bestv, bests);
                } else {
                    Mn[lane + 32 * i] = v;
#pragma unroll
                    for (int l = 0; l < K; ++l) w[i * K + l] = __ballot_sync(0xffffffffu, sb[l] >> 31);
                }
            }
            if constexpr (!LAST) {
                if (lane == 0) {
                    uint32_t* dst = BP + (size_t)t * U * K;
                    if constexpr (U * K == 4) {
                        *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
                    } else {
#pragma unroll
                        for (int q = 0; q < U * K; ++q) dst[q] = w[q];
                    }
                }
                __syncwarp();
            }
        };
        using T0 = std::false_type;
        using T1 = std::true_type;
        float* M0 = Mbuf;
        float* M1 = Mbuf + NU;
        const int n1 = T - 1;  // steps before the last
        int t = 0;
        for (; t + 1 < n1; t += 2) {
            step(M0, M1, t, T0{});
            step(M1, M0, t + 1, T0{});
        }
        if (t < n1) {
            step(M0, M1, t, T0{});
            step(M1, M0, T - 1, T1{});
        } else {
            step(M0, M1, T - 1, T1{});
        }
        // final state: the smallest cost, the smaller state on ties
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bestv, o);
            const uint32_t os = __shfl_xor_sync(0xffffffffu, bests, o);
            keep_best(ov, os, bestv, bests);
        }
        // traceback: bp_t[u] (bit l of its argmin in word (t, u / 32, l), bit u mod 32)
        // decides s_t = (h << (L - k)) | u from u = s_{t+1} >> k
        if (lane == 0) {
            uint32_t s = bests;
            P[T - 1] = (uint16_t)s;
            for (int t = T - 2; t >= 0; --t) {
                const uint32_t u = s >> K;
                const uint32_t* wv = BP + (size_t)t * U * K + (u >> 5) * K;
                uint32_t h = 0;
#pragma unroll
                for (int l = 0; l < K; ++l) h = (h << 1) | ((wv[l] >> (u & 31)) & 1u);
                s = (h << LK) | u;
                P[t] = (uint16_t)s;
            }
        }
        __syncwarp();
        // outputs: packed symbols (MSB first), canonical start s_1 >> k, fp64 cost
        double acc = 0.0;
        for (int t = lane; t < T; t += 32) {
            if (!TCQ_IN_BOUNDS(xb + t - a.x, x_n) || (db && !TCQ_IN_BOUNDS(db + t - a.d, d_n))) continue;
            const double e = (double)xb[t] - (double)load_codeword(a.cb, a.cb_f16, P[t]);
            acc += (double)(db ? db[t] : 1.f) * e * e;
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        const int nbits = T * K;
        for (int w = lane; w < a.W; w += 32) {
            uint32_t word = 0;
            for (int i = 0; i < 32; ++i) {
                const int p = 32 * w + i;
                if (p >= nbits) break;
                const uint32_t sym = P[p / K] & (H - 1);
                word |= ((sym >> (K - 1 - p % K)) & 1u) << (31 - i);
            }
            if (TCQ_IN_BOUNDS(b * a.out_stride * a.W + w, o_n * a.W)) a.bits[b * a.out_stride * a.W + w] = word;
        }
        if (lane == 0 && TCQ_IN_BOUNDS(b * a.out_stride, o_n)) {
            a.start_state[b * a.out_stride] = (uint32_t)P[0] >> K;
            a.path_cost[b * a.out_stride] = (float)acc;
        }
        __syncwarp();  // the warp's buffers are reused by its next block
    }
}

template <int L, int K>
cudaError_t launch_warp_enc(const EncodeArgs& a, int grid, cudaStream_t stream)
{
    const size_t smem = WCfg<L, K>::smem_bytes(L, K, a.T);
    if (a.T > kWarpEncMaxT || a.V != 1) return cudaErrorInvalidValue;
    if (a.fixed_start) {
        cudaError_t e = cudaFuncSetAttribute(acs_warp_kernel<L, K, true>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        acs_warp_kernel<L, K, true><<<grid, kWarpEncWarps * 32, smem, stream>>>(a);
    } else {
        cudaError_t e = cudaFuncSetAttribute(acs_warp_kernel<L, K, false>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        acs_warp_kernel<L, K, false><<<grid, kWarpEncWarps * 32, smem, stream>>>(a);
    }
    return cudaGetLastError();
}

template <int L, int K>
const EncodeKernelInfo* warp_info(const char* name)
{
    static const EncodeKernelInfo info = {
        name, kWarpEncWarps, kWarpEncWarps * 32, 0, &WCfg<L, K>::slot_bytes, &WCfg<L, K>::smem_bytes,
        reinterpret_cast<const void*>(&acs_warp_kernel<L, K, false>), &launch_warp_enc<L, K>};
    return &info;
}

const EncodeKernelInfo* find_warp_kernel(int L, int K, int T)
{
    if (T > kWarpEncMaxT) return nullptr;
    if (L == 8 && K == 2) return warp_info<8, 2>("warp<8,2>");
    return nullptr;
}

}  // namespace tcq
