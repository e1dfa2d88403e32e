// decode.cu -- bitstream -> values for the bitshift trellis.
//
// The 2-bit post describes decoding as "read bits, update state, look up
// values"; with the bitshift trellis of QTIP the state after symbol t is just
// the last L bits of (start || stream[0, tk)), so every output is independent:
// one window extract and one codebook gather, no serial state.
//
// One warp per block in flight, each lane four consecutive weights (one
// 16-byte store when the row allows it).  The codebook is staged once per CTA
// in shared memory (fp32 if it fits in 64 KiB, else as binary16 when the input
// is binary16); a binary32 codebook too large for that is gathered through L1.
// The kernel reads k/8 bytes and writes 4 bytes per weight: HBM bound.
#include "common.cuh"

namespace tcq {

namespace {

enum TableMode { kTableF32 = 0, kTableF16 = 1, kTableGlobal = 2 };

constexpr int kDecodeThreads = 512;

__device__ __forceinline__ uint32_t state_at(const uint32_t* __restrict__ w, int W, uint32_t start,
                                             int t, int K, int L)
{
    const uint32_t mask = (1u << L) - 1u;
    const int pend = t * K;  // stream bits consumed through symbol t
    if (pend >= L) {
        const int p0 = pend - L;
        const int wi = p0 >> 5, off = p0 & 31;
        const unsigned long long hi = w[wi];
        const unsigned long long lo = (off + L > 32 && wi + 1 < W) ? w[wi + 1] : 0ull;
        const unsigned long long v = (hi << 32) | lo;
        return (uint32_t)(v >> (64 - off - L)) & mask;
    }
    // fewer than L stream bits so far: the start state supplies the rest
    return ((start << pend) | (w[0] >> (32 - pend))) & mask;
}

template <int MODE, bool VEC>
__global__ void __launch_bounds__(kDecodeThreads) decode_kernel(DecodeArgs a)
{
    extern __shared__ __align__(16) unsigned char dsm[];
    const int n_entries = 1 << a.L;
    if constexpr (MODE == kTableF32) {
        float* tab = reinterpret_cast<float*>(dsm);
        for (int i = threadIdx.x; i < n_entries; i += blockDim.x) tab[i] = load_codeword(a.cb, a.cb_f16, i);
    } else if constexpr (MODE == kTableF16) {
        __half* tab = reinterpret_cast<__half*>(dsm);
        const __half* src = reinterpret_cast<const __half*>(a.cb);
        for (int i = threadIdx.x; i < n_entries; i += blockDim.x) tab[i] = src[i];
    }
    __syncthreads();

    const int T = a.T, K = a.K, L = a.L, W = a.W;
    const int Q = (T + 3) >> 2;  // quads per block
    const int lane = threadIdx.x & 31;
    const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
    for (long long b = warp; b < a.n_blocks; b += nwarps) {
        const uint32_t* wb = a.bits + b * W;
        const uint32_t start = a.start_state[b];
        float* yb = a.y + b * T;
        for (int q = lane; q < Q; q += 32) {
            float v[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int t = 4 * q + e + 1;
                float val = 0.f;
                if (t <= T) {
                    const uint32_t s = state_at(wb, W, start, t, K, L);
                    if constexpr (MODE == kTableF32)
                        val = reinterpret_cast<const float*>(dsm)[s];
                    else if constexpr (MODE == kTableF16)
                        val = __half2float(reinterpret_cast<const __half*>(dsm)[s]);
                    else
                        val = load_codeword(a.cb, a.cb_f16, s);
                }
                v[e] = val;
            }
            if constexpr (VEC) {
                *reinterpret_cast<float4*>(yb + 4 * q) = make_float4(v[0], v[1], v[2], v[3]);
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (4 * q + e < T) yb[4 * q + e] = v[e];
            }
        }
    }
}

template <int MODE, bool VEC>
cudaError_t launch_mode(const DecodeArgs& a, int grid, size_t smem, cudaStream_t stream)
{
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<MODE, VEC>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    decode_kernel<MODE, VEC><<<grid, kDecodeThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, int num_sms, cudaStream_t stream)
{
    const size_t entries = (size_t)1 << a.L;
    int mode;
    size_t smem;
    if (entries * 4 <= 64 * 1024) {
        mode = kTableF32;
        smem = entries * 4;
    } else if (a.cb_f16) {
        mode = kTableF16;
        smem = entries * 2;
    } else {
        mode = kTableGlobal;
        smem = 0;
    }
    // warps in flight: one per block, capped at what the SMs hold
    const long long warps_needed = a.n_blocks;
    const int per_cta = kDecodeThreads / 32;
    long long grid = (warps_needed + per_cta - 1) / per_cta;
    const int ctas_per_sm = smem > 100 * 1024 ? 1 : (smem > 64 * 1024 ? 2 : 4);
    const long long cap = (long long)num_sms * ctas_per_sm;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    const bool vec = (a.T % 4 == 0) && ((reinterpret_cast<uintptr_t>(a.y) & 15) == 0);
    switch (mode * 2 + (vec ? 1 : 0)) {
    case 0: return launch_mode<kTableF32, false>(a, (int)grid, smem, stream);
    case 1: return launch_mode<kTableF32, true>(a, (int)grid, smem, stream);
    case 2: return launch_mode<kTableF16, false>(a, (int)grid, smem, stream);
    case 3: return launch_mode<kTableF16, true>(a, (int)grid, smem, stream);
    case 4: return launch_mode<kTableGlobal, false>(a, (int)grid, smem, stream);
    default: return launch_mode<kTableGlobal, true>(a, (int)grid, smem, stream);
    }
}

}  // namespace tcq
