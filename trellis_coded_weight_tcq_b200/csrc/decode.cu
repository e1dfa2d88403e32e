// decode.cu -- bitstream -> values for the bitshift trellis.
//
// The 2-bit post's decoder advances the state from the bits and fetches each
// codeword; with the bitshift trellis of QTIP the state after symbol t is just
// the last L bits of (start || stream[0, tk)), so every output is independent:
// one window extract and one codebook gather, no serial state.
//
// Each thread produces four consecutive weights of one block (one 16-byte store
// when the row allows it); a CTA covers as many whole blocks as its threads
// span and strides over the rest, so every thread has independent loads in
// flight.  The codebook is staged once per CTA in shared memory (fp32 if it
// fits in 64 KiB, else as binary16 when the input is binary16); a binary32
// codebook too large for that is gathered through L1.  The kernel reads k/8
// bytes and writes 4 bytes per weight: HBM bound.
#include "codes.cuh"

namespace tcq {

namespace {

enum TableMode { kTableF32 = 0, kTableF16 = 1, kTableGlobal = 2, kTableMad = 3 };

constexpr int kDecodeThreads = 1024;

template <int MODE, bool VEC>
__global__ void __launch_bounds__(kDecodeThreads) decode_kernel(DecodeArgs a)
{
    extern __shared__ __align__(16) unsigned char dsm[];
    const int n_entries = 1 << a.L;
    if constexpr (MODE == kTableF32) {
        float* tab = reinterpret_cast<float*>(dsm);
        for (int i = threadIdx.x; i < n_entries; i += blockDim.x) tab[i] = load_codeword(a.cb, a.cb_f16, i);
    } else if constexpr (MODE == kTableF16) {
        // 16-byte copies when the source allows (the table size, 2^L entries of 2
        // bytes, is a multiple of 16 for L >= 3)
        const __half* src = reinterpret_cast<const __half*>(a.cb);
        if ((reinterpret_cast<uintptr_t>(src) & 15) == 0 && n_entries % 8 == 0) {
            const uint4* s4 = reinterpret_cast<const uint4*>(src);
            uint4* d4 = reinterpret_cast<uint4*>(dsm);
            for (int i = threadIdx.x; i < n_entries / 8; i += blockDim.x) d4[i] = s4[i];
        } else {
            __half* tab = reinterpret_cast<__half*>(dsm);
            for (int i = threadIdx.x; i < n_entries; i += blockDim.x) tab[i] = src[i];
        }
    }
    __syncthreads();

    const int T = a.T, K = a.K, L = a.L, W = a.W;
    const uint32_t mask = (1u << L) - 1u;
#ifdef TCQ_DEBUG
    const long long bits_n = ((a.n_blocks - 1) * a.in_stride + 1) * W;
    const long long st_n = (a.n_blocks - 1) * a.in_stride + 1, y_n = (a.n_blocks - 1) * a.y_stride + T;
#endif
    const int Q = (T + 3) >> 2;  // quads per block
    const bool qpow2 = (Q & (Q - 1)) == 0;
    const int qshift = __ffs(Q) - 1;
    const int per_iter = blockDim.x >= Q ? (int)blockDim.x / Q : 1;  // whole blocks per CTA pass
    const int span = per_iter * Q;  // quads of one pass (i in [0, span) covers per_iter blocks)
    auto lookup = [&](uint32_t s) -> float {
        if constexpr (MODE == kTableF32)
            return reinterpret_cast<const float*>(dsm)[s];
        else if constexpr (MODE == kTableF16)
            return __half2float(reinterpret_cast<const __half*>(dsm)[s]);
        else if constexpr (MODE == kTableMad)
            return mad_codeword(s);
        else
            return load_codeword(a.cb, a.cb_f16, s);
    };
    // Stream word -1 is the start state itself: stream bit p < 0 is bit -p-1 of
    // start, so s_t is the L-bit window ending at stream bit t k for every t,
    // and each thread's four windows [p0 + e k, p0 + e k + L), p0 = (4q+1)k - L
    // >= k - L > -32, lie inside one 64-bit read of words (p0 >> 5, +1).
    constexpr int UNROLL = 4;
    struct Frag {
        unsigned long long win[UNROLL];
        int off[UNROLL];
        int q[UNROLL];
        long long b[UNROLL];
    };
    auto fetch = [&](Frag& f, long long b0, int i0) {
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int i = i0 + u * span;
            const int bl = qpow2 ? (i >> qshift) : i / Q;
            const int q = i - bl * Q;
            const long long b = b0 + bl;
            f.q[u] = q;
            f.b[u] = b;
            f.win[u] = 0ull;
            const int p0 = (4 * q + 1) * K - L;
            f.off[u] = p0 & 31;
            if (b < a.n_blocks) {
                const uint32_t* wb = a.bits + b * a.in_stride * W;
                const int wi = p0 >> 5;  // -1 for the first windows
                const bool ok = wi < 0 ? TCQ_IN_BOUNDS(b * a.in_stride, st_n)
                                       : TCQ_IN_BOUNDS(b * a.in_stride * W + wi, bits_n);
                const bool ok1 = wi + 1 >= W || TCQ_IN_BOUNDS(b * a.in_stride * W + wi + 1, bits_n);
                const unsigned long long hi = !ok ? 0ull : wi < 0 ? a.start_state[b * a.in_stride] : wb[wi];
                const unsigned long long lo = wi + 1 < W && ok1 ? wb[wi + 1] : 0ull;
                f.win[u] = (hi << 32) | lo;
            }
        }
    };
    auto emit = [&](const Frag& f) {
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const long long b = f.b[u];
            if (b >= a.n_blocks) continue;
            const int q = f.q[u];
            float v[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                v[e] = lookup((uint32_t)(f.win[u] >> (64 - f.off[u] - e * K - L)) & mask);
            float* yb = a.y + b * a.y_stride;
            if constexpr (VEC) {
                if (TCQ_IN_BOUNDS(b * a.y_stride + 4 * q + 3, y_n))
                    __stcs(reinterpret_cast<float4*>(yb + 4 * q), make_float4(v[0], v[1], v[2], v[3]));
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (4 * q + e < T && TCQ_IN_BOUNDS(b * a.y_stride + 4 * q + e, y_n)) yb[4 * q + e] = v[e];
            }
        }
    };
    const int blocks_per_pass = per_iter * UNROLL;
    const long long stride = (long long)gridDim.x * blocks_per_pass;
    const long long first = (long long)blockIdx.x * blocks_per_pass;
    if (span <= (int)blockDim.x) {
        // one fragment per thread per pass; the next pass's loads are issued
        // before the current pass's lookups and stores
        if ((int)threadIdx.x >= span) return;
        Frag cur, nxt;
        if (first < a.n_blocks) fetch(cur, first, threadIdx.x);
        for (long long b0 = first; b0 < a.n_blocks; b0 += stride) {
            if (b0 + stride < a.n_blocks) fetch(nxt, b0 + stride, threadIdx.x);
            emit(cur);
            cur = nxt;
        }
    } else {  // blocks longer than 4 * blockDim weights
        for (long long b0 = first; b0 < a.n_blocks; b0 += stride) {
            for (int i0 = threadIdx.x; i0 < span; i0 += blockDim.x) {
                Frag f;
                fetch(f, b0, i0);
                emit(f);
            }
        }
    }
}

// Compile-time (L, k, T) with T / 4 a multiple of 32: a warp decodes whole
// blocks, and lane l always holds quads l, l + 32, ... of a block, so its
// window offsets are constants; the four windows of a quad lie in one 32-bit
// word once it is aligned ((4 - 1) k + L <= 32), so a state is one shift and one
// mask.  The loads decide the speed otherwise (each warp waited on its block's
// words: 14 long-scoreboard stalls per instruction with one block of
// look-ahead), so every warp keeps kDecodeRing blocks' words and start states
// in flight in a shared-memory ring filled by asynchronous 16-byte copies (no
// registers held): cp.async.wait_group then guarantees the oldest slot has
// landed.  A table is staged the same way while the first slots load.
constexpr int kDecodeRing = 8;

// A slot: three unused words, the start state (word 3), the block's W words
// (16-byte aligned, from word 4), a zero word (word W + 4, written once), then
// padding to 16 bytes.  Stream word i (i = -1 the start state) is slot word
// i + 4, so a window's two words are two plain reads whatever the lane.
__host__ __device__ constexpr int decode_ring_slot_bytes(int W) { return 16 + W * 4 + 16; }

template <int L, int K, int T, int MODE>
__global__ void __launch_bounds__(kDecodeThreads) decode_fast_kernel(DecodeArgs a)
{
    constexpr int Q = T / 4;    // quads per block
    constexpr int QPL = Q / 32; // quads per lane per block
    constexpr int W = (T * K + 31) / 32;
    constexpr int D = kDecodeRing;
    constexpr int SLOT = decode_ring_slot_bytes(W);
    constexpr uint32_t MASK = (1u << L) - 1u;
    static_assert(Q % 32 == 0 && 3 * K + L <= 32 && W % 4 == 0 && W / 4 <= 32, "shape");
    extern __shared__ __align__(16) unsigned char dsm[];
    const int n_entries = 1 << L;
    constexpr size_t TAB = MODE == kTableMad ? 0 : ((size_t)1 << L) * (MODE == kTableF16 ? 2 : 4);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned char* ring = dsm + TAB + (size_t)warp * D * SLOT;
    const uint32_t ring_s = (uint32_t)__cvta_generic_to_shared(ring);
    if constexpr (MODE == kTableF16) {
        const char* src = reinterpret_cast<const char*>(a.cb);
        const uint32_t dst = (uint32_t)__cvta_generic_to_shared(dsm);
        for (int i = threadIdx.x; i < n_entries / 8; i += blockDim.x)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + 16 * i),
                         "l"(src + 16 * (size_t)i) : "memory");
        asm volatile("cp.async.commit_group;" ::: "memory");
    } else if constexpr (MODE == kTableF32) {
        float* tab = reinterpret_cast<float*>(dsm);
        for (int i = threadIdx.x; i < n_entries; i += blockDim.x) tab[i] = load_codeword(a.cb, a.cb_f16, i);
    }
    auto lookup = [&](uint32_t s) -> float {
        if constexpr (MODE == kTableF32)
            return reinterpret_cast<const float*>(dsm)[s];
        else if constexpr (MODE == kTableF16)
            return __half2float(reinterpret_cast<const __half*>(dsm)[s]);
        else
            return mad_codeword(s);
    };
    int wi[QPL], off[QPL];
#pragma unroll
    for (int r = 0; r < QPL; ++r) {
        const int p0 = (4 * (lane + 32 * r) + 1) * K - L;  // first window of the quad
        wi[r] = p0 >> 5;                                    // -1: the start state
        off[r] = p0 & 31;
    }
    const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
    const long long b0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
#ifdef TCQ_DEBUG
    const long long bits_n = ((a.n_blocks - 1) * a.in_stride + 1) * W;
    const long long st_n = (a.n_blocks - 1) * a.in_stride + 1, y_n = (a.n_blocks - 1) * a.y_stride + T;
#endif
    // block blk's words and start state into ring slot sl; every lane commits one
    // group (possibly empty) per call, so wait_group counts blocks
    auto prefetch = [&](long long blk, int sl) {
        if (blk < a.n_blocks) {
            if (lane < W / 4 && TCQ_IN_BOUNDS(blk * a.in_stride * W + 4 * lane + 3, bits_n))
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(ring_s + sl * SLOT + 16 + 16 * lane),
                             "l"(a.bits + blk * a.in_stride * W + 4 * lane) : "memory");
            else if (lane == 31 && TCQ_IN_BOUNDS(blk * a.in_stride, st_n))
                asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(ring_s + sl * SLOT + 12),
                             "l"(a.start_state + blk * a.in_stride) : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    if (lane < D) reinterpret_cast<uint32_t*>(ring + lane * SLOT)[W + 4] = 0u;  // never copied over
#pragma unroll
    for (int d = 0; d < D; ++d) prefetch(b0 + d * nwarps, d);
    if constexpr (MODE == kTableF16) {
        // the table's group is older than the ring's: waiting for all but D groups
        asm volatile("cp.async.wait_group %0;" ::"n"(D) : "memory");
    }
    __syncthreads();
    int sl = 0;
    for (long long bb = b0; bb < a.n_blocks; bb += nwarps) {
        asm volatile("cp.async.wait_group %0;" ::"n"(D - 1) : "memory");  // this block's group has landed
        __syncwarp();
        const uint32_t* rw = reinterpret_cast<const uint32_t*>(ring + sl * SLOT);
        float* yb = a.y + bb * a.y_stride;
#pragma unroll
        for (int r = 0; r < QPL; ++r) {
            const uint32_t hi = rw[wi[r] + 4];  // wi = -1: the start state
            const uint32_t lo = rw[wi[r] + 5];  // wi = W - 1: the zero word
            const uint32_t w = __funnelshift_l(lo, hi, off[r]);
            float v[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) v[e] = lookup((w >> (32 - L - e * K)) & MASK);
            if (TCQ_IN_BOUNDS(bb * a.y_stride + 4 * (lane + 32 * r) + 3, y_n))
                __stcs(reinterpret_cast<float4*>(yb + 4 * (lane + 32 * r)), make_float4(v[0], v[1], v[2], v[3]));
        }
        __syncwarp();  // the slot is read: refill it D blocks ahead
        prefetch(bb + D * nwarps, sl);
        sl = sl + 1 == D ? 0 : sl + 1;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
}

template <int L, int K, int T, int MODE>
cudaError_t launch_fast(const DecodeArgs& a, int grid, size_t smem, cudaStream_t stream)
{
    cudaError_t e = cudaFuncSetAttribute(decode_fast_kernel<L, K, T, MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    decode_fast_kernel<L, K, T, MODE><<<grid, kDecodeThreads, smem, stream>>>(a);
    return cudaGetLastError();
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

// Vector trellis: one thread per (block, step); the step's state is the L-bit
// window ending at stream bit t K (K = k V bits per step, stream word -1 the
// start state), and the step writes the V values of its codeword.
__global__ void decode_vec_kernel(DecodeArgs a, int V)
{
    const int K = a.K, L = a.L, W = a.W, NS = a.T / V;
    const uint32_t mask = (1u << L) - 1u;
    const long long total = a.n_blocks * NS;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const long long b = i / NS;
        const int t = (int)(i - b * NS) + 1;
        const int p0 = t * K - L;  // window start, > -32
        const int wi = p0 >> 5;
        const uint32_t* wb = a.bits + b * W;
        const unsigned long long hi = wi < 0 ? a.start_state[b] : wb[wi];
        const unsigned long long lo = wi + 1 < W ? wb[wi + 1] : 0ull;
        const uint32_t s = (uint32_t)((((hi << 32) | lo) >> (64 - (p0 & 31) - L)) & mask);
        float* y = a.y + b * a.T + (long long)(t - 1) * V;
        for (int v = 0; v < V; ++v) y[v] = load_codeword(a.cb, a.cb_f16, s * V + v);
    }
}

// The vector trellis at L = 16, four bits per step (k = 2, V = 2), binary16
// pairs, one 32-bit word per state.  The 256 KiB table does not fit in shared
// memory; its first seven eighths (states below 0xE000, 224 KiB) are copied
// there once per CTA and the rest is read through the read-only cache: a warp's
// 32 random shared-memory reads cost a few bank passes where 32 random cache
// lines cost 32 tag lookups (the all-cache version reached 0.32 of HBM, three
// quarters in shared memory 0.46, seven eighths 0.53).
// A warp decodes 128 steps of a block at a time, lane l steps 4l+1 .. 4l+4:
// their 16-bit windows end at stream bits 16l+3 .. 16l+15, so they lie in the
// 64 bits of words (l >> 1) - 1 and l >> 1 of the chunk (word -1 of a block is
// its start state), and the lane writes its 8 values as two 16-byte streaming
// stores.  Needs T % 8 == 0 and a 16-byte aligned output; other shapes take
// decode_vec_kernel.
constexpr int kVec2DecThreads = 1024;
constexpr uint32_t kVec2DecSmemStates = 0xE000u;

__global__ void __launch_bounds__(kVec2DecThreads) decode_vec2_kernel(DecodeArgs a)
{
    extern __shared__ __align__(16) uint32_t tab[];  // [kVec2DecSmemStates]
    const uint32_t* cb = reinterpret_cast<const uint32_t*>(a.cb);
    {
        // the table by asynchronous 16-byte copies, all in flight at once (a load
        // and a store per thread and round would wait on each load in turn)
        const uint32_t dst = (uint32_t)__cvta_generic_to_shared(tab);
        for (int i = threadIdx.x; i < (int)(kVec2DecSmemStates / 4); i += blockDim.x)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + 16 * i),
                         "l"(cb + 4 * (size_t)i) : "memory");
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
    const int NS = a.T >> 1;
    const int chunks = (NS + 127) >> 7;
    const long long items = a.n_blocks * chunks;
    const int lane = threadIdx.x & 31;
    const long long stride = ((long long)gridDim.x * blockDim.x) >> 5;
    // the two words of item it that the lane's windows lie in (word -1 of a block
    // is its start state); a lane with no steps in the item reads nothing
    auto fetch = [&](long long it, unsigned long long& v) {
        if (it >= items) return;
        const long long b = chunks == 1 ? it : it / chunks;
        const int c = (int)(it - b * chunks);
        if ((c << 7) + 4 * lane + 4 > NS) return;
        const uint32_t* wb = a.bits + b * a.W;
        const int wi = (c << 4) + (lane >> 1);  // word holding the lane's last window end
        const unsigned long long hi = wi >= 1 ? __ldg(wb + wi - 1) : __ldg(a.start_state + b);
        v = (hi << 32) | __ldg(wb + wi);
    };
    long long it = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    unsigned long long v = 0, vn = 0;
    fetch(it, v);  // the first item's words load while the table is copied
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    for (; it < items; it += stride) {
        fetch(it + stride, vn);  // the next item's words are in flight during this one
        const long long b = chunks == 1 ? it : it / chunks;
        const int c = (int)(it - b * chunks);
        const int t0 = (c << 7) + 4 * lane;  // steps t0+1 .. t0+4
        if (t0 + 4 <= NS) {                  // NS % 4 == 0: a lane's steps are all in or all out
            float y[8];
#pragma unroll
            for (int q = 1; q <= 4; ++q) {
                // window start relative to bit 0 of v: 16 (lane & 1) + 4q + 16
                const int sh = 48 - (16 * (lane & 1) + 4 * q + 16);
                const uint32_t s = (uint32_t)(v >> sh) & 0xffffu;
                const uint32_t w = s < kVec2DecSmemStates ? tab[s] : __ldg(cb + s);
                const __half2 h2 = *reinterpret_cast<const __half2*>(&w);
                const float2 f = __half22float2(h2);
                y[2 * q - 2] = f.x;
                y[2 * q - 1] = f.y;
            }
            float4* dst = reinterpret_cast<float4*>(a.y + b * a.y_stride + 2 * (long long)t0);
            __stcs(dst, make_float4(y[0], y[1], y[2], y[3]));
            __stcs(dst + 1, make_float4(y[4], y[5], y[6], y[7]));
        }
        v = vn;
    }
}

cudaError_t launch_decode_vec(const DecodeArgs& a, int V, int num_sms, cudaStream_t stream)
{
    if (a.L == 16 && a.K == 4 && V == 2 && a.cb_f16 == 1 && a.T % 8 == 0 && a.y_stride % 4 == 0 &&
        (reinterpret_cast<uintptr_t>(a.y) & 15) == 0 && (reinterpret_cast<uintptr_t>(a.cb) & 15) == 0) {
        const size_t smem = kVec2DecSmemStates * sizeof(uint32_t);
        const cudaError_t e = cudaFuncSetAttribute(decode_vec2_kernel,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        const long long warps = a.n_blocks * ((a.T / 2 + 127) / 128);
        long long grid = (warps + kVec2DecThreads / 32 - 1) / (kVec2DecThreads / 32);
        if (grid > num_sms) grid = num_sms;  // one CTA per SM: the table copy is paid once per SM
        if (grid < 1) grid = 1;
        decode_vec2_kernel<<<(int)grid, kVec2DecThreads, smem, stream>>>(a);
        return cudaGetLastError();
    }
    const long long total = a.n_blocks * (a.T / V);
    long long grid = (total + 255) / 256;
    const long long cap = (long long)num_sms * 8;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    decode_vec_kernel<<<(int)grid, 256, 0, stream>>>(a, V);
    return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs& a, int num_sms, cudaStream_t stream)
{
    const size_t entries = (size_t)1 << a.L;
    int mode;
    size_t smem;
    if (a.cb_f16 == kMadCodebook) {
        mode = kTableMad;
        smem = 0;
    } else if (entries * 4 <= 64 * 1024) {
        mode = kTableF32;
        smem = entries * 4;
    } else if (a.cb_f16) {
        mode = kTableF16;
        smem = entries * 2;
    } else {
        mode = kTableGlobal;
        smem = 0;
    }
    // CTAs: enough to cover every block once, capped at what the SMs hold
    const int Q = (a.T + 3) / 4;
    const long long per_cta = 4 * (kDecodeThreads >= Q ? kDecodeThreads / Q : 1);
    long long grid = (a.n_blocks + per_cta - 1) / per_cta;
    const int ctas_per_sm = smem > 100 * 1024 ? 1 : 2;
    const long long cap = (long long)num_sms * ctas_per_sm;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    const bool vec = (a.T % 4 == 0) && (a.y_stride % 4 == 0) &&
                     ((reinterpret_cast<uintptr_t>(a.y) & 15) == 0);
    // compile-time shapes: whole blocks per warp, constant per-lane offsets
    if (vec && mode != kTableGlobal && a.T == 256) {
        long long fg = (long long)num_sms * ctas_per_sm;
        const long long need = (a.n_blocks + kDecodeThreads / 32 - 1) / (kDecodeThreads / 32);
        if (fg > need) fg = need;
        if (fg < 1) fg = 1;
        const bool cb16_ok = (mode != kTableF16 || (reinterpret_cast<uintptr_t>(a.cb) & 15) == 0) &&
                             (reinterpret_cast<uintptr_t>(a.bits) & 15) == 0;
        // the table, then one ring of blocks per warp
        const size_t ring = (size_t)(kDecodeThreads / 32) * kDecodeRing * decode_ring_slot_bytes(a.K * 256 / 32);
#define TCQ_DECODE_FAST(LL, KK, MM) \
        if (a.L == LL && a.K == KK && mode == MM && cb16_ok) return launch_fast<LL, KK, 256, MM>(a, (int)fg, smem + ring, stream);
        TCQ_DECODE_FAST(16, 2, kTableF16)
        TCQ_DECODE_FAST(16, 2, kTableMad)
        TCQ_DECODE_FAST(16, 3, kTableF16)
        TCQ_DECODE_FAST(16, 3, kTableMad)
        TCQ_DECODE_FAST(12, 2, kTableF32)
        TCQ_DECODE_FAST(12, 2, kTableMad)
#undef TCQ_DECODE_FAST
    }
    switch (mode * 2 + (vec ? 1 : 0)) {
    case 0: return launch_mode<kTableF32, false>(a, (int)grid, smem, stream);
    case 1: return launch_mode<kTableF32, true>(a, (int)grid, smem, stream);
    case 2: return launch_mode<kTableF16, false>(a, (int)grid, smem, stream);
    case 3: return launch_mode<kTableF16, true>(a, (int)grid, smem, stream);
    case 4: return launch_mode<kTableGlobal, false>(a, (int)grid, smem, stream);
    case 5: return launch_mode<kTableGlobal, true>(a, (int)grid, smem, stream);
    case 6: return launch_mode<kTableMad, false>(a, (int)grid, smem, stream);
    default: return launch_mode<kTableMad, true>(a, (int)grid, smem, stream);
    }
}

}  // namespace tcq
