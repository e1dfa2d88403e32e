// gemv.cu -- matrix-vector product with a trellis-coded matrix, decoding the
// bits on the fly.
//
// The 2-bit post's Pingala-8 section describes the inference side: a fused kernel
// decodes inside the matrix-vector product (advance the state from the bits,
// fetch the codeword), so the weights are never written out.  Here the
// matrix is rows x cols, stored as coding blocks of T consecutive columns per
// row (block (r, j) = r * (cols / T) + j, the layout tcq_encode produces when
// fed the row-major matrix reshaped to [rows * cols / T, T]), each with its
// start state, its bits and an optional fp32 scale:
//     y[r] = sum_j scale[r, j] * sum_t c[s_{r,j,t}] * x[jT + t].
//
// One warp per row.  A lane takes quads of four consecutive weights; as in the
// decoder, the four states are L-bit windows of one 64-bit read (stream word -1
// being the start state).  The codebook and x are staged in shared memory (x
// from L1 when it does not fit); four quads' loads are issued before their
// lookups.  Per weight: a window extract, a table lookup (random addresses, so
// shared-memory bank conflicts bound the kernel), a widening and an FMA; the
// bits are k/8 bytes per weight from HBM.
#include "codes.cuh"

namespace tcq {

namespace {

constexpr int kGemvThreads = 1024;
constexpr int kGemvUnroll = 4;

// CODE: kCodeF32 / kCodeF16 (the table staged in shared memory as fp32 or
// binary16) or kCodeMad (the computed code, no table).
enum GemvCode { kCodeF32 = 0, kCodeF16 = 1, kCodeMad = 2 };

template <int CODE, bool XSMEM>
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_kernel(GemvArgs a)
{
    constexpr bool CB16 = CODE == kCodeF16;
    extern __shared__ __align__(16) unsigned char gsm[];
    const int n_entries = 1 << a.L;
    const size_t tab_bytes = CODE == kCodeMad ? 0 : (size_t)n_entries * (CB16 ? 2 : 4);
    float* xs = reinterpret_cast<float*>(gsm + ((tab_bytes + 15) & ~(size_t)15));
    // stage the codebook (16-byte copies when possible) and x
    if constexpr (CODE == kCodeMad) {
        if constexpr (XSMEM)
            for (long long i = threadIdx.x; i < a.cols; i += blockDim.x) xs[i] = a.x[i];
    } else {
        const unsigned char* src = reinterpret_cast<const unsigned char*>(a.cb);
        if (CB16 || !a.cb_f16) {  // same representation in and out
            if ((reinterpret_cast<uintptr_t>(src) & 15) == 0 && tab_bytes % 16 == 0) {
                const uint4* s4 = reinterpret_cast<const uint4*>(src);
                uint4* d4 = reinterpret_cast<uint4*>(gsm);
                for (int i = threadIdx.x; i < (int)(tab_bytes / 16); i += blockDim.x) d4[i] = s4[i];
            } else {
                for (int i = threadIdx.x; i < (int)tab_bytes; i += blockDim.x) gsm[i] = src[i];
            }
        } else {  // fp16 input held as fp32
            float* tab = reinterpret_cast<float*>(gsm);
            for (int i = threadIdx.x; i < n_entries; i += blockDim.x)
                tab[i] = load_codeword(a.cb, 1, (uint32_t)i);
        }
        if constexpr (XSMEM)
            for (long long i = threadIdx.x; i < a.cols; i += blockDim.x) xs[i] = a.x[i];
    }
    __syncthreads();

    const int L = a.L, K = a.K, T = a.T, W = a.W;
    const int Q = T >> 2;                 // quads per block (T % 4 == 0)
    const bool qpow2 = (Q & (Q - 1)) == 0;
    const int qshift = __ffs(Q) - 1;
    const long long nb = a.cols / T;      // blocks per row
    const int nq = (int)(a.cols >> 2);    // quads per row
    const int lane = threadIdx.x & 31;
    const long long warp0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;

    // A warp's work is the sequence of (row, iteration) items of its rows; the
    // next item's window and scale loads are issued before the current item's
    // lookups, so every lane keeps loads in flight across row boundaries.
    // Per-quad index arithmetic is 32-bit off per-row base pointers, and each
    // state is one funnel shift of the 64-bit window (hi:lo).
    struct Frag {
        uint32_t hi[kGemvUnroll], lo[kGemvUnroll];
        float sc[kGemvUnroll];
        int off[kGemvUnroll];
        int g[kGemvUnroll];
    };
    const int iters = (nq + 32 * kGemvUnroll - 1) / (32 * kGemvUnroll);
    auto fetch = [&](Frag& f, long long r, int it) {
        const uint32_t* rbits = a.bits + r * nb * W;
        const uint32_t* rstart = a.start_state + r * nb;
        const float* rscale = a.scale ? a.scale + r * nb : nullptr;
#pragma unroll
        for (int u = 0; u < kGemvUnroll; ++u) {
            const int g = it * 32 * kGemvUnroll + 32 * u + lane;  // quad index within the row
            const int j = qpow2 ? (g >> qshift) : g / Q;
            const int q = g - j * Q;
            const int p0 = (4 * q + 1) * K - L;
            f.g[u] = g;
            f.off[u] = p0 & 31;
            f.hi[u] = 0u;
            f.lo[u] = 0u;
            f.sc[u] = 0.f;
            if (g < nq) {
                const uint32_t* wb = rbits + j * W;
                const int wi = p0 >> 5;  // -1: the start state is stream word -1
                f.hi[u] = wi < 0 ? rstart[j] : wb[wi];
                f.lo[u] = wi + 1 < W ? wb[wi + 1] : 0u;
                f.sc[u] = rscale ? rscale[j] : 1.f;
            }
        }
    };
    auto consume = [&](const Frag& f) -> float {
        float acc = 0.f;
#pragma unroll
        for (int u = 0; u < kGemvUnroll; ++u) {
            const int g = f.g[u];
            if (g >= nq) break;
            float4 xv;
            if constexpr (XSMEM)
                xv = reinterpret_cast<const float4*>(xs)[g];
            else
                xv = __ldg(reinterpret_cast<const float4*>(a.x) + g);
            // align the window: (hi:lo) << off puts the first state's bits at the
            // top; the four windows then start at bits e k <= 12 of the aligned
            // pair and end before bit 12 + L <= 28 of its high word's range + 32
            const uint32_t ahi = __funnelshift_l(f.lo[u], f.hi[u], f.off[u]);  // off <= 31
            const uint32_t alo = f.lo[u] << f.off[u];
            float c[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint32_t top = e == 0 ? ahi : __funnelshift_l(alo, ahi, e * K);  // e k <= 12
                const uint32_t s = top >> (32 - L);
                if constexpr (CODE == kCodeMad)
                    c[e] = mad_codeword(s);
                else if constexpr (CB16)
                    c[e] = __half2float(reinterpret_cast<const __half*>(gsm)[s]);
                else
                    c[e] = reinterpret_cast<const float*>(gsm)[s];
            }
            const float part = fmaf(c[3], xv.w, fmaf(c[2], xv.z, fmaf(c[1], xv.y, c[0] * xv.x)));
            acc = fmaf(f.sc[u], part, acc);
        }
        return acc;
    };

    long long r = warp0;
    int it = 0;
    Frag cur, nxt;
    if (r < a.rows) fetch(cur, r, it);
    float acc = 0.f;
    while (r < a.rows) {  // r and it are the same in every lane of the warp
        long long rn = r;
        int itn = it + 1;
        if (itn == iters) {
            itn = 0;
            rn += nwarps;
        }
        if (rn < a.rows) fetch(nxt, rn, itn);
        acc += consume(cur);
        if (itn == 0) {  // row r complete
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == 0) a.y[r] = acc;
            acc = 0.f;
        }
        r = rn;
        it = itn;
        cur = nxt;
    }
}

// Compile-time (L, k): an item is N consecutive weights of a block whose N
// state windows all lie in the high word of the 64-bit read once it is aligned
// to the first window, (N-1)k + L <= 32, so a state is one shift and one mask.
// Everything else as gemv_kernel; each item's sum runs as two FMA chains.
template <int L, int K, int N, int CODE, bool XSMEM>
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_fast_kernel(GemvArgs a)
{
    static_assert((N - 1) * K + L <= 32 && N % 4 == 0, "item windows must share one word");
    constexpr bool CB16 = CODE == kCodeF16;
    constexpr int U = 2;  // items per lane per fetch
    constexpr uint32_t MASK = (1u << L) - 1u;
    extern __shared__ __align__(16) unsigned char gsm[];
    const int n_entries = 1 << L;
    const size_t tab_bytes = CODE == kCodeMad ? 0 : (size_t)n_entries * (CB16 ? 2 : 4);
    float* xs = reinterpret_cast<float*>(gsm + ((tab_bytes + 15) & ~(size_t)15));
    if constexpr (CODE == kCodeMad) {
        if constexpr (XSMEM)
            for (long long i = threadIdx.x; i < a.cols; i += blockDim.x) xs[i] = a.x[i];
    } else {
        const unsigned char* src = reinterpret_cast<const unsigned char*>(a.cb);
        if (CB16 || !a.cb_f16) {
            if ((reinterpret_cast<uintptr_t>(src) & 15) == 0 && tab_bytes % 16 == 0) {
                const uint4* s4 = reinterpret_cast<const uint4*>(src);
                uint4* d4 = reinterpret_cast<uint4*>(gsm);
                for (int i = threadIdx.x; i < (int)(tab_bytes / 16); i += blockDim.x) d4[i] = s4[i];
            } else {
                for (int i = threadIdx.x; i < (int)tab_bytes; i += blockDim.x) gsm[i] = src[i];
            }
        } else {
            float* tab = reinterpret_cast<float*>(gsm);
            for (int i = threadIdx.x; i < n_entries; i += blockDim.x)
                tab[i] = load_codeword(a.cb, 1, (uint32_t)i);
        }
        if constexpr (XSMEM)
            for (long long i = threadIdx.x; i < a.cols; i += blockDim.x) xs[i] = a.x[i];
    }
    __syncthreads();

    const int T = a.T, W = a.W;
    const int ipb = T / N;  // items per block
    const bool ipow2 = (ipb & (ipb - 1)) == 0;
    const int ishift = __ffs(ipb) - 1;
    const long long nb = a.cols / T;
    const int ni = (int)(a.cols / N);  // items per row
    const int lane = threadIdx.x & 31;
    const long long warp0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;

    struct Frag {
        uint32_t hi[U], lo[U];
        float sc[U];
        int off[U], i[U];
    };
    const int iters = (ni + 32 * U - 1) / (32 * U);
    auto fetch = [&](Frag& f, long long r, int it) {
        const uint32_t* rbits = a.bits + r * nb * W;
        const uint32_t* rstart = a.start_state + r * nb;
        const float* rscale = a.scale ? a.scale + r * nb : nullptr;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = it * 32 * U + 32 * u + lane;  // item index within the row
            const int j = ipow2 ? (i >> ishift) : i / ipb;
            const int p = i - j * ipb;
            const int p0 = (N * p + 1) * K - L;  // first window of the item
            f.i[u] = i;
            f.off[u] = p0 & 31;
            f.hi[u] = 0u;
            f.lo[u] = 0u;
            f.sc[u] = 0.f;
            if (i < ni) {
                const uint32_t* wb = rbits + j * W;
                const int wi = p0 >> 5;  // -1: the start state is stream word -1
                f.hi[u] = wi < 0 ? rstart[j] : wb[wi];
                f.lo[u] = wi + 1 < W ? wb[wi + 1] : 0u;
                f.sc[u] = rscale ? rscale[j] : 1.f;
            }
        }
    };
    auto consume = [&](const Frag& f) -> float {
        float acc = 0.f;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = f.i[u];
            if (i >= ni) break;
            const uint32_t w = __funnelshift_l(f.lo[u], f.hi[u], f.off[u]);  // off <= 31
            float c[N], xv[N];
#pragma unroll
            for (int e = 0; e < N; ++e) {
                const uint32_t s = (w >> (32 - L - e * K)) & MASK;
                if constexpr (CODE == kCodeMad)
                    c[e] = mad_codeword(s);
                else if constexpr (CB16)
                    c[e] = __half2float(reinterpret_cast<const __half*>(gsm)[s]);
                else
                    c[e] = reinterpret_cast<const float*>(gsm)[s];
            }
#pragma unroll
            for (int e = 0; e < N; e += 4) {
                float4 v;
                if constexpr (XSMEM)
                    v = reinterpret_cast<const float4*>(xs)[(i * N + e) >> 2];
                else
                    v = __ldg(reinterpret_cast<const float4*>(a.x) + ((i * N + e) >> 2));
                xv[e] = v.x;
                xv[e + 1] = v.y;
                xv[e + 2] = v.z;
                xv[e + 3] = v.w;
            }
            float p0 = c[0] * xv[0], p1 = c[N / 2] * xv[N / 2];
#pragma unroll
            for (int e = 1; e < N / 2; ++e) {
                p0 = fmaf(c[e], xv[e], p0);
                p1 = fmaf(c[N / 2 + e], xv[N / 2 + e], p1);
            }
            acc = fmaf(f.sc[u], p0 + p1, acc);
        }
        return acc;
    };

    long long r = warp0;
    int it = 0;
    Frag cur, nxt;
    if (r < a.rows) fetch(cur, r, it);
    float acc = 0.f;
    while (r < a.rows) {  // r and it are the same in every lane of the warp
        long long rn = r;
        int itn = it + 1;
        if (itn == iters) {
            itn = 0;
            rn += nwarps;
        }
        if (rn < a.rows) fetch(nxt, rn, itn);
        acc += consume(cur);
        if (itn == 0) {
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == 0) a.y[r] = acc;
            acc = 0.f;
        }
        r = rn;
        it = itn;
        cur = nxt;
    }
}

// Compile-time (L, k, N) and T: a warp takes whole rows, and within a
// row lane l always holds the same positions of every block (items l, l + 32,
// ... of N weights), so each lane's window offsets are constants and a block's
// words sit at fixed offsets from its base.  A warp walks its rows CH blocks at
// a time and loads the next CH blocks' words (row boundaries included) while
// it sums the current ones, so every lane keeps 2 CH loads in flight.  Per
// weight: the state (a shift and a mask), the codeword, one FMA.  The computed
// code's codeword is one multiply, one byte dot product and n - 255 as a float
// by its bits (the 2^-7 applies once per block with the block scale); a table
// code's is a shared-memory lookup.
// 16 warps of up to 128 registers: eight blocks' words in flight per lane
// (measured 27.1 us on the 14336 x 4096 matrix, against 29.0 us with four
// blocks and 30.0 us with 32 warps of 64 registers)
constexpr int kMadRowsChunk = 8;  // blocks per fetch of gemv_rows_kernel
constexpr int kMadRowsThreads = 512;

template <int L, int K, int N, int T, int CODE>
__global__ void __launch_bounds__(kMadRowsThreads, 1) gemv_rows_kernel(GemvArgs a)
{
    constexpr int IPB = T / N;  // items per block
    static_assert(IPB % 32 == 0 && (N - 1) * K + L <= 32 && N % 4 == 0, "shape");
    constexpr int IPL = IPB / 32;  // items per lane per block
    constexpr int W = (T * K + 31) / 32;
    constexpr int CH = kMadRowsChunk;
    constexpr uint32_t MASK = (1u << L) - 1u;
    extern __shared__ __align__(16) unsigned char gsm[];
    constexpr size_t TAB = CODE == kCodeMad ? 0 : ((size_t(1) << L) * (CODE == kCodeF16 ? 2 : 4) + 15) & ~size_t(15);
    float* xs = reinterpret_cast<float*>(gsm + TAB);
    if constexpr (CODE == kCodeF16) {  // binary16 input, binary16 table
        const uint4* s4 = reinterpret_cast<const uint4*>(a.cb);
        uint4* d4 = reinterpret_cast<uint4*>(gsm);
        for (int i = threadIdx.x; i < (1 << L) / 8; i += blockDim.x) d4[i] = s4[i];
    } else if constexpr (CODE == kCodeF32) {
        float* tab = reinterpret_cast<float*>(gsm);
        for (int i = threadIdx.x; i < (1 << L); i += blockDim.x) tab[i] = load_codeword(a.cb, a.cb_f16, (uint32_t)i);
    }
    for (long long i = threadIdx.x; i < a.cols; i += blockDim.x) xs[i] = a.x[i];
    __syncthreads();

    const int lane = threadIdx.x & 31;
    const long long nb = a.cols / T;
    const long long nch = nb / CH;  // chunks per row
    int wi[IPL], off[IPL];
#pragma unroll
    for (int q = 0; q < IPL; ++q) {
        const int p0 = (N * (lane + 32 * q) + 1) * K - L;  // first window of the item
        wi[q] = p0 >> 5;                                    // -1: the start state
        off[q] = p0 & 31;
    }
    const long long warp0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;

    struct Chunk {
        uint32_t hi[CH][IPL], lo[CH][IPL];
        float sc[CH];
    };
    // words of blocks [c CH, c CH + CH) of row r (the host guarantees CH | nb)
    auto fetch = [&](Chunk& f, long long r, long long c) {
        const uint32_t* rbits = a.bits + (r * nb + c * CH) * W;
        const uint32_t* rstart = a.start_state + r * nb + c * CH;
        const float* rscale = a.scale ? a.scale + r * nb + c * CH : nullptr;
#pragma unroll
        for (int b = 0; b < CH; ++b) {
#pragma unroll
            for (int q = 0; q < IPL; ++q) {
                f.hi[b][q] = wi[q] < 0 ? rstart[b] : rbits[b * W + wi[q]];
                f.lo[b][q] = wi[q] + 1 < W ? rbits[b * W + wi[q] + 1] : 0u;
            }
            f.sc[b] = rscale ? rscale[b] : 1.f;
        }
    };
    auto consume = [&](const Chunk& f, long long c) -> float {
        float acc = 0.f;
        const float* xc = xs + c * (CH * T) + N * lane;
#pragma unroll
        for (int b = 0; b < CH; ++b) {
            float part = 0.f;
#pragma unroll
            for (int q = 0; q < IPL; ++q) {
                const uint32_t w = __funnelshift_l(f.lo[b][q], f.hi[b][q], off[q]);
                const float* xv = xc + b * T + N * 32 * q;
                float p0 = 0.f, p1 = 0.f;
#pragma unroll
                for (int e = 0; e < N; e += 4) {
                    const float4 v = *reinterpret_cast<const float4*>(xv + e);
                    const float xe[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const uint32_t st = (w >> (32 - L - (e + g) * K)) & MASK;
                        float cv;
                        if constexpr (CODE == kCodeMad) {
                            // the byte sum lands on the bits of 2^23: 2^23 + n exactly
                            const uint32_t nb23 = __dp4a(st * kMadA, 0x01010000u, 0x4B000000u);
                            cv = __uint_as_float(nb23) - 8388863.0f;  // n - 255
                        } else if constexpr (CODE == kCodeF16) {
                            cv = __half2float(reinterpret_cast<const __half*>(gsm)[st]);
                        } else {
                            cv = reinterpret_cast<const float*>(gsm)[st];
                        }
                        if (g & 1)
                            p1 = fmaf(cv, xe[g], p1);
                        else
                            p0 = fmaf(cv, xe[g], p0);
                    }
                }
                part += p0 + p1;
            }
            // (n - 255) / 128 for the computed code
            acc = fmaf(CODE == kCodeMad ? f.sc[b] * 0.0078125f : f.sc[b], part, acc);
        }
        return acc;
    };

    // the warp's (row, chunk) sequence, two chunks per turn so that the buffers
    // alternate without copies: A is summed while B loads, then the reverse
    long long r = warp0, c = 0;
    auto advance = [&](long long& rr, long long& cc) {
        if (++cc == nch) {
            cc = 0;
            rr += nwarps;
        }
    };
    Chunk A, B;
    if (r < a.rows) fetch(A, r, c);
    float acc = 0.f;
    auto finish_row = [&](long long row) {
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) a.y[row] = acc;
        acc = 0.f;
    };
    while (r < a.rows) {  // r and c are the same in every lane of the warp
        long long r1 = r, c1 = c;
        advance(r1, c1);
        if (r1 < a.rows) fetch(B, r1, c1);
        acc += consume(A, c);
        if (c1 == 0) finish_row(r);
        if (r1 >= a.rows) break;
        long long r2 = r1, c2 = c1;
        advance(r2, c2);
        if (r2 < a.rows) fetch(A, r2, c2);
        acc += consume(B, c1);
        if (c2 == 0) finish_row(r1);
        r = r2;
        c = c2;
    }
}

template <int L, int K, int N, int T, int CODE>
cudaError_t launch_gemv_rows(const GemvArgs& a, int grid, cudaStream_t stream)
{
    const size_t tab = CODE == kCodeMad ? 0 : (((size_t)1 << L) * (CODE == kCodeF16 ? 2 : 4) + 15) & ~(size_t)15;
    const size_t smem = tab + (size_t)a.cols * 4;
    cudaError_t e = cudaFuncSetAttribute(gemv_rows_kernel<L, K, N, T, CODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    gemv_rows_kernel<L, K, N, T, CODE><<<grid, kMadRowsThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

template <int L, int K, int N, int CODE, bool XSMEM>
cudaError_t launch_gemv_fast_t(const GemvArgs& a, int grid, size_t smem, cudaStream_t stream)
{
    cudaError_t e = cudaFuncSetAttribute(gemv_fast_kernel<L, K, N, CODE, XSMEM>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    gemv_fast_kernel<L, K, N, CODE, XSMEM><<<grid, kGemvThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

template <int CODE, bool XSMEM>
cudaError_t launch_gemv_t(const GemvArgs& a, int grid, size_t smem, cudaStream_t stream)
{
    cudaError_t e = cudaFuncSetAttribute(gemv_kernel<CODE, XSMEM>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    gemv_kernel<CODE, XSMEM><<<grid, kGemvThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemv(const GemvArgs& a, int num_sms, cudaStream_t stream)
{
    const size_t entries = (size_t)1 << a.L;
    const bool mad = a.cb_f16 == kMadCodebook;
    // the table as fp32 when it fits in 64 KiB, else as binary16 (binary16 input only;
    // the host refuses a binary32 table of 2^15 or more entries); none for the computed code
    const bool cb16 = !mad && entries * 4 > 64 * 1024;
    const int code = mad ? kCodeMad : cb16 ? kCodeF16 : kCodeF32;
    const size_t tab = mad ? 0 : (entries * (cb16 ? 2 : 4) + 15) & ~(size_t)15;
    const size_t xbytes = (size_t)a.cols * 4;
    const bool xsmem = tab + xbytes <= 200 * 1024;
    const size_t smem = tab + (xsmem ? xbytes : 0);
    const long long warps_per_cta = kGemvThreads / 32;
    long long grid = (a.rows + warps_per_cta - 1) / warps_per_cta;
    if (grid > num_sms) grid = num_sms;
    if (grid < 1) grid = 1;
    // computed code at T = 256: whole rows per warp, constant per-lane offsets
    // T = 256: whole rows per warp, constant per-lane offsets
    const bool rows_ok = xsmem && a.T == 256 && (a.cols / 256) % kMadRowsChunk == 0;
#define TCQ_GEMV_ROWS(LL, KK, NN, CC) \
    if (rows_ok && a.L == LL && a.K == KK && code == CC) return launch_gemv_rows<LL, KK, NN, 256, CC>(a, (int)grid, stream);
    TCQ_GEMV_ROWS(16, 2, 8, kCodeMad)
    TCQ_GEMV_ROWS(16, 3, 4, kCodeMad)
    TCQ_GEMV_ROWS(16, 2, 8, kCodeF16)
    TCQ_GEMV_ROWS(16, 3, 4, kCodeF16)
    TCQ_GEMV_ROWS(12, 2, 8, kCodeF32)
#undef TCQ_GEMV_ROWS
    // specialised (L, k): compile-time shifts and masks, 8 or 4 weights per item
#define TCQ_GEMV_FAST(LL, KK, NN, CC)                                                         \
    if (a.L == LL && a.K == KK && code == CC && a.T % NN == 0)                                 \
        return xsmem ? launch_gemv_fast_t<LL, KK, NN, CC, true>(a, (int)grid, smem, stream) \
                     : launch_gemv_fast_t<LL, KK, NN, CC, false>(a, (int)grid, smem, stream);
    TCQ_GEMV_FAST(16, 2, 8, kCodeF16)
    TCQ_GEMV_FAST(16, 3, 4, kCodeF16)
    TCQ_GEMV_FAST(12, 2, 8, kCodeF32)
    TCQ_GEMV_FAST(8, 2, 8, kCodeF32)
    TCQ_GEMV_FAST(16, 2, 8, kCodeMad)
    TCQ_GEMV_FAST(16, 3, 4, kCodeMad)
#undef TCQ_GEMV_FAST
    if (mad)
        return xsmem ? launch_gemv_t<kCodeMad, true>(a, (int)grid, smem, stream)
                     : launch_gemv_t<kCodeMad, false>(a, (int)grid, smem, stream);
    if (cb16)
        return xsmem ? launch_gemv_t<kCodeF16, true>(a, (int)grid, smem, stream)
                     : launch_gemv_t<kCodeF16, false>(a, (int)grid, smem, stream);
    return xsmem ? launch_gemv_t<kCodeF32, true>(a, (int)grid, smem, stream)
                 : launch_gemv_t<kCodeF32, false>(a, (int)grid, smem, stream);
}

}  // namespace tcq
