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
#ifdef TCQ_DEBUG
    const long long nblk = a.rows * nb;
#endif

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
            if (g < nq && TCQ_IN_BOUNDS(r * nb + j, nblk)) {
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
            if (lane == 0 && TCQ_IN_BOUNDS(r, a.rows)) a.y[r] = acc;
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
#ifdef TCQ_DEBUG
    const long long nblk = a.rows * nb;
#endif

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
            if (i < ni && TCQ_IN_BOUNDS(r * nb + j, nblk)) {
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
            if (lane == 0 && TCQ_IN_BOUNDS(r, a.rows)) a.y[r] = acc;
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
        if (!TCQ_IN_BOUNDS(r * nb + c * CH + CH - 1, a.rows * nb)) return;
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
        if (lane == 0 && TCQ_IN_BOUNDS(row, a.rows)) a.y[row] = acc;
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

// ---------------------------------------------------------------------------
// L = 16, k = 2, T = 256, cols a multiple of 4096: the layout for the matrices
// a model layer has.  A warp's lane (j, h) = (lane >> 1, lane & 1) takes half h
// (128 weights, 8 stream words) of the coding block j of a 16-block (4096
// column) chunk, for three rows at a time: the lane's x values are then the
// same for the three rows (measured: 35.3 us against 37.3 us with two rows per
// item for the table code, the same 21.0 us for the computed code, at 128
// registers without spills), its words are two 16-byte loads per row (a half-warp reads
// 1 KiB of one row contiguously), the window before its first weight is the
// block's start state (h = 0) or the block's word 7 (h = 1), and the row sums
// need one 5-step warp reduction per row.  x sits in shared memory with 16
// bytes of padding after every 128 values, so the 16-byte loads of 8
// consecutive lanes hit 8 different bank quads.
//
// States, 16 windows per stream word lo (with hi the word before): window i
// (i = 1..16) is bits [32 - 2i, 48 - 2i) of the 64-bit hi:lo.  Seven funnel
// shifts give "views" of the pair at bit offsets 2, 4, 6, 16, 18, 20, 22, in
// which every window starts at bit 0, 8 or 16, so each state is then one
// byte permutation, mask or shift (23 instructions per 16 states instead of 2
// per state).
//
// Rows: phase A gives every warp of the grid the same number of row groups
// (three rows); when the rows of the last, partial round are at most one per
// CTA, they are phase B, one row per CTA, its stream words spread over all the
// CTA's threads (each computes one word's two FMA chains) and then combined by
// one warp in phase A's order, so that the last round costs a fraction of a row
// instead of a whole row group.  Otherwise (fewer row groups than warps, or a
// large remainder) the partial round stays in phase A, the first warps taking
// one group more, and phase B takes only the rows of no whole group.  A row's
// result is the same bits whichever phase computes it, and every sum has a
// fixed order: the result does not depend on timing.
//
// Rounding depth of a product (the tolerance tests/test_gpu_gemv.py uses):
// 8 in a word's FMA chain, 8 over the words into the half-block sum, 1 for the
// two half-block sums, 1 for the scale, c = cols / 4096 over the chunks, 5 in
// the warp reduction: 23 + c <= 13 + cols / 256.
// ---------------------------------------------------------------------------
constexpr int kPairThreads = 512;
constexpr int kPairWarps = kPairThreads / 32;
// rows per warp item: three when every warp has at least three rows (the x
// loads serve three rows), else one, so that every warp has work
constexpr int kPairRowsMax = 3;

// padded position of x[i] in shared memory: 4 floats of padding per 128
__device__ __forceinline__ int xpad(int i) { return i + ((i >> 7) << 2); }

// byte permutation of (b:a) with selector sel (PTX prmt, default mode)
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// The 16 states of stream word lo (hi is the word before), in stream order.
__device__ __forceinline__ void states16(uint32_t hi, uint32_t lo, uint32_t (&s)[16])
{
    const uint32_t v2 = __funnelshift_r(lo, hi, 2), v4 = __funnelshift_r(lo, hi, 4);
    const uint32_t v6 = __funnelshift_r(lo, hi, 6), v16 = __funnelshift_r(lo, hi, 16);
    const uint32_t v18 = __funnelshift_r(lo, hi, 18), v20 = __funnelshift_r(lo, hi, 20);
    const uint32_t v22 = __funnelshift_r(lo, hi, 22);
    // window i starts at bit 32 - 2i of hi:lo; 0x4421 picks bytes 1, 2 and two zero
    // bytes of the second operand (0): bits 8..23
    s[0] = prmt(v22, 0u, 0x4421);   // i = 1, bit 30 = 22 + 8
    s[1] = prmt(v20, 0u, 0x4421);   // i = 2, bit 28
    s[2] = prmt(v18, 0u, 0x4421);   // i = 3, bit 26
    s[3] = prmt(v16, 0u, 0x4421);   // i = 4, bit 24
    s[4] = v22 & 0xFFFFu;           // i = 5, bit 22
    s[5] = v20 & 0xFFFFu;           // i = 6, bit 20
    s[6] = v18 & 0xFFFFu;           // i = 7, bit 18
    s[7] = v16 & 0xFFFFu;           // i = 8, bit 16
    s[8] = prmt(v6, 0u, 0x4421);    // i = 9, bit 14
    s[9] = prmt(v4, 0u, 0x4421);    // i = 10, bit 12
    s[10] = prmt(v2, 0u, 0x4421);   // i = 11, bit 10
    s[11] = prmt(lo, 0u, 0x4421);   // i = 12, bit 8
    s[12] = v6 & 0xFFFFu;           // i = 13, bit 6
    s[13] = v4 & 0xFFFFu;           // i = 14, bit 4
    s[14] = v2 & 0xFFFFu;           // i = 15, bit 2
    s[15] = lo & 0xFFFFu;           // i = 16, bit 0
}

// Codeword of state s: the computed code as 128 c (n - 255, exact; the 2^-7 goes
// with the block scale), or the binary16 table entry.
template <int CODE>
__device__ __forceinline__ float pair_codeword(uint32_t s, const __half* tab)
{
    if constexpr (CODE == kCodeMad) {
        const uint32_t nb23 = __dp4a(s * kMadA, 0x01010000u, 0x4B000000u);  // bits of 2^23 + n
        return __uint_as_float(nb23) - 8388863.0f;
    } else {
        return __half2float(tab[s]);
    }
}

__device__ __forceinline__ unsigned long long pack2(float a, float b)
{
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}

__device__ __forceinline__ void unpack2(unsigned long long v, float& a, float& b)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}

// sum over the 16 weights of stream word lo of c[s] x, as two chains of 8
template <int CODE>
__device__ __forceinline__ void word_dot(uint32_t hi, uint32_t lo, const float* __restrict__ xq,
                                         const __half* tab, float& acc0, float& acc1)
{
    uint32_t st[16];
    states16(hi, lo, st);
    if constexpr (CODE == kCodeMad) {
        // two weights per instruction for the float part: (n - 255) of both by
        // one packed subtraction, both products into the pair of chains by one
        // packed FMA (each half rounds like the scalar operation, so the sums
        // are those of two scalar chains)
        const unsigned long long off = pack2(-8388863.0f, -8388863.0f);
        unsigned long long p = 0ull;
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
            const float4 v = *reinterpret_cast<const float4*>(xq + e);
#pragma unroll
            for (int h = 0; h < 4; h += 2) {
                const uint32_t n0 = __dp4a(st[e + h] * kMadA, 0x01010000u, 0x4B000000u);
                const uint32_t n1 = __dp4a(st[e + h + 1] * kMadA, 0x01010000u, 0x4B000000u);
                unsigned long long c2;
                asm("add.rn.f32x2 %0, %1, %2;" : "=l"(c2) : "l"(pack2(__uint_as_float(n0), __uint_as_float(n1))), "l"(off));
                const unsigned long long x2 = h == 0 ? pack2(v.x, v.y) : pack2(v.z, v.w);
                if (e == 0 && h == 0)
                    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(p) : "l"(c2), "l"(x2));
                else
                    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(p) : "l"(c2), "l"(x2), "l"(p));
            }
        }
        float p0, p1;
        unpack2(p, p0, p1);
        acc0 += p0;
        acc1 += p1;
    } else {
        float xv[16];
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
            const float4 v = *reinterpret_cast<const float4*>(xq + e);
            xv[e] = v.x;
            xv[e + 1] = v.y;
            xv[e + 2] = v.z;
            xv[e + 3] = v.w;
        }
        float p0 = pair_codeword<CODE>(st[0], tab) * xv[0];
        float p1 = pair_codeword<CODE>(st[1], tab) * xv[1];
#pragma unroll
        for (int e = 2; e < 16; e += 2) {
            p0 = fmaf(pair_codeword<CODE>(st[e], tab), xv[e], p0);
            p1 = fmaf(pair_codeword<CODE>(st[e + 1], tab), xv[e + 1], p1);
        }
        acc0 += p0;
        acc1 += p1;
    }
}

template <int CODE, int R>
__global__ void __launch_bounds__(kPairThreads, 1) gemv_pair_kernel(GemvArgs a)
{
    constexpr int kPairRows = R;  // rows per warp item
    constexpr int T = 256, W = 16;
    extern __shared__ __align__(16) unsigned char gsm[];
    constexpr size_t TAB = CODE == kCodeMad ? 0 : ((size_t)1 << 16) * 2;
    const __half* tab = reinterpret_cast<const __half*>(gsm);
    float* xs = reinterpret_cast<float*>(gsm + TAB);
    float* wsum = xs + xpad((int)a.cols);  // phase B: the (p0, p1) of every word of a row
    // stage the table (16-byte asynchronous copies) and x (padded)
    if constexpr (CODE != kCodeMad) {
        const char* src = reinterpret_cast<const char*>(a.cb);
        const uint32_t dst = (uint32_t)__cvta_generic_to_shared(gsm);
        for (int i = threadIdx.x; i < (int)(TAB / 16); i += blockDim.x)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + 16 * i),
                         "l"(src + 16 * (size_t)i) : "memory");
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
    for (int i = threadIdx.x; i < (int)(a.cols / 4); i += blockDim.x) {
        const float4 v = reinterpret_cast<const float4*>(a.x)[i];
        *reinterpret_cast<float4*>(xs + xpad(4 * i)) = v;
    }

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int jl = lane >> 1, h = lane & 1;  // block of the 16-block chunk, half
    const long long nb = a.cols / T;
    const int nch = (int)(nb / 16);          // 4096-column chunks per row
    const float sc_code = CODE == kCodeMad ? 0.0078125f : 1.f;
    // warps ranked warp-major over the CTAs, so that a partial round's groups
    // (ranks below `extra`) spread over every SM instead of filling the first CTAs
    const long long gw = (long long)warp * gridDim.x + blockIdx.x;
    const long long nw = (long long)gridDim.x * kPairWarps;
    const long long pairs = a.rows / kPairRows;  // row groups
    const long long rounds = pairs / nw;     // whole rounds of phase A
    const long long extra = pairs - rounds * nw;  // groups of the partial round
    // the partial round in phase A unless its rows (and the rows of no group)
    // are at most one per CTA
    const bool partial = extra * kPairRows + (a.rows - pairs * kPairRows) > (long long)gridDim.x;

    // ---- phase A
    struct Item {
        uint4 w[kPairRows][2];
        uint32_t prev[kPairRows];
        float sc[kPairRows];
    };
    auto fetch = [&](Item& it, long long r0, int c) {
#pragma unroll
        for (int i = 0; i < kPairRows; ++i) {
            const long long b = (r0 + i) * nb + 16LL * c + jl;
            if (!TCQ_IN_BOUNDS(b, a.rows * nb)) continue;
            const uint4* wp = reinterpret_cast<const uint4*>(a.bits + b * W + 8 * h);
            it.w[i][0] = wp[0];
            it.w[i][1] = wp[1];
            it.prev[i] = h ? a.bits[b * W + 7] : a.start_state[b];
            it.sc[i] = (a.scale ? a.scale[b] : 1.f) * sc_code;
        }
    };
    auto consume = [&](const Item& it, int c, float (&row)[kPairRows]) {
        const float* xl = xs + xpad(c * 4096 + 128 * lane);  // the lane's 128 x values, unpadded inside
        float a0[kPairRows], a1[kPairRows];
#pragma unroll
        for (int i = 0; i < kPairRows; ++i) a0[i] = a1[i] = 0.f;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
#pragma unroll
            for (int i = 0; i < kPairRows; ++i) {
                const uint32_t* wd = reinterpret_cast<const uint32_t*>(&it.w[i][0]);
                const uint32_t hi = q == 0 ? it.prev[i] : wd[q - 1];
                word_dot<CODE>(hi, wd[q], xl + 16 * q, tab, a0[i], a1[i]);
            }
        }
#pragma unroll
        for (int i = 0; i < kPairRows; ++i) row[i] = fmaf(it.sc[i], a0[i] + a1[i], row[i]);
    };
    // items (pair, chunk) of this warp in order; two buffers, no copies.  The
    // first item's loads are in flight while the table and x are staged.
    const long long n_items = (rounds + (partial && gw < extra ? 1 : 0)) * nch;
    auto item_row = [&](long long t) { return (gw + (t / nch) * nw) * kPairRows; };
    Item A, B;
    if (n_items > 0) fetch(A, item_row(0), 0);
    // phase B's first row: each thread's first task's two words, loaded before
    // the staging barrier so that their latency overlaps it
    const long long first_b = (partial ? pairs : rounds * nw) * kPairRows;
    const long long rb0 = first_b + blockIdx.x;
    uint32_t pre_hi = 0u, pre_lo = 0u;
    if (rb0 < a.rows && (int)threadIdx.x < nch * 256) {
        const int c = threadIdx.x >> 8, ln = (threadIdx.x >> 3) & 31, q = threadIdx.x & 7;
        const long long b = rb0 * nb + 16LL * c + (ln >> 1);
        if (TCQ_IN_BOUNDS(b, a.rows * nb)) {
            const uint32_t* wb = a.bits + b * W;
            pre_hi = q > 0 ? wb[8 * (ln & 1) + q - 1] : (ln & 1) ? wb[7] : a.start_state[b];
            pre_lo = wb[8 * (ln & 1) + q];
        }
    }
    if constexpr (CODE != kCodeMad) asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    // ---- phase B, first: the rows phase A leaves, one per CTA at a time (their
    // loads overlap the staging and phase A's first loads; warp 0's final sums
    // overlap the other warps' phase A).  The row's arithmetic is phase A's
    // exactly, so that a row's result does not depend on the phase that
    // computes it: every thread takes stream words (the word's two FMA chains,
    // word_dot from zero), then warp 0, lane = half block, adds the eight words
    // of its half in order, scales per chunk, and runs the same five-step
    // butterfly.
    for (long long r = rb0; r < a.rows; r += gridDim.x) {
        if (r != rb0) __syncthreads();  // warp 0 has read the previous row's sums
        for (int task = threadIdx.x; task < nch * 256; task += blockDim.x) {
            const int c = task >> 8, ln = (task >> 3) & 31, q = task & 7;  // chunk, half block (lane), word
            const int jb = ln >> 1, hb = ln & 1;
            const long long b = r * nb + 16LL * c + jb;
            float p0 = 0.f, p1 = 0.f;
            if (TCQ_IN_BOUNDS(b, a.rows * nb)) {
                const uint32_t* wb = a.bits + b * W;
                const bool pre = r == rb0 && task == (int)threadIdx.x;
                const uint32_t hi = pre ? pre_hi : q > 0 ? wb[8 * hb + q - 1] : hb ? wb[7] : a.start_state[b];
                const uint32_t lo = pre ? pre_lo : wb[8 * hb + q];
                word_dot<CODE>(hi, lo, xs + xpad(c * 4096 + 128 * ln) + 16 * q, tab, p0, p1);
            }
            wsum[2 * task] = p0;
            wsum[2 * task + 1] = p1;
        }
        __syncthreads();
        if (warp == 0) {
            float v = 0.f;
            for (int c = 0; c < nch; ++c) {
                const long long b = r * nb + 16LL * c + jl;
                float a0 = 0.f, a1 = 0.f;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int task = (c << 8) | (lane << 3) | q;
                    a0 += wsum[2 * task];
                    a1 += wsum[2 * task + 1];
                }
                const float sc = (a.scale && TCQ_IN_BOUNDS(b, a.rows * nb) ? a.scale[b] : 1.f) * sc_code;
                v = fmaf(sc, a0 + a1, v);
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0 && TCQ_IN_BOUNDS(r, a.rows)) a.y[r] = v;
        }
    }

    if (n_items > 0) {
        float row[kPairRows];
#pragma unroll
        for (int i = 0; i < kPairRows; ++i) row[i] = 0.f;
        auto finish = [&](long long t) {  // item t was the last chunk of its pair
            const long long r0 = item_row(t);
#pragma unroll
            for (int i = 0; i < kPairRows; ++i) {
                float v = row[i];
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0 && TCQ_IN_BOUNDS(r0 + i, a.rows)) a.y[r0 + i] = v;
                row[i] = 0.f;
            }
        };
        for (long long t = 0; t < n_items; t += 2) {
            if (t + 1 < n_items) fetch(B, item_row(t + 1), (int)((t + 1) % nch));
            consume(A, (int)(t % nch), row);
            if ((t + 1) % nch == 0) finish(t);
            if (t + 1 >= n_items) break;
            if (t + 2 < n_items) fetch(A, item_row(t + 2), (int)((t + 2) % nch));
            consume(B, (int)((t + 1) % nch), row);
            if ((t + 2) % nch == 0) finish(t + 1);
        }
    }


}

cudaError_t launch_gemv_pair(const GemvArgs& a, int num_sms, cudaStream_t stream, bool mad)
{
    const size_t tab = mad ? 0 : ((size_t)1 << 16) * 2;
    // x padded, then phase B's two floats per stream word of a row (cols / 16 words)
    const size_t smem = tab + (size_t)(a.cols + (a.cols / 128) * 4) * 4 + (size_t)(a.cols / 16) * 2 * 4;
    int grid = num_sms;  // one CTA of 16 warps per SM
    const bool three = a.rows >= (long long)kPairRowsMax * grid * kPairWarps;
    const void* fn = mad ? (three ? reinterpret_cast<const void*>(&gemv_pair_kernel<kCodeMad, 3>)
                                  : reinterpret_cast<const void*>(&gemv_pair_kernel<kCodeMad, 1>))
                         : (three ? reinterpret_cast<const void*>(&gemv_pair_kernel<kCodeF16, 3>)
                                  : reinterpret_cast<const void*>(&gemv_pair_kernel<kCodeF16, 1>));
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (mad && three)
        gemv_pair_kernel<kCodeMad, 3><<<grid, kPairThreads, smem, stream>>>(a);
    else if (mad)
        gemv_pair_kernel<kCodeMad, 1><<<grid, kPairThreads, smem, stream>>>(a);
    else if (three)
        gemv_pair_kernel<kCodeF16, 3><<<grid, kPairThreads, smem, stream>>>(a);
    else
        gemv_pair_kernel<kCodeF16, 1><<<grid, kPairThreads, smem, stream>>>(a);
    return cudaGetLastError();
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
    // L = 16, k = 2, T = 256 and 4096-column chunks: three rows per warp item, lanes on
    // half blocks (16-byte loads of the bits and, for the table, of the codebook)
    if (a.L == 16 && a.K == 2 && a.T == 256 && a.cols % 4096 == 0 && (code == kCodeMad || code == kCodeF16) &&
        (reinterpret_cast<uintptr_t>(a.bits) & 15) == 0 &&
        (code == kCodeMad || (reinterpret_cast<uintptr_t>(a.cb) & 15) == 0) &&
        (code == kCodeMad ? 0 : 131072) + (size_t)(a.cols + a.cols / 32) * 4 + (size_t)(a.cols / 8) * 4 <= 220 * 1024)
        return launch_gemv_pair(a, num_sms, stream, code == kCodeMad);
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
