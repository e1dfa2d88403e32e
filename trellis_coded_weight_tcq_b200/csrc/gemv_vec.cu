// gemv_vec.cu -- decode-in-matvec for the vector trellis (V weights per step):
// y = (trellis-coded matrix) x with the weights decoded in registers, as
// tcq_gemv does for V = 1 (the 2-bit post's Pingala-8 section: the decoder runs
// inside the matrix-vector product, so the weights are never materialised).
//
// Block (r, j) of the rows x cols matrix covers columns [jT, jT + T) of row r;
// its step t (1-based) holds weights (t-1)V .. tV-1 of the block, the V entries
// of the codeword of the L-bit window ending at stream bit t kV - 1 (word -1 of
// the stream is the start state).
//     y[r] = sum_j scale[r, j] * sum_t sum_v c[s_{r,j,t}][v] x[jT + (t-1)V + v]
//
// Two kernels, both one warp per row:
//   gemv_vec2_kernel  L = 16, k = 2, V = 2, binary16 pairs (16-byte aligned),
//                     T % 8 == 0: lane l takes steps 4l+1 .. 4l+4 of each
//                     128-step chunk (two stream words, as in the vector
//                     decoder), the pair table's first seven eighths in shared
//                     memory and the rest through the read-only cache, x in
//                     16-byte loads through the cache, the loads of two
//                     (block, chunk) items in flight together (measured best
//                     of 1, 2 and 4);
//   gemv_vec_kernel   any supported (L, k, V) and dtype: lanes stride over a
//                     block's steps, codewords through the cache.
#include "common.cuh"

namespace tcq {

namespace {

constexpr int kGemvVec2Threads = 1024;
constexpr uint32_t kGemvVec2SmemStates = 0xE000u;
constexpr int kGemvVec2Unroll = 2;  // (block, chunk) items whose loads are in flight together

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// One (block, chunk) item of row r for this lane: its share of the item's dot
// product (four steps, eight weights, one FMA chain) and the block's scale.
// `on` is false (and part 0) when the lane has no steps in the item.
struct Vec2Item {
    unsigned long long v;
    float4 x0, x1;
    float sc;
    bool on;
};

__device__ __forceinline__ void vec2_item_load(const GemvArgs& a, long long r, long long i, int chunks,
                                               int NS, long long nb, long long items, int lane, Vec2Item& it)
{
    const long long j = chunks == 1 ? i : i / chunks;
    const int c = (int)(i - j * chunks);
    const int t0 = (c << 7) + 4 * lane;  // steps t0+1 .. t0+4
    it.on = i < items && t0 + 4 <= NS;   // NS % 4 == 0
    it.v = 0ull;
    it.x0 = it.x1 = make_float4(0.f, 0.f, 0.f, 0.f);
    it.sc = 0.f;
    if (it.on) {
        const long long b = r * nb + j;
        const uint32_t* wb = a.bits + b * a.W;
        const int wi = (c << 4) + (lane >> 1);
        const unsigned long long hi = wi >= 1 ? __ldg(wb + wi - 1) : __ldg(a.start_state + b);
        it.v = (hi << 32) | __ldg(wb + wi);
        const float* xb = a.x + j * a.T + 2 * t0;
        it.x0 = __ldg(reinterpret_cast<const float4*>(xb));
        it.x1 = __ldg(reinterpret_cast<const float4*>(xb + 4));
        it.sc = a.scale ? __ldg(a.scale + b) : 1.f;
    }
}

__device__ __forceinline__ float vec2_item_part(const Vec2Item& it, const uint32_t* tab, const uint32_t* cb,
                                                int lane)
{
    const float xs[8] = {it.x0.x, it.x0.y, it.x0.z, it.x0.w, it.x1.x, it.x1.y, it.x1.z, it.x1.w};
    float part = 0.f;
#pragma unroll
    for (int q = 1; q <= 4; ++q) {
        const int sh = 48 - (16 * (lane & 1) + 4 * q + 16);
        const uint32_t s = (uint32_t)(it.v >> sh) & 0xffffu;
        const uint32_t w = s < kGemvVec2SmemStates ? tab[s] : __ldg(cb + s);
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w));
        part = fmaf(f.x, xs[2 * q - 2], part);
        part = fmaf(f.y, xs[2 * q - 1], part);
    }
    return part;
}

// Rows: whole rounds give every warp one row at a time; the rows of the last,
// partial round, when they are at most one per CTA and a row's items fit the
// shared memory left beside the table, go one per CTA with its items spread
// over the CTA's warps, each lane's share of each item stored and then summed
// by one warp in item order with the same FMAs, so that a row's result is the
// same bits either way (14336 rows over 4736 warps left 64 warps a fourth row
// while the others idled).
constexpr int kGemvVec2MaxSplitItems = 23;  // items x (32 + 1) floats in the 3 KiB left

__global__ void __launch_bounds__(kGemvVec2Threads) gemv_vec2_kernel(GemvArgs a)
{
    extern __shared__ __align__(16) uint32_t tab[];  // [kGemvVec2SmemStates], then the split row's shares
    const uint32_t* cb = reinterpret_cast<const uint32_t*>(a.cb);
    {
        // the table by asynchronous 16-byte copies, all in flight at once
        const uint32_t dst = (uint32_t)__cvta_generic_to_shared(tab);
        for (int i = threadIdx.x; i < (int)(kGemvVec2SmemStates / 4); i += blockDim.x)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + 16 * i),
                         "l"(cb + 4 * (size_t)i) : "memory");
        asm volatile("cp.async.commit_group;" ::: "memory");
        asm volatile("cp.async.wait_all;" ::: "memory");
    }
    __syncthreads();
    const int NS = a.T >> 1;
    const int chunks = (NS + 127) >> 7;
    const long long nb = a.cols / a.T;  // blocks per row
    const long long items = nb * chunks;  // (block, 128-step chunk) pairs of a row
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
    const long long full = (a.rows / nw) * nw;
    const bool split = items <= kGemvVec2MaxSplitItems && a.rows - full <= (long long)gridDim.x;
    const long long rows_a = split ? full : a.rows;
    for (long long r = (long long)blockIdx.x * (blockDim.x >> 5) + warp; r < rows_a; r += nw) {
        float acc = 0.f;
        // kGemvVec2Unroll items at a time: all their loads issue before any use
        for (long long i0 = 0; i0 < items; i0 += kGemvVec2Unroll) {
            Vec2Item it[kGemvVec2Unroll];
#pragma unroll
            for (int u = 0; u < kGemvVec2Unroll; ++u)
                vec2_item_load(a, r, i0 + u, chunks, NS, nb, items, lane, it[u]);
#pragma unroll
            for (int u = 0; u < kGemvVec2Unroll; ++u)
                if (it[u].on) acc = fmaf(it[u].sc, vec2_item_part(it[u], tab, cb, lane), acc);
        }
        acc = warp_sum(acc);
        if (lane == 0) a.y[r] = acc;
    }
    if (!split) return;
    float* share = reinterpret_cast<float*>(tab + kGemvVec2SmemStates);  // [items][33]: 32 lanes, the scale
    for (long long r = full + blockIdx.x; r < a.rows; r += gridDim.x) {
        for (long long i = warp; i < items; i += blockDim.x >> 5) {
            Vec2Item it;
            vec2_item_load(a, r, i, chunks, NS, nb, items, lane, it);
            share[i * 33 + lane] = it.on ? vec2_item_part(it, tab, cb, lane) : 0.f;
            if (lane == 0) share[i * 33 + 32] = it.sc;
        }
        __syncthreads();
        if (warp == 0) {
            float acc = 0.f;
            for (long long i = 0; i < items; ++i) {
                const long long j = chunks == 1 ? i : i / chunks;
                const int c = (int)(i - j * chunks);
                if ((c << 7) + 4 * lane + 4 <= NS)  // the lanes with steps in the item, as in phase A
                    acc = fmaf(share[i * 33 + 32], share[i * 33 + lane], acc);
            }
            acc = warp_sum(acc);
            if (lane == 0) a.y[r] = acc;
        }
        __syncthreads();
    }
}

__global__ void __launch_bounds__(256) gemv_vec_kernel(GemvArgs a, int V)
{
    const int L = a.L, K = a.K, NS = a.T / V;
    const uint32_t mask = (1u << L) - 1u;
    const long long nb = a.cols / a.T;
    const int lane = threadIdx.x & 31;
    for (long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < a.rows;
         r += ((long long)gridDim.x * blockDim.x) >> 5) {
        float acc = 0.f;
        for (long long j = 0; j < nb; ++j) {
            const long long b = r * nb + j;
            const uint32_t* wb = a.bits + b * a.W;
            const float* xb = a.x + j * a.T;
            float part = 0.f;
            for (int t = lane + 1; t <= NS; t += 32) {
                const int p0 = t * K - L;  // window start, > -32
                const int wi = p0 >> 5;
                const unsigned long long hi = wi < 0 ? a.start_state[b] : wb[wi];
                const unsigned long long lo = wi + 1 < a.W ? wb[wi + 1] : 0ull;
                const uint32_t s = (uint32_t)((((hi << 32) | lo) >> (64 - (p0 & 31) - L)) & mask);
                for (int v = 0; v < V; ++v)
                    part = fmaf(load_codeword(a.cb, a.cb_f16, s * V + v), xb[(t - 1) * V + v], part);
            }
            acc = a.scale ? fmaf(a.scale[b], part, acc) : acc + part;
        }
        acc = warp_sum(acc);
        if (lane == 0) a.y[r] = acc;
    }
}

}  // namespace

cudaError_t launch_gemv_vec(const GemvArgs& a, int V, int num_sms, cudaStream_t stream)
{
    if (a.L == 16 && a.K == 4 && V == 2 && a.cb_f16 == 1 && a.T % 8 == 0 &&
        (reinterpret_cast<uintptr_t>(a.cb) & 15) == 0) {
        const long long items = (long long)(a.cols / a.T) * ((a.T / 2 + 127) / 128);
        const size_t smem = kGemvVec2SmemStates * sizeof(uint32_t) +
                            (items <= kGemvVec2MaxSplitItems ? (size_t)items * 33 * sizeof(float) : 0);
        const cudaError_t e = cudaFuncSetAttribute(gemv_vec2_kernel,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        long long grid = (a.rows + kGemvVec2Threads / 32 - 1) / (kGemvVec2Threads / 32);
        if (grid > num_sms) grid = num_sms;  // one CTA per SM: the table copy is paid once per SM
        if (grid < 1) grid = 1;
        gemv_vec2_kernel<<<(int)grid, kGemvVec2Threads, smem, stream>>>(a);
        return cudaGetLastError();
    }
    long long grid = (a.rows + 7) / 8;
    const long long cap = (long long)num_sms * 8;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    gemv_vec_kernel<<<(int)grid, 256, 0, stream>>>(a, V);
    return cudaGetLastError();
}

}  // namespace tcq
