// acs_vec2.cu -- Viterbi encoder for the vector trellis at L = 16, k = 2, V = 2:
// two weights per step, four bits shifted in per step, codebook [2^16][2] in
// binary16 (a computed code is not vector-valued, so only tables come here).
//
// Recurrence (QTIP's bitshift trellis with V weights per step, CurveTQ's
// weighted metric, free start), in the u-formulation of the scalar encoders
// with K = kV = 4 bits per step: u = s mod 2^12 and
//     M_t[u] = min_h M_{t-1}[s >> 4] + d_{2t-1}(x_{2t-1} - c[s][0])^2
//                                    + d_{2t}  (x_{2t}   - c[s][1])^2,
// s = (h << 12) | u, h the top four bits.  Group g = u >> 4 covers the 16 values
// u = (g << 4) | j, whose 256 candidate states all read the 16 metrics
// M_{t-1}[(h << 8) | g].
//
// Layout.  512 threads, one block per CTA at a time, persistent over blocks.
// Thread tid takes half a group: g = tid >> 1 and j = 8 (tid & 1) + jj, jj < 8,
// i.e. 8 u values and their 128 states.  A state's two codewords are one 32-bit
// word (two binary16 halves); of a thread's 128 words, those of the first
// kV2HR predecessors stay in registers for the whole kernel and the rest sit in
// shared memory, thread-interleaved so that a warp's 16-byte loads are
// contiguous.  Path metrics ping-pong in shared memory (2 x 16 KiB), read as
// 16 scalars per thread and step (conflict free: consecutive threads read
// consecutive g) and written as two float4 per thread.  The kernel takes the
// scalar encoders' 128-byte argument block.
//
// Per node: two mixed-precision subtractions (binary16 codeword minus fp32 x),
// one product and two FMAs, with the metrics carried divided by the step's
// first weight d_{2t-1} (floored at max(2^-60 max d, FLT_MIN) per block as in
// the scalar kernels), so cand = M' r + e1^2 + (d_{2t}/d_{2t-1}) e2^2 with
// r = d_{2t-3}/d_{2t-1}; then the scalar kernels' sign-bit tournament over the
// 16 candidates of each u.  The backpointers of a thread and step are one
// 32-bit word (four bit planes of eight bits), double buffered by round; the
// traceback of a block runs one step per forward step of the next block on the
// first warp, and the whole CTA then forms its bits and its fp64 cost.
#include "acs_grouped.cuh"

namespace tcq {

namespace {

constexpr int kV2Threads = 512;
constexpr int kV2NU = 4096;                    // u values: 2^(L - kV)
// predecessors whose codewords stay in registers: 4 (32 registers) measured 13 %
// faster than 8 (11.74 vs 13.29 ms on 4736 blocks); fewer would overflow the
// 227 KiB of shared memory
constexpr int kV2HR = 4;
constexpr int kV2SW = 16 - kV2HR;              // predecessors with codewords in shared memory
constexpr int kV2ChunksPerJ = kV2SW / 4;       // 16-byte chunks per u value
constexpr int kV2Chunks = 8 * kV2ChunksPerJ;   // 16-byte chunks per thread
constexpr int kV2Stage = 128;                  // steps staged at a time
static_assert(kV2SW % 4 == 0, "shared-memory codewords come in 16-byte chunks per u");

struct V2Smem {
    uint4 cbs[kV2Chunks][kV2Threads];  // codewords of predecessors kV2HR..15
    float M[2][kV2NU];                 // path metrics, ping-pong
    float4 stage[kV2Stage];            // (-x_{2t-1}, -x_{2t}, r_t, rho_t)
    float redv[kV2Threads / 32];
    uint32_t reds[kV2Threads / 32];
    double redd[kV2Threads / 32];
    uint32_t fin;
};

__host__ __device__ inline size_t v2_round256(size_t v) { return (v + 255) & ~(size_t)255; }

// backpointer words of one block: steps 1 .. NS-1, one word per thread and step
__host__ __device__ inline size_t v2_rec_bytes(int NS)
{
    return v2_round256((size_t)(NS > 1 ? NS - 1 : 0) * kV2Threads * sizeof(uint32_t));
}
__host__ __device__ inline size_t v2_path_bytes(int NS) { return v2_round256((size_t)NS * 2); }

// (L, bits per step, steps per block), as for the runtime kernel's vector path
size_t v2_slot_bytes(int, int, int NS) { return 2 * v2_rec_bytes(NS) + v2_path_bytes(NS); }
size_t v2_smem_bytes(int, int, int) { return sizeof(V2Smem); }

// cand = M' + e1^2 + rho e2^2 for the state whose codeword pair is w
template <bool WEIGHTED>
__device__ __forceinline__ float v2_node(uint32_t w, const float4& st, float m)
{
    float e1, e2;
    asm("{.reg .f16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
        "add.rn.f32.f16 %0, lo, %3;\n\tadd.rn.f32.f16 %1, hi, %4;}"
        : "=f"(e1), "=f"(e2) : "r"(w), "f"(st.x), "f"(st.y));
    return fmaf(e1, e1, fmaf(WEIGHTED ? e2 * st.w : e2, e2, m));
}

// One trellis step of one thread (see acs_step in the scalar encoder).  The
// backpointer word: bit 8 l + 7 - jj is bit 3 - l of the argmin h of u value jj.
template <bool WEIGHTED, bool FIRST, bool LAST>
__device__ __forceinline__ void v2_step(const uint32_t (&cw)[kV2HR][8],
                                        const uint4* __restrict__ cbs, const float4 st,
                                        const float* __restrict__ Mp, float* __restrict__ Mn,
                                        int g, int half, uint32_t& rec, float& bestv,
                                        uint32_t& bests)
{
    float Mh[16];
#pragma unroll
    for (int h = 0; h < 16; ++h) Mh[h] = FIRST ? 0.f : (WEIGHTED ? Mp[(h << 8) | g] * st.z : Mp[(h << 8) | g]);
    uint32_t planes[4] = {0u, 0u, 0u, 0u};
    float mn[4];
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
        float cand[16];
#pragma unroll
        for (int h = 0; h < kV2HR; ++h) cand[h] = v2_node<WEIGHTED>(cw[h][jj], st, Mh[h]);
#pragma unroll
        for (int c = 0; c < kV2ChunksPerJ; ++c) {
            const uint4 q = cbs[(jj * kV2ChunksPerJ + c) * kV2Threads];
            cand[kV2HR + 4 * c + 0] = v2_node<WEIGHTED>(q.x, st, Mh[kV2HR + 4 * c + 0]);
            cand[kV2HR + 4 * c + 1] = v2_node<WEIGHTED>(q.y, st, Mh[kV2HR + 4 * c + 1]);
            cand[kV2HR + 4 * c + 2] = v2_node<WEIGHTED>(q.z, st, Mh[kV2HR + 4 * c + 2]);
            cand[kV2HR + 4 * c + 3] = v2_node<WEIGHTED>(q.w, st, Mh[kV2HR + 4 * c + 3]);
        }
        uint32_t sb[4];
        const float v = SignTree<16, 0>::template run<16, 4>(cand, sb);
        if constexpr (LAST) {
            uint32_t idx = 0;
#pragma unroll
            for (int l = 0; l < 4; ++l) idx = (idx << 1) | (sb[l] >> 31);
            const uint32_t s = (idx << 12) | ((uint32_t)g << 4) | (uint32_t)(8 * half + jj);
            keep_best(v, s, bestv, bests);
        } else {
            mn[jj & 3] = v;
#pragma unroll
            for (int l = 0; l < 4; ++l) planes[l] = __funnelshift_l(sb[l], planes[l], 1);
            if ((jj & 3) == 3)
                *reinterpret_cast<float4*>(Mn + ((g << 4) | (8 * half + (jj & 4)))) =
                    make_float4(mn[0], mn[1], mn[2], mn[3]);
        }
    }
    if constexpr (!LAST) rec = planes[0] | (planes[1] << 8) | (planes[2] << 16) | (planes[3] << 24);
}

// Traceback of one block by the first warp (all lanes hold the same state and
// load the same word): issue() before a forward step, retire() after it.
struct V2Tracer {
    long long b;  // block being traced, -1: none
    const uint32_t* bp;
    uint16_t* path;
    uint32_t s;   // s_tau
    int tau;
    uint32_t unit;

    __device__ __forceinline__ void issue()
    {
        if (tau > 1) {  // the word of u = s_tau >> 4 at step tau - 1 decides s_{tau-1}
            const uint32_t u = s >> 4;
            const uint32_t owner = ((u >> 4) << 1) | ((u >> 3) & 1u);
            unit = bp[(size_t)(tau - 2) * kV2Threads + owner];
        }
    }
    __device__ __forceinline__ bool retire(bool store)
    {
        if (store) path[tau - 1] = (uint16_t)s;
        if (tau == 1) return true;
        const uint32_t u = s >> 4, jj = u & 7u;
        uint32_t h = 0;
#pragma unroll
        for (int l = 0; l < 4; ++l) h = (h << 1) | ((unit >> (8 * l + 7 - jj)) & 1u);
        s = (h << 12) | u;
        --tau;
        return false;
    }
};

// Bits, start state and fp64 cost of a traced block, by the whole CTA.
__device__ __forceinline__ void v2_finish(const GroupedArgs& a, long long b,
                                          const uint16_t* __restrict__ path, V2Smem& S, int NS)
{
    const int tid = threadIdx.x;
    const float* xb = a.x + b * opaque(a.x_stride);
    const float* db = a.d ? a.d + b * opaque(a.d_stride) : nullptr;
    const __half* cbh = reinterpret_cast<const __half*>(a.cb);
    double acc = 0.0;
    for (int t = tid; t < NS; t += kV2Threads) {
        const uint32_t s = path[t];
#pragma unroll
        for (int v = 0; v < 2; ++v) {
            const double e = (double)xb[2 * t + v] - (double)__half2float(cbh[2 * s + v]);
            acc += (double)(db ? db[2 * t + v] : 1.f) * e * e;
        }
    }
    for (int w = tid; w < a.W; w += kV2Threads) {  // 8 symbols of 4 bits per word
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int t = 8 * w + i;
            if (t < NS) word |= ((uint32_t)path[t] & 15u) << (28 - 4 * i);
        }
        a.bits[b * a.W + w] = word;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if ((tid & 31) == 0) S.redd[tid >> 5] = acc;
    __syncthreads();
    if (tid == 0) {
        double total = 0.0;
        for (int w = 0; w < kV2Threads / 32; ++w) total += S.redd[w];
        a.start_state[b] = (uint32_t)path[0] >> 4;
        a.path_cost[b] = (float)total;
    }
    __syncthreads();
}

// LONG: blocks of more than kRenormAfter steps, whose metrics are shifted
// towards 0 every 64 steps (a separate instantiation, as in the scalar kernel).
// WEIGHTED = false (no d): every ratio is 1, so a node saves its product and a
// metric read its rescale (9.76 vs 11.59 ms on 4736 unweighted blocks).
template <bool LONG, bool WEIGHTED>
__global__ void __launch_bounds__(kV2Threads, 1) acs_vec2_kernel(GroupedArgs a)
{
    extern __shared__ __align__(16) unsigned char smem[];
    V2Smem& S = *reinterpret_cast<V2Smem*>(smem);
    const int tid = threadIdx.x;
    const int g = tid >> 1, half = tid & 1;
    const int NS = a.T >> 1;
    const long long nb = a.n_blocks;
    const long long stride = gridDim.x;
    const long long first = blockIdx.x;
    const int R = first < nb ? (int)((nb - first + stride - 1) / stride) : 0;
    unsigned char* slot = a.ws + (size_t)blockIdx.x * a.slot_bytes;
    const size_t recb = v2_rec_bytes(NS);
    uint16_t* path = reinterpret_cast<uint16_t*>(slot + 2 * recb);

    // codeword pairs of the thread's 128 states, one 32-bit word per state
    const uint32_t* cb32 = reinterpret_cast<const uint32_t*>(a.cb);
    uint32_t cw[kV2HR][8];
#pragma unroll
    for (int h = 0; h < 16; ++h)
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
            const uint32_t w = cb32[((uint32_t)h << 12) | ((uint32_t)g << 4) | (uint32_t)(8 * half + jj)];
            if (h < kV2HR) {
                cw[h][jj] = w;
            } else {
                const int q = jj * kV2SW + (h - kV2HR);
                reinterpret_cast<uint32_t*>(&S.cbs[q >> 2][tid])[q & 3] = w;
            }
        }
    const uint4* cbs = &S.cbs[0][tid];

    V2Tracer tr;
    tr.b = -1;
    long long done = -1;  // block whose path is complete, to be finished
    const bool tracer = tid < 32;

    for (int r = 0; r < R; ++r) {
        const long long b = first + (long long)r * stride;
        uint32_t* bp = reinterpret_cast<uint32_t*>(slot + (size_t)(r & 1) * recb);
        const float* xb = a.x + b * opaque(a.x_stride);
        const float* db = a.d ? a.d + b * opaque(a.d_stride) : nullptr;
        float dm = 0.f;
        for (int q = tid; q < a.T; q += kV2Threads) dm = fmaxf(dm, db ? db[q] : 1.f);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) dm = fmaxf(dm, __shfl_xor_sync(0xffffffffu, dm, o));
        if ((tid & 31) == 0) S.redv[tid >> 5] = dm;
        __syncthreads();
        dm = S.redv[0];
        for (int w = 1; w < kV2Threads / 32; ++w) dm = fmaxf(dm, S.redv[w]);
        const float dfloor = fmaxf(dm * 0x1p-60f, 1.17549435e-38f);
        float bestv = __int_as_float(0x7f800000);
        uint32_t bests = 0xffffffffu;
        uint32_t* bpw = bp + tid;

        auto step = [&](auto first_tag, auto last_tag, int t) {
            constexpr bool FIRST = decltype(first_tag)::value;
            constexpr bool LAST = decltype(last_tag)::value;
            const int tc = (t - 1) % kV2Stage;
            if (tc == 0) {
                for (int q = tid; q < kV2Stage && t + q <= NS; q += kV2Threads) {
                    const int i = 2 * (t - 1 + q);
                    const float d1 = fmaxf(db ? db[i] : 1.f, dfloor);
                    const float d2 = db ? db[i + 1] : 1.f;
                    const float d1p = i > 0 ? fmaxf(db ? db[i - 2] : 1.f, dfloor) : d1;
                    S.stage[q] = make_float4(-xb[i], -xb[i + 1], d1p / d1, d2 / d1);
                }
                __syncthreads();
            }
            const bool tracing = tracer && tr.b >= 0;
            if (tracing) tr.issue();
            const float4 st = S.stage[tc];
            uint32_t rec = 0;
            v2_step<WEIGHTED, FIRST, LAST>(cw, cbs, st, S.M[(t - 1) & 1], S.M[t & 1], g, half, rec, bestv,
                                 bests);
            if constexpr (!LAST) {
                *bpw = rec;
                bpw += kV2Threads;
            }
            if (tracing && tr.retire(tid == 0)) tr.b = -1;
            if constexpr (!LAST) {
                __syncthreads();
                if constexpr (LONG) {
                    if ((t & 63) == 0) {  // shift by state 0's metric
                        float* Mn = S.M[t & 1];
                        const float o = Mn[0];
                        const float off = (o < __int_as_float(0x7f800000)) ? o : 0.f;
                        __syncthreads();
#pragma unroll
                        for (int jj = 0; jj < 8; ++jj) Mn[(g << 4) | (8 * half + jj)] -= off;
                        __syncthreads();
                    }
                }
            }
        };
        using T0 = std::false_type;
        using T1 = std::true_type;
        if (NS == 1) {
            step(T1{}, T1{}, 1);
        } else {
            step(T1{}, T0{}, 1);
            for (int t = 2; t < NS; ++t) step(T0{}, T0{}, t);
            step(T0{}, T1{}, NS);
        }

        // final state of the block: lexicographic (cost, state) minimum over the CTA
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bestv, o);
            const uint32_t os = __shfl_xor_sync(0xffffffffu, bests, o);
            keep_best(ov, os, bestv, bests);
        }
        if ((tid & 31) == 0) {
            S.redv[tid >> 5] = bestv;
            S.reds[tid >> 5] = bests;
        }
        __syncthreads();
        if (tid == 0) {
            float bv = S.redv[0];
            uint32_t bs = S.reds[0];
            for (int w = 1; w < kV2Threads / 32; ++w) keep_best(S.redv[w], S.reds[w], bv, bs);
            S.fin = bs;
        }
        // the previous block's walk ended with this round's last step
        if (done >= 0) v2_finish(a, done, path, S, NS);  // syncs the CTA (S.fin visible)
        else __syncthreads();
        if (tracer) {
            tr.b = b;
            tr.bp = bp;
            tr.path = path;
            tr.s = S.fin;
            tr.tau = NS;
        }
        done = b;
        __syncthreads();  // S.fin is rewritten by the next round
    }
    if (R > 0) {  // the last block: walk alone, then finish
        if (tracer) {
            while (true) {
                tr.issue();
                if (tr.retire(tid == 0)) break;
            }
        }
        __syncthreads();
        v2_finish(a, done, path, S, NS);
    }
}

template <bool LONG, bool WEIGHTED>
cudaError_t v2_launch_t(const EncodeArgs& a, int grid, cudaStream_t stream)
{
    const size_t smem = sizeof(V2Smem);
    cudaError_t e = cudaFuncSetAttribute(acs_vec2_kernel<LONG, WEIGHTED>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    acs_vec2_kernel<LONG, WEIGHTED><<<grid, kV2Threads, smem, stream>>>(grouped_args(a));
    return cudaGetLastError();
}

cudaError_t v2_launch(const EncodeArgs& a, int grid, cudaStream_t stream)
{
    if (a.T / 2 > kRenormAfter) return v2_launch_t<true, true>(a, grid, stream);
    return a.d ? v2_launch_t<false, true>(a, grid, stream) : v2_launch_t<false, false>(a, grid, stream);
}

const EncodeKernelInfo kVec2Info = {"vec2<16,2,f16x2,512>", 1, kV2Threads, 1, &v2_slot_bytes,
                                    &v2_smem_bytes,
                                    reinterpret_cast<const void*>(&acs_vec2_kernel<false, true>),
                                    &v2_launch};

}  // namespace

// The compile-time vector-trellis kernel for (L, k, V, codebook dtype), or nullptr.
const EncodeKernelInfo* find_vec_kernel(int L, int k, int V, int cb_f16)
{
    if (L == 16 && k == 2 && V == 2 && cb_f16) return &kVec2Info;
    return nullptr;
}

}  // namespace tcq
