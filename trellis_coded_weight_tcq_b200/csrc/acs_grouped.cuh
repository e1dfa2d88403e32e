// acs_grouped.cuh -- specialised Viterbi add-compare-select (ACS) encoder for the
// bitshift trellis, compile-time (L, k).
//
// Method: Viterbi search (the 2-bit post's Viterbi section) over the QTIP
// bitshift trellis (QTIP abstract) with CurveTQ's weighted branch metric
// d_t (x_t - c[s])^2 and a free start state (CurveTQ abstract).
//
// Reformulation used on the GPU.  The branch metric depends only on the
// destination state s, and the predecessors of s are the 2^k states
// (h << (L-k)) | (s >> k).  Writing u = s & (2^(L-k) - 1) for the part of a state
// that survives into its successors,
//     C_t[s]  = M_{t-1}[s >> k] + d_t (x_t - c[s])^2,
//     M_t[u]  = min_h C_t[(h << (L-k)) | u],     bp_t[u] = argmin_h,
// so the recurrence carries 2^(L-k) path metrics instead of 2^L, and one k-bit
// backpointer per u.  A thread owns "groups": group g covers the 2^k values
// u = (g << k) | j, whose 2^(2k) candidate states all read the same 2^k metrics
// M_{t-1}[(h << (L-2k)) | g].  The codewords of a thread's states are fixed for
// every step and every block, so they live in registers for the whole kernel.
//
// Branch metric, two forms, both without cancellation so the path metrics stay
// the true partial costs:
//   fp32 codewords: a = -sqrt(d_t), xs = sqrt(d_t) x_t per step,
//                   e = fma(a, c, xs) = sqrt(d_t)(x_t - c), cand = fma(e, e, M);
//   fp16 codewords: e = c - x_t in one mixed-precision add,
//                   cand = fma(d_t e, e, M) (the product is skipped when d = 1).
//
// CTA layout: NTEAM teams of NT threads; each team advances one block per
// round and the CTA loops over rounds (persistent).  Backpointers go to the
// workspace, double buffered by round parity.  Thread 0 of each team traces
// back the team's previous block one step per forward step of the current
// block: the dependent backpointer load of a trace step is issued before the
// step's add-compare-select work and consumed after it, so the serial traceback
// hides behind the forward pass and needs no warp of its own.  Only the last
// block of each team is traced after the loop.  The per-step __syncthreads is
// the only wait, and no wait depends on another CTA.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace tcq {

template <int L_, int K_, int NT_, int GPT_, int NTEAM_, bool CB16_>
struct GCfg {
    static constexpr int L = L_, K = K_, NT = NT_, GPT = GPT_, NTEAM = NTEAM_;
    static constexpr bool CB16 = CB16_;        // codewords held as fp16 pairs
    static constexpr int H = 1 << K;           // predecessors per state / symbols
    static constexpr int LK = L - K;           // bits of u
    static constexpr int NU = 1 << LK;         // path metrics per block
    static constexpr int G = 1 << (L - 2 * K); // groups per block
    static constexpr int REC_BITS = GPT * H * K;  // backpointer bits per thread per step
    static constexpr int UNIT_BITS = REC_BITS <= 32 ? 32 : 64;
    static constexpr int SPU = UNIT_BITS / REC_BITS;  // steps per stored unit
    static constexpr int NCOMP = NT * NTEAM;
    static constexpr int NTHREADS = NCOMP;
    static constexpr int TCHUNK = 256;         // steps of (a, xs) staged at a time
    using unit_t = typename std::conditional<UNIT_BITS == 32, uint32_t, unsigned long long>::type;

    static_assert(L >= 2 * K, "grouped kernel needs L >= 2k");
    static_assert(NT * GPT == G, "threads x groups per thread must cover every group");
    static_assert(REC_BITS <= 64, "backpointer record must fit 64 bits");
    static_assert(NCOMP % 32 == 0, "compute threads must be whole warps");
    static_assert(NT >= 32 ? (NT % 32 == 0) : (32 % NT == 0), "teams tile warps");
    static_assert(NTEAM == 1 || NT <= 32, "multi-team CTAs use sub-warp teams");

    // bytes of one team's backpointers for one block, rounded to 256
    static __host__ __device__ size_t team_bytes(int T)
    {
        size_t units = (size_t)((T - 1 + SPU - 1) / SPU) * NT;
        return (units * (UNIT_BITS / 8) + 255) & ~(size_t)255;
    }
    static __host__ __device__ size_t slot_bytes(int, int, int T) { return 2 * NTEAM * team_bytes(T); }
    static __host__ __device__ size_t smem_bytes(int, int, int)
    {
        return sizeof(float) * NTEAM * 2 * NU       // path metrics, ping-pong
               + sizeof(float2) * NTEAM * TCHUNK    // staged (a, xs)
               + 8 * (NCOMP / 32)                   // per-warp reduction
               + 8 * NTEAM;                         // final states
    }
};

// ---------------------------------------------------------------------------
// codewords of a thread's states, resident in registers
// ---------------------------------------------------------------------------
template <class C, bool F16>
struct Codewords;

template <class C>
struct Codewords<C, false> {  // fp32
    float w[C::GPT][C::H][C::H];
    __device__ __forceinline__ void load(const void* cb, int f16, int tid)
    {
#pragma unroll
        for (int i = 0; i < C::GPT; ++i)
#pragma unroll
            for (int h = 0; h < C::H; ++h)
#pragma unroll
                for (int j = 0; j < C::H; ++j) {
                    const uint32_t g = (uint32_t)(tid + i * C::NT);
                    const uint32_t s = ((uint32_t)h << C::LK) | (g << C::K) | (uint32_t)j;
                    w[i][h][j] = load_codeword(cb, f16, s);
                }
    }
    __device__ __forceinline__ float get(int i, int h, int j) const { return w[i][h][j]; }
};

template <class C>
struct Codewords<C, true> {  // binary16 pairs; the input codebook is binary16
    static_assert(C::H % 2 == 0, "pairs of codewords");
    uint32_t w[C::GPT][C::H][C::H / 2];
    __device__ __forceinline__ void load(const void* cb, int, int tid)
    {
        const unsigned short* c = reinterpret_cast<const unsigned short*>(cb);
#pragma unroll
        for (int i = 0; i < C::GPT; ++i)
#pragma unroll
            for (int h = 0; h < C::H; ++h)
#pragma unroll
                for (int j = 0; j < C::H; j += 2) {
                    const uint32_t g = (uint32_t)(tid + i * C::NT);
                    const uint32_t s = ((uint32_t)h << C::LK) | (g << C::K) | (uint32_t)j;
                    w[i][h][j / 2] = (uint32_t)c[s] | ((uint32_t)c[s + 1] << 16);
                }
    }
    // c - x in one rounding: sm_100's mixed-precision add takes the binary16
    // codeword straight from its half of the register, so there is no
    // separate (and loop-invariant, hence hoistable) widening.
    __device__ __forceinline__ float diff(int i, int h, int j, float nx) const
    {
        float e;
        if (j & 1)
            asm("{.reg .f16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tadd.rn.f32.f16 %0, hi, %2;}"
                : "=f"(e) : "r"(w[i][h][j / 2]), "f"(nx));
        else
            asm("{.reg .f16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tadd.rn.f32.f16 %0, lo, %2;}"
                : "=f"(e) : "r"(w[i][h][j / 2]), "f"(nx));
        return e;
    }
};

// ---------------------------------------------------------------------------
// argmin over N consecutive candidates by a tournament; the smallest index wins
// a tie (strict compare), like the textbook recurrence.
// ---------------------------------------------------------------------------
template <int N, int OFF, int H>
struct ArgminTree {
    static __device__ __forceinline__ float run(const float (&c)[H], int& idx)
    {
        int il, ir;
        const float vl = ArgminTree<N / 2, OFF, H>::run(c, il);
        const float vr = ArgminTree<N / 2, OFF + N / 2, H>::run(c, ir);
        const bool p = vr < vl;
        idx = p ? ir : il;
        return p ? vr : vl;
    }
};
template <int OFF, int H>
struct ArgminTree<1, OFF, H> {
    static __device__ __forceinline__ float run(const float (&c)[H], int& idx)
    {
        idx = OFF;
        return c[OFF];
    }
};

template <int H>
__device__ __forceinline__ void store_metrics(float* dst, const float (&v)[H])
{
    if constexpr (H % 4 == 0) {
#pragma unroll
        for (int j = 0; j < H; j += 4)
            *reinterpret_cast<float4*>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
    } else if constexpr (H == 2) {
        *reinterpret_cast<float2*>(dst) = make_float2(v[0], v[1]);
    } else {
#pragma unroll
        for (int j = 0; j < H; ++j) dst[j] = v[j];
    }
}

// One trellis step for one thread.  FIRST: M_0 = 0 (free start).  LAST: no
// metrics or backpointers are stored; the thread keeps its best final state.
// (p0, p1) is the step's staged pair: (a, xs) for fp32 codewords, (-x_t, d_t)
// for fp16 codewords.
template <class C, bool WEIGHTED, bool FIRST, bool LAST>
__device__ __forceinline__ void acs_step(const Codewords<C, C::CB16>& cw, float p0, float p1,
                                         const float* __restrict__ Mp, float* __restrict__ Mn,
                                         int tid, uint32_t& rec_lo, uint32_t& rec_hi,
                                         float& bestv, uint32_t& bests)
{
    rec_lo = 0;
    rec_hi = 0;
#pragma unroll
    for (int i = 0; i < C::GPT; ++i) {
        const int g = tid + i * C::NT;
        float Mh[C::H];
#pragma unroll
        for (int h = 0; h < C::H; ++h) Mh[h] = FIRST ? 0.f : Mp[(h << (C::L - 2 * C::K)) | g];
        float mn[C::H];
#pragma unroll
        for (int j = 0; j < C::H; ++j) {
            float cand[C::H];
#pragma unroll
            for (int h = 0; h < C::H; ++h) {
                if constexpr (C::CB16) {
                    const float e = cw.diff(i, h, j, p0);
                    cand[h] = fmaf(WEIGHTED ? e * p1 : e, e, Mh[h]);
                } else {
                    const float e = fmaf(p0, cw.get(i, h, j), p1);
                    cand[h] = fmaf(e, e, Mh[h]);
                }
            }
            int idx;
            const float v = ArgminTree<C::H, 0, C::H>::run(cand, idx);
            mn[j] = v;
            if constexpr (LAST) {
                const uint32_t s = ((uint32_t)idx << C::LK) | ((uint32_t)g << C::K) | (uint32_t)j;
                keep_best(v, s, bestv, bests);
            } else {
                const int pos = (i * C::H + j) * C::K;  // compile-time after unrolling
                if (pos < 32) {
                    rec_lo |= (uint32_t)idx << pos;
                    if (pos + C::K > 32) rec_hi |= (uint32_t)idx >> (32 - pos);
                } else {
                    rec_hi |= (uint32_t)idx << (pos - 32);
                }
            }
        }
        if constexpr (!LAST) store_metrics<C::H>(Mn + ((size_t)g << C::K), mn);
    }
}

// Traceback of one block, advanced one trellis step at a time by one thread.
// issue() starts the loads of the current step; retire() consumes them, emits
// the symbol, adds d_t (x_t - c[s_t])^2 to the fp64 cost and moves to s_{t-1}.
template <class C>
struct Tracer {
    using unit_t = typename C::unit_t;
    long long b;        // block being traced, -1 when idle
    const unit_t* bp;   // its backpointers
    uint32_t s;         // s_tau
    int tau;            // step about to be emitted (T .. 1)
    double cost;
    int widx;           // backward bit writer state
    uint32_t wcur;
    // loads in flight
    unit_t unit;
    float cval, xval, dval;

    __device__ __forceinline__ void start(long long blk, uint32_t sT, const unit_t* p, int T, int W)
    {
        b = blk;
        bp = p;
        s = sT;
        tau = T;
        cost = 0.0;
        widx = W - 1;
        wcur = 0;
    }

    __device__ __forceinline__ void issue(const EncodeArgs& a)
    {
        const int T = a.T;
        if (tau > 1) {  // bp_{tau-1}[s_tau >> k] decides s_{tau-1}
            const uint32_t u = s >> C::K;
            const uint32_t g = u >> C::K;
            unit = bp[(size_t)((tau - 2) / C::SPU) * C::NT + (g % C::NT)];
        }
        cval = load_codeword(a.cb, a.cb_f16, s);
        xval = a.x[b * T + tau - 1];
        dval = a.d ? a.d[b * T + tau - 1] : 1.f;
    }

    // returns true when the block is finished
    __device__ __forceinline__ bool retire(const EncodeArgs& a)
    {
        const double e = (double)xval - (double)cval;
        cost += (double)dval * e * e;
        BackwardBitWriter bw(a.bits + b * a.W, 0);
        bw.idx = widx;
        bw.cur = wcur;
        bw.put(tau, C::K, s & (C::H - 1));
        if (tau > 1) {
            const uint32_t u = s >> C::K;
            const uint32_t g = u >> C::K, j = u & (C::H - 1);
            const int off = ((tau - 2) % C::SPU) * C::REC_BITS + (int)((g / C::NT) * C::H + j) * C::K;
            const uint32_t h = (uint32_t)(unit >> off) & (C::H - 1);
            s = (h << C::LK) | u;
            widx = bw.idx;
            wcur = bw.cur;
            --tau;
            return false;
        }
        bw.finish();
        a.start_state[b] = s >> C::K;
        a.path_cost[b] = (float)cost;
        return true;
    }
};

template <class C, bool WEIGHTED>
__global__ void __launch_bounds__(C::NTHREADS, 1) acs_grouped_kernel(EncodeArgs a)
{
    using unit_t = typename C::unit_t;
    extern __shared__ __align__(16) unsigned char smem[];
    float* Mall = reinterpret_cast<float*>(smem);
    float2* stage_all = reinterpret_cast<float2*>(Mall + C::NTEAM * 2 * C::NU);
    float* redv = reinterpret_cast<float*>(stage_all + C::NTEAM * C::TCHUNK);
    uint32_t* reds = reinterpret_cast<uint32_t*>(redv + C::NCOMP / 32);
    uint32_t* fin_state = reds + C::NCOMP / 32;  // [NTEAM]

    const int T = a.T;
    const long long nb = a.n_blocks;
    const long long stride = (long long)gridDim.x * C::NTEAM;
    const long long first = (long long)blockIdx.x * C::NTEAM;
    const int R = first < nb ? (int)((nb - first + stride - 1) / stride) : 0;
    unsigned char* slot = a.ws + (size_t)blockIdx.x * a.slot_bytes;
    const size_t team_bytes = C::team_bytes(T);

    const int m = threadIdx.x / C::NT;    // team
    const int tid = threadIdx.x % C::NT;  // thread within the team
    const bool tracer = tid == 0;
    float* Mteam = Mall + m * 2 * C::NU;
    float2* stage = stage_all + m * C::TCHUNK;
    Codewords<C, C::CB16> cw;
    cw.load(a.cb, a.cb_f16, tid);
    Tracer<C> tr;
    tr.b = -1;

    for (int r = 0; r < R; ++r) {
        const int par = r & 1;
        const long long b = first + (long long)r * stride + m;
        const bool valid = b < nb;
        unit_t* bp = reinterpret_cast<unit_t*>(slot + (size_t)(par * C::NTEAM + m) * team_bytes);
        const float* xb = a.x + (valid ? b : 0) * T;
        const float* db = a.d ? a.d + (valid ? b : 0) * T : nullptr;
        unit_t acc = 0;
        float bestv = __int_as_float(0x7f800000);  // +inf
        uint32_t bests = 0xffffffffu;

        for (int t = 1; t <= T; ++t) {
            const int tc = (t - 1) % C::TCHUNK;
            if (tc == 0) {
                if (valid) {
                    for (int q = tid; q < C::TCHUNK && t + q <= T; q += C::NT) {
                        const float xv = xb[t - 1 + q];
                        const float dv = WEIGHTED ? db[t - 1 + q] : 1.f;
                        if constexpr (C::CB16) {
                            stage[q] = make_float2(-xv, dv);
                        } else {
                            const float sd = WEIGHTED ? sqrtf(dv) : 1.f;
                            stage[q] = make_float2(-sd, sd * xv);
                        }
                    }
                }
                __syncthreads();
            }
            const bool tracing = tracer && tr.b >= 0;
            if (tracing) tr.issue(a);
            if (valid) {
                const float2 ax = stage[tc];
                const float* Mp = Mteam + ((t - 1) & 1) * C::NU;
                float* Mn = Mteam + (t & 1) * C::NU;
                uint32_t lo, hi;
                if (t == T) {
                    if (t == 1)
                        acs_step<C, WEIGHTED, true, true>(cw, ax.x, ax.y, Mp, Mn, tid, lo, hi, bestv, bests);
                    else
                        acs_step<C, WEIGHTED, false, true>(cw, ax.x, ax.y, Mp, Mn, tid, lo, hi, bestv, bests);
                } else {
                    if (t == 1)
                        acs_step<C, WEIGHTED, true, false>(cw, ax.x, ax.y, Mp, Mn, tid, lo, hi, bestv, bests);
                    else
                        acs_step<C, WEIGHTED, false, false>(cw, ax.x, ax.y, Mp, Mn, tid, lo, hi, bestv, bests);
                    unit_t rec;
                    if constexpr (C::UNIT_BITS == 64)
                        rec = ((unit_t)hi << 32) | (unit_t)lo;
                    else
                        rec = (unit_t)lo;
                    const int q = (t - 1) % C::SPU;
                    acc |= rec << (q * C::REC_BITS);
                    if (q == C::SPU - 1 || t == T - 1) {
                        bp[(size_t)((t - 1) / C::SPU) * C::NT + tid] = acc;
                        acc = 0;
                    }
                }
            }
            if (tracing && tr.retire(a)) tr.b = -1;
            if (t < T) __syncthreads();
        }

        // ---- final state of the block: lexicographic (cost, state) minimum over the team
        if constexpr (C::NT >= 32) {
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bestv, o);
                const uint32_t os = __shfl_xor_sync(0xffffffffu, bests, o);
                keep_best(ov, os, bestv, bests);
            }
            const int warp = threadIdx.x >> 5;
            if ((threadIdx.x & 31) == 0) {
                redv[warp] = bestv;
                reds[warp] = bests;
            }
            __syncthreads();
            if (tid == 0) {
                const int w0 = (m * C::NT) >> 5;
                float bv = redv[w0];
                uint32_t bs = reds[w0];
                for (int w = 1; w < C::NT / 32; ++w) keep_best(redv[w0 + w], reds[w0 + w], bv, bs);
                bests = bs;
            }
        } else {
#pragma unroll
            for (int o = C::NT / 2; o >= 1; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bestv, o);
                const uint32_t os = __shfl_xor_sync(0xffffffffu, bests, o);
                keep_best(ov, os, bestv, bests);
            }
        }
        // the team's thread 0 holds the final state; its trace runs during the next round
        if (tracer && valid) tr.start(b, bests, bp, T, a.W);
        __syncthreads();  // backpointers of this round visible to the tracer; redv reusable
    }
    // the last block of each team has no next round to hide behind
    if (tracer && tr.b >= 0) {
        while (true) {
            tr.issue(a);
            if (tr.retire(a)) break;
        }
    }
    (void)fin_state;
}

template <class C, bool WEIGHTED>
cudaError_t launch_grouped_w(const EncodeArgs& a, int grid, cudaStream_t stream)
{
    const size_t smem = C::smem_bytes(a.L, a.K, a.T);
    cudaError_t e = cudaFuncSetAttribute(acs_grouped_kernel<C, WEIGHTED>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    acs_grouped_kernel<C, WEIGHTED><<<grid, C::NTHREADS, smem, stream>>>(a);
    return cudaGetLastError();
}

template <class C>
cudaError_t launch_grouped(const EncodeArgs& a, int grid, cudaStream_t stream)
{
    return a.d ? launch_grouped_w<C, true>(a, grid, stream) : launch_grouped_w<C, false>(a, grid, stream);
}

template <class C>
const EncodeKernelInfo* grouped_info(const char* name)
{
    static const EncodeKernelInfo info = {
        name, C::NTEAM, C::NTHREADS, 0, &C::slot_bytes, &C::smem_bytes,
        reinterpret_cast<const void*>(&acs_grouped_kernel<C, true>), &launch_grouped<C>};
    return &info;
}

}  // namespace tcq
