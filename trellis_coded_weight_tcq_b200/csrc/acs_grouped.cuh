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
// Branch metric, two forms, both without cancellation:
//   fp32 codewords: a = -sqrt(d_t), xs = sqrt(d_t) x_t per step,
//                   e = fma(a, c, xs) = sqrt(d_t)(x_t - c), cand = fma(e, e, M);
//   fp16 codewords: e = c - x_t in one mixed-precision add and cand = fma(e, e, M'),
//                   where the path metrics are carried divided by the current
//                   weight, M'_t = M_t / d_t.  Dividing every candidate of a step
//                   by the same d_t > 0 leaves the step's argmins unchanged, and
//                   the per-node product by d_t becomes one product per metric
//                   read, M'_{t-1} * (d_{t-1} / d_t).  To keep the ratio finite,
//                   d_t is floored at max(2^-60 max_t d_t, FLT_MIN) per block: the
//                   change to the cost is below 2^-60 T max d (x - c)^2, far under
//                   any fp32 tolerance, and an all-zero d becomes a plain
//                   Euclidean search, where every path costs 0 anyway.
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

// The grouped kernels' own copy of the encoder arguments, without the fields
// only the runtime kernel reads.  Measured: the same kernel code with a
// 136-byte argument block ran 16 % slower than with this 128-byte one (182.4 vs
// 157.3 ms on 59,200 blocks), and 3 % slower with 32-bit strides packed into
// 128 bytes, so the layout stays exactly this.
struct GroupedArgs {
    const float* x;
    const float* d;
    const void* cb;
    int cb_f16;
    int L, K, T, W;
    long long n_blocks;
    uint32_t* start_state;
    uint32_t* bits;
    float* path_cost;
    long long x_stride, d_stride, out_stride;
    const uint32_t* fixed_start;
    unsigned char* ws;
    size_t slot_bytes;
};
static_assert(sizeof(GroupedArgs) == 128, "the measured layout");

inline GroupedArgs grouped_args(const EncodeArgs& e)
{
    GroupedArgs g;
    g.x = e.x;
    g.d = e.d;
    g.cb = e.cb;
    g.cb_f16 = e.cb_f16;
    g.L = e.L;
    g.K = e.K;
    g.T = e.T;
    g.W = e.W;
    g.n_blocks = e.n_blocks;
    g.start_state = e.start_state;
    g.bits = e.bits;
    g.path_cost = e.path_cost;
    g.x_stride = e.x_stride;
    g.d_stride = e.d_stride;
    g.out_stride = e.out_stride;
    g.fixed_start = e.fixed_start;
    g.ws = e.ws;
    g.slot_bytes = e.slot_bytes;
    return g;
}

template <int L_, int K_, int NT_, int GPT_, int NTEAM_, bool CB16_>
struct GCfg {
    static constexpr int L = L_, K = K_, NT = NT_, GPT = GPT_, NTEAM = NTEAM_;
    static constexpr bool CB16 = CB16_;        // codewords held as fp16 pairs
    static constexpr int H = 1 << K;           // predecessors per state / symbols
    static constexpr int LK = L - K;           // bits of u
    static constexpr int NU = 1 << LK;         // path metrics per block
    static constexpr int G = 1 << (L - 2 * K); // groups per block
    static constexpr int P = GPT * H;             // u values per thread (bits per plane)
    static constexpr int REC_BITS = K * P;        // backpointer bits per thread per step
    static constexpr int UNIT_BITS = REC_BITS <= 32 ? 32 : 64;
    static constexpr int SPU = UNIT_BITS / REC_BITS;  // steps per stored unit
    static constexpr int NCOMP = NT * NTEAM;
    static constexpr int NTHREADS = NCOMP;
    // resident CTAs per SM the register allocation must allow: 128 registers
    // per thread for every configuration (the fp16-pair codewords alone take 64)
    static constexpr int MINB = NTHREADS >= 512 ? 1 : 512 / NTHREADS;
    static constexpr int TCHUNK = 256;         // steps of (a, xs) staged at a time
    using unit_t = typename std::conditional<UNIT_BITS == 32, uint32_t, unsigned long long>::type;

    static_assert(L >= 2 * K, "grouped kernel needs L >= 2k");
    static_assert(NT * GPT == G, "threads x groups per thread must cover every group");
    static_assert(REC_BITS <= 64, "backpointer record must fit 64 bits");
    static_assert(P <= 32, "a bit plane is one 32-bit register");
    static_assert(NCOMP % 32 == 0, "compute threads must be whole warps");
    static_assert(NT >= 32 ? (NT % 32 == 0) : (32 % NT == 0), "teams tile warps");

    // bytes of one team's backpointers for one block, rounded to 256
    static __host__ __device__ size_t team_bytes(int T)
    {
        size_t units = (size_t)((T - 1 + SPU - 1) / SPU) * NT;
        return (units * (UNIT_BITS / 8) + 255) & ~(size_t)255;
    }
    // states s_1..s_T of the block being traced, one buffer per team
    static __host__ __device__ size_t path_bytes(int T) { return ((size_t)T * 2 + 255) & ~(size_t)255; }
    static __host__ __device__ size_t slot_bytes(int, int, int T)
    {
        return 2 * NTEAM * team_bytes(T) + NTEAM * path_bytes(T);
    }
    static __host__ __device__ size_t smem_bytes(int, int, int)
    {
        return sizeof(float) * NTEAM * 2 * NU       // path metrics, ping-pong
               + sizeof(float2) * NTEAM * TCHUNK    // staged (a, xs)
               + 8 * (NCOMP / 32)                   // per-warp reduction (value, state)
               + 8 * (NCOMP / 32);                  // per-warp reduction (fp64 cost)
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
                    w[i][h][j] = TCQ_IN_BOUNDS(s, 1 << C::L) ? load_codeword(cb, f16, s) : 0.f;
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
                    w[i][h][j / 2] = TCQ_IN_BOUNDS(s + 1, 1 << C::L)
                                         ? (uint32_t)c[s] | ((uint32_t)c[s + 1] << 16) : 0u;
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
// Minimum of N consecutive candidates by a tournament, with the argmin given
// as sign bits: sb[0] is a register whose sign bit is the argmin's most
// significant bit (1: the right half won), sb[1] the next bit, and so on.  Each
// match is decided by the sign of the fp32 difference right - left, which is
// exact (a difference of distinct finite floats never rounds to zero with
// gradual underflow), and a tie leaves the bit at 0, so the smallest index
// wins like the textbook recurrence's strict compare.  The differences run on
// the FMA pipe; only the minima and one LOP3 mux per lower bit use the ALU.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t mux_sign(uint32_t s, uint32_t r, uint32_t l)
{
    return (s & r) | (~s & l);  // bitwise: where s has its sign bit set take r, else l
}

template <int N, int OFF>
struct SignTree {
    template <int H, int K>
    static __device__ __forceinline__ float run(const float (&c)[H], uint32_t (&sb)[K])
    {
        constexpr int D = (N >= 2) + (N >= 4) + (N >= 8) + (N >= 16);  // log2 N
        uint32_t l[K], r[K];
        const float vl = SignTree<N / 2, OFF>::template run<H, K>(c, l);
        const float vr = SignTree<N / 2, OFF + N / 2>::template run<H, K>(c, r);
        const uint32_t s = __float_as_uint(vr - vl);
        sb[0] = s;
#pragma unroll
        for (int q = 1; q < D; ++q) sb[q] = mux_sign(s, r[q - 1], l[q - 1]);
        return fminf(vl, vr);
    }
};
// Four candidates: m01 = min(c0, c1) and the three-input m = min(m01, c2, c3)
// give the minimum without forming min(c2, c3); the top bit is the sign of
// m - m01 (negative exactly when the right pair holds a strictly smaller
// value, +0 on a tie, so the left pair wins ties as required).
template <int OFF>
struct SignTree<4, OFF> {
    template <int H, int K>
    static __device__ __forceinline__ float run(const float (&c)[H], uint32_t (&sb)[K])
    {
        const float m01 = fminf(c[OFF], c[OFF + 1]);
        float m;
        asm("min.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(m01), "f"(c[OFF + 2]), "f"(c[OFF + 3]));
        const uint32_t s = __float_as_uint(m - m01);
        sb[0] = s;
        sb[1] = mux_sign(s, __float_as_uint(c[OFF + 3] - c[OFF + 2]),
                         __float_as_uint(c[OFF + 1] - c[OFF]));
        return m;
    }
};
template <int OFF>
struct SignTree<2, OFF> {
    template <int H, int K>
    static __device__ __forceinline__ float run(const float (&c)[H], uint32_t (&sb)[K])
    {
        sb[0] = __float_as_uint(c[OFF + 1] - c[OFF]);
        return fminf(c[OFF], c[OFF + 1]);
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

// One trellis step for one thread.  FIRST: M_0 = 0 (free start), or, for a
// start fixed at s_0 (s0 = its low L-k bits), 0 at u = s0 and +inf elsewhere,
// so only the successors of s_0 are reachable at step 1.  LAST: no
// metrics or backpointers are stored; the thread keeps its best final state.
// (p0, p1) is the step's staged pair: (a, xs) for fp32 codewords,
// (-x_t, d_{t-1} / d_t) for fp16 codewords.  Backpointers come back as K bit planes: bit P-1-q of
// plane l is bit K-1-l of the argmin h of the thread's q-th u value
// (q = i * 2^k + j).
template <class C, bool WEIGHTED, bool FIRST, bool LAST>
__device__ __forceinline__ void acs_step(const Codewords<C, C::CB16>& cw, float p0, float p1,
                                         const float* __restrict__ Mp, float* __restrict__ Mn,
                                         int tid, uint32_t (&planes)[C::K], float& bestv,
                                         uint32_t& bests, uint32_t s0 = 0xffffffffu)
{
#pragma unroll
    for (int l = 0; l < C::K; ++l) planes[l] = 0;
#pragma unroll
    for (int i = 0; i < C::GPT; ++i) {
        const int g = tid + i * C::NT;
        float Mh[C::H];
#pragma unroll
        for (int h = 0; h < C::H; ++h) {
            if constexpr (FIRST)
                Mh[h] = (s0 == 0xffffffffu || (uint32_t)((h << (C::L - 2 * C::K)) | g) == s0)
                            ? 0.f : __int_as_float(0x7f800000);
            else
                Mh[h] = Mp[(h << (C::L - 2 * C::K)) | g];
            if constexpr (C::CB16 && WEIGHTED) Mh[h] *= p1;  // M_{t-1}/d_{t-1} -> M_{t-1}/d_t
        }
        float mn[C::H];
#pragma unroll
        for (int j = 0; j < C::H; ++j) {
            float cand[C::H];
#pragma unroll
            for (int h = 0; h < C::H; ++h) {
                if constexpr (C::CB16) {
                    const float e = cw.diff(i, h, j, p0);
                    cand[h] = fmaf(e, e, Mh[h]);
                } else {
                    const float e = fmaf(p0, cw.get(i, h, j), p1);
                    cand[h] = fmaf(e, e, Mh[h]);
                }
            }
            uint32_t sb[C::K];
            const float v = SignTree<C::H, 0>::template run<C::H, C::K>(cand, sb);
            mn[j] = v;
            if constexpr (LAST) {
                uint32_t idx = 0;
#pragma unroll
                for (int l = 0; l < C::K; ++l) idx = (idx << 1) | (sb[l] >> 31);
                const uint32_t s = (idx << C::LK) | ((uint32_t)g << C::K) | (uint32_t)j;
                keep_best(v, s, bestv, bests);
            } else {
#pragma unroll
                for (int l = 0; l < C::K; ++l) planes[l] = __funnelshift_l(sb[l], planes[l], 1);
            }
        }
        if constexpr (!LAST) store_metrics<C::H>(Mn + ((size_t)g << C::K), mn);
    }
}

// Traceback of one block, advanced one trellis step at a time by one thread:
// only the dependent walk through the backpointers, storing s_tau per step.
// issue() starts the load that decides s_{tau-1}; retire() stores s_tau and
// moves on.  Bits, start state and cost are formed afterwards by the whole team
// (finish_block), so the per-step work on the tracing thread stays small.
template <class C>
struct Tracer {
    using unit_t = typename C::unit_t;
    long long b;        // block being traced, -1 when idle
    const unit_t* bp;   // its backpointers
    uint16_t* path;     // its states s_1..s_T
    uint32_t s;         // s_tau
    int tau;            // step about to be stored (T .. 1)
    unit_t unit;        // load in flight
#ifdef TCQ_DEBUG
    const unsigned char* ws;  // the workspace and its size, for the index checks
    long long ws_n;
#endif

    __device__ __forceinline__ void start(long long blk, uint32_t sT, const unit_t* p,
                                          uint16_t* pth, int T)
    {
        b = blk;
        bp = p;
        path = pth;
        s = sT;
        tau = T;
    }

    __device__ __forceinline__ void issue()
    {
        if (tau > 1) {  // bp_{tau-1}[s_tau >> k] decides s_{tau-1}
            const uint32_t g = s >> (2 * C::K);
            const unit_t* p = bp + (size_t)((tau - 2) / C::SPU) * C::NT + (g % C::NT);
            unit = TCQ_IN_BOUNDS((const unsigned char*)p - ws, ws_n - (long long)sizeof(unit_t) + 1) ? *p : unit_t(0);
        }
    }

    // returns true when the block's path is complete; every lane running the
    // tracer holds the same state, thread 0 of the team stores it
    __device__ __forceinline__ bool retire(bool store)
    {
        if (store && TCQ_IN_BOUNDS((const unsigned char*)(path + tau - 1) - ws, ws_n - 1)) path[tau - 1] = (uint16_t)s;
        if (tau == 1) return true;
        const uint32_t u = s >> C::K;
        const uint32_t g = u >> C::K, j = u & (C::H - 1);
        const int q = (int)((g / C::NT) * C::H + j);  // position of u among its thread's
        const int off = ((tau - 2) % C::SPU) * C::REC_BITS + (C::P - 1 - q);
        uint32_t h = 0;
#pragma unroll
        for (int l = 0; l < C::K; ++l) h = (h << 1) | ((uint32_t)(unit >> (off + l * C::P)) & 1u);
        s = (h << C::LK) | u;
        --tau;
        return false;
    }
};

// CTA warp index of the w-th warp of team m (see the team mapping in the kernel)
template <class C>
__device__ __forceinline__ int team_warp(int m, int w)
{
    constexpr bool STRIDED = C::NTEAM > 1 && C::NT % 32 == 0 && C::NTEAM % 4 == 0;
    return STRIDED ? m + C::NTEAM * w : ((m * C::NT) >> 5) + w;
}

// Sum of v over a team; the team's thread 0 gets the total.  Called by all
// threads of the CTA (it contains __syncthreads for multi-warp teams).
template <class C>
__device__ __forceinline__ double team_sum(double v, double* redd, int m, int tid)
{
    if constexpr (C::NT >= 32) {
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if ((threadIdx.x & 31) == 0) redd[threadIdx.x >> 5] = v;
        __syncthreads();
        double r = 0.0;
        if (tid == 0) {
            for (int w = 0; w < C::NT / 32; ++w) r += redd[team_warp<C>(m, w)];
        }
        __syncthreads();
        return r;
    } else {
#pragma unroll
        for (int o = C::NT / 2; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        return v;
    }
}

// Outputs of one traced block, formed by its whole team from the stored path:
// packed symbols (stream bit p is bit 31 - p mod 32 of word p / 32, symbol t at
// bits [(t-1)k, tk), most significant first, zero padding), the canonical start
// state s_1 >> k, and the cost sum_t d_t (x_t - c[s_t])^2 accumulated in fp64.
// All threads of the CTA call it; b < 0 marks a team with nothing to finish.
template <class C>
__device__ __forceinline__ void finish_block(const GroupedArgs& a, long long b,
                                             const uint16_t* __restrict__ path, double* redd,
                                             int m, int tid)
{
    const int T = a.T;
    double acc = 0.0;
#ifdef TCQ_DEBUG
    const long long x_n = (a.n_blocks - 1) * a.x_stride + T, d_n = (a.n_blocks - 1) * a.d_stride + T;
    const long long o_n = (a.n_blocks - 1) * a.out_stride + 1;
    const long long ws_n = (long long)gridDim.x * (long long)a.slot_bytes;
#endif
    if (b >= 0) {
        const float* xb = a.x + b * opaque(a.x_stride);
        const float* db = a.d ? a.d + b * opaque(a.d_stride) : nullptr;
        for (int t = tid; t < T; t += C::NT) {
            if (!TCQ_IN_BOUNDS(xb + t - a.x, x_n) || !TCQ_IN_BOUNDS((const unsigned char*)(path + t) - a.ws, ws_n - 1) ||
                (db && !TCQ_IN_BOUNDS(db + t - a.d, d_n)) || !TCQ_IN_BOUNDS(path[t], 1 << C::L))
                continue;
            const double e = (double)xb[t] - (double)load_codeword(a.cb, a.cb_f16, path[t]);
            acc += (double)(db ? db[t] : 1.f) * e * e;
        }
        const int nbits = T * C::K;
        for (int w = tid; w < a.W; w += C::NT) {
            uint32_t word = 0;
            for (int i = 0; i < 32; ++i) {
                const int p = 32 * w + i;
                if (p >= nbits) break;
                const uint32_t sym = path[p / C::K] & (C::H - 1);
                word |= ((sym >> (C::K - 1 - p % C::K)) & 1u) << (31 - i);
            }
            if (TCQ_IN_BOUNDS(b * a.out_stride * a.W + w, o_n * a.W)) a.bits[b * opaque(a.out_stride) * a.W + w] = word;
        }
    }
    const double total = team_sum<C>(acc, redd, m, tid);
    if (b >= 0 && tid == 0 && TCQ_IN_BOUNDS(b * a.out_stride, o_n)) {
        a.start_state[b * opaque(a.out_stride)] = (uint32_t)path[0] >> C::K;
        a.path_cost[b * opaque(a.out_stride)] = (float)total;
    }
}

// Maximum of v over a team (every team thread gets it).  Called by all threads.
template <class C>
__device__ __forceinline__ float team_max(float v, float* redv, int m)
{
    if constexpr (C::NT >= 32) {
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if ((threadIdx.x & 31) == 0) redv[threadIdx.x >> 5] = v;
        __syncthreads();
        float r = redv[team_warp<C>(m, 0)];
        for (int w = 1; w < C::NT / 32; ++w) r = fmaxf(r, redv[team_warp<C>(m, w)]);
        __syncthreads();
        return r;
    } else {
#pragma unroll
        for (int o = C::NT / 2; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        return v;
    }
}

// FIXED: every block starts in a.fixed_start[b] (a separate instantiation, so the
// free-start kernel carries none of it).  LONG: blocks of more than kRenormAfter
// steps, whose metrics are shifted every 64 steps; it reads a fixed start, if
// any, at run time.
template <class C, bool WEIGHTED, bool FIXED = false, bool LONG = false>
__global__ void __launch_bounds__(C::NTHREADS, C::MINB) acs_grouped_kernel(GroupedArgs a)
{
    using unit_t = typename C::unit_t;
    extern __shared__ __align__(16) unsigned char smem[];
    float* Mall = reinterpret_cast<float*>(smem);
    float2* stage_all = reinterpret_cast<float2*>(Mall + C::NTEAM * 2 * C::NU);
    float* redv = reinterpret_cast<float*>(stage_all + C::NTEAM * C::TCHUNK);
    uint32_t* reds = reinterpret_cast<uint32_t*>(redv + C::NCOMP / 32);
    double* redd = reinterpret_cast<double*>(reds + C::NCOMP / 32);  // 8-byte aligned

    const int T = a.T;
    const long long nb = a.n_blocks;
    const long long stride = (long long)gridDim.x * C::NTEAM;
    const long long first = (long long)blockIdx.x * C::NTEAM;
    const int R = first < nb ? (int)((nb - first + stride - 1) / stride) : 0;
    unsigned char* slot = a.ws + (size_t)blockIdx.x * a.slot_bytes;
    const size_t team_bytes = C::team_bytes(T);

    // teams of whole warps take warps m, m + NTEAM, ...: a team's warps then share
    // a scheduler (warp w issues from scheduler w mod 4) and wait for each other
    // less at the team barrier
    constexpr bool STRIDED = C::NTEAM > 1 && C::NT % 32 == 0 && C::NTEAM % 4 == 0;
    const int m = STRIDED ? (int)((threadIdx.x >> 5) % C::NTEAM) : threadIdx.x / C::NT;  // team
    const int tid = STRIDED ? (int)(((threadIdx.x >> 5) / C::NTEAM) * 32 + (threadIdx.x & 31))
                            : threadIdx.x % C::NT;  // thread within the team
    // the team's first warp (or whole sub-warp team) runs the traceback in
    // lockstep: no divergent branch, the loads of all lanes hit one address
    const bool tracer = tid < 32;
    float* Mteam = Mall + m * 2 * C::NU;
    float2* stage = stage_all + m * C::TCHUNK;
    uint16_t* path = reinterpret_cast<uint16_t*>(slot + 2 * C::NTEAM * team_bytes +
                                                 (size_t)m * C::path_bytes(T));
    Codewords<C, C::CB16> cw;
    cw.load(a.cb, a.cb_f16, tid);
    Tracer<C> tr;
    tr.b = -1;
#ifdef TCQ_DEBUG
    const long long x_n = (a.n_blocks - 1) * a.x_stride + T, d_n = (a.n_blocks - 1) * a.d_stride + T;
    const long long ws_n = (long long)gridDim.x * (long long)a.slot_bytes;
    tr.ws = a.ws;
    tr.ws_n = ws_n;
#endif

    for (int r = 0; r < R; ++r) {
        const int par = r & 1;
        const long long b = first + (long long)r * stride + m;
        const bool valid = b < nb;
        unit_t* bp = reinterpret_cast<unit_t*>(slot + (size_t)(par * C::NTEAM + m) * team_bytes);
        const float* xb = a.x + (valid ? b : 0) * opaque(a.x_stride);
        const float* db = a.d ? a.d + (valid ? b : 0) * opaque(a.d_stride) : nullptr;
        float dfloor = 0.f;
        if constexpr (C::CB16 && WEIGHTED) {
            float dm = 0.f;
            if (valid)
                for (int q = tid; q < T; q += C::NT)
                    dm = fmaxf(dm, db && TCQ_IN_BOUNDS(db + q - a.d, d_n) ? db[q] : 1.f);
            dfloor = fmaxf(team_max<C>(dm, redv, m) * 0x1p-60f, 1.17549435e-38f);
        }
        unit_t acc = 0;
        float bestv = __int_as_float(0x7f800000);  // +inf
        uint32_t bests = 0xffffffffu;

        unit_t* bpw = bp + tid;  // next backpointer record of this thread
        // a team's steps depend only on its own metrics and staged inputs: with
        // several warp-wide teams per CTA each syncs alone on a named barrier
        auto team_sync = [&]() {
            if constexpr (C::NTEAM == 1) {
                __syncthreads();
            } else if constexpr (C::NT % 32 == 0) {
                named_barrier(1 + m, C::NT);
            } else {  // teams narrower than a warp: measured faster with the CTA barrier
                __syncthreads();
            }
        };
        // one trellis step; FIRST and LAST select the variant
        auto step = [&](auto first_tag, auto last_tag, int t) {
            constexpr bool FIRST = decltype(first_tag)::value;
            constexpr bool LAST = decltype(last_tag)::value;
            const int tc = (t - 1) % C::TCHUNK;
            if (tc == 0) {
                if (valid) {
                    for (int q = tid; q < C::TCHUNK && t + q <= T; q += C::NT) {
                        if (!TCQ_IN_BOUNDS(xb + t - 1 + q - a.x, x_n) ||
                            (db && !TCQ_IN_BOUNDS(db + t - 1 + q - a.d, d_n)) ||
                            (db && t - 1 + q > 0 && !TCQ_IN_BOUNDS(db + t - 2 + q - a.d, d_n)))
                            continue;
                        const float xv = xb[t - 1 + q];
                        const float dv = (WEIGHTED && db) ? db[t - 1 + q] : 1.f;
                        if constexpr (C::CB16) {
                            float rr = 1.f;  // d_{t-1} / d_t, applied to the metrics read at step t
                            if (WEIGHTED) {
                                const float dc = fmaxf(dv, dfloor);
                                const float dp = (t - 1 + q) > 0 ? fmaxf(db ? db[t - 2 + q] : 1.f, dfloor) : dc;
                                rr = dp / dc;
                            }
                            stage[q] = make_float2(-xv, rr);
                        } else {
                            const float sd = WEIGHTED ? sqrtf(dv) : 1.f;
                            stage[q] = make_float2(-sd, sd * xv);
                        }
                    }
                }
                team_sync();
            }
            const bool tracing = tracer && tr.b >= 0;
            if (tracing) tr.issue();
            if (valid) {
                const float2 ax = stage[tc];
                const float* Mp = Mteam + ((t - 1) & 1) * C::NU;
                float* Mn = Mteam + (t & 1) * C::NU;
                uint32_t planes[C::K];
                uint32_t s0 = 0xffffffffu;
                if constexpr (FIRST && FIXED)
                    if (TCQ_IN_BOUNDS(b, a.n_blocks)) s0 = a.fixed_start[b] & (uint32_t)(C::NU - 1);
                if constexpr (FIRST && LONG)
                    if (a.fixed_start && TCQ_IN_BOUNDS(b, a.n_blocks)) s0 = a.fixed_start[b] & (uint32_t)(C::NU - 1);
                acs_step<C, WEIGHTED, FIRST, LAST>(cw, ax.x, ax.y, Mp, Mn, tid, planes, bestv, bests,
                                                   s0);
                if constexpr (!LAST) {
                    unit_t rec = 0;
#pragma unroll
                    for (int l = 0; l < C::K; ++l) rec |= (unit_t)planes[l] << (l * C::P);
                    if constexpr (C::SPU == 1) {
                        if (TCQ_IN_BOUNDS((const unsigned char*)bpw - a.ws, ws_n - (long long)sizeof(unit_t) + 1)) *bpw = rec;
                        bpw += C::NT;
                    } else {
                        const int q = (t - 1) % C::SPU;
                        acc |= rec << (q * C::REC_BITS);
                        if (q == C::SPU - 1 || t == T - 1) {
                            if (TCQ_IN_BOUNDS((const unsigned char*)bpw - a.ws, ws_n - (long long)sizeof(unit_t) + 1)) *bpw = acc;
                            bpw += C::NT;
                            acc = 0;
                        }
                    }
                }
            }
            if (tracing && tr.retire(tid == 0)) tr.b = -1;
            if (!LAST) team_sync();
            if constexpr (LONG && !LAST) {
                // long blocks: shift the team's metrics by state 0's every 64 steps
                if ((t & 63) == 0) {
                    float* Mn = Mteam + (t & 1) * C::NU;
                    const float o = Mn[0];
                    const float off = (o < __int_as_float(0x7f800000)) ? o : 0.f;
                    team_sync();
#pragma unroll
                    for (int i = 0; i < C::GPT; ++i) {
                        float* row = Mn + ((size_t)(tid + i * C::NT) << C::K);
#pragma unroll
                        for (int j = 0; j < C::H; ++j) row[j] -= off;
                    }
                    team_sync();
                }
            }
        };
        using T0 = std::false_type;
        using T1 = std::true_type;
        if (T == 1) {
            step(T1{}, T1{}, 1);
        } else {
            step(T1{}, T0{}, 1);
            for (int t = 2; t < T; ++t) step(T0{}, T0{}, t);
            step(T0{}, T1{}, T);
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
                float bv = redv[team_warp<C>(m, 0)];
                uint32_t bs = reds[team_warp<C>(m, 0)];
                for (int w = 1; w < C::NT / 32; ++w)
                    keep_best(redv[team_warp<C>(m, w)], reds[team_warp<C>(m, w)], bv, bs);
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
        // the previous round's block was traced during this round's T steps:
        // its path is complete, the team forms its outputs
        __syncthreads();
        if (r > 0) {
            const long long pb = b - stride;  // this team's block of round r-1 (always valid)
            finish_block<C>(a, pb, path, redd, m, tid);
        }
        __syncthreads();  // path consumed; this round's backpointers visible to the tracer
        // the team's thread 0 holds the final state; its trace runs during the next round
        if (tracer && valid) tr.start(b, bests, bp, path, T);
    }
    // the last block of each team has no next round to hide behind
    if constexpr (C::NT <= 64 && C::UNIT_BITS == 32) {
        // small teams: the walk's dependent loads would each wait an L2 round
        // trip, so the team copies its records into its metric buffer (dead
        // now) a chunk of rows at a time, with coalesced loads, and the walk
        // reads them there; every team takes the same barriers (T is common)
        constexpr int CHR = (2 * C::NU) / C::NT;  // record rows per chunk
        static_assert(CHR >= 1, "a chunk holds at least one row of records");
        uint32_t* buf = reinterpret_cast<uint32_t*>(Mteam);
        const int rows = (T - 2 + C::SPU) / C::SPU;  // rows of records of T - 1 steps
        // the same in every thread of the team (only the tracer lanes hold tr)
        const bool walking = R > 0 && first + (long long)(R - 1) * stride + m < nb;
        const uint32_t* bpt = reinterpret_cast<const uint32_t*>(
            slot + (size_t)(((R - 1) & 1) * C::NTEAM + m) * team_bytes);
        for (int hi = rows - 1; hi >= 0; hi -= CHR) {
            const int lo = hi - CHR + 1 > 0 ? hi - CHR + 1 : 0;
            if (walking)
                for (int i = tid; i < (hi - lo + 1) * C::NT; i += C::NT)
                    if (TCQ_IN_BOUNDS((const unsigned char*)(bpt + (size_t)lo * C::NT + i) - a.ws, ws_n - 3))
                        buf[i] = bpt[(size_t)lo * C::NT + i];
            if constexpr (C::NTEAM == 1 || C::NT % 32 != 0) __syncthreads(); else named_barrier(1 + m, C::NT);
            if (tracer && walking) {
                while (tr.tau > 1 && (tr.tau - 2) / C::SPU >= lo) {
                    const uint32_t g = tr.s >> (2 * C::K);
                    tr.unit = buf[((tr.tau - 2) / C::SPU - lo) * C::NT + (g % C::NT)];
                    tr.retire(tid == 0);
                }
            }
            if constexpr (C::NTEAM == 1 || C::NT % 32 != 0) __syncthreads(); else named_barrier(1 + m, C::NT);
        }
        if (tracer && walking) tr.retire(tid == 0);  // stores s_1
    } else if (tracer && tr.b >= 0) {
        while (true) {
            tr.issue();
            if (tr.retire(tid == 0)) break;
        }
    }
    __syncthreads();
    if (R > 0) {
        const long long lb = first + (long long)(R - 1) * stride + m;
        finish_block<C>(a, lb < nb ? lb : -1, path, redd, m, tid);
    }
}

template <class C, bool WEIGHTED, bool FIXED = false, bool LONG = false>
cudaError_t launch_grouped_w(const EncodeArgs& a, int grid, cudaStream_t stream)
{
    const size_t smem = C::smem_bytes(a.L, a.K, a.T);
    cudaError_t e = cudaFuncSetAttribute(acs_grouped_kernel<C, WEIGHTED, FIXED, LONG>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    acs_grouped_kernel<C, WEIGHTED, FIXED, LONG><<<grid, C::NTHREADS, smem, stream>>>(grouped_args(a));
    return cudaGetLastError();
}

template <class C>
cudaError_t launch_grouped(const EncodeArgs& a, int grid, cudaStream_t stream)
{
    // The fp16-pair kernels always run the weighted form (an absent d reads as 1,
    // every ratio d_{t-1}/d_t is then 1): measured faster than a separate
    // unweighted instantiation, whose schedule came out worse.
    // blocks of more than kRenormAfter steps: the renormalising instantiation
    // (weighted form, free or fixed start read at run time), kept apart so that
    // the code of short blocks does not change
    if (a.T > kRenormAfter) return launch_grouped_w<C, true, false, true>(a, grid, stream);
    if (a.fixed_start)  // weighted form: an absent d reads as 1
        return launch_grouped_w<C, true, true>(a, grid, stream);
    if constexpr (C::CB16)
        return launch_grouped_w<C, true>(a, grid, stream);
    else
        return a.d ? launch_grouped_w<C, true>(a, grid, stream)
                   : launch_grouped_w<C, false>(a, grid, stream);
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
