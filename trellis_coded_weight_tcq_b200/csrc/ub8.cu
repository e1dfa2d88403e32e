// ub8.cu -- trellis-coded quantization over Ungerboeck's 8-state
// set-partitioned trellis, and its decoder.
//
// Source: the 2-bit post ("How do you fit a 4B LLM in 1.24 GB? Trellis-coded
// 2-bit"), Pingala-8 section: an 8-state set-partitioned trellis with
// Ungerboeck's labels over symbols of several weights at about 2 bits per
// weight; its section on trellis-coded quantization: the state selects the
// subset the next symbol may use, the written bits pick a value inside it and
// set the next state.  The labels are those of Marcellin and Fischer's TCQ on
// Ungerboeck's 8-state code for one-dimensional signals (parity-check
// polynomials 13 and 04 octal), with V weights per symbol:
//   - union codebook of 4 * 2^m rows of V values, row r in subset D_{r mod 4};
//   - state sigma = 4p + 2q + r; the branch with bit z uses subset 2z + p and
//     leads to 4(p ^ q) + 2(r ^ z) + p;
//   - a step codes V weights with 1 + m bits, symbol (z << m) | i, row 4i + 2z + p.
//
// Encoder, one warp per coding block (CTAs of several warps loop over blocks):
//   1. branch metrics: lane l takes steps l, l + 32, ... two at a time; for
//      each it scans the union codebook (staged in shared memory as fp32, every
//      lane reading the same row, so each read is a broadcast) and keeps the
//      nearest entry of every subset, d-weighted, in fp32 with the error formed
//      as fma(-sqrt d, c, sqrt(d) x) (no cancellation) and ties to the smaller
//      entry;
//   2. the Viterbi recursion over the 8 states on lanes 0..7: each state has two
//      predecessors, sigma_a = 4r' + 2(p' ^ r') and sigma_a + 1, whose metrics
//      come by shuffle; a strict compare keeps the smaller predecessor on ties
//      and the choice bits of the 8 states are one ballot byte per step;
//   3. lane 0 traces back from the smallest final state (lexicographic, so the
//      smaller state wins ties), then the warp packs the symbols MSB first and
//      sums the path's cost in fp64.
// Nothing needs a workspace: per step the warp keeps 4 metrics, 4 entry
// indices, one backpointer byte, the symbol and the row in shared memory, which
// bounds a block to TCQ_UB8_MAX_STEPS steps.
//
// Decoder: the state at every step depends on all earlier branch bits, so a
// warp first walks 32 blocks at once (one lane per block, only the branch bit
// of each symbol read) and records each step's subset half p; then it writes
// the 32 blocks one after the other with the whole warp, lane l emitting steps
// l, l + 32, ... (coalesced rows of V floats).
#include "common.cuh"

namespace tcq {

namespace {

constexpr int kUb8Warps = 8;    // warps (blocks in flight) per encoder CTA
constexpr int kUb8Unroll = 2;   // steps a lane scores per pass over the codebook

// shared memory per encoder warp and step: 4 metrics, 4 entry indices (bytes),
// the backpointer byte, the symbol and the row (16-bit each)
constexpr size_t kUb8StepBytes = 4 * 4 + 4 + 1 + 2 + 2;

__host__ __device__ constexpr int ub8_next(int s, int z)
{
    return 4 * (((s >> 2) & 1) ^ ((s >> 1) & 1)) + 2 * ((s & 1) ^ z) + ((s >> 2) & 1);
}

// the successors of states 0..7 as nibbles (nibble s = ub8_next(s, z)), one table per z
__host__ __device__ constexpr uint32_t ub8_next_table(int z)
{
    uint32_t t = 0;
    for (int s = 0; s < 8; ++s) t |= (uint32_t)ub8_next(s, z) << (4 * s);
    return t;
}
constexpr uint32_t kUb8Next0 = ub8_next_table(0), kUb8Next1 = ub8_next_table(1);

// Stages the union codebook (rows x V, fp32 or binary16) into shared memory as fp32.
__device__ __forceinline__ void ub8_stage_codebook(float* dst, const void* cb, int cb_f16, int n)
{
    for (int i = threadIdx.x; i < n; i += blockDim.x) dst[i] = load_codeword(cb, cb_f16, (uint32_t)i);
}

// The encoder's copy of the union codebook pairs the subsets (D_0, D_1) and
// (D_2, D_3) of every entry coordinate by coordinate, so that one packed f32x2
// operation works on two candidates: value v of row r = 4 i + j sits at
// ((2 i + (j >> 1)) V + v) 2 + (j & 1).
__device__ __forceinline__ int ub8_pair_index(int r, int v, int V)
{
    return ((2 * (r >> 2) + ((r >> 1) & 1)) * V + v) * 2 + (r & 1);
}

__device__ __forceinline__ void ub8_stage_pairs(float* dst, const void* cb, int cb_f16, int rows, int V)
{
    for (int i = threadIdx.x; i < rows * V; i += blockDim.x)
        dst[ub8_pair_index(i / V, i % V, V)] = load_codeword(cb, cb_f16, (uint32_t)i);
}

__device__ __forceinline__ unsigned long long ub8_pack(float a, float b)
{
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}

template <int V>
__global__ void __launch_bounds__(kUb8Warps * 32) ub8_encode_kernel(Ub8EncodeArgs a)
{
    extern __shared__ __align__(16) unsigned char smem[];
    const int rows = 4 << a.m;
    float* cbs = reinterpret_cast<float*>(smem);
    const int S = a.T / V;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned char* wbase = smem + (((size_t)rows * V * 4 + 15) & ~(size_t)15) +
                           (size_t)warp * (((size_t)S * kUb8StepBytes + 15) & ~(size_t)15);
    float* E = reinterpret_cast<float*>(wbase);                    // [S][4]
    uint8_t* I = reinterpret_cast<uint8_t*>(E + 4 * S);           // [S][4]
    uint16_t* SYM = reinterpret_cast<uint16_t*>(I + 4 * S);       // [S]
    uint16_t* ROW = SYM + S;                                       // [S]
    uint8_t* BP = reinterpret_cast<uint8_t*>(ROW + S);             // [S]

    ub8_stage_pairs(cbs, a.cb, a.cb_f16, rows, V);
    __syncthreads();

    const int n_sub = 1 << a.m;
    const int K = 1 + a.m;
    for (long long b = (long long)blockIdx.x * kUb8Warps + warp; b < a.n_blocks;
         b += (long long)gridDim.x * kUb8Warps) {
        const float* xb = a.x + b * a.T;
        const float* db = a.d ? a.d + b * a.T : nullptr;

        // ---- 1. nearest entry of every subset, per step
        for (int t0 = lane; t0 < S; t0 += 32 * kUb8Unroll) {
            // per step and coordinate the packed pairs (-sqrt d, -sqrt d) and
            // (sqrt(d) x, sqrt(d) x): both candidates of a subset pair see them
            unsigned long long nsd2[kUb8Unroll][V], xs2[kUb8Unroll][V];
#pragma unroll
            for (int u = 0; u < kUb8Unroll; ++u) {
                const int t = t0 + 32 * u < S ? t0 + 32 * u : t0;  // a spare lane repeats a valid step
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    const bool ok = TCQ_IN_BOUNDS(b * a.T + t * V + v, a.n_blocks * a.T);
                    const float dv = db && ok ? db[t * V + v] : 1.f;
                    const float sd = sqrtf(dv);
                    const float xs = ok ? sd * xb[t * V + v] : 0.f;
                    nsd2[u][v] = ub8_pack(-sd, -sd);
                    xs2[u][v] = ub8_pack(xs, xs);
                }
            }
            float best[kUb8Unroll][4];
            int bi[kUb8Unroll][4];
#pragma unroll
            for (int u = 0; u < kUb8Unroll; ++u)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    best[u][j] = __int_as_float(0x7f800000);
                    bi[u][j] = 0;
                }
            // entries two at a time when there are two (m >= 1): half the loop overhead
#pragma unroll 2
            for (int i = 0; i < n_sub; ++i) {
                const unsigned long long* grp =
                    reinterpret_cast<const unsigned long long*>(cbs) + (size_t)(2 * i) * V;
#pragma unroll
                for (int pp = 0; pp < 2; ++pp) {  // subsets (2pp, 2pp + 1)
                    unsigned long long c2[V];
                    if constexpr (V % 2 == 0) {  // 16-byte loads: two coordinates' pairs each
#pragma unroll
                        for (int v = 0; v < V; v += 2) {
                            const ulonglong2 q = *reinterpret_cast<const ulonglong2*>(grp + pp * V + v);
                            c2[v] = q.x;
                            c2[v + 1] = q.y;
                        }
                    } else {
#pragma unroll
                        for (int v = 0; v < V; ++v) c2[v] = grp[pp * V + v];
                    }
#pragma unroll
                    for (int u = 0; u < kUb8Unroll; ++u) {
                        // e = fma(-sqrt d, c, sqrt(d) x), dist = fma(e, e, dist) in each half
                        unsigned long long dist2 = 0ull;
#pragma unroll
                        for (int v = 0; v < V; ++v) {
                            unsigned long long e2;
                            asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(e2) : "l"(nsd2[u][v]), "l"(c2[v]), "l"(xs2[u][v]));
                            if (v == 0)
                                asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(dist2) : "l"(e2), "l"(e2));
                            else
                                asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(dist2) : "l"(e2), "l"(e2), "l"(dist2));
                        }
                        float d0, d1;
                        asm("mov.b64 {%0, %1}, %2;" : "=f"(d0), "=f"(d1) : "l"(dist2));
                        if (d0 < best[u][2 * pp]) {
                            best[u][2 * pp] = d0;
                            bi[u][2 * pp] = i;
                        }
                        if (d1 < best[u][2 * pp + 1]) {
                            best[u][2 * pp + 1] = d1;
                            bi[u][2 * pp + 1] = i;
                        }
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < kUb8Unroll; ++u) {
                const int t = t0 + 32 * u;
                if (t < S) {
                    *reinterpret_cast<float4*>(E + 4 * t) =
                        make_float4(best[u][0], best[u][1], best[u][2], best[u][3]);
                    *reinterpret_cast<uint32_t*>(I + 4 * t) =
                        (uint32_t)bi[u][0] | ((uint32_t)bi[u][1] << 8) | ((uint32_t)bi[u][2] << 16) |
                        ((uint32_t)bi[u][3] << 24);
                }
            }
        }
        __syncwarp();

        // ---- 2. Viterbi over the 8 states (lanes 0..7 hold one state each; the
        // other lanes follow along on state lane & 7 so every shuffle is full)
        const int sg = lane & 7;
        const int p2 = (sg >> 2) & 1, q2 = (sg >> 1) & 1, r2 = sg & 1;
        const int sa = 4 * r2 + 2 * (p2 ^ r2);  // predecessor with r = 0; the other is sa + 1
        const int ja = 2 * q2 + r2;             // its subset (z = q2, p = r2)
        const int jb = 2 * (q2 ^ 1) + r2;       // the subset from sa + 1 (z = q2 ^ 1)
        float M = 0.f;
        if (a.fixed_start && TCQ_IN_BOUNDS(b, a.n_blocks))
            M = (sg == (int)(a.fixed_start[b] & 7u)) ? 0.f : __int_as_float(0x7f800000);
        for (int t = 0; t < S; ++t) {
            const float ma = __shfl_sync(0xffffffffu, M, sa);
            const float mb = __shfl_sync(0xffffffffu, M, sa + 1);
            const float ca = ma + E[4 * t + ja];
            const float cb = mb + E[4 * t + jb];
            const bool takeb = cb < ca;
            M = takeb ? cb : ca;
            const uint32_t ch = __ballot_sync(0xffffffffu, takeb);
            if (lane == 0) BP[t] = (uint8_t)(ch & 0xffu);
        }
        // smallest final metric, the smaller state on ties
        float bv = M;
        int bs = sg;
#pragma unroll
        for (int o = 4; o >= 1; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int os = __shfl_xor_sync(0xffffffffu, bs, o);
            if (ov < bv || (ov == bv && os < bs)) {
                bv = ov;
                bs = os;
            }
        }
        __syncwarp();

        // ---- 3. traceback on lane 0: backpointer bytes and index words are read
        // at addresses that do not depend on the walk
        if (lane == 0) {
            int s = bs;
            for (int t = S - 1; t >= 0; --t) {
                const int bsel = (BP[t] >> s) & 1;
                const uint32_t iw = *reinterpret_cast<const uint32_t*>(I + 4 * t);
                const int sp = (s >> 2) & 1, sq = (s >> 1) & 1, sr = s & 1;
                const int prev = 4 * sr + 2 * (sp ^ sr) + bsel;
                const int z = sq ^ bsel;
                const int j = 2 * z + sr;  // p(prev) = sr
                const int i = (int)((iw >> (8 * j)) & 0xffu);
                SYM[t] = (uint16_t)((z << a.m) | i);
                ROW[t] = (uint16_t)(4 * i + j);
                s = prev;
            }
            if (TCQ_IN_BOUNDS(b, a.n_blocks)) a.start_state[b] = (uint32_t)s;
        }
        __syncwarp();

        // packed symbols, MSB first: symbol t at stream bits [tK, tK + K)
        const int nbits = S * K;
        uint32_t* wb = a.bits + b * a.W;
        for (int w = lane; w < a.W; w += 32) {
            uint32_t word = 0;
            int p = 32 * w;
            const int pend = min(32 * w + 32, nbits);
            while (p < pend) {
                const int t = p / K, off = p - t * K;
                const int take = min(K - off, pend - p);
                const uint32_t bits = ((uint32_t)SYM[t] >> (K - off - take)) & ((1u << take) - 1u);
                word |= bits << (32 * w + 32 - p - take);
                p += take;
            }
            if (TCQ_IN_BOUNDS(b * a.W + w, a.n_blocks * a.W)) wb[w] = word;
        }
        // the path's cost, summed in fp64
        double acc = 0.0;
        for (int t = lane; t < S; t += 32) {
            const int r = ROW[t];
#pragma unroll
            for (int v = 0; v < V; ++v) {
                if (!TCQ_IN_BOUNDS(b * a.T + t * V + v, a.n_blocks * a.T)) continue;
                const double e = (double)xb[t * V + v] - (double)cbs[ub8_pair_index(r, v, V)];
                acc += (double)(db ? db[t * V + v] : 1.f) * e * e;
            }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0 && TCQ_IN_BOUNDS(b, a.n_blocks)) a.path_cost[b] = (float)acc;
        __syncwarp();  // the warp's arrays are reused by its next block
    }
}

// ---- decoder
constexpr int kUb8DecWarps = 8;

// STAGED: the 32 blocks' stream words (W <= kUb8DecStageWords each) are first
// copied into shared memory with coalesced loads (the walk's loads would
// otherwise each wait on memory in turn), rows padded by one word so that the
// walk's lanes, one per block, hit distinct banks.  VSTORE: rows of V = 2, 4
// or 8 values leave as 8- or 16-byte stores (the output is aligned for them).
constexpr int kUb8DecStageWords = 32;

// six CTAs per SM (at most 40 registers); the shapes that would spill at 40
// registers keep the default register count
template <int V, bool STAGED, bool VSTORE>
constexpr int ub8_dec_min_blocks() { return STAGED && !(V == 8 && VSTORE) ? 6 : 1; }

template <int V, bool STAGED, bool VSTORE>
__global__ void __launch_bounds__(kUb8DecWarps * 32, (ub8_dec_min_blocks<V, STAGED, VSTORE>())) ub8_decode_kernel(Ub8DecodeArgs a)
{
    extern __shared__ __align__(16) unsigned char smem[];
    const int rows = 4 << a.m;
    float* cbs = reinterpret_cast<float*>(smem);
    const int S = a.T / V;
    const int PW = (S + 31) / 32;  // words of subset-half bits per block
    const int WP = a.W + 1;        // padded row of staged words
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t* P = reinterpret_cast<uint32_t*>(smem + (((size_t)rows * V * 4 + 15) & ~(size_t)15)) +
                  (size_t)warp * 32 * PW;  // [32 blocks][PW]
    uint32_t* WB = reinterpret_cast<uint32_t*>(smem + (((size_t)rows * V * 4 + 15) & ~(size_t)15)) +
                   (size_t)kUb8DecWarps * 32 * PW + (size_t)warp * 32 * WP;  // [32 blocks][W + 1]
    ub8_stage_codebook(cbs, a.cb, a.cb_f16, rows * V);
    __syncthreads();

    const int K = 1 + a.m;
    const uint32_t imask = (1u << a.m) - 1u;
    const long long groups = (a.n_blocks + 31) / 32;
    for (long long g = (long long)blockIdx.x * kUb8DecWarps + warp; g < groups;
         g += (long long)gridDim.x * kUb8DecWarps) {
        const long long b0 = g * 32;
        const int nb = (int)min(32LL, a.n_blocks - b0);
        if constexpr (STAGED) {
            // the group's words, row by row (lane w of a row loads word w; the
            // group's rows are contiguous, so a row is one coalesced read), eight
            // rows in flight per lane, then stored into the padded rows
            const uint32_t* src = a.bits + b0 * a.W + lane;
            uint32_t* dst = WB + lane;
            for (int q0 = 0; q0 < nb; q0 += 8) {
                uint32_t r[8];
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    r[u] = lane < a.W && q0 + u < nb && TCQ_IN_BOUNDS((b0 + q0 + u) * a.W + lane, a.n_blocks * a.W)
                               ? src[(q0 + u) * a.W] : 0u;
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    if (lane < a.W && q0 + u < nb) dst[(q0 + u) * WP] = r[u];
            }
            __syncwarp();
        }
        auto word = [&](int q, int w) -> uint32_t {
            if constexpr (STAGED) return WB[q * WP + w];
            else return TCQ_IN_BOUNDS((b0 + q) * a.W + w, a.n_blocks * a.W) ? a.bits[(b0 + q) * a.W + w] : 0u;
        };
        // walk: lane l follows block b0 + l and records p of the state before each
        // step; the successor of state s on branch bit z is nibble s of kUb8Next[z]
        if (lane < nb) {
            const long long b = b0 + lane;
            uint32_t* Pl = P + lane * PW;
            uint32_t s = TCQ_IN_BOUNDS(b, a.n_blocks) ? (a.start_state[b] & 7u) : 0u;
            uint32_t acc = 0;
            int pos = 0;  // the branch bit is the symbol's first bit
            for (int t = 0; t < S; ++t, pos += K) {
                const uint32_t z = (word(lane, pos >> 5) >> (31 - (pos & 31))) & 1u;
                acc = __funnelshift_r(acc, s >> 2, 1);  // p of step t into bit 31, earlier steps down
                if ((t & 31) == 31) {
                    Pl[t >> 5] = acc;
                    acc = 0;
                }
                s = ((z ? kUb8Next1 : kUb8Next0) >> (4 * s)) & 7u;
            }
            if (S & 31) Pl[S >> 5] = acc >> (32 - (S & 31));
        }
        __syncwarp();
        // emit: the whole warp writes one block at a time, lane l the steps
        // t = l + 32 r; a step's stream position, word and P bit depend only on
        // (lane, r), so they are set once per r and the inner loop runs over blocks
        for (int r = 0; 32 * r < S; ++r) {
            const int t = lane + 32 * r;
            if (t >= S) break;
            const int pos = t * K;
            const int w0 = pos >> 5, off = pos & 31;
            const bool two = off + K > 32;  // K <= 9 bits: at most two words
            float* yt = a.y + b0 * a.T + t * V;   // block q's values at yt + q T
            const uint32_t* pr = P + r;           // block q's P word at pr + q PW
            const uint32_t* wq = WB + w0;         // staged: block q's word w0 at wq + q WP
            for (int q = 0; q < nb; ++q, yt += a.T, pr += PW, wq += WP) {
                uint32_t hi, lo = 0u;
                if constexpr (STAGED) {
                    hi = wq[0];
                    if (two) lo = wq[1];
                } else {
                    hi = word(q, w0);
                    if (two) lo = word(q, w0 + 1);
                }
                const uint32_t sym = __funnelshift_l(lo, hi, off) >> (32 - K);
                const uint32_t z = sym >> a.m;
                const uint32_t p = (*pr >> lane) & 1u;
                const float* row = cbs + (size_t)(((sym & imask) << 2) | (z << 1) | p) * V;
                if (!TCQ_IN_BOUNDS((b0 + q) * a.T + t * V + V - 1, a.n_blocks * a.T)) continue;
                if constexpr (VSTORE && V == 4) {
                    *reinterpret_cast<float4*>(yt) = *reinterpret_cast<const float4*>(row);
                } else if constexpr (VSTORE && V == 8) {
                    reinterpret_cast<float4*>(yt)[0] = reinterpret_cast<const float4*>(row)[0];
                    reinterpret_cast<float4*>(yt)[1] = reinterpret_cast<const float4*>(row)[1];
                } else if constexpr (VSTORE && V == 2) {
                    *reinterpret_cast<float2*>(yt) = *reinterpret_cast<const float2*>(row);
                } else {
#pragma unroll
                    for (int v = 0; v < V; ++v) yt[v] = row[v];
                }
            }
        }
        __syncwarp();
    }
}

template <int V>
cudaError_t launch_ub8_encode_v(const Ub8EncodeArgs& a, int num_sms, cudaStream_t stream)
{
    const size_t smem = ub8_encode_smem_bytes(V, a.m, a.T);
    cudaError_t e = cudaFuncSetAttribute(ub8_encode_kernel<V>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, ub8_encode_kernel<V>, kUb8Warps * 32, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const long long need = (a.n_blocks + kUb8Warps - 1) / kUb8Warps;
    const long long resident = (long long)num_sms * per_sm;
    const int grid = (int)(need < resident ? need : resident);
    ub8_encode_kernel<V><<<grid, kUb8Warps * 32, smem, stream>>>(a);
    return cudaGetLastError();
}

template <int V, bool STAGED, bool VSTORE>
cudaError_t launch_ub8_decode_sv(const Ub8DecodeArgs& a, int num_sms, cudaStream_t stream)
{
    const size_t smem = ub8_decode_smem_bytes(V, a.m, a.T);
    cudaError_t e = cudaFuncSetAttribute(ub8_decode_kernel<V, STAGED, VSTORE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, ub8_decode_kernel<V, STAGED, VSTORE>,
                                                      kUb8DecWarps * 32, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const long long groups = (a.n_blocks + 31) / 32;
    const long long need = (groups + kUb8DecWarps - 1) / kUb8DecWarps;
    const long long resident = (long long)num_sms * per_sm;
    const int grid = (int)(need < resident ? need : resident);
    ub8_decode_kernel<V, STAGED, VSTORE><<<grid, kUb8DecWarps * 32, smem, stream>>>(a);
    return cudaGetLastError();
}

template <int V>
cudaError_t launch_ub8_decode_v(const Ub8DecodeArgs& a, int num_sms, cudaStream_t stream)
{
    // vector stores when V is 2, 4 or 8 and every row of V values is aligned for them
    const size_t vb = (V == 2 ? 8 : 16);
    const bool vst = (V == 2 || V == 4 || V == 8) && (reinterpret_cast<uintptr_t>(a.y) % vb) == 0 &&
                     ((size_t)a.T * 4) % vb == 0;
    const bool staged = a.W <= kUb8DecStageWords;
    if (staged)
        return vst ? launch_ub8_decode_sv<V, true, true>(a, num_sms, stream)
                   : launch_ub8_decode_sv<V, true, false>(a, num_sms, stream);
    return vst ? launch_ub8_decode_sv<V, false, true>(a, num_sms, stream)
               : launch_ub8_decode_sv<V, false, false>(a, num_sms, stream);
}

}  // namespace

size_t ub8_encode_smem_bytes(int V, int m, int T)
{
    const size_t cb = ((size_t)(4 << m) * V * 4 + 15) & ~(size_t)15;
    const size_t per_warp = ((size_t)(T / V) * kUb8StepBytes + 15) & ~(size_t)15;
    return cb + kUb8Warps * per_warp;
}

size_t ub8_decode_smem_bytes(int V, int m, int T)
{
    const size_t cb = ((size_t)(4 << m) * V * 4 + 15) & ~(size_t)15;
    const size_t pw = (size_t)((T / V + 31) / 32);
    const size_t W = (size_t)((T / V * (1 + m) + 31) / 32);
    const size_t staged = W <= (size_t)kUb8DecStageWords ? (size_t)kUb8DecWarps * 32 * (W + 1) * 4 : 0;
    return cb + (size_t)kUb8DecWarps * 32 * pw * 4 + staged;
}

cudaError_t launch_ub8_encode(const Ub8EncodeArgs& a, int num_sms, cudaStream_t stream)
{
    switch (a.V) {
    case 1: return launch_ub8_encode_v<1>(a, num_sms, stream);
    case 2: return launch_ub8_encode_v<2>(a, num_sms, stream);
    case 3: return launch_ub8_encode_v<3>(a, num_sms, stream);
    case 4: return launch_ub8_encode_v<4>(a, num_sms, stream);
    case 5: return launch_ub8_encode_v<5>(a, num_sms, stream);
    case 6: return launch_ub8_encode_v<6>(a, num_sms, stream);
    case 7: return launch_ub8_encode_v<7>(a, num_sms, stream);
    case 8: return launch_ub8_encode_v<8>(a, num_sms, stream);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_ub8_decode(const Ub8DecodeArgs& a, int num_sms, cudaStream_t stream)
{
    switch (a.V) {
    case 1: return launch_ub8_decode_v<1>(a, num_sms, stream);
    case 2: return launch_ub8_decode_v<2>(a, num_sms, stream);
    case 3: return launch_ub8_decode_v<3>(a, num_sms, stream);
    case 4: return launch_ub8_decode_v<4>(a, num_sms, stream);
    case 5: return launch_ub8_decode_v<5>(a, num_sms, stream);
    case 6: return launch_ub8_decode_v<6>(a, num_sms, stream);
    case 7: return launch_ub8_decode_v<7>(a, num_sms, stream);
    case 8: return launch_ub8_decode_v<8>(a, num_sms, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace tcq
