// acs_grouped.cu -- the specialised encoder instantiations and their lookup.
//
// Each configuration is chosen so that a thread's codewords fit in registers
// next to its working set, and the ping-pong path metrics fit in shared memory:
//   L=16 k=2: 512 threads x 8 groups x 16 states, codewords as fp16 pairs
//             (64 registers), 128 KiB of metrics, one CTA per SM;
//   L=16 k=3: 512 threads x 2 groups x 64 states, fp16 pairs, 64 KiB of metrics;
//   L=12 k=2: 4 teams of 64 threads x 4 groups x 16 states, fp32, two CTAs per SM;
//   L=8  k=2: 8 teams of 16 threads, one block per team, fp32 (CTAs of one
//             warp with 2 teams measured the same on 256 blocks: 38.9 vs 38.0 us).
// The fp16-pair kernels need a binary16 codebook (the widening is exact); the
// fp32 kernels accept either dtype.
#include "acs_grouped.cuh"

namespace tcq {

using CfgL16K2 = GCfg<16, 2, 512, 8, 1, true>;
using CfgL16K3 = GCfg<16, 3, 512, 2, 1, true>;
using CfgL12K2 = GCfg<12, 2, 64, 4, 4, false>;
using CfgL8K2 = GCfg<8, 2, 16, 1, 8, false>;

const EncodeKernelInfo* find_grouped_kernel(int L, int K, int cb_f16)
{
    if (L == 16 && K == 2 && cb_f16) return grouped_info<CfgL16K2>("grouped<16,2,f16x2,512x8>");
    if (L == 16 && K == 3 && cb_f16) return grouped_info<CfgL16K3>("grouped<16,3,f16x2,512x2>");
    if (L == 12 && K == 2) return grouped_info<CfgL12K2>("grouped<12,2,f32,64x4x4>");
    if (L == 8 && K == 2) return grouped_info<CfgL8K2>("grouped<8,2,f32,16x1x8>");
    return nullptr;
}

}  // namespace tcq
