// codes.cu -- materialises the computed code as a binary16 table, for the
// kernels that keep codewords in registers or shared memory (the encoders and
// the soft quantizer).
#include "codes.cuh"

namespace tcq {

namespace {

__global__ void mad_table_kernel(int L, __half* table)
{
    const uint32_t n = 1u << L;
    for (uint32_t s = blockIdx.x * blockDim.x + threadIdx.x; s < n; s += gridDim.x * blockDim.x)
        table[s] = __float2half_rn(mad_codeword(s));
}

}  // namespace

cudaError_t launch_mad_table(int L, void* table, cudaStream_t stream)
{
    const int threads = 256;
    int blocks = (int)(((1u << L) + threads - 1) / threads);
    if (blocks > 1024) blocks = 1024;
    mad_table_kernel<<<blocks, threads, 0, stream>>>(L, static_cast<__half*>(table));
    return cudaGetLastError();
}

}  // namespace tcq
