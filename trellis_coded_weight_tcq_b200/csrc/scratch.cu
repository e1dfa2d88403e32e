// scratch.cu -- the encoder's backpointer scratch is dead once the traceback has
// read it, yet its last ~100 MB of lines are still dirty in L2 when the encode
// ends, and whatever runs next (the decoder, typically) pays for their write-back
// to HBM.  discard.global.L2 drops a 128-byte line from L2 without writing it
// back; the next encode writes every record before reading it, so nothing reads
// the discarded contents.
#include "common.cuh"

namespace tcq {

namespace {

__global__ void discard_l2_kernel(unsigned char* base, size_t lines)
{
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < lines;
         i += (size_t)gridDim.x * blockDim.x)
        asm volatile("discard.global.L2 [%0], 128;" ::"l"(base + i * 128) : "memory");
}

}  // namespace

cudaError_t launch_discard_l2(void* base, size_t bytes, int num_sms, cudaStream_t stream)
{
    const size_t lines = bytes / 128;  // whole lines only (base is 256-byte aligned)
    if (lines == 0) return cudaSuccess;
    long long grid = (long long)((lines + 255) / 256);
    const long long cap = (long long)(num_sms > 0 ? num_sms : 148) * 8;
    if (grid > cap) grid = cap;
    discard_l2_kernel<<<(int)grid, 256, 0, stream>>>(static_cast<unsigned char*>(base), lines);
    return cudaGetLastError();
}

}  // namespace tcq
