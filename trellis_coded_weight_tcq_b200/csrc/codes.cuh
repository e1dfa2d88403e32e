// codes.cuh -- the computed (lookup-free) trellis code.
//
// QTIP (abstract) introduces codes for the bitshift trellis that range from
// lookup-only tables to codewords computed from the state; it gives no formula.
// This library's computed code: a multiplicative hash of the state, whose high
// half is a well-mixed function of every state bit, and the sum of that half's
// two bytes, centred and scaled by 2^-7 so that every codeword is exact in
// binary16 and fp32:
//     v = 0x9E3779B1 s mod 2^32,   c[s] = (v_2 + v_3 - 255) / 128.
// One multiply and one byte dot product give n = v_2 + v_3; n << 13 added to
// the bits of 1.0f gives 1 + n / 1024 exactly, with no integer-to-float
// conversion.
#pragma once

#include "common.cuh"

namespace tcq {

constexpr uint32_t kMadA = 0x9E3779B1u;
constexpr int kMadCodebook = 2;  // cb_f16 value that selects the computed code

// v_2 + v_3 in [0, 510]
__device__ __forceinline__ uint32_t mad_sum(uint32_t s)
{
    return __dp4a(s * kMadA, 0x01010000u, 0u);
}

// 1 + n / 1024 for n = mad_sum(s): the codeword is 8 (f - 1) - 255 / 128
__device__ __forceinline__ float mad_unit(uint32_t s)
{
    return __uint_as_float(0x3F800000u + (mad_sum(s) << 13));
}

// the codeword itself, exact
__device__ __forceinline__ float mad_codeword(uint32_t s)
{
    return (__uint_as_float(0x4B000000u | mad_sum(s)) - 8388863.0f) * 0.0078125f;  // (n - 255) / 128
}

// Writes the 2^L codewords as binary16 (exact) to table.
cudaError_t launch_mad_table(int L, void* table, cudaStream_t stream);

}  // namespace tcq
