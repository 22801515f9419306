// The bf16-mode master copy of the Newton-Schulz iterate X, as two bf16 parts:
//
//   X = hi + lo,   hi = bf16(X),   lo = bf16(X - hi)      (both round to nearest even)
//
// hi is also the GEMM operand.  X - hi is exact in fp32 (Sterbenz) and at most
// half an ulp of hi, 2^-8 |X|; rounding it to bf16 errs by at most 2^-8 of
// itself, so hi + lo (exact in fp32) is within 2^-16 |X| of X, against 2^-8
// for hi alone.  One element costs 4 bytes, two of them the operand, against
// the 4 + 2 of an fp32 master beside a bf16 operand.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace mfsdp {

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ float master_value(uint16_t hi_bits, uint16_t lo_bits) {
    return bf16_bits_to_float(hi_bits) + bf16_bits_to_float(lo_bits);
}

// Two elements at once, packed as bf16 pairs (element 0 in the low half); each
// element's parts are exactly those of master_split.
__device__ __forceinline__ void master_split2(float x0, float x1, uint32_t& hi_pair, uint32_t& lo_pair) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    hi_pair = *reinterpret_cast<const uint32_t*>(&h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - __uint_as_float(hi_pair << 16),
                                                   x1 - __uint_as_float(hi_pair & 0xFFFF0000u));
    lo_pair = *reinterpret_cast<const uint32_t*>(&l);
}

__device__ __forceinline__ void master_split(float x, uint16_t& hi_bits, uint16_t& lo_bits) {
    hi_bits = __bfloat16_as_ushort(__float2bfloat16_rn(x));
    lo_bits = __bfloat16_as_ushort(__float2bfloat16_rn(x - bf16_bits_to_float(hi_bits)));
}

}  // namespace mfsdp
