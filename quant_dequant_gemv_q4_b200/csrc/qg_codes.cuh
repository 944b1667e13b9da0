// qg_codes.cuh -- quantized codes as tensor-core A operands (sm_100a).
//
// The K-quant GEMV kernels on the tensor cores multiply unsigned integer codes q (4, 5 or 6 bits)
// by fp16 x.  A mask (one LOP3) leaves each code in the low mantissa bits of an fp16 half, where it
// reads as the subnormal q * 2^-24 (a high nibble left in place reads as q * 2^-20).  The tensor
// core keeps its full fp32 accumulation precision only on normal operands (on subnormal ones its
// sums kept about 12 bits below the largest product, measured), so one packed fp16 multiply by a
// power of two, or by a sub-block scale times a power of two, makes every code a normal fp16 number
// (or zero) before the MMA.  Each product is exact: the result is an integer of at most 11 bits
// times a power of two, so the multiply rounds nothing and no subnormal input is flushed
// (mul.rn.f16x2 without .ftz keeps subnormals).
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

namespace qg {

// two fp16 codes (low / high half of v) times the fp16 pair m, rounded to nearest (exact here)
__device__ __forceinline__ uint32_t f16x2_mul(uint32_t v, uint32_t m)
{
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(v), "r"(m));
    return r;
}

// the fp16 pair (v, v); v must be exact in fp16
__device__ __forceinline__ uint32_t f16x2_dup(float v)
{
    const uint32_t b = __half_as_ushort(__float2half_rn(v));
    return b | (b << 16);
}

constexpr uint32_t kF16x2_2p14 = 0x74007400u;  // (2^14, 2^14): q 2^-24 -> q 2^-10
constexpr uint32_t kF16x2_2p10 = 0x64006400u;  // (2^10, 2^10): q 2^-20 -> q 2^-10

}  // namespace qg
