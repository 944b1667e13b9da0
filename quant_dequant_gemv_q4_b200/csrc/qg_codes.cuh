// qg_codes.cuh -- quantized codes as tensor-core A operands (sm_100a).
//
// The K-quant GEMV kernels on the tensor cores multiply unsigned integer codes q (4, 5 or 6 bits)
// by fp16 x.  The codes enter the MMA as fp16 numbers equal to q: exact, normal (or zero), and no
// larger than the code itself, so every product is exact and the tensor core's fp32 sums keep
// their full precision.  Two instructions per register of two codes: one LOP3 masks the codes of
// two bytes under the exponent of 1024 (the fp16 pair 1024 + s*q), and one packed fp16 FMA takes
// the offset back out.
#pragma once

#include <cstdint>

namespace qg {

// A-operand codes.  v holds two fp16 numbers 1024 + s*q (the exponent of 1024 OR-ed over codes q
// in the mantissa, s = 1 or 16); one f16x2 FMA returns the fp16 integers q exactly:
// (1024 + s q) * (1/s) - 1024/s, every term and the result exact in fp16.
__device__ __forceinline__ uint32_t f16x2_code(uint32_t v)  // s = 1
{
    uint32_t r;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(v), "r"(0x3C003C00u), "r"(0xE400E400u));
    return r;
}
__device__ __forceinline__ uint32_t f16x2_code16(uint32_t v)  // s = 16
{
    uint32_t r;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(v), "r"(0x2C002C00u), "r"(0xD400D400u));
    return r;
}
constexpr uint32_t kE1024 = 0x64006400u;  // the fp16 pair (1024, 1024)

}  // namespace qg
