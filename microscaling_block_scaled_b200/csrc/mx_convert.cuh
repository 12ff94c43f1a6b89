// mx_convert.cuh -- device helpers of the OCP MX conversion shared by the
// quantiser kernel (quant.cu) and the GEMM's quantised-output epilogue
// (gemm.cu): the block scale exponent from the FP32 bits of the block amax,
// and the hardware round-to-nearest-even conversions with saturation.
#pragma once

#include <cstdint>

namespace mxg {

// One E4M3 code (RNE, saturating at +-448) of an FP32 value.
__device__ __forceinline__ uint32_t cvt_e4m3(float x)
{
    uint16_t h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(0.0f), "f"(x));
    return h & 0xFFu;            // second source lands in the low byte
}

// Two E2M1 codes in one byte (RNE, saturating at +-6): `lo` in bits 0..3,
// `hi` in bits 4..7.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float hi, float lo)
{
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\t.reg .b16 h;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
        "cvt.u16.u8 h, t;\n\t"
        "cvt.u32.u16 %0, h;\n\t}"
        : "=r"(r)
        : "f"(hi), "f"(lo));
    return r & 0xFFu;
}

// floor(log2 v) for a positive finite FP32 value given by its bits.
__device__ __forceinline__ int floor_log2_bits(uint32_t bits)
{
    const int e = static_cast<int>(bits >> 23);
    if (e > 0)
        return e - 127;
    return (31 - __clz(static_cast<int>(bits))) - 149;   // subnormal: m * 2^-149
}

// The block scale of the OCP MX rule from the block's largest magnitude,
// given as FP32 bits with the sign cleared (NaN > Inf > finite as integers).
// Returns the E8M0 byte and sets *inv to 2^-s, the exact factor that maps
// the block onto the element grid (0 for a block holding NaN or Inf, whose
// codes are all zero).
template <int EMAX>
__device__ __forceinline__ uint32_t mx_block_scale(uint32_t amax_bits, float *inv)
{
    if (amax_bits >= 0x7F800000u) {
        *inv = 0.0f;
        return 0xFFu;
    }
    int s;
    if (amax_bits == 0u) {
        s = -127;
    } else {
        s = floor_log2_bits(amax_bits) - EMAX;
        s = s < -127 ? -127 : (s > 127 ? 127 : s);
    }
    // 2^-s is a normal FP32 number: s lies in [-127, 119] for any finite amax.
    *inv = __uint_as_float(static_cast<uint32_t>(127 - s) << 23);
    return static_cast<uint32_t>(s + 127);
}

}  // namespace mxg
