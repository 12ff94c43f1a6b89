// quant.cu -- OCP MX quantiser on the device (FP32 -> E4M3 / E2M1 codes plus
// one E8M0 scale per 32 elements).  It generates the pre-quantised inputs the
// GEMM is measured on; the devotd.net page (section 2) and the 5ulink.com
// page (support-matrix preamble) state that the MX timings start from
// already-quantised inputs, so this kernel is not on the timed path.
//
// Rule per 32-element block of a row: amax = max |x|; scale exponent
// s = floor(log2 amax) - emax (emax = 8 for E4M3, 2 for E2M1) taken from the
// FP32 exponent bits, clamped to [-127, 127] (s = -127 for an all-zero
// block); each element is x * 2^-s rounded to nearest even and saturated to
// the format's largest finite value by the hardware conversion
// (cvt.rn.satfinite); a block holding NaN or Inf gets scale 0xFF and zero
// codes.
#include <cuda_runtime.h>

#include <cstdint>

#include "mx_internal.h"

namespace mxg {

namespace {

__device__ __forceinline__ uint32_t cvt_e4m3(float x)
{
    uint16_t h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(0.0f), "f"(x));
    return h & 0xFFu;            // second source lands in the low byte
}

// Two E2M1 codes in one byte: `lo` in bits 0..3, `hi` in bits 4..7.
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

template <int FMT>
__global__ void __launch_bounds__(256) mx_quantize_kernel(const float *__restrict__ X, uint8_t *__restrict__ Q,
                                                          uint8_t *__restrict__ S, int64_t R, int64_t K)
{
    constexpr int kEmax = FMT == kFmtMXFP8 ? 8 : 2;
    const int lane = threadIdx.x & 31;
    const int64_t nb = K / 32;
    const int64_t nblocks = R * nb;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x / 32);
    for (int64_t blk = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32; blk < nblocks;
         blk += warps) {
        const int64_t r = blk / nb, j = blk - r * nb;
        const float x = X[r * K + j * 32 + lane];
        const uint32_t mag = __float_as_uint(x) & 0x7FFFFFFFu;
        const uint32_t amax = __reduce_max_sync(0xffffffffu, mag);   // NaN > Inf > finite as integers
        int s;
        uint32_t sbyte;
        const bool nonfinite = amax >= 0x7F800000u;
        if (nonfinite) {
            s = 0;
            sbyte = 0xFFu;
        } else if (amax == 0u) {
            s = -127;
            sbyte = 0u;
        } else {
            s = floor_log2_bits(amax) - kEmax;
            s = s < -127 ? -127 : (s > 127 ? 127 : s);
            sbyte = static_cast<uint32_t>(s + 127);
        }
        // 2^-s is a normal FP32 number: s lies in [-127, 119] for any finite amax.
        const float inv = __uint_as_float(static_cast<uint32_t>(127 - s) << 23);
        const float q = nonfinite ? 0.0f : __fmul_rn(x, inv);
        if (lane == 0)
            S[r * nb + j] = static_cast<uint8_t>(sbyte);
        if (FMT == kFmtMXFP8) {
            Q[r * K + j * 32 + lane] = static_cast<uint8_t>(cvt_e4m3(q));
        } else {
            const float hi = __shfl_down_sync(0xffffffffu, q, 1);
            if ((lane & 1) == 0)
                Q[r * (K / 2) + j * 16 + lane / 2] = static_cast<uint8_t>(cvt_e2m1x2(hi, q));
        }
    }
}

}  // namespace

cudaError_t launch_quantize(int fmt, int64_t R, int64_t K, const float *X, uint8_t *Q, uint8_t *S,
                            cudaStream_t stream)
{
    const int64_t nblocks = R * (K / 32);
    if (nblocks == 0)
        return cudaSuccess;
    const int threads = 256;
    int64_t grid = (nblocks + 7) / 8;
    if (grid > 148 * 64)
        grid = 148 * 64;
    if (fmt == kFmtMXFP8)
        mx_quantize_kernel<kFmtMXFP8><<<static_cast<unsigned>(grid), threads, 0, stream>>>(X, Q, S, R, K);
    else
        mx_quantize_kernel<kFmtMXFP4><<<static_cast<unsigned>(grid), threads, 0, stream>>>(X, Q, S, R, K);
    return cudaGetLastError();
}

}  // namespace mxg
