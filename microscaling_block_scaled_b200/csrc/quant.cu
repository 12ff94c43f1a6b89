// quant.cu -- OCP MX quantiser on the device (FP32 or BF16 -> E4M3 / E2M1
// codes plus one E8M0 scale per 32 elements).  With FP32 input it generates
// the pre-quantised inputs the GEMM is measured on; the devotd.net page
// (section 2) and the 5ulink.com page (support-matrix preamble) state that
// the MX timings start from already-quantised inputs, so that use is not on
// the timed path.  With BF16 input it is the activation quantiser that turns
// a layer's BF16 output into the next layer's MX operand -- the conversion
// copy the devotd.net page (section 4) counts against layouts the kernel
// does not take directly.
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

#include "mx_convert.cuh"
#include "mx_internal.h"

namespace mxg {

namespace {

// Input element as FP32: FP32 as is, BF16 bit patterns widened exactly.
__device__ __forceinline__ float widen(float x) { return x; }
__device__ __forceinline__ float widen(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

// One warp per 32-element block; T = float (FP32 input) or uint16_t (BF16
// bit patterns, widened exactly to FP32 before the rule applies).
template <int FMT, typename T>
__global__ void __launch_bounds__(256) mx_quantize_kernel(const T *__restrict__ X, uint8_t *__restrict__ Q,
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
        const float x = widen(X[r * K + j * 32 + lane]);
        const uint32_t mag = __float_as_uint(x) & 0x7FFFFFFFu;
        const uint32_t amax = __reduce_max_sync(0xffffffffu, mag);   // NaN > Inf > finite as integers
        float inv;
        const uint32_t sbyte = mx_block_scale<kEmax>(amax, &inv);
        const float q = sbyte == 0xFFu ? 0.0f : __fmul_rn(x, inv);
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
                            cudaStream_t stream, const uint16_t *X_bf16)
{
    const int64_t nblocks = R * (K / 32);
    if (nblocks == 0)
        return cudaSuccess;
    const int threads = 256;
    int64_t grid = (nblocks + 7) / 8;
    if (grid > 148 * 64)
        grid = 148 * 64;
    const unsigned g = static_cast<unsigned>(grid);
    if (X_bf16) {
        if (fmt == kFmtMXFP8)
            mx_quantize_kernel<kFmtMXFP8, uint16_t><<<g, threads, 0, stream>>>(X_bf16, Q, S, R, K);
        else
            mx_quantize_kernel<kFmtMXFP4, uint16_t><<<g, threads, 0, stream>>>(X_bf16, Q, S, R, K);
    } else {
        if (fmt == kFmtMXFP8)
            mx_quantize_kernel<kFmtMXFP8, float><<<g, threads, 0, stream>>>(X, Q, S, R, K);
        else
            mx_quantize_kernel<kFmtMXFP4, float><<<g, threads, 0, stream>>>(X, Q, S, R, K);
    }
    return cudaGetLastError();
}

}  // namespace mxg
