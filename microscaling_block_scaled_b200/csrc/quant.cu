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

// The input viewed as one flat sequence of 32-element blocks: K is a
// multiple of 32, so a block never straddles two rows, and codes and scales
// are row-major and contiguous too (block b's codes start at byte 32 b for
// E4M3 and 16 b for E2M1, its scale is byte b).
//
// Each lane converts the E values of 32 input bytes (8 FP32 or 16 BF16,
// two 16-byte loads); the L = 32 / E lanes of a block reduce its amax with
// shuffles, so a warp tile covers 1 KB of input with contiguous loads and
// stores.  A warp loads U = 4 tiles (128 input bytes per lane) before
// converting any.  The kernel streams from DRAM, but with one value per lane
// it also ran out of issue slots at the power-capped SM clock: the values of
// a lane share one amax reduction and scale, and the E4M3 codes are
// converted in pairs.
constexpr int kQuantThreads = 256;
constexpr int kQuantCtasPerSm = 4;   // 64 registers a thread at most

template <typename T>
struct QuantShape {
    static constexpr int E = 32 / static_cast<int>(sizeof(T));   // values a lane: 8 FP32, 16 BF16
    static constexpr int V = 2;                                  // 16-byte loads a lane and tile
    static constexpr int U = 4;                                  // tiles a warp pass
};

// Two E4M3 codes (RNE, saturating at +-448): `lo` in bits 0..7, `hi` in 8..15.
__device__ __forceinline__ uint32_t cvt_e4m3_pair(float hi, float lo)
{
    uint16_t h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(hi), "f"(lo));
    return h;
}

// The E values of one lane from its 16-byte loads: FP32 as they are, BF16
// bit patterns widened exactly (element 2i in the low half of word i).
template <typename T>
__device__ __forceinline__ void widen(const uint4 (&v)[QuantShape<T>::V], float (&x)[QuantShape<T>::E])
{
#pragma unroll
    for (int w = 0; w < QuantShape<T>::V; ++w) {
        const uint32_t wd[4] = {v[w].x, v[w].y, v[w].z, v[w].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if constexpr (sizeof(T) == 4) {
                x[4 * w + i] = __uint_as_float(wd[i]);
            } else {
                x[8 * w + 2 * i] = __uint_as_float(wd[i] << 16);
                x[8 * w + 2 * i + 1] = __uint_as_float(wd[i] & 0xFFFF0000u);
            }
        }
    }
}

template <int FMT, typename T>
__global__ void __launch_bounds__(kQuantThreads, kQuantCtasPerSm)
    mx_quantize_kernel(const T *__restrict__ X, uint8_t *__restrict__ Q, uint8_t *__restrict__ S, int64_t total)
{
    constexpr int kEmax = FMT == kFmtMXFP8 ? 8 : 2;
    constexpr int E = QuantShape<T>::E, L = 32 / E;
    constexpr int V = QuantShape<T>::V, U = QuantShape<T>::U;
    const int lane = threadIdx.x & 31;
    const int64_t chunks = total / E;                 // lane chunks: a multiple of L
    const int64_t tiles = (chunks + 31) / 32;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t t0 = warp * U; t0 < tiles; t0 += nwarps * U) {   // warp-uniform
        const int64_t c0 = t0 * 32;
        const int rem = chunks - c0 < 32 * U ? static_cast<int>(chunks - c0) : 32 * U;
        const uint4 *src = reinterpret_cast<const uint4 *>(X) + c0 * V;
        uint4 v[U][V];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = u * 32 + lane;
#pragma unroll
            for (int w = 0; w < V; ++w)
                v[u][w] = c < rem ? __ldcs(src + c * V + w) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = u * 32 + lane;
            float x[E];
            widen<T>(v[u], x);
            uint32_t m = 0;
#pragma unroll
            for (int k = 0; k < E; ++k) {
                const uint32_t mag = __float_as_uint(x[k]) & 0x7FFFFFFFu;   // NaN > Inf > finite
                m = mag > m ? mag : m;
            }
#pragma unroll
            for (int off = L / 2; off >= 1; off /= 2) {
                const uint32_t o = __shfl_xor_sync(0xffffffffu, m, off);
                m = o > m ? o : m;
            }
            float inv;
            const uint32_t sbyte = mx_block_scale<kEmax>(m, &inv);
            if (c >= rem)
                continue;
            float q[E];
#pragma unroll
            for (int k = 0; k < E; ++k)
                q[k] = sbyte == 0xFFu ? 0.0f : __fmul_rn(x[k], inv);
            const int64_t gc = c0 + c;
            if (lane % L == 0)
                S[gc / L] = static_cast<uint8_t>(sbyte);
            if constexpr (FMT == kFmtMXFP8) {
                uint32_t w[E / 4];   // 4 codes a word
#pragma unroll
                for (int i = 0; i < E / 4; ++i)
                    w[i] = cvt_e4m3_pair(q[4 * i + 1], q[4 * i]) | (cvt_e4m3_pair(q[4 * i + 3], q[4 * i + 2]) << 16);
                if constexpr (E == 8)
                    *reinterpret_cast<uint2 *>(Q + gc * E) = make_uint2(w[0], w[1]);
                else
                    *reinterpret_cast<uint4 *>(Q + gc * E) = make_uint4(w[0], w[1], w[2], w[3]);
            } else {
                uint32_t w[E / 8];   // 8 codes a word
#pragma unroll
                for (int i = 0; i < E / 8; ++i)
                    w[i] = cvt_e2m1x2(q[8 * i + 1], q[8 * i]) | (cvt_e2m1x2(q[8 * i + 3], q[8 * i + 2]) << 8) |
                           (cvt_e2m1x2(q[8 * i + 5], q[8 * i + 4]) << 16) | (cvt_e2m1x2(q[8 * i + 7], q[8 * i + 6]) << 24);
                if constexpr (E == 8)
                    *reinterpret_cast<uint32_t *>(Q + gc * (E / 2)) = w[0];
                else
                    *reinterpret_cast<uint2 *>(Q + gc * (E / 2)) = make_uint2(w[0], w[1]);
            }
        }
    }
}

}  // namespace

cudaError_t launch_quantize(int fmt, int64_t R, int64_t K, const float *X, uint8_t *Q, uint8_t *S,
                            cudaStream_t stream, const uint16_t *X_bf16)
{
    const int64_t total = R * K;
    if (total == 0)
        return cudaSuccess;
    // lane chunks of 32 input bytes, 32 per warp tile, U tiles per warp and
    // pass; one wave of kQuantCtasPerSm CTAs on each of 148 SMs at most
    const int U = X_bf16 ? QuantShape<uint16_t>::U : QuantShape<float>::U;
    const int64_t chunks = total / (X_bf16 ? QuantShape<uint16_t>::E : QuantShape<float>::E);
    const int64_t per_cta = 32LL * U * (kQuantThreads / 32);
    int64_t grid = (chunks + per_cta - 1) / per_cta;
    if (grid > 148 * kQuantCtasPerSm)
        grid = 148 * kQuantCtasPerSm;
    const unsigned g = static_cast<unsigned>(grid);
    if (X_bf16) {
        if (fmt == kFmtMXFP8)
            mx_quantize_kernel<kFmtMXFP8, uint16_t><<<g, kQuantThreads, 0, stream>>>(X_bf16, Q, S, total);
        else
            mx_quantize_kernel<kFmtMXFP4, uint16_t><<<g, kQuantThreads, 0, stream>>>(X_bf16, Q, S, total);
    } else {
        if (fmt == kFmtMXFP8)
            mx_quantize_kernel<kFmtMXFP8, float><<<g, kQuantThreads, 0, stream>>>(X, Q, S, total);
        else
            mx_quantize_kernel<kFmtMXFP4, float><<<g, kQuantThreads, 0, stream>>>(X, Q, S, total);
    }
    return cudaGetLastError();
}

}  // namespace mxg
