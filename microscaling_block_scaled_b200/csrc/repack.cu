// repack.cu -- scale-layout repack: canonical row-major E8M0 scales
// [R][K/32] -> the tensor-core scale layout the GEMM streams per stage.
//
// The devotd.net page (section 4) notes that low-precision inputs whose
// layout does not match what the kernel needs get an extra conversion copy;
// this is that copy for the scales, launched by mxgemm_run before the GEMM
// and timed on its own.
//
// Output of one operand: [ceil(R/256)*2][ka][512 bytes], row blocks of 128
// rows, ka scale atoms per row block (K/128 rounded up to whole pipeline
// stages).  A 512-byte atom holds the 4 scales (K blocks 4a..4a+3) of each of
// its 128 rows; the 4 bytes of row r sit at byte offset (r%32)*16 + (r/32)*4,
// ascending K block in ascending byte.  Rows past R and atoms past K/128 are
// zero (scale 2^-127, multiplied only by zero elements).
#include <cuda_runtime.h>

#include <cstdint>

#include "mx_internal.h"

namespace mxg {

namespace {

struct RepackOperand {
    const uint8_t *src;
    uint32_t *dst;
    int64_t rows;          // R
    int64_t words;         // output 32-bit words
    int64_t ka;            // atoms per row block (padded)
    int64_t ka_real;       // K / 128
    int64_t src_ld;        // K / 32 bytes per source row
};

__global__ void __launch_bounds__(256) mx_repack_kernel(RepackOperand a, RepackOperand b)
{
    const int64_t total = a.words + b.words;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
         t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const bool is_a = t < a.words;
        const RepackOperand &op = is_a ? a : b;
        const int64_t wi = is_a ? t : t - a.words;
        const int64_t atom = wi / 128;              // (row block, k atom) pair
        const int i = static_cast<int>(wi % 128);    // word inside the atom
        const int64_t rb = atom / op.ka, ka = atom - rb * op.ka;
        const int64_t r = rb * 128 + (i % 4) * 32 + i / 4;
        uint32_t v = 0u;
        if (r < op.rows && ka < op.ka_real)
            v = *reinterpret_cast<const uint32_t *>(op.src + r * op.src_ld + ka * 4);
        op.dst[wi] = v;
    }
}

RepackOperand describe(int fmt, const uint8_t *src, uint8_t *dst, int64_t R, int64_t K)
{
    RepackOperand o;
    o.src = src;
    o.dst = reinterpret_cast<uint32_t *>(dst);
    o.rows = R;
    o.ka = sf_atoms_per_rowblock(fmt, K);
    o.ka_real = K / 128;
    o.words = sf_repacked_bytes(fmt, R, K) / 4;
    o.src_ld = K / 32;
    return o;
}

}  // namespace

cudaError_t launch_repack(int fmt, int64_t M, int64_t N, int64_t K, const uint8_t *sa, const uint8_t *sb,
                          uint8_t *sa_out, uint8_t *sb_out, cudaStream_t stream)
{
    RepackOperand a = describe(fmt, sa, sa_out, M, K);
    RepackOperand b = describe(fmt, sb, sb_out, N, K);
    const int64_t total = a.words + b.words;
    int64_t grid = (total + 255) / 256;
    if (grid > 148 * 16)
        grid = 148 * 16;
    mx_repack_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(a, b);
    return cudaGetLastError();
}

}  // namespace mxg
