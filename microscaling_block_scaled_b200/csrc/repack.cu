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
//
// One 128-thread block moves a 128-row x 32-atom tile: coalesced 128-byte
// row reads into shared memory, then contiguous 16 KB of atoms out.
#include <cuda_runtime.h>

#include <cstdint>

#include "mx_internal.h"

namespace mxg {

namespace {

constexpr int kTileAtoms = 32;              // atoms per block along K (128 bytes of scales per row)

struct RepackOperand {
    const uint8_t *src;
    uint32_t *dst;
    int64_t rows;          // R
    int64_t row_blocks;    // padded 128-row blocks
    int64_t ka;            // atoms per row block (padded)
    int64_t ka_real;       // K / 128
    int64_t src_ld;        // K / 32 bytes per source row
    int64_t chunks;        // ceil(ka / kTileAtoms)
    int64_t blocks;        // row_blocks * chunks
};

__global__ void __launch_bounds__(128) mx_repack_kernel(RepackOperand a, RepackOperand b)
{
    // The scales being rewritten may still be read by a GEMM launched before
    // this kernel; then let the next GEMM start its prologue early.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    __shared__ uint32_t tile[128][kTileAtoms + 1];
    const bool is_a = blockIdx.x < a.blocks;
    const RepackOperand &op = is_a ? a : b;
    const int64_t bid = is_a ? blockIdx.x : blockIdx.x - a.blocks;
    const int64_t rb = bid / op.chunks, chunk = bid - rb * op.chunks;
    const int64_t ka0 = chunk * kTileAtoms;
    const int nka = static_cast<int>((op.ka - ka0) < kTileAtoms ? (op.ka - ka0) : kTileAtoms);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    // rows of the tile: each warp reads 32 rows, one 128-byte row segment per instruction
    for (int r = warp; r < 128; r += 4) {
        const int64_t row = rb * 128 + r;
        const int64_t atom = ka0 + lane;
        uint32_t v = 0u;
        if (lane < nka && row < op.rows && atom < op.ka_real)
            v = *reinterpret_cast<const uint32_t *>(op.src + row * op.src_ld + atom * 4);
        tile[r][lane] = v;
    }
    __syncthreads();
    // out: nka consecutive atoms of 128 words each
    uint32_t *dst = op.dst + (rb * op.ka + ka0) * 128;
    for (int i = threadIdx.x; i < nka * 128; i += 128) {
        const int atom = i / 128, w = i % 128;
        const int r = (w % 4) * 32 + w / 4;
        dst[i] = tile[r][atom];
    }
}

RepackOperand describe(int fmt, const uint8_t *src, uint8_t *dst, int64_t R, int64_t K)
{
    RepackOperand o;
    o.src = src;
    o.dst = reinterpret_cast<uint32_t *>(dst);
    o.rows = R;
    o.row_blocks = (R + 255) / 256 * 2;
    o.ka = sf_atoms_per_rowblock(fmt, K);
    o.ka_real = K / 128;
    o.src_ld = K / 32;
    o.chunks = (o.ka + kTileAtoms - 1) / kTileAtoms;
    o.blocks = o.row_blocks * o.chunks;
    return o;
}

}  // namespace

cudaError_t launch_repack(int fmt, int64_t M, int64_t N, int64_t K, const uint8_t *sa, const uint8_t *sb,
                          uint8_t *sa_out, uint8_t *sb_out, cudaStream_t stream)
{
    RepackOperand a = describe(fmt, sa, sa_out, M, K);
    RepackOperand b = describe(fmt, sb, sb_out, N, K);
    const int64_t grid = a.blocks + b.blocks;
    if (grid > 0x7FFFFFFF)
        return cudaErrorInvalidValue;
    mx_repack_kernel<<<static_cast<unsigned>(grid), 128, 0, stream>>>(a, b);
    return cudaGetLastError();
}

}  // namespace mxg
