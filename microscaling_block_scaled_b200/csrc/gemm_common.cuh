// gemm_common.cuh -- what the one-CTA kernel (gemm_kernel.cuh) and the
// CTA-pair kernel (gemm_pair_kernel.cuh) share: the kernel parameter block,
// the device error word, BF16 packing, and the host-side tensor-map
// builders.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <cstdlib>

#include "mx_convert.cuh"
#include "mx_internal.h"
#include "sm100_ptx.cuh"

namespace mxg {

struct KParams {
    __nv_bfloat16 *C;
    float *partials;
    uint32_t *counters;
    int *error;
    int64_t P, Q;          // valid rows of the two MMA operands
    int64_t ldc;           // = N
    uint32_t tilesP, kt, iters, workers;   // host guarantees iters * workers < 2^32
    int dp;                // workers == tiles: worker w is exactly tile w
    uint64_t limit_ns;
    int swap;
    int inject;
    int tma_store;         // 1: epilogue stores C through shared memory with TMA
    // Fused scale conversion (1-CTA kernel): the scale producers gather each
    // stage's atoms from the row-major scales [rows][K/32] themselves instead
    // of loading the repacked layout.
    int fused_sf;
    const uint8_t *rawP, *rawQ;   // row-major scales of the row / column operand
    int64_t ldS;                  // K / 32: scale bytes per row
    // Operands that may be read before the prerequisite grid (the previous
    // kernel on the stream, when launched as its programmatic dependent) has
    // completed: bit 0 the row operand (P) with its row-major scales, bit 1
    // the column operand (Q) with its row-major scales.  Repacked scales and
    // C are always accessed after it.
    int early;
    // Fused epilogue: out = act(acc + bias[n]) + residual[m][n] (BF16 bias
    // and residual), then BF16 C, or with qfmt >= 0 the MX codes and E8M0
    // scales of out rounded to BF16 (one scale per 32 consecutive n).
    const uint16_t *bias;
    const uint16_t *residual;
    int act;               // 0 none, 1 ReLU, 2 SiLU, 3 GELU
    int has_ops;           // bias, residual or act present
    int qfmt;              // -1: BF16 C
    uint8_t *Cq, *Cs;
    // Grouped GEMM (non-swapped, whole tiles): group g owns rows
    // [goff[g], goff[g+1]) of the row operand and of C, and rows
    // [g*ldc, g*ldc + ldc) of the column operand.
    const int64_t *goff;
    uint32_t groups;
    uint32_t tilesQ;       // column tiles (grouped: per group), ceil(N / BN)
    uint32_t band;         // CTA-pair plans: tile rows per band of the tile order
    // CTA-pair plans: tiles from tail_first on (the last, partial wave) are
    // split into tail_split K ranges, each its own work unit (1: no split)
    uint32_t tail_first, tail_split;
    // One-CTA plans: > 1 when each tile's K range is split over a cluster of
    // ksplit CTAs (blockIdx.x = tile * ksplit + cluster rank) whose partial
    // accumulators are summed through distributed shared memory by rank 0.
    int ksplit;
};

// Error site codes written to the device error word.
enum : int {
    kErrProducerEmpty = 1,
    kErrMmaFull = 2,
    kErrMmaAccEmpty = 3,
    kErrEpiAccFull = 4,
    kErrDrain = 5,
    kErrLaunch = 6,        // launched with a block size the kernel was not built for
    kErrReduce = 7,        // cluster K split: a partial sum or the leader's go-ahead never came
};

__device__ __forceinline__ void record_error(int *err, int code, volatile int *abort_flag)
{
    atomicCAS(err, 0, code);
    *abort_flag = 1;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b)
{
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// ---------------------------------------------------------- host helpers

namespace {


using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2-D uint8 map over [rows][row_bytes] with a box of 128 bytes x box_rows,
// 128-byte swizzle, zero fill out of bounds.
bool make_operand_map(CUtensorMap *map, const void *base, int64_t rows, int64_t rbytes, int box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(rbytes), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(rbytes)};
    cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 3-D uint8 map viewing [rows][row_bytes] as {128-byte piece, row, chunk}
// (strides: row_bytes between rows, 128 bytes between chunks) with a box of
// 128 bytes x box_rows x kc chunks, 128-byte swizzle, zero fill out of
// bounds.  Needs row_bytes % 128 == 0.
bool make_operand_map_3d(CUtensorMap *map, const void *base, int64_t rows, int64_t rbytes, int box_rows, int kc)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn || rbytes % 128 != 0)
        return false;
    cuuint64_t dims[3] = {128u, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(rbytes / 128)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(rbytes), 128u};
    cuuint32_t box[3] = {128u, static_cast<cuuint32_t>(box_rows), static_cast<cuuint32_t>(kc)};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 3-D uint32 map over a repacked scale buffer [row blocks][ka][512 bytes]:
// {128 words of an atom, atom, 128-row block}, box {128, atoms, row blocks}.
bool make_sf_map(CUtensorMap *map, const uint8_t *base, int64_t ka, int64_t row_blocks, int atoms, int rbs)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    cuuint64_t dims[3] = {128u, static_cast<cuuint64_t>(ka), static_cast<cuuint64_t>(row_blocks)};
    cuuint64_t strides[2] = {512u, static_cast<cuuint64_t>(ka) * 512u};
    cuuint32_t box[3] = {128u, static_cast<cuuint32_t>(atoms), static_cast<cuuint32_t>(rbs)};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint8_t *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

inline int64_t sf_row_blocks(int64_t rows) { return (rows + 255) / 256 * 2; }

// 2-D BF16 map over C [M][N] with a box of box_x (inner, along N) x box_y
// rows, no swizzle; used by the epilogue's TMA stores.
bool make_output_map(CUtensorMap *map, void *C, int64_t M, int64_t N, int box_x, int box_y)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(N) * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(box_x), static_cast<cuuint32_t>(box_y)};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, C, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

}  // namespace mxg
