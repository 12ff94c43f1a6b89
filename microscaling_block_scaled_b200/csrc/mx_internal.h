// mx_internal.h -- declarations shared by the library's translation units
// (not part of the public C ABI, which is include/mxgemm.h).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace mxg {

constexpr int kFmtMXFP8 = 0;
constexpr int kFmtMXFP4 = 1;
constexpr int kFmtBF16 = 2;     // dense BF16 operands, no scales (kind::f16 MMA)

// Bytes of one operand row of K elements.
inline int64_t row_bytes(int fmt, int64_t K) { return fmt == kFmtMXFP8 ? K : (fmt == kFmtMXFP4 ? K / 2 : 2 * K); }

// 512-byte scale atoms per 128-row block per 128-byte K chunk of the
// operands (128 E4M3 elements = 4 scale blocks, or 256 E2M1 elements = 8
// scale blocks; BF16 operands carry none); a pipeline stage holds 1, 2 or 4
// chunks.
inline int atoms_per_stage(int fmt) { return fmt == kFmtMXFP8 ? 1 : (fmt == kFmtMXFP4 ? 2 : 0); }

// Repacked scale layout of one operand with R rows: [ceil(R/256)*2][ka][512]
// (row blocks of 128, padded to an even count so a 256-row tile never reads
// past the end), ka = atoms per 128-row block (K/128 rounded up to whole
// stages).  Inside a
// 512-byte atom the scale of row r (0..127) and block j (0..3) sits at byte
// (r % 32) * 16 + (r / 32) * 4 + j: the layout tcgen05.cp .32x128b.warpx4
// expects for block-scale factors.
inline int64_t sf_atoms_per_rowblock(int fmt, int64_t K)
{
    if (fmt == kFmtBF16)
        return 0;
    const int64_t a = K / 128, s = 4 * atoms_per_stage(fmt);   // room for up to 4 chunks per stage
    return (a + s - 1) / s * s;
}
inline int64_t sf_repacked_bytes(int fmt, int64_t R, int64_t K)
{
    return (R + 255) / 256 * 2 * sf_atoms_per_rowblock(fmt, K) * 512;
}

// Launch the repack of both operands' scales (one kernel launch).
cudaError_t launch_repack(int fmt, int64_t M, int64_t N, int64_t K, const uint8_t *sa, const uint8_t *sb,
                          uint8_t *sa_out, uint8_t *sb_out, cudaStream_t stream);

// Launch the OCP MX quantiser (FP32 input, or BF16 input when X_bf16 is set
// and X is NULL).
cudaError_t launch_quantize(int fmt, int64_t R, int64_t K, const float *X, uint8_t *Q, uint8_t *S,
                            cudaStream_t stream, const uint16_t *X_bf16 = nullptr);

// Scheduling plan of one GEMM.
struct GemmPlan {
    int fmt = 0;
    int swap = 0;          // 1: MMA rows come from B (C^T = B * A^T)
    int bn = 0;            // MMA N (columns of one output tile)
    int kc = 1;            // 128-byte K chunks per pipeline stage
    int pair = 0;          // 1: 256x256 tiles on CTA pairs (tcgen05 cta_group::2)
    int stages = 0;
    int64_t M = 0, N = 0, K = 0;
    int64_t P = 0, Q = 0;  // rows of the MMA's row operand / column operand
    int64_t tilesP = 0, tilesQ = 0, kt = 0, tiles = 0, iters = 0;
    int64_t workers = 0;
    int grid = 0;
    int sched = 0;         // resolved schedule (MXGEMM_SCHED_*)
    int64_t kaP = 0, kaQ = 0;
    int64_t partial_bytes = 0;  // workspace for split partials
    bool valid = true;          // false: the shape exceeds the kernel's 32-bit scheduler range
    int64_t counter_bytes = 0;
    int64_t groups = 0;         // > 0: grouped plan (make_grouped_plan)
    int64_t band = 0;           // CTA-pair plans: tile rows per band of the tile order
    int64_t ksplit = 1;         // one-CTA plans: CTAs of a cluster sharing one tile's K range (0: all)
    // CTA-pair plans: the tiles from tail_first on (the last, partial wave)
    // are each split into tail_split K ranges (1: whole tiles only)
    int64_t tail_first = 0, tail_split = 1;
};

// Build the plan for a shape.  sched/splits/workers as mxgemm_set_schedule.
// allow_pair = false keeps the plan on one-CTA tiles (the paths whose
// epilogue or tile walk only the one-CTA kernel implements).
GemmPlan make_plan(int fmt, int64_t M, int64_t N, int64_t K, int num_sms, int sched, int splits,
                   int workers, int force_kc = 0, bool allow_pair = true);

// Plan of a grouped GEMM: G groups sharing N and K, group g owning rows
// [off[g], off[g+1]) of A and C (M_total rows in all) and rows [g*N, g*N+N)
// of B.  Whole 128 x 128 tiles, never swapped; W is an upper bound on the
// number of tiles ((ceil(M_total/128) + G) * ceil(N/128)), the kernel skips
// what the group sizes leave empty.
GemmPlan make_grouped_plan(int fmt, int64_t G, int64_t M_total, int64_t N, int64_t K, int num_sms);

// Fused epilogue of the one-CTA kernel: out = act(acc + bias[n]) +
// residual[m][n], then either BF16 C or the next layer's MX operand (codes
// plus E8M0 scales, one per 32 consecutive n of a row).
struct Epilogue {
    const uint16_t *bias = nullptr;       // BF16 [N] or NULL
    const uint16_t *residual = nullptr;   // BF16 [M][N] or NULL
    int act = 0;                          // 0 none, 1 ReLU, 2 SiLU, 3 GELU (erf form)
    int qfmt = -1;                        // -1 BF16 C; kFmtMXFP8 / kFmtMXFP4 quantised output
    uint8_t *Cq = nullptr;                // codes [M][row_bytes(qfmt, N)]
    uint8_t *Cs = nullptr;                // E8M0 scales [M][N/32]
};

// Launch the GEMM kernel for `plan`.
struct GemmBuffers {
    const void *A, *B;
    const uint8_t *sfA, *sfB;   // repacked scales of A and of B
    // row-major scales of A and B: when set (1-CTA plans only), the GEMM
    // converts them itself and sfA / sfB are not read
    const uint8_t *rawA = nullptr, *rawB = nullptr;
    void *C;
    float *partials;
    uint32_t *counters;
    int *error;
    // With pdl: operands that may be read before the preceding kernel has
    // completed (bit 0 A, bit 1 B, each with its row-major scales).  Only
    // safe where that kernel does not write them: the scale repack, or a
    // caller's promise that B is constant.
    int early = 0;
    Epilogue epi;
    const int64_t *group_offsets = nullptr;   // grouped plans: device [G+1]
};
// pdl: launch as a programmatic dependent of the preceding kernel, letting
// the prologue (and the operands named in buf.early) overlap its tail; every
// other global access waits for it to complete.
cudaError_t launch_gemm(const GemmPlan &plan, const GemmBuffers &buf, uint64_t wait_limit_ns, int inject, int pdl,
                        cudaStream_t stream);

// Per-(fmt, BN) kernel attribute setup; returns cudaSuccess once done.
cudaError_t prepare_gemm_kernels();

// The kernel instantiations, one translation unit per operand type
// (gemm_mxfp8.cu, gemm_mxfp4.cu, gemm_bf16.cu: one-CTA kernel;
// gemm_pair.cu: CTA-pair kernel): ring depth of a configuration, launch,
// and shared-memory attribute setup.
int stages_mxfp8(int bn, int kc);
int stages_mxfp4(int bn, int kc);
int stages_bf16(int bn, int kc);
int stages_pair(int fmt, int kc);
cudaError_t launch_gemm_mxfp8(const GemmPlan &pl, const GemmBuffers &b, uint64_t limit_ns, int inject, int pdl,
                              cudaStream_t st);
cudaError_t launch_gemm_mxfp4(const GemmPlan &pl, const GemmBuffers &b, uint64_t limit_ns, int inject, int pdl,
                              cudaStream_t st);
cudaError_t launch_gemm_bf16(const GemmPlan &pl, const GemmBuffers &b, uint64_t limit_ns, int inject, int pdl,
                             cudaStream_t st);
cudaError_t launch_gemm_pair(const GemmPlan &pl, const GemmBuffers &b, uint64_t limit_ns, int inject, int pdl,
                             cudaStream_t st);
cudaError_t prepare_mxfp8();
cudaError_t prepare_mxfp4();
cudaError_t prepare_bf16();
cudaError_t prepare_pair();

}  // namespace mxg
