/*
 * mxgemm.h -- C ABI of the B200 (sm_100a) MX block-scaled matrix multiply.
 *
 * Operation (all entry points below serve it):
 *
 *     C[m][n] = sum_k  dec(A[m][k]) * 2^(SA[m][k/32]-127)
 *                    * dec(B[n][k]) * 2^(SB[n][k/32]-127)
 *
 * accumulated in FP32 and stored as BF16.  This is the "MXFP scaled GEMM" of
 * the 5ulink.com page "PyTorch 接上 FlyDSL" (support-matrix table: A
 * row-major, B column-major i.e. NT, K a multiple of 128; note under the
 * table: one E8M0 scale per 32 values "BlockWise1x32", FP32 accumulation,
 * FP16/BF16 output -- this library writes BF16).  The devotd.net page, section
 * 2, reports the MXFP8 and MXFP4 NT suites this operation is measured on.
 *
 * Formats (OCP Microscaling v1.0 encodings; the pages only name them):
 *   MXGEMM_FMT_MXFP8: elements FP8 E4M3 (max 448, S.1111.111 = NaN), one byte
 *                     each; a row of K elements is K bytes.
 *   MXGEMM_FMT_MXFP4: elements FP4 E2M1, two per byte, element 2j in the low
 *                     nibble of byte j; a row of K elements is K/2 bytes.
 *   scales:           E8M0 bytes, value 2^(e-127), 0xFF = NaN, one per 32
 *                     consecutive K elements.
 *
 * Canonical layouts (caller-owned, dense, row-major, device memory unless an
 * entry point says "host"):
 *   A        [M][row_bytes(K)]   row_bytes = K (MXFP8) or K/2 (MXFP4)
 *   A_scales [M][K/32]           uint8
 *   B        [N][row_bytes(K)]   (B stored as N rows of K: "column-major K x N")
 *   B_scales [N][K/32]           uint8
 *   C        [M][N]              bfloat16 bits (uint16)
 *
 * Requirements checked before any launch: K > 0 and K % 128 == 0; M, N >= 1;
 * every pointer non-NULL and 16-byte aligned; fmt one of the two formats.
 * Violations return an error status and launch nothing.  The calls are
 * stream-ordered and do not synchronise the host unless stated.  A handle is
 * not thread-safe: use one handle per host thread / stream.
 */
#ifndef MXGEMM_H
#define MXGEMM_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MXGEMM_API __attribute__((visibility("default")))
#else
#define MXGEMM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct mxgemm_ctx *mxgemm_handle;

/* Element formats.  MXGEMM_FMT_BF16 (dense BF16 operands, no scales) is
 * taken only where an entry point says so. */
enum {
    MXGEMM_FMT_MXFP8_E4M3 = 0,
    MXGEMM_FMT_MXFP4_E2M1 = 1,
    MXGEMM_FMT_BF16 = 2
};

/* Activations of the fused epilogue (mxgemm_run_fused / _quantized). */
enum {
    MXGEMM_ACT_NONE = 0,
    MXGEMM_ACT_RELU = 1,       /* x < 0 ? 0 : x                                  */
    MXGEMM_ACT_SILU = 2,       /* x * sigmoid(x) = x / (1 + e^-x)                */
    MXGEMM_ACT_GELU = 3        /* x * Phi(x), Phi the standard normal CDF (erf form) */
};

/* Status codes.  Every entry point returns one of these. */
enum {
    MXGEMM_OK = 0,
    MXGEMM_ERR_INVALID_ARG = 1,        /* bad size, format, NULL pointer or handle */
    MXGEMM_ERR_ALIGNMENT = 2,          /* a pointer is not 16-byte aligned */
    MXGEMM_ERR_UNSUPPORTED_DEVICE = 3, /* current device is not compute capability 10.0 */
    MXGEMM_ERR_OOM = 4,                /* workspace allocation failed */
    MXGEMM_ERR_CUDA = 5,               /* a CUDA runtime/driver call failed */
    MXGEMM_ERR_TIMEOUT = 6,            /* a kernel gave up on a bounded wait */
    MXGEMM_ERR_TOO_LARGE = 7,          /* exceeds mxgemm_run_noalloc's fixed scratch */
    MXGEMM_ERR_CAPTURE = 8             /* the workspace would have to grow during stream capture */
};

/* Schedules for the GEMM's persistent tile scheduler (mxgemm_set_schedule). */
enum {
    MXGEMM_SCHED_AUTO = 0,     /* pick per shape (default) */
    MXGEMM_SCHED_DP = 1,       /* one whole output tile per work unit */
    MXGEMM_SCHED_SPLITK = 2,   /* each tile split into `splits` equal K ranges */
    MXGEMM_SCHED_STREAMK = 3,  /* K iterations of all tiles split evenly over the SMs */
    MXGEMM_SCHED_KSPLIT = 4    /* decode tiles: each tile's K range split over a cluster of
                                  `splits` (2 or 4) CTAs, summed in distributed shared memory */
};

/* Create a handle bound to the current CUDA device.  The device must be an
 * sm_100 part (B200).  The handle owns a lazily grown device workspace
 * (repacked scales, split-K partials and tile counters).
 * out: receives the handle (host pointer, not NULL).
 *
 * Workspace and CUDA graphs: the first run of a shape that needs more
 * workspace than the handle holds grows it with cudaFree + cudaMalloc, which
 * synchronises the device and cannot be recorded by a stream capture.  Run
 * each shape once (or call mxgemm_reserve for it) before capturing; a run
 * that would have to grow the workspace while its stream is capturing
 * returns MXGEMM_ERR_CAPTURE and launches nothing. */
MXGEMM_API int mxgemm_create(mxgemm_handle *out);

/* Free the handle and its workspace (synchronises the device first).
 * NULL is accepted and ignored. */
MXGEMM_API int mxgemm_destroy(mxgemm_handle h);

/* Full hot path on `stream`: convert A_scales and B_scales from the
 * canonical row-major layout into the tensor-core scale layout and run the
 * block-scaled GEMM writing C.  Where the plan allows (see
 * mxgemm_describe_plan, "scales=fused") the GEMM gathers the scales itself:
 * one kernel launch.  Otherwise the scales are repacked into the handle's
 * workspace first: two launches.  No host synchronisation.  All buffers are
 * device memory.  `stream` is a cudaStream_t (NULL = legacy default stream).
 * The GEMM launches as a programmatic dependent of the work before it on
 * `stream`: when that is a GEMM of this library, the new GEMM's CTAs set up
 * while it finishes, and read or write no buffer before it has completed
 * (except B under mxgemm_set_prefetch_b). */
MXGEMM_API int mxgemm_run(mxgemm_handle h, int fmt, int64_t M, int64_t N, int64_t K,
               const void *A, const uint8_t *A_scales,
               const void *B, const uint8_t *B_scales,
               void *C, void *stream);

/* Grow the handle's workspace now to what mxgemm_run needs for this shape
 * under the handle's current schedule settings (an addition; the pages have
 * no counterpart), so that later runs of this shape or smaller ones allocate
 * nothing and can be captured into a CUDA graph.  Synchronises the device
 * when it allocates.  Returns MXGEMM_ERR_OOM when the allocation fails. */
MXGEMM_API int mxgemm_reserve(mxgemm_handle h, int fmt, int64_t M, int64_t N, int64_t K);

/* GEMM epilogue fusion (the roadmap item "GEMM 尾部融合", GEMM epilogue
 * fusion, at the end of section 怎么用起来 of the 5ulink.com page; an
 * addition to the operation above): mxgemm_run's product followed, in the
 * kernel's epilogue and before the one rounding to BF16, by
 *
 *     C[m][n] = bf16( act( acc[m][n] + bias[n] ) + residual[m][n] )
 *
 * with each step in FP32.  bias: BF16 [N] or NULL (no bias).  residual: BF16
 * [M][N] or NULL; it may be the same buffer as C (each element is read
 * before it is written, by the same thread).  act: MXGEMM_ACT_*.  Same
 * operands, layouts, requirements and stream semantics as mxgemm_run; non-
 * NULL bias / residual must be 16-byte aligned.  Runs on one-CTA tiles for
 * every shape (the CTA-pair kernel has no fused epilogue). */
MXGEMM_API int mxgemm_run_fused(mxgemm_handle h, int fmt, int64_t M, int64_t N, int64_t K,
                     const void *A, const uint8_t *A_scales, const void *B, const uint8_t *B_scales,
                     const void *bias, int act, const void *residual, void *C, void *stream);

/* Quantised output (the next layer's MX operand written by the GEMM's
 * epilogue instead of a BF16 C, saving the conversion copy the devotd.net
 * page, section 4, counts against layouts the kernel does not take; an
 * addition): the fused-epilogue result of mxgemm_run_fused, rounded to BF16,
 * then MX-quantised by the rule of mxgemm_quantize along n -- one E8M0 scale
 * per 32 consecutive values of a row of C, as the 5ulink.com support-matrix
 * note fixes for MX operands (BlockWise1x32).  out_fmt: MXGEMM_FMT_MXFP8_E4M3
 * or MXGEMM_FMT_MXFP4_E2M1.  C_codes: [M][row_bytes(N)] device; C_scales:
 * [M][N/32] device.  N % 32 == 0.  bias / residual / act as mxgemm_run_fused
 * (NULL, NULL, MXGEMM_ACT_NONE for the plain product). */
MXGEMM_API int mxgemm_run_quantized(mxgemm_handle h, int fmt, int64_t M, int64_t N, int64_t K,
                         const void *A, const uint8_t *A_scales, const void *B, const uint8_t *B_scales,
                         const void *bias, int act, const void *residual, int out_fmt,
                         void *C_codes, uint8_t *C_scales, void *stream);

/* Dense BF16 NT GEMM on the same kernel and scheduler (the comparison suite
 * "BF16 稠密 GEMM" of the 内核级成绩 table of the 5ulink.com page, which
 * calls out 64x4096x4096; the support-matrix row "稠密 GEMM" takes FP16 and
 * BF16 -- this entry point takes BF16, NT only):
 *
 *     C[m][n] = bf16( sum_k A[m][k] * B[n][k] ),  FP32 accumulation
 *
 * A: BF16 [M][K], B: BF16 [N][K], C: BF16 [M][N], all device, dense
 * row-major.  K % 8 == 0 (16-byte rows), M, N >= 1, pointers 16-byte
 * aligned.  No scales, no repack: one launch.  Stream semantics as
 * mxgemm_run (programmatic dependent of the work before it). */
MXGEMM_API int mxgemm_run_bf16(mxgemm_handle h, int64_t M, int64_t N, int64_t K,
                    const void *A, const void *B, void *C, void *stream);

/* Grouped GEMM (the 5ulink.com page: support-matrix row "Grouped GEMM" --
 * A rows of uneven length per group, empty groups skipped; the Grouped GEMM
 * row of the 内核级成绩 table; "MXFP8 Grouped GEMM" on the roadmap at the
 * end of 怎么用起来).  G groups share N and K; group g owns rows
 * [off[g], off[g+1]) of A and of C and its own B_g:
 *
 *     C[m][n] = sum_k A[m][k] * B[g][n][k]     for off[g] <= m < off[g+1]
 *
 * with MX scales as mxgemm_run (fmt MXGEMM_FMT_MXFP8_E4M3 / _MXFP4_E2M1) or
 * dense BF16 operands (fmt MXGEMM_FMT_BF16; scale pointers ignored, may be
 * NULL).  group_offsets: int64 [G+1] in DEVICE memory (a router's output
 * need not come back to the host), off[0] = 0, non-decreasing, off[G] =
 * M_total; offsets outside [0, M_total] are clamped, and a group whose end
 * lies before its start is empty (results for such offsets are unspecified,
 * but no access leaves the buffers).  A: [M_total][row_bytes(K)], A_scales:
 * [M_total][K/32], B: [G][N][row_bytes(K)], B_scales: [G][N][K/32], C: BF16
 * [M_total][N].  One launch; a persistent grid walks the groups' 128x128
 * tiles in order.  1 <= G <= 65536, G * N <= 2^24, M_total >= 0 (0: no
 * launch). */
MXGEMM_API int mxgemm_run_grouped(mxgemm_handle h, int fmt, int64_t G, int64_t M_total, int64_t N, int64_t K,
                       const int64_t *group_offsets, const void *A, const uint8_t *A_scales,
                       const void *B, const uint8_t *B_scales, void *C, void *stream);

/* The plan text of mxgemm_run_grouped for a device with num_sms SMs, without
 * a handle or a GPU (as mxgemm_describe_plan_for); `tiles` there is the
 * upper bound the launch is sized for. */
MXGEMM_API int mxgemm_describe_grouped_plan(int num_sms, int fmt, int64_t G, int64_t M_total, int64_t N,
                                 int64_t K, char *buf, size_t cap);

/* The first half of mxgemm_run on its own: the scale repack into the
 * handle's workspace.  Sizes as for mxgemm_run. */
MXGEMM_API int mxgemm_repack(mxgemm_handle h, int fmt, int64_t M, int64_t N, int64_t K,
                  const uint8_t *A_scales, const uint8_t *B_scales, void *stream);

/* The second half of mxgemm_run on its own: the GEMM, reading the scales the
 * last mxgemm_repack on this handle (same fmt, M, N, K) left in the
 * workspace.  Returns MXGEMM_ERR_INVALID_ARG if the shape differs from the
 * last repack. */
MXGEMM_API int mxgemm_gemm(mxgemm_handle h, int fmt, int64_t M, int64_t N, int64_t K,
                const void *A, const void *B, void *C, void *stream);

/* mxgemm_run with HOST buffers (pinned or pageable): copies the operands and
 * scales to device staging buffers owned by the handle, runs the hot path and
 * copies C back to the host buffer C_host, after the work already queued on
 * `stream`, then synchronises the stream.  Host buffers use the canonical
 * layouts above.  A product with 32 MB or more of copies runs in blocks of C
 * (an addition; the pages have no counterpart): row bands of A and of B go
 * up on a copy stream of the handle, each block's GEMM runs on `stream` once
 * its two bands have landed, and the block goes down on a second copy stream
 * of the handle while later bands still go up.  Blocks are multiples of 256
 * rows and columns with at most 4 parts of M and of N, each at least 2^22
 * elements.  With profiling on, or while `stream` is capturing, the product
 * runs as one block.  On return (success or error) no copy of this call is
 * still in flight. */
MXGEMM_API int mxgemm_run_host(mxgemm_handle h, int fmt, int64_t M, int64_t N, int64_t K,
                    const void *A_host, const uint8_t *A_scales_host,
                    const void *B_host, const uint8_t *B_scales_host,
                    void *C_host, void *stream);

/* Profiling switch (an addition; the pages have no counterpart): with `on`
 * = 1, mxgemm_run and mxgemm_run_host record CUDA events on their stream
 * before the scale repack, between repack and GEMM, and after the GEMM.  The
 * middle event keeps the GEMM from overlapping the repack, so profiled runs
 * are slightly slower than unprofiled ones.  `on` = 0 turns it off.  Returns
 * MXGEMM_ERR_INVALID_ARG for a NULL handle or another value of `on`. */
MXGEMM_API int mxgemm_set_profiling(mxgemm_handle h, int on);

/* Device times of the last profiled mxgemm_run / mxgemm_run_host on this
 * handle: *repack_ms for the scale repack, *gemm_ms for the GEMM.  Waits for
 * that run to finish.  MXGEMM_ERR_INVALID_ARG when profiling was off for the
 * last run, or for NULL arguments. */
MXGEMM_API int mxgemm_last_timing(mxgemm_handle h, float *repack_ms, float *gemm_ms);

/* Prefetch-B promise (an addition; the pages have no counterpart): with
 * `on` = 1 the caller promises that B and B_scales of every later
 * mxgemm_run on this handle are not written by the work queued before that
 * call on its stream, as for the constant weights of a decode layer.  A
 * one-launch mxgemm_run may then stream B into its pipeline while a
 * preceding GEMM of this library still runs; A, A_scales and C still wait
 * for it.  Results are unchanged; breaking the promise gives undefined
 * results.  `on` = 0 (the default) withdraws it.  Returns
 * MXGEMM_ERR_INVALID_ARG for a NULL handle or another value of `on`. */
MXGEMM_API int mxgemm_set_prefetch_b(mxgemm_handle h, int on);

/* OCP MX quantisation (the input generator; not part of the timed path).
 * X: FP32 [R][K] device.  Q: codes [R][row_bytes(K)] device.  scales: E8M0
 * [R][K/32] device.  Per 32-element block: amax = max|x|, scale exponent
 * s = floor(log2 amax) - emax (emax 8 for E4M3, 2 for E2M1) clamped to
 * [-127, 127] (all-zero block: s = -127), elements x / 2^s rounded to nearest
 * even with saturation at +-448 / +-6, the sign of a zero kept.  A block that
 * holds a NaN or an infinity gets scale 0xFF and zero codes.  K % 32 == 0. */
MXGEMM_API int mxgemm_quantize(int fmt, int64_t R, int64_t K, const float *X,
                    void *Q, uint8_t *scales, void *stream);

/* The same quantisation of BF16 input (bit patterns [R][K], device): each
 * value widens exactly to FP32, then the rule above applies.  This is the
 * activation quantiser that turns a layer's BF16 output into the next
 * layer's MX operand -- the conversion copy of the devotd.net page, section
 * 4 -- as a stand-alone op (an addition). */
MXGEMM_API int mxgemm_quantize_bf16(int fmt, int64_t R, int64_t K, const void *X,
                         void *Q, uint8_t *scales, void *stream);

/* Force a schedule for later mxgemm_run / mxgemm_gemm calls on this handle.
 * splits is used by MXGEMM_SCHED_SPLITK (>= 1) and MXGEMM_SCHED_KSPLIT
 * (2 or 4; 3 takes 2; shapes that are not decode tiles, or whose clusters
 * would not all fit on the GPU at once, take MXGEMM_SCHED_SPLITK instead);
 * workers by MXGEMM_SCHED_STREAMK (0 = number of SMs). */
MXGEMM_API int mxgemm_set_schedule(mxgemm_handle h, int schedule, int splits, int workers);

/* Force the number of 128-byte K chunks each pipeline stage of later GEMMs
 * on this handle loads: 1, 2 or 4 (2 and 4 apply only when an operand row is
 * a whole number of 128-byte chunks; 4 only to tiles of at most 64 columns),
 * 0 = automatic (the default). */
MXGEMM_API int mxgemm_set_kchunks(mxgemm_handle h, int kc);

/* Describe the plan mxgemm_gemm would use for a shape: writes up to `cap`
 * bytes of a NUL-terminated text such as
 * "fmt=1 swap=1 pair=0 BN=32 kc=2 stages=5 tiles=112 kt=8 workers=112
 * grid=112 sched=dp partial_bytes=0 scales=fused".  "scales" says how
 * mxgemm_run treats the scales for this shape: "fused" (the GEMM converts
 * the row-major scales itself, one launch) or "repack" (scale repack, then
 * the GEMM).  sched is dp (whole tiles), splitk, streamk, ksplit (the K
 * range of each tile split over a cluster of `ksplit` CTAs, field appended),
 * or for CTA-pair plans dptail: whole tiles, except that the tiles of the
 * last, partial wave (from tail_first on, fields appended) are split into
 * tail_split K ranges over the pairs that wave would leave idle.  fmt
 * MXGEMM_FMT_BF16 describes the plan of mxgemm_run_bf16 (K % 8 == 0). */
MXGEMM_API int mxgemm_describe_plan(mxgemm_handle h, int fmt, int64_t M, int64_t N, int64_t K,
                         char *buf, size_t cap);

/* The same text for a device with `num_sms` SMs (2 to 4096) and the
 * automatic schedule, without a handle: it touches no GPU, so the planner
 * can be queried for capacity planning on any host.  fmt MXGEMM_FMT_BF16
 * describes the plan of mxgemm_run_bf16 (K % 8 == 0).  Returns
 * MXGEMM_ERR_INVALID_ARG for a NULL or empty buffer, an SM count out of
 * range, or a shape mxgemm_run would reject. */
MXGEMM_API int mxgemm_describe_plan_for(int num_sms, int fmt, int64_t M, int64_t N, int64_t K,
                             char *buf, size_t cap);

/* Read and clear the device error word that kernels set when a bounded wait
 * runs out.  Synchronises the device.  *code receives 0 if no kernel gave
 * up, else a nonzero site code (1 producer waiting for a free stage, 2 MMA
 * waiting for a loaded stage, 3 MMA waiting for a free accumulator,
 * 4 epilogue waiting for a finished accumulator, 5 end-of-kernel drain,
 * 6 kernel launched with a block size it was not built for, 7 cluster K
 * split waiting for a partial tile or for the go-ahead to write one); the return
 * value is MXGEMM_ERR_TIMEOUT in that case, else MXGEMM_OK. */
MXGEMM_API int mxgemm_check_device_error(mxgemm_handle h, int *code);

/* Set the per-wait time limit of the kernels' bounded waits in nanoseconds
 * (default 2e9).  0 restores the default. */
MXGEMM_API int mxgemm_set_wait_limit(mxgemm_handle h, uint64_t ns);

/* Test hook: when `mode` is 1 the next GEMM launch on this handle arms no
 * TMA load for its first pipeline stage, so the consumer's bounded wait runs
 * out and the kernel reports MXGEMM_ERR_TIMEOUT through
 * mxgemm_check_device_error.  The hook disarms itself after one launch. */
MXGEMM_API int mxgemm_debug_inject(mxgemm_handle h, int mode);

/* mxgemm_run without a handle and without allocating device memory, for
 * callers that cannot call cudaMalloc when they run the product: code inside
 * an allocator or memory-pool hook that must not re-enter the allocator, or
 * runtimes that make every allocation up front.  (The pages have no
 * counterpart; this is a property of this library's interface.)
 *
 * Same operation, layouts and requirements as mxgemm_run, except:
 *  - the repacked scales live in a fixed 8 MiB array inside the library
 *    (held by every GPU that loads it until exit): (ceil(M/256) +
 *    ceil(N/256)) * 2 * ka * 512 bytes must fit, where ka = K/128 rounded up
 *    to a multiple of 4 (MXFP8) or 8 (MXFP4); larger problems return
 *    MXGEMM_ERR_TOO_LARGE and launch nothing;
 *  - the GEMM always computes whole output tiles (no split-K);
 *  - the first call on a device sets that device up (checks it is sm_100,
 *    looks up the array's device address); make that first call before any
 *    stream capture;
 *  - all calls share the array: calls whose work overlaps on the GPU race
 *    and give wrong results, so order them on one stream;
 *  - device timeouts of the bounded waits are not reported.
 * Buffers are device memory; `stream` is a cudaStream_t. */
MXGEMM_API int mxgemm_run_noalloc(int fmt, int64_t M, int64_t N, int64_t K,
                       const void *A, const uint8_t *A_scales,
                       const void *B, const uint8_t *B_scales,
                       void *C, void *stream);

/* Static description of a status code. */
MXGEMM_API const char *mxgemm_status_string(int status);

/* Library version as "major.minor.patch". */
MXGEMM_API const char *mxgemm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MXGEMM_H */
