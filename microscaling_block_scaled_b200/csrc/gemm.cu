// gemm.cu -- the sm_100a MX block-scaled GEMM: C = A * B^T, BF16 out.
//
// Operation: the "MXFP scaled GEMM" of the 5ulink.com page "PyTorch 接上
// FlyDSL" (support-matrix table; note under it: one E8M0 scale per 32
// values, FP32 accumulation, BF16 output).  The page's own kernel design
// (HTI pipeline with staged LDS, MFMA atoms, "operand and scale-factor
// lifetime pairing", section "三条路") targets another GPU; here the same
// ideas take Blackwell form: a TMA-fed shared-memory ring whose every stage
// carries an operand tile pair together with the scale tiles of exactly
// those K elements, released by one mbarrier.
//
// Structure of one persistent CTA (192 threads, one per SM):
//   warp 0      TMA producer: per stage, the 128x128-byte row-operand tile,
//               the BNx128-byte column-operand tile (both 128B-swizzled) and
//               the matching repacked scale atoms (plain bulk copies).
//   warp 1      MMA issuer and TMEM owner: tcgen05.cp of the stage's scales
//               into TMEM, then four tcgen05.mma block_scale instructions
//               (kind::mxf8f6f4 K=32 / kind::mxf4 K=64) into an FP32 TMEM
//               accumulator; tcgen05.commit releases the stage.
//   warps 2..5  epilogue: tcgen05.ld of the accumulator, BF16 (RNE) stores;
//               for split tiles an FP32 partial plus a last-arriver fixup.
//
// Work decomposition (stream-K family): the I = tiles * kt K-iterations of
// all output tiles, tile-major, are cut into W contiguous ranges, one per
// virtual worker; worker w owns [floor(w*I/W), floor((w+1)*I/W)).  W = tiles
// gives plain data-parallel tiles, W = tiles*s split-K, W = #SMs stream-K.
// A tile covered by several workers is reduced by whichever of them arrives
// last (an atomic counter per tile), summing the partials in worker order so
// the result does not depend on arrival order.  No CTA ever waits for
// another CTA.
//
// Decode shapes (M <= 64) swap the operands (C^T = B * A^T) so that the N
// rows of B fill the MMA's 128-row side and the small M becomes the MMA's N.
//
// Every wait is bounded in time; a wait that runs out records a site code in
// a device error word, the CTA drains its in-flight copies and MMAs, frees
// its tensor memory and exits normally.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>

#include "mx_internal.h"
#include "sm100_ptx.cuh"

namespace mxg {

// ------------------------------------------------------------ configuration

template <int FMT, int BN>
struct Cfg {
    static constexpr int kBM = 128;
    static constexpr int kStageKBytes = 128;                  // K bytes per stage per row
    static constexpr int kAtoms = FMT == kFmtMXFP8 ? 1 : 2;   // 512B scale atoms per 128 rows
    static constexpr int kRBQ = (BN + 127) / 128;             // 128-row blocks of the column operand
    static constexpr int kABytes = kBM * kStageKBytes;
    static constexpr int kBBytes = BN * kStageKBytes;
    static constexpr int kSFABytes = kAtoms * 512;
    static constexpr int kSFBBytes = kRBQ * kAtoms * 512;
    static constexpr int kStageBytes = kABytes + kBBytes + kSFABytes + kSFBBytes;
    static constexpr int kSmemBudget = 227 * 1024 - 2048;
    static constexpr int kStagesRaw = kSmemBudget / kStageBytes;
    static constexpr int kStages = kStagesRaw > 12 ? 12 : kStagesRaw;
    static constexpr int kSFACols = kAtoms * 4;
    static constexpr int kSFBCols = kRBQ * kAtoms * 4;
    static constexpr int kSFCols = kStages * (kSFACols + kSFBCols);
    static constexpr int kNumAcc = (2 * BN + kSFCols <= 512) ? 2 : 1;
    static constexpr int kAccCols = kNumAcc * BN;
    static constexpr int kTmemCols = 512;
    static constexpr int kMmaPerStage = 4;                    // 32 bytes of K per MMA
    static constexpr uint32_t kTxBytes = kStageBytes;
    // shared memory layout (offsets from a 1024-aligned base)
    static constexpr int kOffA = 0;
    static constexpr int kOffB = kOffA + kStages * kABytes;
    static constexpr int kOffSFA = kOffB + kStages * kBBytes;
    static constexpr int kOffSFB = kOffSFA + kStages * kSFABytes;
    static constexpr int kOffBar = kOffSFB + kStages * kSFBBytes;
    static constexpr int kNumBars = 2 * kStages + 2 * kNumAcc + 1;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kSmemBytes = kOffMisc + 64 + 1024;   // + alignment slack

    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N must be a multiple of 16 in [16, 256]");
    static_assert(kStages >= 2, "at least two pipeline stages");
    static_assert(kAccCols + kSFCols <= kTmemCols, "TMEM budget");
    static_assert(kBBytes % 1024 == 0, "tiles must keep 1024-byte alignment");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

// Instruction descriptor of the block-scaled MMA (PTX ISA, instruction
// descriptor for .kind::mxf8f6f4 / .kind::mxf4): A/B type at bits [7,10) and
// [10,13) (E4M3 = 0 under mxf8f6f4, E2M1 = 1 under mxf4), both K-major (bits
// 15, 16 = 0), N >> 3 at [17,23), scale type UE8M0 at bit 23, M >> 4 at
// [24,29); scale-factor ids of B at [4,6) and of A at [29,31) are added per
// instruction.
template <int FMT, int BN>
__host__ __device__ constexpr uint32_t idesc_base()
{
    constexpr uint32_t t = FMT == kFmtMXFP8 ? 0u : 1u;
    return (t << 7) | (t << 10) | (static_cast<uint32_t>(BN >> 3) << 17) | (1u << 23) |
           (static_cast<uint32_t>(128 >> 4) << 24);
}

struct KParams {
    const uint8_t *sfP;   // repacked scales of the MMA row operand
    const uint8_t *sfQ;   // repacked scales of the MMA column operand
    __nv_bfloat16 *C;
    float *partials;
    uint32_t *counters;
    int *error;
    int64_t P, Q;          // valid rows of the two MMA operands
    int64_t ldc;           // = N
    int64_t tilesP, kt, iters, workers;
    int64_t kaP, kaQ;      // scale atoms per 128-row block
    uint64_t limit_ns;
    int swap;
    int inject;
};

// Error site codes written to the device error word.
enum : int {
    kErrProducerEmpty = 1,
    kErrMmaFull = 2,
    kErrMmaAccEmpty = 3,
    kErrEpiAccFull = 4,
    kErrDrain = 5,
};

__device__ __forceinline__ void record_error(int *err, int code, volatile int *abort_flag)
{
    atomicCAS(err, 0, code);
    *abort_flag = 1;
}

// Which worker owns K-iteration i (largest g with floor(g*I/W) <= i).
__device__ __forceinline__ int64_t worker_of(int64_t i, int64_t I, int64_t W)
{
    return ((i + 1) * W - 1) / I;
}

__device__ __forceinline__ int64_t worker_begin(int64_t g, int64_t I, int64_t W) { return g * I / W; }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Store CW FP32 values as BF16 into C.  Non-swapped: thread's row p = C row,
// values are C[p][q0 .. q0+CW).  Swapped: thread's row p = C column, values
// are C[q0 .. q0+CW)[p].
template <int CW>
__device__ __forceinline__ void store_bf16(const KParams &kp, int64_t p, int64_t q0, const float (&v)[CW])
{
    if (p >= kp.P)
        return;
    if (!kp.swap) {
        __nv_bfloat16 *dst = kp.C + p * kp.ldc + q0;
        const int64_t nvalid = kp.Q - q0;
        if (nvalid >= CW && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
#pragma unroll
            for (int j = 0; j < CW / 8; ++j) {
                uint4 w;
                w.x = pack_bf16x2(v[8 * j + 0], v[8 * j + 1]);
                w.y = pack_bf16x2(v[8 * j + 2], v[8 * j + 3]);
                w.z = pack_bf16x2(v[8 * j + 4], v[8 * j + 5]);
                w.w = pack_bf16x2(v[8 * j + 6], v[8 * j + 7]);
                reinterpret_cast<uint4 *>(dst)[j] = w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < CW; ++j)
                if (j < nvalid)
                    dst[j] = __float2bfloat16_rn(v[j]);
        }
    } else {
#pragma unroll
        for (int j = 0; j < CW; ++j) {
            const int64_t q = q0 + j;
            if (q < kp.Q)
                kp.C[q * kp.ldc + p] = __float2bfloat16_rn(v[j]);
        }
    }
}

template <int FMT, int BN>
__global__ void __launch_bounds__(192, 1)
    mx_gemm_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmQ,
                   const KParams kp)
{
    using C_ = Cfg<FMT, BN>;
    constexpr int S = C_::kStages;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + C_::kOffBar;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
    auto accf_bar = [&](int a) { return bar0 + 8u * (2 * S + a); };
    auto acce_bar = [&](int a) { return bar0 + 8u * (2 * S + C_::kNumAcc + a); };
    const uint32_t drain_bar = bar0 + 8u * (2 * S + 2 * C_::kNumAcc);
    volatile uint32_t *s_tmem = reinterpret_cast<volatile uint32_t *>(smem + C_::kOffMisc);
    volatile int *s_abort = reinterpret_cast<volatile int *>(smem + C_::kOffMisc + 4);
    volatile int *s_last = reinterpret_cast<volatile int *>(smem + C_::kOffMisc + 8);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int a = 0; a < C_::kNumAcc; ++a) {
            mbar_init(accf_bar(a), 1);
            mbar_init(acce_bar(a), 4);
        }
        mbar_init(drain_bar, 1);
        *s_abort = 0;
        *s_last = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(sbase + C_::kOffMisc, C_::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    const int64_t I = kp.iters, W = kp.workers, KT = kp.kt;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmP);
            tma_prefetch_desc(&tmQ);
        }
        const uint64_t pol_stream = policy_evict_first();
        int s = 0;
        uint32_t ph = 0;
        int64_t armed = 0;          // loads armed so far (round-robin over stages)
        int skipped_stage = -1;
        bool inject = kp.inject == 1;
        bool ok = true;
        for (int64_t w = blockIdx.x; w < W && ok; w += gridDim.x) {
            int64_t it = worker_begin(w, I, W);
            const int64_t end = worker_begin(w + 1, I, W);
            while (it < end && ok) {
                const int64_t tile = it / KT;
                const int64_t kb = it - tile * KT;
                const int64_t ke = (kb + (end - it) < KT) ? kb + (end - it) : KT;
                const int64_t tp = tile % kp.tilesP, tq = tile / kp.tilesP;
                for (int64_t k = kb; k < ke; ++k) {
                    int good = 1;
                    if (lane == 0)
                        good = mbar_wait_bounded(empty_bar(s), ph ^ 1u, s_abort, kp.limit_ns);
                    good = __shfl_sync(0xffffffffu, good, 0);
                    if (!good) {
                        if (lane == 0)
                            record_error(kp.error, kErrProducerEmpty, s_abort);
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        if (inject) {
                            inject = false;          // leave this stage unarmed
                            skipped_stage = s;
                        } else {
                            const uint32_t fb = full_bar(s);
                            mbar_arrive_expect_tx(fb, C_::kTxBytes);
                            const int32_t x = static_cast<int32_t>(k * C_::kStageKBytes);
                            tma_load_2d(sbase + C_::kOffA + s * C_::kABytes, &tmP, x,
                                        static_cast<int32_t>(tp * 128), fb, pol_stream);
                            tma_load_2d(sbase + C_::kOffB + s * C_::kBBytes, &tmQ, x,
                                        static_cast<int32_t>(tq * BN), fb, pol_stream);
                            const uint8_t *sfa = kp.sfP + (tp * kp.kaP + k * C_::kAtoms) * 512;
                            bulk_load(sbase + C_::kOffSFA + s * C_::kSFABytes, sfa, C_::kSFABytes, fb);
                            const int64_t rb0 = (tq * BN) / 128;
#pragma unroll
                            for (int rb = 0; rb < C_::kRBQ; ++rb) {
                                const uint8_t *sfb = kp.sfQ + ((rb0 + rb) * kp.kaQ + k * C_::kAtoms) * 512;
                                bulk_load(sbase + C_::kOffSFB + s * C_::kSFBBytes + rb * C_::kAtoms * 512, sfb,
                                          C_::kAtoms * 512, fb);
                            }
                        }
                        ++armed;
                    }
                    __syncwarp();
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                it += ke - kb;
            }
        }
        // Let every armed copy land before the CTA can exit: wait for the
        // latest armed phase of each stage (already complete on the normal
        // path, where the MMA warp consumed every stage).
        if (lane == 0) {
            for (int st = 0; st < S; ++st) {
                const int64_t n = armed / S + (st < armed % S ? 1 : 0);
                if (n == 0 || (st == skipped_stage && n == 1))
                    continue;
                const uint32_t parity = static_cast<uint32_t>((n - 1) & 1);
                int dummy_abort = 0;
                if (!mbar_wait_bounded(full_bar(st), parity, &dummy_abort, kp.limit_ns))
                    atomicCAS(kp.error, 0, kErrDrain);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        constexpr uint32_t kIdesc = idesc_base<FMT, BN>();
        const uint32_t t_sfa0 = tmem + C_::kAccCols;
        const uint32_t t_sfb0 = t_sfa0 + S * C_::kSFACols;
        int s = 0;
        uint32_t ph = 0;
        int acc = 0;
        uint32_t acc_ph = 0;
        bool ok = true;
        for (int64_t w = blockIdx.x; w < W && ok; w += gridDim.x) {
            int64_t it = worker_begin(w, I, W);
            const int64_t end = worker_begin(w + 1, I, W);
            while (it < end && ok) {
                const int64_t tile = it / KT;
                const int64_t kb = it - tile * KT;
                const int64_t ke = (kb + (end - it) < KT) ? kb + (end - it) : KT;
                int good = 1;
                if (lane == 0)
                    good = mbar_wait_bounded(acce_bar(acc), acc_ph ^ 1u, s_abort, kp.limit_ns);
                good = __shfl_sync(0xffffffffu, good, 0);
                if (!good) {
                    if (lane == 0)
                        record_error(kp.error, kErrMmaAccEmpty, s_abort);
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t t_acc = tmem + acc * BN;
                for (int64_t k = kb; k < ke; ++k) {
                    good = 1;
                    if (lane == 0)
                        good = mbar_wait_bounded(full_bar(s), ph, s_abort, kp.limit_ns);
                    good = __shfl_sync(0xffffffffu, good, 0);
                    if (!good) {
                        if (lane == 0)
                            record_error(kp.error, kErrMmaFull, s_abort);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t t_sfa = t_sfa0 + s * C_::kSFACols;
                        const uint32_t t_sfb = t_sfb0 + s * C_::kSFBCols;
                        const uint32_t s_sfa = sbase + C_::kOffSFA + s * C_::kSFABytes;
                        const uint32_t s_sfb = sbase + C_::kOffSFB + s * C_::kSFBBytes;
#pragma unroll
                        for (int a = 0; a < C_::kAtoms; ++a)
                            tmem_cp_32x128b_x4(t_sfa + 4 * a, sdesc_rows16(s_sfa + 512 * a));
#pragma unroll
                        for (int rb = 0; rb < C_::kRBQ; ++rb)
#pragma unroll
                            for (int a = 0; a < C_::kAtoms; ++a)
                                tmem_cp_32x128b_x4(t_sfb + a * 4 * C_::kRBQ + 4 * rb,
                                                   sdesc_rows16(s_sfb + (rb * C_::kAtoms + a) * 512));
                        const uint64_t adesc = sdesc_sw128_kmajor(sbase + C_::kOffA + s * C_::kABytes);
                        const uint64_t bdesc = sdesc_sw128_kmajor(sbase + C_::kOffB + s * C_::kBBytes);
#pragma unroll
                        for (int j = 0; j < C_::kMmaPerStage; ++j) {
                            // MXFP8: one scale block per MMA, id j of the atom's 4 bytes.
                            // MXFP4: two scale blocks per MMA, atom j/2, byte pair 2*(j%2).
                            const int atom = FMT == kFmtMXFP8 ? 0 : j / 2;
                            const uint32_t sf_id = FMT == kFmtMXFP8 ? j : 2 * (j % 2);
                            const uint32_t idesc = kIdesc | (sf_id << 4) | (sf_id << 29);
                            const uint32_t acc_flag = (k > kb || j > 0) ? 1u : 0u;
                            const uint64_t koff = static_cast<uint64_t>(j * 32) >> 4;
                            if (FMT == kFmtMXFP8)
                                mma_mxf8f6f4(t_acc, adesc + koff, bdesc + koff, idesc, t_sfa + 4 * atom,
                                             t_sfb + atom * 4 * C_::kRBQ, acc_flag);
                            else
                                mma_mxf4(t_acc, adesc + koff, bdesc + koff, idesc, t_sfa + 4 * atom,
                                         t_sfb + atom * 4 * C_::kRBQ, acc_flag);
                        }
                        tc_commit(empty_bar(s));
                    }
                    __syncwarp();
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok)
                    break;
                if (lane == 0)
                    tc_commit(accf_bar(acc));
                __syncwarp();
                if (++acc == C_::kNumAcc) {
                    acc = 0;
                    acc_ph ^= 1u;
                }
                it += ke - kb;
            }
        }
        // Drain: every tcgen05 operation this thread issued has completed.
        if (lane == 0) {
            tc_commit(drain_bar);
            int dummy_abort = 0;
            if (!mbar_wait_bounded(drain_bar, 0, &dummy_abort, kp.limit_ns))
                atomicCAS(kp.error, 0, kErrDrain);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------- epilogue
        constexpr int CW = BN < 32 ? BN : 32;  // accumulator columns per tcgen05.ld
        const int quad = warp & 3;             // TMEM lanes 32*quad .. +31
        const int row = quad * 32 + lane;      // accumulator row = MMA row in tile
        const int etid = threadIdx.x - 64;     // 0..127
        int acc = 0;
        uint32_t acc_ph = 0;
        bool stop = false;
        for (int64_t w = blockIdx.x; w < W && !stop; w += gridDim.x) {
            int64_t it = worker_begin(w, I, W);
            const int64_t end = worker_begin(w + 1, I, W);
            bool first = true;
            while (it < end) {
                const int64_t tile = it / KT;
                const int64_t kb = it - tile * KT;
                const int64_t ke = (kb + (end - it) < KT) ? kb + (end - it) : KT;
                const int64_t tp = tile % kp.tilesP, tq = tile / kp.tilesP;
                int good = 1;
                if (lane == 0)
                    good = mbar_wait_bounded(accf_bar(acc), acc_ph, s_abort, kp.limit_ns);
                good = __shfl_sync(0xffffffffu, good, 0);
                if (!good && lane == 0)
                    record_error(kp.error, kErrEpiAccFull, s_abort);
                // One decision for all four epilogue warps.
                if (named_bar_or(1, 128, (!good || *s_abort) ? 1 : 0)) {
                    stop = true;
                    break;
                }
                tc_fence_after();
                const uint32_t t_acc = tmem + acc * BN + (static_cast<uint32_t>(quad * 32) << 16);
                const int64_t p = tp * 128 + row;
                const int64_t g_first = worker_of(tile * KT, I, W);
                const int64_t g_last = worker_of(tile * KT + KT - 1, I, W);
                if (g_first == g_last) {
#pragma unroll 1
                    for (int c = 0; c < BN; c += CW) {
                        uint32_t r[CW];
                        tmem_ld_cols<CW>(t_acc + c, r);
                        tmem_ld_wait();
                        float v[CW];
#pragma unroll
                        for (int j = 0; j < CW; ++j)
                            v[j] = __uint_as_float(r[j]);
                        store_bf16<CW>(kp, p, tq * BN + c, v);
                    }
                } else {
                    const int64_t slot = 2 * w + (first ? 0 : 1);
                    float *mine = kp.partials + (slot * 128 + row) * BN;
#pragma unroll 1
                    for (int c = 0; c < BN; c += CW) {
                        uint32_t r[CW];
                        tmem_ld_cols<CW>(t_acc + c, r);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < CW / 4; ++j)
                            reinterpret_cast<uint4 *>(mine + c)[j] =
                                make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
                    }
                    __threadfence();
                    named_bar_sync(1, 128);
                    if (etid == 0) {
                        const int64_t nseg = g_last - g_first + 1;
                        const uint32_t old = atomicAdd(kp.counters + tile, 1u);
                        const int last = (static_cast<int64_t>(old) == nseg - 1) ? 1 : 0;
                        if (last)
                            kp.counters[tile] = 0u;
                        *s_last = last;
                    }
                    named_bar_sync(1, 128);
                    if (*s_last) {
                        __threadfence();
#pragma unroll 1
                        for (int c = 0; c < BN; c += CW) {
                            uint32_t r[CW];
                            tmem_ld_cols<CW>(t_acc + c, r);
                            tmem_ld_wait();
                            float v[CW];
#pragma unroll
                            for (int j = 0; j < CW; ++j)
                                v[j] = 0.0f;
                            for (int64_t g = g_first; g <= g_last; ++g) {
                                if (g == w) {
#pragma unroll
                                    for (int j = 0; j < CW; ++j)
                                        v[j] += __uint_as_float(r[j]);
                                } else {
                                    const int64_t gslot =
                                        2 * g + ((worker_begin(g, I, W) / KT == tile) ? 0 : 1);
                                    const float4 *src = reinterpret_cast<const float4 *>(
                                        kp.partials + (gslot * 128 + row) * BN + c);
#pragma unroll
                                    for (int j = 0; j < CW / 4; ++j) {
                                        const float4 x = __ldcg(src + j);
                                        v[4 * j + 0] += x.x;
                                        v[4 * j + 1] += x.y;
                                        v[4 * j + 2] += x.z;
                                        v[4 * j + 3] += x.w;
                                    }
                                }
                            }
                            store_bf16<CW>(kp, p, tq * BN + c, v);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(acce_bar(acc));
                if (++acc == C_::kNumAcc) {
                    acc = 0;
                    acc_ph ^= 1u;
                }
                first = false;
                it += ke - kb;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        tmem_dealloc(tmem, C_::kTmemCols);
}

// ------------------------------------------------------------------- host

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

template <int FMT, int BN>
cudaError_t set_attrs()
{
    return cudaFuncSetAttribute(mx_gemm_kernel<FMT, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Cfg<FMT, BN>::kSmemBytes);
}

template <int FMT, int BN>
cudaError_t launch_t(const GemmPlan &pl, const GemmBuffers &b, uint64_t limit_ns, int inject, cudaStream_t st)
{
    using C_ = Cfg<FMT, BN>;
    const int64_t rbytes = row_bytes(FMT, pl.K);
    const void *Pptr = pl.swap ? b.B : b.A;
    const void *Qptr = pl.swap ? b.A : b.B;
    CUtensorMap tmP, tmQ;
    if (!make_operand_map(&tmP, Pptr, pl.P, rbytes, 128) || !make_operand_map(&tmQ, Qptr, pl.Q, rbytes, BN))
        return cudaErrorInvalidValue;
    KParams kp;
    kp.sfP = pl.swap ? b.sfB : b.sfA;
    kp.sfQ = pl.swap ? b.sfA : b.sfB;
    kp.C = reinterpret_cast<__nv_bfloat16 *>(b.C);
    kp.partials = b.partials;
    kp.counters = b.counters;
    kp.error = b.error;
    kp.P = pl.P;
    kp.Q = pl.Q;
    kp.ldc = pl.N;
    kp.tilesP = pl.tilesP;
    kp.kt = pl.kt;
    kp.iters = pl.iters;
    kp.workers = pl.workers;
    kp.kaP = pl.kaP;
    kp.kaQ = pl.kaQ;
    kp.limit_ns = limit_ns;
    kp.swap = pl.swap;
    kp.inject = inject;
    mx_gemm_kernel<FMT, BN><<<pl.grid, 192, C_::kSmemBytes, st>>>(tmP, tmQ, kp);
    return cudaGetLastError();
}

template <int FMT>
cudaError_t dispatch_bn(const GemmPlan &pl, const GemmBuffers &b, uint64_t limit_ns, int inject, cudaStream_t st)
{
    switch (pl.bn) {
    case 16: return launch_t<FMT, 16>(pl, b, limit_ns, inject, st);
    case 32: return launch_t<FMT, 32>(pl, b, limit_ns, inject, st);
    case 64: return launch_t<FMT, 64>(pl, b, limit_ns, inject, st);
    case 128: return launch_t<FMT, 128>(pl, b, limit_ns, inject, st);
    case 256: return launch_t<FMT, 256>(pl, b, limit_ns, inject, st);
    default: return cudaErrorInvalidValue;
    }
}

template <int FMT>
int stages_for(int bn)
{
    switch (bn) {
    case 16: return Cfg<FMT, 16>::kStages;
    case 32: return Cfg<FMT, 32>::kStages;
    case 64: return Cfg<FMT, 64>::kStages;
    case 128: return Cfg<FMT, 128>::kStages;
    case 256: return Cfg<FMT, 256>::kStages;
    default: return 0;
    }
}

}  // namespace

cudaError_t prepare_gemm_kernels()
{
    cudaError_t e = cudaSuccess;
#define MXG_ATTR(F, B)                 \
    if (e == cudaSuccess)              \
        e = set_attrs<F, B>();
    MXG_ATTR(0, 16) MXG_ATTR(0, 32) MXG_ATTR(0, 64) MXG_ATTR(0, 128) MXG_ATTR(0, 256)
    MXG_ATTR(1, 16) MXG_ATTR(1, 32) MXG_ATTR(1, 64) MXG_ATTR(1, 128) MXG_ATTR(1, 256)
#undef MXG_ATTR
    return e;
}

GemmPlan make_plan(int fmt, int64_t M, int64_t N, int64_t K, int num_sms, int sched, int splits, int workers)
{
    GemmPlan pl;
    pl.fmt = fmt;
    pl.M = M;
    pl.N = N;
    pl.K = K;
    pl.swap = M <= 64 ? 1 : 0;
    if (pl.swap) {
        pl.P = N;
        pl.Q = M;
        pl.bn = M <= 16 ? 16 : (M <= 32 ? 32 : 64);
    } else {
        pl.P = M;
        pl.Q = N;
        pl.bn = 128;
    }
    pl.stages = fmt == kFmtMXFP8 ? stages_for<0>(pl.bn) : stages_for<1>(pl.bn);
    pl.tilesP = (pl.P + 127) / 128;
    pl.tilesQ = (pl.Q + pl.bn - 1) / pl.bn;
    pl.kt = (row_bytes(fmt, K) + 127) / 128;
    pl.tiles = pl.tilesP * pl.tilesQ;
    pl.iters = pl.tiles * pl.kt;
    const int64_t sms = num_sms > 0 ? num_sms : 1;
    int s = sched;
    if (s == 0)   // auto
        s = pl.tiles >= sms ? 1 : 3;
    pl.sched = s;
    if (s == 1) {
        pl.workers = pl.tiles;
    } else if (s == 2) {
        const int64_t sp = splits < 1 ? 1 : (splits > pl.kt ? pl.kt : splits);
        pl.workers = pl.tiles * sp;
    } else {
        int64_t w = workers > 0 ? workers : sms;
        if (w > pl.iters)
            w = pl.iters;
        if (w < pl.tiles && workers <= 0)
            w = pl.tiles;
        pl.workers = w;
    }
    if (pl.workers < 1)
        pl.workers = 1;
    pl.grid = static_cast<int>(pl.workers < sms ? pl.workers : sms);
    pl.kaP = sf_atoms_per_rowblock(fmt, K);
    pl.kaQ = pl.kaP;
    pl.partial_bytes = (pl.workers == pl.tiles) ? 0 : 2 * pl.workers * 128 * pl.bn * 4;
    pl.counter_bytes = pl.tiles * 4;
    return pl;
}

cudaError_t launch_gemm(const GemmPlan &plan, const GemmBuffers &buf, uint64_t wait_limit_ns, int inject,
                        cudaStream_t stream)
{
    if (plan.fmt == kFmtMXFP8)
        return dispatch_bn<0>(plan, buf, wait_limit_ns, inject, stream);
    return dispatch_bn<1>(plan, buf, wait_limit_ns, inject, stream);
}

}  // namespace mxg
