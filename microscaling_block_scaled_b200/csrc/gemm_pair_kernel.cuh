// gemm_pair_kernel.cuh -- the sm_100a CTA-pair GEMM kernel (256x256 tiles
// on two CTAs with tcgen05.mma.cta_group::2) for large M, and its host
// launch template; instantiated in gemm_pair.cu.  The operation, the
// bounded waits and launch chaining are as described at the top of
// gemm_kernel.cuh.
#pragma once

#include "gemm_common.cuh"

namespace mxg {

// ------------------------------------------------------ CTA-pair kernel
//
// Large-M form: a cluster of two CTAs computes a 256x256 output tile with
// tcgen05.mma.cta_group::2 (M = 256, N = 256).  Each CTA loads its own 128
// rows of A and its own 128 rows of B (no multicast), the scale atoms of its
// A rows and of all 256 B rows; the even CTA (the leader) issues the scale
// copies and MMAs for both and its commits arrive in both CTAs.  Per CTA this
// halves the operand bytes per MMA against a 128x256 tile on one SM.
//
// Hand-offs across the pair: both CTAs' TMA loads count their bytes on the
// leader's full barrier (the 2-SM form of the tensor copy signals an
// mbarrier of either CTA of the pair), so the leader learns that a stage has
// landed in both CTAs from one barrier; the MMA commits release the stage in
// both CTAs; both CTAs' epilogues tell the leader when the accumulator may
// be reused with remote arrives.
//
// Tile order: tiles are taken in bands of `band` tile rows, every column
// tile of a band before the next band, column by column inside a band, so
// the pairs at work at one time share a few hundred rows of A and of B in L2.

template <int FMT, int KC>
struct PairCfg {
    static constexpr int kAtomsPerChunk = FMT == kFmtMXFP8 ? 1 : 2;
    static constexpr int kAtoms = kAtomsPerChunk * KC;
    static constexpr int kChunk = 128 * 128;                  // 128 rows x 128 bytes of K
    static constexpr int kABytes = kChunk * KC;               // this CTA's 128 rows of A
    static constexpr int kBBytes = kChunk * KC;               // this CTA's 128 rows of B
    static constexpr int kSFABytes = kAtoms * 512;            // scales of this CTA's A rows
    static constexpr int kSFBBytes = 2 * kAtoms * 512;        // scales of all 256 B rows
    static constexpr int kStageBytes = kABytes + kBBytes + kSFABytes + kSFBBytes;
    // output staging: two BF16 chunks of 128 rows x kCW columns; 16-column
    // chunks when the smaller staging buys the ring another stage
    static constexpr int stages_with(int cw)
    {
        return (227 * 1024 - 2048 - 2 * 128 * cw * 2) / kStageBytes;
    }
    static constexpr int kCW = stages_with(16) > stages_with(32) ? 16 : 32;
    static constexpr int kOutBytes = 128 * kCW * 2;
    static constexpr int kSmemBudget = 227 * 1024 - 2048 - 2 * kOutBytes;
    static constexpr int kStagesRaw = kSmemBudget / kStageBytes;
    static constexpr int kStages = kStagesRaw > 12 ? 12 : kStagesRaw;
    static constexpr int kSFACols = kAtoms * 4;
    static constexpr int kSFBCols = 2 * kAtoms * 4;
    static constexpr int kAccCols = 256;
    static constexpr int kTmemCols = 512;
    static constexpr int kOffA = 0;
    static constexpr int kOffB = kOffA + kStages * kABytes;
    static constexpr int kOffSFA = kOffB + kStages * kBBytes;
    static constexpr int kOffSFB = kOffSFA + kStages * kSFABytes;
    static constexpr int kOffOut = (kOffSFB + kStages * kSFBBytes + 1023) / 1024 * 1024;
    static constexpr int kOffBar = kOffOut + 2 * kOutBytes;
    static constexpr int kNumBars = 3 * kStages + 3;   // full, empty, scales-ready per stage; accf, acce, drain
    static constexpr int kThreads = 256;                 // warps 0, 6 TMA; 1 MMA; 2..5 epilogue; 7 scale copies
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kSmemBytes = kOffMisc + 64 + 1024;

    static_assert(kStages >= 2, "at least two pipeline stages");
    static_assert(kAccCols + kStages * (kSFACols + kSFBCols) <= kTmemCols, "TMEM budget");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

template <int FMT>
__host__ __device__ constexpr uint32_t idesc_pair()
{
    constexpr uint32_t t = FMT == kFmtMXFP8 ? 0u : 1u;
    return (t << 7) | (t << 10) | (static_cast<uint32_t>(256 >> 3) << 17) | (1u << 23) |
           (static_cast<uint32_t>(256 >> 4) << 24);
}

// Tile t of a pair plan -> (tp, tq), bands of `band` tile rows (see above);
// band >= tilesP is the plain column-major order.
__device__ __forceinline__ void pair_tile(uint32_t t, uint32_t tilesP, uint32_t tilesQ, uint32_t band, uint32_t &tp,
                                          uint32_t &tq)
{
    const uint32_t per_band = band * tilesQ;
    const uint32_t b = t / per_band;
    const uint32_t rows = (tilesP - b * band) < band ? (tilesP - b * band) : band;
    const uint32_t w = t - b * per_band;
    tq = w / rows;
    tp = b * band + (w - tq * rows);
}

// Work unit w of a pair plan: whole tiles first; then, for the tiles of the
// last, partial wave, `split` units per tile, each a contiguous range of its
// K iterations.  A split tile's units write FP32 partials to slots
// [slot0, slot0 + nseg) and the last to finish sums them in slot order.
struct PairUnit {
    uint32_t tile, kb, ke, seg, nseg, slot0;
};

__device__ __forceinline__ PairUnit pair_unit(uint32_t w, uint32_t first, uint32_t split, uint32_t KT)
{
    PairUnit u;
    if (w < first || split <= 1) {
        u.tile = w;
        u.kb = 0;
        u.ke = KT;
        u.seg = 0;
        u.nseg = 1;
        u.slot0 = 0;
    } else {
        const uint32_t v = w - first, ti = v / split;
        u.tile = first + ti;
        u.seg = v - ti * split;
        u.kb = u.seg * KT / split;
        u.ke = (u.seg + 1) * KT / split;
        u.nseg = split;
        u.slot0 = ti * split;
    }
    return u;
}

template <int FMT, int KC>
__global__ void __launch_bounds__(256, 1)
    mx_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmSP, const __grid_constant__ CUtensorMap tmSQ,
                        const __grid_constant__ CUtensorMap tmC, const KParams kp_in)
{
    using C_ = PairCfg<FMT, KC>;
    constexpr int S = C_::kStages;
    const KParams kp = kp_in;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + C_::kOffBar;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };              // leader: both CTAs' stage landed
    auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
    auto sfr_bar = [&](int s) { return bar0 + 8u * (2 * S + s); };     // leader: stage's scales in TMEM
    const uint32_t accf_bar = bar0 + 8u * (3 * S);
    const uint32_t acce_bar = bar0 + 8u * (3 * S + 1);
    const uint32_t drain_bar = bar0 + 8u * (3 * S + 2);
    volatile uint32_t *s_tmem = reinterpret_cast<volatile uint32_t *>(smem + C_::kOffMisc);
    volatile int *s_abort = reinterpret_cast<volatile int *>(smem + C_::kOffMisc + 4);
    volatile int *s_last = reinterpret_cast<volatile int *>(smem + C_::kOffMisc + 8);

    if (blockDim.x != C_::kThreads) {     // uniform over the cluster: both CTAs return
        if (threadIdx.x == 0)
            atomicCAS(kp.error, 0, kErrLaunch);
        return;
    }
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const uint32_t pair = blockIdx.x / 2, npairs = gridDim.x / 2;
    const uint32_t units = kp.workers, tilesP = kp.tilesP, tilesQ = kp.tilesQ, KT = kp.kt;
    const uint32_t band = kp.band, tail_first = kp.tail_first, tail_split = kp.tail_split;

    if (threadIdx.x == 0) {
        tma_prefetch_desc(&tmP);
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmSP);
        tma_prefetch_desc(&tmSQ);
        tma_prefetch_desc(&tmC);
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 2);          // the leader's two producer warps arm it (both CTAs' bytes)
            mbar_init(empty_bar(s), 1);
            mbar_init(sfr_bar(s), 1);
        }
        mbar_init(accf_bar, 1);
        mbar_init(acce_bar, 8);
        mbar_init(drain_bar, 2);            // MMA warp and scale-copy warp of the leader
        *s_abort = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc_pair(sbase + C_::kOffMisc, C_::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp != 0 && warp != 6)
        grid_dependency_wait();

    if (warp == 0 || warp == 6) {
        // ----------------------------------------------------- TMA producers
        // Warp 0: this CTA's 128 rows of A and their scale atoms; warp 6: its
        // 128 rows of B and the scale atoms of all 256 B rows of the tile.
        // Every copy counts its bytes on the leader's full barrier; the
        // leader's warps arm it for both CTAs' bytes.
        const bool sideA = warp == 0;
        if (lane == 0) {
            const uint64_t pol = policy_evict_normal();
            const CUtensorMap *tmOp = sideA ? &tmP : &tmQ;
            const CUtensorMap *tmSf = sideA ? &tmSP : &tmSQ;
            const uint32_t opBytes = sideA ? C_::kABytes : C_::kBBytes;
            const uint32_t sfBytes = sideA ? C_::kSFABytes : C_::kSFBBytes;
            const uint32_t offOp = sideA ? C_::kOffA : C_::kOffB;
            const uint32_t offSf = sideA ? C_::kOffSFA : C_::kOffSFB;
            uint32_t armed = 0;
            int skipped_stage = -1;
            bool inject = sideA && leader && kp.inject == 1;
            int s = 0;
            uint32_t ph = 0;
            bool first = true;
            for (uint32_t w = pair; w < units; w += npairs) {
                const PairUnit un = pair_unit(w, tail_first, tail_split, KT);
                uint32_t tp, tq;
                pair_tile(un.tile, tilesP, tilesQ, band, tp, tq);
                const int32_t row = static_cast<int32_t>((sideA ? tp : tq) * 256 + rank * 128);
                const int32_t sf_rb = sideA ? static_cast<int32_t>(tp * 2 + rank) : static_cast<int32_t>(tq * 2);
                bool ok = true;
                for (uint32_t k = un.kb; k < un.ke; ++k) {
                    if (!mbar_wait_parked(empty_bar(s), ph ^ 1u, s_abort, kp.limit_ns)) {
                        record_error(kp.error, kErrProducerEmpty, s_abort);
                        ok = false;
                        break;
                    }
                    const uint32_t fb = cluster_addr(full_bar(s), 0);      // the leader's barrier
                    if (inject) {
                        inject = false;
                        skipped_stage = s;
                    } else {
                        if (leader)
                            mbar_arrive_expect_tx(full_bar(s), 2 * (opBytes + sfBytes));
                        if constexpr (KC == 1)
                            tma_load_2d_pair(sbase + offOp + s * opBytes, tmOp, static_cast<int32_t>(k * 128), row, fb,
                                             pol);
                        else
                            tma_load_3d_pair(sbase + offOp + s * opBytes, tmOp, 0, row, static_cast<int32_t>(k * KC),
                                             fb, pol);
                        if (first) {            // operands of stage 0 may overlap the preceding kernel
                            grid_dependency_wait();
                            first = false;
                        }
                        tma_load_3d_pair(sbase + offSf + s * sfBytes, tmSf, 0, static_cast<int32_t>(k * C_::kAtoms),
                                         sf_rb, fb, pol);
                    }
                    ++armed;
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok)
                    break;
            }
            if (first)
                grid_dependency_wait();
            // Let every copy land before the CTAs can exit.  The leader waits
            // for the last armed phase of each stage, which counts both CTAs'
            // bytes; the other CTA cannot exit before the leader (the final
            // cluster barrier).
            if (leader) {
                for (int st = 0; st < S; ++st) {
                    const uint32_t n = armed / S + (static_cast<uint32_t>(st) < armed % S ? 1u : 0u);
                    if (n == 0 || (st == skipped_stage && n == 1))
                        continue;
                    int dummy_abort = 0;
                    if (!mbar_wait_cluster_parked(full_bar(st), (n - 1) & 1u, &dummy_abort, kp.limit_ns))
                        atomicCAS(kp.error, 0, kErrDrain);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1 && leader) {
        // ------------------------------------------- MMA issuer (leader CTA)
        constexpr uint32_t kIdesc = idesc_pair<FMT>();
        const uint32_t t_sfa0 = tmem + C_::kAccCols;
        const uint32_t t_sfb0 = t_sfa0 + S * C_::kSFACols;
        int s = 0;
        uint32_t ph = 0;
        uint32_t acc_ph = 0;
        bool ok = true;
        for (uint32_t w = pair; w < units && ok; w += npairs) {
            const PairUnit un = pair_unit(w, tail_first, tail_split, KT);
            int good = 1;
            if (lane == 0)
                good = mbar_wait_cluster_bounded(acce_bar, acc_ph ^ 1u, s_abort, kp.limit_ns);
            good = __shfl_sync(0xffffffffu, good, 0);
            if (!good) {
                if (lane == 0)
                    record_error(kp.error, kErrMmaAccEmpty, s_abort);
                break;
            }
            tc_fence_after();
            for (uint32_t k = un.kb; k < un.ke; ++k) {
                good = 1;
                if (lane == 0)
                    // the MMA warp alone spins: it feeds the tensor pipe
                    good = mbar_wait_bounded(sfr_bar(s), ph, s_abort, kp.limit_ns);
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
#pragma unroll
                    for (int c = 0; c < KC; ++c) {
                        const uint64_t adesc = sdesc_sw128_kmajor(sbase + C_::kOffA + s * C_::kABytes + c * C_::kChunk);
                        const uint64_t bdesc = sdesc_sw128_kmajor(sbase + C_::kOffB + s * C_::kBBytes + c * C_::kChunk);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int atom = FMT == kFmtMXFP8 ? c : 2 * c + j / 2;
                            const uint32_t sf_id = FMT == kFmtMXFP8 ? j : 2 * (j % 2);
                            const uint32_t idesc = kIdesc | (sf_id << 4) | (sf_id << 29);
                            const uint32_t acc_flag = (k > un.kb || c > 0 || j > 0) ? 1u : 0u;
                            const uint64_t koff = static_cast<uint64_t>(j * 32) >> 4;
                            if (FMT == kFmtMXFP8)
                                mma_mxf8f6f4_pair(tmem, adesc + koff, bdesc + koff, idesc, t_sfa + 4 * atom,
                                                  t_sfb + atom * 8, acc_flag);
                            else
                                mma_mxf4_pair(tmem, adesc + koff, bdesc + koff, idesc, t_sfa + 4 * atom,
                                              t_sfb + atom * 8, acc_flag);
                        }
                    }
                    tc_commit_pair(empty_bar(s), 0x3);
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
                tc_commit_pair(accf_bar, 0x3);
            __syncwarp();
            acc_ph ^= 1u;
        }
        if (lane == 0) {
            tc_commit_pair(drain_bar, 0x1);
            int dummy_abort = 0;
            if (!mbar_wait_parked(drain_bar, 0, &dummy_abort, kp.limit_ns))
                atomicCAS(kp.error, 0, kErrDrain);
        }
        __syncwarp();
    } else if (warp == 7 && leader) {
        // ------------------------------ scale copies into TMEM (leader CTA)
        // Once both CTAs' stage has landed, copy the scale atoms of both
        // CTAs' A rows and of the tile's B rows into the stage's TMEM slots
        // (cta_group::2 copies write both CTAs' TMEM), then signal the MMA
        // warp.  Issuing the copies beside the MMAs keeps them off the MMA
        // warp's issue stream, where they would add to every stage.
        const uint32_t t_sfa0 = tmem + C_::kAccCols;
        const uint32_t t_sfb0 = t_sfa0 + S * C_::kSFACols;
        int s = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (uint32_t w = pair; w < units && ok; w += npairs) {
            const PairUnit un = pair_unit(w, tail_first, tail_split, KT);
            for (uint32_t k = un.kb; k < un.ke; ++k) {
                int good = 1;
                if (lane == 0)
                    good = mbar_wait_cluster_parked(full_bar(s), ph, s_abort, kp.limit_ns);
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
                        tmem_cp_32x128b_x4_pair(t_sfa + 4 * a, sdesc_rows16(s_sfa + 512 * a));
#pragma unroll
                    for (int rb = 0; rb < 2; ++rb)
#pragma unroll
                        for (int a = 0; a < C_::kAtoms; ++a)
                            tmem_cp_32x128b_x4_pair(t_sfb + a * 8 + 4 * rb,
                                                    sdesc_rows16(s_sfb + (rb * C_::kAtoms + a) * 512));
                    tc_commit_pair(sfr_bar(s), 0x1);
                }
                __syncwarp();
                if (++s == S) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
        if (lane == 0) {
            tc_commit_pair(drain_bar, 0x1);
            int dummy_abort = 0;
            if (!mbar_wait_parked(drain_bar, 0, &dummy_abort, kp.limit_ns))
                atomicCAS(kp.error, 0, kErrDrain);
        }
        __syncwarp();
    } else if (warp >= 2 && warp <= 5) {
        // ---------------------------------------------------------- epilogue
        constexpr int CW = C_::kCW;
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const int etid = threadIdx.x - 64;
        uint32_t acc_ph = 0;
        uint32_t out_chunks = 0;
        // one CW-column chunk of BF16 pairs to C through shared memory and a TMA store
        auto store_chunk = [&](const uint32_t *pk, uint32_t tp, uint32_t tq, int c) {
            const int b = static_cast<int>(out_chunks & 1u);
            uint8_t *buf = smem + C_::kOffOut + b * C_::kOutBytes;
            if (etid == 0)
                bulk_wait_group_read<1>();
            named_bar_sync(1, 128);
            uint4 *dst = reinterpret_cast<uint4 *>(buf + row * CW * 2);
#pragma unroll
            for (int j = 0; j < CW / 8; ++j)
                dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            if (etid == 0) {
                tma_store_2d(&tmC, smem_u32(buf), static_cast<int32_t>(tq * 256 + c),
                             static_cast<int32_t>(tp * 256 + rank * 128));
                bulk_commit_group();
            }
            ++out_chunks;
        };
        for (uint32_t w = pair; w < units; w += npairs) {
            const PairUnit un = pair_unit(w, tail_first, tail_split, KT);
            uint32_t tp, tq;
            pair_tile(un.tile, tilesP, tilesQ, band, tp, tq);
            int good = 1;
            if (lane == 0)
                good = mbar_wait_parked(accf_bar, acc_ph, s_abort, kp.limit_ns);
            good = __shfl_sync(0xffffffffu, good, 0);
            if (!good && lane == 0)
                record_error(kp.error, kErrEpiAccFull, s_abort);
            if (named_bar_or(1, 128, (!good || *s_abort) ? 1 : 0))
                break;
            tc_fence_after();
            const uint32_t t_acc = tmem + (static_cast<uint32_t>(quad * 32) << 16);
            if (un.nseg == 1) {
                // Drain the whole accumulator row into registers (BF16 pairs), 64
                // columns per TMEM load, and hand the accumulator back to the MMA
                // warp before any store, so the next tile's MMAs overlap this
                // tile's output traffic.
                uint32_t packed[128];
#pragma unroll
                for (int c = 0; c < 256; c += 64) {
                    uint32_t r[64];
                    tmem_ld_32x32b_x64(t_acc + c, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        packed[c / 2 + j] = pack_bf16x2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (leader)
                        mbar_arrive(acce_bar);
                    else
                        mbar_arrive_remote(acce_bar, 0);
                }
#pragma unroll
                for (int c = 0; c < 256; c += CW)
                    store_chunk(packed + c / 2, tp, tq, c);
            } else {
                // A K range of a split tile: its FP32 partial (this CTA's 128
                // rows) goes to its slot; the unit that completes the tile
                // sums all slots in order and stores C.
                float *mine = kp.partials + ((static_cast<int64_t>(un.slot0 + un.seg) * 2 + rank) * 128 + row) * 256;
#pragma unroll 1
                for (int c = 0; c < 256; c += 64) {
                    uint32_t r[64];
                    tmem_ld_32x32b_x64(t_acc + c, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        reinterpret_cast<float4 *>(mine + c)[j] =
                            make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                        __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (leader)
                        mbar_arrive(acce_bar);
                    else
                        mbar_arrive_remote(acce_bar, 0);
                }
                __threadfence();
                named_bar_sync(1, 128);
                if (etid == 0) {
                    uint32_t *ctr = kp.counters + (un.tile - tail_first) * 2 + rank;
                    const uint32_t old = atomicAdd(ctr, 1u);
                    const int last = (old == un.nseg - 1) ? 1 : 0;
                    if (last)
                        *ctr = 0u;          // counters stay zero between launches
                    *s_last = last;
                }
                named_bar_sync(1, 128);
                if (*s_last) {
                    __threadfence();
#pragma unroll 1
                    for (int c = 0; c < 256; c += CW) {
                        float v[CW];
#pragma unroll
                        for (int j = 0; j < CW; ++j)
                            v[j] = 0.0f;
                        for (uint32_t g = 0; g < un.nseg; ++g) {
                            const float4 *src = reinterpret_cast<const float4 *>(
                                kp.partials + ((static_cast<int64_t>(un.slot0 + g) * 2 + rank) * 128 + row) * 256 + c);
#pragma unroll
                            for (int j = 0; j < CW / 4; ++j) {
                                const float4 x = __ldcg(src + j);
                                v[4 * j + 0] += x.x;
                                v[4 * j + 1] += x.y;
                                v[4 * j + 2] += x.z;
                                v[4 * j + 3] += x.w;
                            }
                        }
                        uint32_t pk[CW / 2];
#pragma unroll
                        for (int j = 0; j < CW / 2; ++j)
                            pk[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
                        store_chunk(pk, tp, tq, c);
                    }
                }
            }
            acc_ph ^= 1u;
        }
        if (etid == 0)
            bulk_wait_group<0>();
    }

    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    if (warp == 1)
        tmem_dealloc_pair(tmem, C_::kTmemCols);
}

// ------------------------------------------------------------------- host

namespace {

template <int FMT, int KC>
cudaError_t launch_pair_t(const GemmPlan &pl, const GemmBuffers &b, uint64_t limit_ns, int inject, int pdl,
                          cudaStream_t st)
{
    using C_ = PairCfg<FMT, KC>;
    const int64_t rbytes = row_bytes(FMT, pl.K);
    CUtensorMap tmP, tmQ, tmC;
    if (KC == 1) {
        if (!make_operand_map(&tmP, b.A, pl.M, rbytes, 128) || !make_operand_map(&tmQ, b.B, pl.N, rbytes, 128))
            return cudaErrorInvalidValue;
    } else {
        if (!make_operand_map_3d(&tmP, b.A, pl.M, rbytes, 128, KC) ||
            !make_operand_map_3d(&tmQ, b.B, pl.N, rbytes, 128, KC))
            return cudaErrorInvalidValue;
    }
    if (!make_output_map(&tmC, b.C, pl.M, pl.N, C_::kCW, 128))
        return cudaErrorInvalidValue;
    CUtensorMap tmSP, tmSQ;
    if (!make_sf_map(&tmSP, b.sfA, pl.kaP, sf_row_blocks(pl.M), C_::kAtoms, 1) ||
        !make_sf_map(&tmSQ, b.sfB, pl.kaQ, sf_row_blocks(pl.N), C_::kAtoms, 2))
        return cudaErrorInvalidValue;
    KParams kp;
    kp.C = reinterpret_cast<__nv_bfloat16 *>(b.C);
    kp.partials = b.partials;
    kp.counters = b.counters;
    kp.error = b.error;
    kp.P = pl.M;
    kp.Q = pl.N;
    kp.ldc = pl.N;
    kp.tilesP = static_cast<uint32_t>(pl.tilesP);
    kp.kt = static_cast<uint32_t>(pl.kt);
    kp.iters = static_cast<uint32_t>(pl.iters);
    kp.workers = static_cast<uint32_t>(pl.workers);
    kp.dp = 1;
    kp.limit_ns = limit_ns;
    kp.swap = 0;
    kp.inject = inject;
    kp.tma_store = 1;
    kp.fused_sf = 0;
    kp.rawP = nullptr;
    kp.rawQ = nullptr;
    kp.ldS = pl.K / 32;
    kp.early = 3;              // this kernel's operand producers never wait (it follows the repack)
    kp.bias = nullptr;
    kp.residual = nullptr;
    kp.act = 0;
    kp.has_ops = 0;
    kp.qfmt = -1;
    kp.Cq = nullptr;
    kp.Cs = nullptr;
    kp.goff = nullptr;
    kp.groups = 0;
    kp.tilesQ = static_cast<uint32_t>(pl.tilesQ);
    kp.band = static_cast<uint32_t>(pl.band > 0 ? pl.band : pl.tilesP);
    kp.tail_first = static_cast<uint32_t>(pl.tail_first);
    kp.tail_split = static_cast<uint32_t>(pl.tail_split > 1 ? pl.tail_split : 1);
    kp.ksplit = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(pl.grid));
    cfg.blockDim = dim3(C_::kThreads);
    cfg.dynamicSmemBytes = C_::kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, mx_gemm_pair_kernel<FMT, KC>, tmP, tmQ, tmSP, tmSQ, tmC, kp);
}

}  // namespace

}  // namespace mxg
