// gemm.cu -- the GEMM's host planner and launch dispatch.
//
// The planner picks, from the shape and the SM count alone, the operand
// swap for decode shapes (M <= 64: C^T = B * A^T), the output tile width,
// the 128-byte K chunks per pipeline stage, CTA pairs for large M, and the
// schedule (whole tiles, split-K or stream-K).  The kernels and their launch
// templates are in gemm_kernel.cuh, instantiated per operand type in
// gemm_mxfp8.cu, gemm_mxfp4.cu, gemm_bf16.cu and gemm_pair.cu.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdlib>

#include "mx_internal.h"

namespace mxg {

namespace {

int stages_for(int fmt, int bn, int kc)
{
    return fmt == kFmtMXFP8 ? stages_mxfp8(bn, kc) : (fmt == kFmtMXFP4 ? stages_mxfp4(bn, kc) : stages_bf16(bn, kc));
}

}  // namespace

cudaError_t prepare_gemm_kernels()
{
    cudaError_t e = prepare_mxfp8();
    if (e == cudaSuccess)
        e = prepare_mxfp4();
    if (e == cudaSuccess)
        e = prepare_bf16();
    if (e == cudaSuccess)
        e = prepare_pair();
    return e;
}

GemmPlan make_plan(int fmt, int64_t M, int64_t N, int64_t K, int num_sms, int sched, int splits, int workers,
                   int force_kc, bool allow_pair)
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
        // measurement knob: MXGEMM_BN=256 selects 128x256 output tiles
        if (const char *e = getenv("MXGEMM_BN"))
            if (atoi(e) == 256 && N >= 256)
                pl.bn = 256;
    }
    // Two 128-byte K chunks per stage halve the TMA operations per byte (each
    // costs ~0.2 us of the SM's copy engine); rows must be whole chunks.
    const int64_t chunks = (row_bytes(fmt, K) + 127) / 128;
    const bool whole = row_bytes(fmt, K) % 128 == 0;
    pl.kc = (whole && chunks >= 2) ? 2 : 1;
    // (four chunks per stage, mxgemm_set_kchunks(4), fit only two ring
    // stages on 64-column decode tiles and measured slower in chained steps:
    // MXFP8 64x4096x4096 15.2 us against 13.0 us with two chunks, MXFP4
    // 11.5 us against 10.3 us)
    if (force_kc == 1 || (force_kc == 2 && whole))
        pl.kc = force_kc;
    if (force_kc == 4 && whole && pl.bn <= 64)
        pl.kc = 4;
    // Large M: 256x256 tiles on CTA pairs (cta_group::2) when they fill the GPU.
    {
        const int64_t ptiles = ((M + 255) / 256) * ((N + 255) / 256);
        const char *e = getenv("MXGEMM_PAIR");
        const bool allow = allow_pair && fmt != kFmtBF16 && !(e && atoi(e) == 0);
        if (allow && !pl.swap && M >= 512 && N >= 256 && N % 8 == 0 && ptiles >= 64)
            pl.pair = 1;
    }
    if (pl.pair) {
        pl.bn = 256;
        if (force_kc == 0)
            pl.kc = (whole && chunks >= 2) ? 2 : 1;
        else
            pl.kc = (force_kc == 2 && whole) ? 2 : 1;
        pl.stages = stages_pair(fmt, pl.kc);
        pl.tilesP = (M + 255) / 256;
        pl.tilesQ = (N + 255) / 256;
        pl.kt = (chunks + pl.kc - 1) / pl.kc;
        pl.tiles = pl.tilesP * pl.tilesQ;
        pl.iters = pl.tiles * pl.kt;
        // Tile order: bands of 8 tile rows (2048 rows of A).  In plain
        // column-major order the pairs at work at one time span all tile
        // rows, so every wave re-reads A from DRAM: MXFP8 8192x8192x8192
        // read 946 MB per launch against 273 MB of A, B, scales and C.  In a
        // band of 8 rows, A's rows stay in L2 while the band's columns pass.
        // Measurement knob MXGEMM_BAND.
        pl.band = pl.tilesP < 8 ? pl.tilesP : 8;
        if (const char *e = getenv("MXGEMM_BAND"))
            if (atoi(e) > 0)
                pl.band = atoi(e) < pl.tilesP ? atoi(e) : pl.tilesP;
        const int64_t pairs = (num_sms > 0 ? num_sms : 2) / 2;
        const int64_t npairs = pl.tiles < pairs ? pl.tiles : pairs;
        pl.workers = pl.tiles;
        pl.grid = static_cast<int>(2 * npairs);
        pl.sched = 1;
        pl.kaP = sf_atoms_per_rowblock(fmt, K);
        pl.kaQ = pl.kaP;
        pl.partial_bytes = 0;
        pl.counter_bytes = 4;
        pl.tail_first = pl.tiles;
        pl.tail_split = 1;
        // Last-wave split (measurement knob MXGEMM_TAIL=1): when the last
        // wave of whole tiles would leave pairs idle, split each of its tiles
        // into up to four K ranges over them; the split tiles' FP32 partials
        // (128 KB per CTA and range) are summed by the range that finishes
        // last.  Off by default: in chained steps, where the next GEMM's CTAs
        // start on the pairs the last wave leaves idle, it measured slower
        // (MXFP4 2048x28672x8192: 4418 TFLOPS whole tiles, 3703 split).
        const char *tail = getenv("MXGEMM_TAIL");
        if (sched == 0 && tail && atoi(tail) == 1) {
            const int64_t full = pl.tiles / npairs * npairs, rest = pl.tiles - full;
            int64_t sp = rest > 0 ? npairs / rest : 1;
            sp = sp > 4 ? 4 : sp;
            sp = sp > pl.kt ? pl.kt : sp;
            if (rest > 0 && sp >= 2) {
                pl.tail_first = full;
                pl.tail_split = sp;
                pl.workers = full + rest * sp;
                pl.sched = 5;
                pl.partial_bytes = rest * sp * 2 * 128 * 256 * 4;
                pl.counter_bytes = rest * 2 * 4;
            }
        }
        pl.valid = pl.iters < (int64_t(1) << 31);
        return pl;
    }
    pl.stages = stages_for(fmt, pl.bn, pl.kc);
    pl.tilesP = (pl.P + 127) / 128;
    pl.tilesQ = (pl.Q + pl.bn - 1) / pl.bn;
    pl.kt = (chunks + pl.kc - 1) / pl.kc;
    pl.tiles = pl.tilesP * pl.tilesQ;
    pl.iters = pl.tiles * pl.kt;
    const int64_t sms = num_sms > 0 ? num_sms : 1;
    int s = sched;
    int auto_splits = 1;
    int64_t ks = 1;                    // CTAs of a cluster sharing one tile's K range
    if (s == 0) {
        // auto: decode tiles (swapped, at most 64 columns) that fill at most
        // half the GPU split each tile's K range over a cluster of 4 or 2
        // CTAs, every CTA with at least four K steps (the hand-off of the
        // partial tiles costs ~3 us, which fewer steps do not repay); the
        // partials are summed through distributed shared memory, so the
        // split costs no global round trip.  Chained steps, 64x4096x4096:
        // MXFP8 (16 K steps) 14.7 us whole, 12.4 us in clusters of 2 or 4;
        // MXFP4 (8 K steps) 11.9 us whole, 10.2 us in 2, 11.7 us in 4; BF16
        // (32 K steps) 20.2 us whole, 14.3 us in 2, 13.7 us in 4.
        if (pl.swap)
            for (int64_t c = 4; c >= 2; c /= 2)
                if (pl.tiles * c <= sms && pl.kt >= 4 * c) {
                    ks = c;
                    break;
                }
        if (ks > 1) {
            s = 4;
        } else if (pl.tiles * 4 <= sms && pl.kt >= 32) {
            // other shapes with few tiles and many K steps: a two-way split
            // with the partials summed through global memory (the dense BF16
            // 64x4096x4096 measured 18.0 against 18.9 us whole)
            s = 2;
            auto_splits = 2;
        } else {
            s = 1;
        }
    } else if (s == 4) {
        // forced cluster split: 2 or 4 CTAs per tile (3 takes 2), decode tiles
        // only, all clusters in one wave; otherwise the global-memory split
        const int64_t c = splits >= 4 ? 4 : 2;
        if (pl.swap && pl.tiles * c <= sms && pl.kt >= c) {
            ks = c;
        } else {
            s = 2;
            splits = static_cast<int>(c);
        }
    }
    if (sched == 0 && s == 2)
        splits = auto_splits;
    pl.sched = s;
    if (s == 1) {
        pl.workers = pl.tiles;
    } else if (s == 2) {
        const int64_t sp = splits < 1 ? 1 : (splits > pl.kt ? pl.kt : splits);
        pl.workers = pl.tiles * sp;
    } else if (s == 4) {
        pl.workers = pl.tiles * ks;
        pl.ksplit = ks;
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
    // the kernel's scheduler arithmetic is 32-bit: iters * workers < 2^32
    // unless whole tiles are scheduled (which needs no products)
    const int64_t lim = (int64_t(1) << 32) - 1;
    if (pl.ksplit > 1 && pl.iters * pl.workers > lim) {
        pl.ksplit = 1;                 // too long for one cluster wave's arithmetic: whole tiles
        pl.sched = 1;
        pl.workers = pl.tiles;
    }
    if (pl.workers != pl.tiles && pl.iters * pl.workers > lim) {
        const int64_t w = lim / pl.iters;
        pl.workers = w > pl.tiles ? w : pl.tiles;
        if (pl.workers != pl.tiles && pl.iters * pl.workers > lim)
            pl.workers = pl.tiles;
    }
    pl.valid = pl.iters < (int64_t(1) << 31) && pl.tiles < (int64_t(1) << 31);
    pl.grid = static_cast<int>(pl.workers < sms ? pl.workers : sms);
    pl.kaP = sf_atoms_per_rowblock(fmt, K);
    pl.kaQ = pl.kaP;
    pl.partial_bytes = (pl.workers == pl.tiles || pl.ksplit > 1) ? 0 : 2 * pl.workers * 128 * pl.bn * 4;
    pl.counter_bytes = pl.tiles * 4;
    return pl;
}

GemmPlan make_grouped_plan(int fmt, int64_t G, int64_t M_total, int64_t N, int64_t K, int num_sms)
{
    GemmPlan pl;
    pl.fmt = fmt;
    pl.M = M_total;
    pl.N = N;
    pl.K = K;
    pl.swap = 0;
    pl.pair = 0;
    pl.bn = 128;        // 128 x 256 tiles fit two ring stages only: measured slower (1157 vs 1325 TFLOPS)
    pl.P = M_total;
    pl.Q = N;
    const int64_t chunks = (row_bytes(fmt, K) + 127) / 128;
    const bool whole = row_bytes(fmt, K) % 128 == 0;
    pl.kc = (whole && chunks >= 2) ? 2 : 1;
    pl.stages = stages_for(fmt, pl.bn, pl.kc);
    pl.tilesQ = (N + pl.bn - 1) / pl.bn;
    pl.tilesP = (M_total + 127) / 128 + G;        // each group adds at most one partial row tile
    pl.kt = (chunks + pl.kc - 1) / pl.kc;
    pl.tiles = pl.tilesP * pl.tilesQ;
    pl.iters = pl.tiles * pl.kt;
    pl.workers = pl.tiles;
    pl.sched = 1;
    const int64_t sms = num_sms > 0 ? num_sms : 1;
    pl.grid = static_cast<int>(pl.tiles < sms ? pl.tiles : sms);
    pl.kaP = sf_atoms_per_rowblock(fmt, K);
    pl.kaQ = pl.kaP;
    pl.partial_bytes = 0;
    pl.counter_bytes = 4;
    pl.groups = G;
    pl.valid = pl.iters < (int64_t(1) << 31) && pl.tiles < (int64_t(1) << 31);
    return pl;
}

cudaError_t launch_gemm(const GemmPlan &plan, const GemmBuffers &buf, uint64_t wait_limit_ns, int inject, int pdl,
                        cudaStream_t stream)
{
    if (plan.pair)
        return launch_gemm_pair(plan, buf, wait_limit_ns, inject, pdl, stream);
    if (plan.fmt == kFmtMXFP8)
        return launch_gemm_mxfp8(plan, buf, wait_limit_ns, inject, pdl, stream);
    if (plan.fmt == kFmtMXFP4)
        return launch_gemm_mxfp4(plan, buf, wait_limit_ns, inject, pdl, stream);
    return launch_gemm_bf16(plan, buf, wait_limit_ns, inject, pdl, stream);
}

}  // namespace mxg
