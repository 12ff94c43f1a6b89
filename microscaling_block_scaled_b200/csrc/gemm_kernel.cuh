// gemm_kernel.cuh -- the sm_100a one-CTA GEMM kernel C = A * B^T, BF16 out,
// and its host launch template.  Included by the translation units that
// instantiate it per operand type (gemm_mxfp8.cu, gemm_mxfp4.cu,
// gemm_bf16.cu), so the instantiations compile in parallel; the CTA-pair
// kernel is in gemm_pair_kernel.cuh, the planner and dispatch in gemm.cu.
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
// Two kernels.  mx_gemm_kernel: one persistent CTA per SM, 128-row tiles.
//   warps 0, 6  TMA producers of the row / column operand tile of each stage
//               (128B-swizzled, KC 128-byte K chunks per 3-D box);
//   warps 7, 8  their scale atoms: a TMA box of the repacked layout, or, with
//               the scale conversion fused (mxgemm_run), 4-byte cp.async
//               gathers from the row-major scales;
//   warps 1, 9.. MMA warps, up to four: each owns a run of the stage's scale
//               atoms, copies them into TMEM (tcgen05.cp) and issues the
//               block-scaled MMAs (kind::mxf8f6f4 K=32 / kind::mxf4 K=64) that
//               read them into its own FP32 accumulator; its tcgen05.commit
//               counts toward releasing the stage;
//   warps 2..5  epilogue: tcgen05.ld of the accumulators, summed in FP32,
//               BF16 (RNE) through shared memory and TMA stores; for split
//               tiles an FP32 partial plus a last-arriver fixup.
// mx_gemm_pair_kernel (gemm_pair_kernel.cuh): a cluster of two CTAs per
// 256x256 tile (tcgen05.mma.cta_group::2); both CTAs' TMA copies count on
// the leader's barrier, the leader's warp 7 copies both CTAs' scale atoms and
// its warp 1 issues the MMAs.  Every instruction-issuing role has its own
// warp because a TMA or tcgen05 instruction holds the issuing thread for
// tens to hundreds of ns.
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
//
// Launch chaining (programmatic dependent launch): mx_gemm_kernel lets the
// next launch on its stream start as soon as its own CTAs are set up.  A
// launch that starts early sets up its CTA (barriers, tensor memory, tensor
// maps) while the previous kernel finishes, and every role waits for that
// kernel (griddepcontrol.wait) before it touches global memory, except the
// operand producers named in KParams::early, which may stream their operand
// into the ring first.  They wait before their first blocking ring wait, so
// no bounded wait ever spans the previous kernel's run time.
#pragma once

#include "gemm_common.cuh"

namespace mxg {

// ------------------------------------------------------------ configuration

template <int FMT, int BN, int KC>
struct Cfg {
    static constexpr int kBM = 128;
    static constexpr bool kScaled = FMT != kFmtBF16;          // MX operands carry E8M0 block scales
    // 512B scale atoms per 128-byte K chunk (BF16 operands: none)
    static constexpr int kAtomsPerChunk = FMT == kFmtMXFP8 ? 1 : (FMT == kFmtMXFP4 ? 2 : 0);
    static constexpr int kAtoms = kAtomsPerChunk * KC;        // scale atoms per 128 rows per stage
    static constexpr int kRBQ = (BN + 127) / 128;             // 128-row blocks of the column operand
    static constexpr int kAChunk = kBM * 128;                 // one 128-byte K chunk of the row-operand tile
    static constexpr int kBChunk = BN * 128;
    static constexpr int kABytes = kAChunk * KC;
    static constexpr int kBBytes = kBChunk * KC;
    static constexpr int kSFABytes = kAtoms * 512;
    static constexpr int kSFBBytes = kRBQ * kAtoms * 512;
    static constexpr int kStageBytes = kABytes + kBBytes + kSFABytes + kSFBBytes;
    static constexpr int kCW = BN < 32 ? BN : 32;             // accumulator columns per epilogue chunk
    // Output staging for TMA stores: two BF16 chunks of the 128-row tile.
    // Tiles of at most 32 columns (decode, M <= 32) have none of their own
    // and give the space to a fifth ring stage: a CTA's final tile stages its
    // output in the then idle first ring stage, an earlier one stores from
    // registers.
    static constexpr bool kStaged = BN > 32;
    static constexpr int kChunkOutBytes = 128 * kCW * 2;      // one BF16 output chunk
    static constexpr int kOutBytes = kStaged ? kChunkOutBytes : 0;
    static constexpr int kSmemBudget = 227 * 1024 - 2048 - 2 * kOutBytes;
    static constexpr int kStagesRaw = kSmemBudget / kStageBytes;
    static constexpr int kStages = kStagesRaw > 12 ? 12 : kStagesRaw;
    static constexpr int kSFACols = kAtoms * 4;
    static constexpr int kSFBCols = kRBQ * kAtoms * 4;
    static constexpr int kSFCols = kStages * (kSFACols + kSFBCols);
    // A tcgen05 instruction holds its issuing thread ~40 ns, so a stage's
    // scale copies and MMAs are split over kNMma MMA warps, each with its own
    // accumulator (summed by the epilogue).  Warp m owns a contiguous run of
    // the stage's work units -- scale atoms for MX operands, 128-byte K
    // chunks for BF16 ones: it copies their scales and issues exactly the
    // MMAs that read them, so no warp's MMA depends on another warp's copy.
    // Narrow (decode) tiles take up to four warps where TMEM holds one
    // accumulator set; wider ones keep two accumulator sets.
    static constexpr int kMmaPerAtom = FMT == kFmtMXFP8 ? 4 : 2;   // MMAs reading one 512B atom
    static constexpr int kUnits = kScaled ? kAtoms : KC;
    static constexpr int kMmaPerUnit = kScaled ? kMmaPerAtom : 4;  // BF16: K = 16 (32 bytes) per MMA
    static constexpr int pick_nmma()
    {
        for (int nm = 4; nm > 1; nm /= 2)
            if (kUnits % nm == 0 && (BN <= 64 ? nm * BN : 2 * nm * BN) + kSFCols <= 512)
                return nm;
        return 1;
    }
    static constexpr int kNMma = pick_nmma();
    static constexpr int kUnitsPerMma = kUnits / kNMma;
    static constexpr int kNumAcc = (2 * kNMma * BN + kSFCols <= 512) ? 2 : 1;
    static constexpr int kAccCols = kNumAcc * kNMma * BN;
    static constexpr int kTmemCols = 512;
    // warps: 0 row-operand TMA, 1 MMA, 2..5 epilogue, 6 column-operand TMA,
    // 7 row-scale TMA, 8 column-scale TMA, 9.. further MMA warps
    static constexpr int kWarps = 9 + kNMma - 1;
    static constexpr int kThreads = 32 * kWarps;
    static constexpr int kMmaPerChunk = 4;                    // 32 bytes of K per MMA
    static constexpr uint32_t kTxBytes = kStageBytes;
    // shared memory layout (offsets from a 1024-aligned base)
    static constexpr int kOffA = 0;
    static constexpr int kOffB = kOffA + kStages * kABytes;
    static constexpr int kOffSFA = kOffB + kStages * kBBytes;
    static constexpr int kOffSFB = kOffSFA + kStages * kSFABytes;
    static constexpr int kOffOut = (kOffSFB + kStages * kSFBBytes + 1023) / 1024 * 1024;
    static constexpr int kOffBar = kOffOut + 2 * kOutBytes;
    // Cluster K split (decode tiles, BN <= 64): rank r of a cluster of S = 2
    // or 4 CTAs owns the tile rows of 4/S of the epilogue warps' 32-row TMEM
    // lane quarters.  The other ranks ship their partials of those rows into
    // its drained ring (FP32, 16-byte column groups: group g of quarter row i
    // at (g * 32 + i) * 16): incoming quarters from kRedOff (slot s, quarter
    // j at (s * 4/S + j) * kQuadBytes), this rank's outgoing quarters from
    // kRedOut, per-quarter output staging (two chunks each) from kRedStage.
    static constexpr int kRedOff = kOffA + 16384;
    static constexpr int kQuadBytes = 32 * BN * 4;
    static constexpr int kRedOut = kRedOff + 3 * kQuadBytes;
    static constexpr int kRedStage = kRedOut + 4 * kQuadBytes;
    static constexpr int kQStageBytes = BN * 32 * 2;          // a lane quarter's [BN][32] BF16 output
    static constexpr bool kCanKsplit = BN <= 64;
    static constexpr int kNumBars = 2 * kStages + 2 * kNumAcc + 3;   // + drain, go-ahead, reduction
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kSmemBytes = kOffMisc + 64 + 1024;   // + alignment slack

    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N must be a multiple of 16 in [16, 256]");
    static_assert(KC == 1 || KC == 2 || KC == 4, "1, 2 or 4 K chunks per stage");
    static_assert(kStages >= 2, "at least two pipeline stages");
    static_assert(kAccCols + kSFCols <= kTmemCols, "TMEM budget");
    static_assert(kBChunk % 1024 == 0, "tiles must keep 1024-byte alignment");
    static_assert(kStaged || 2 * kChunkOutBytes <= kABytes, "ring stage 0 holds two output chunks");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
    static_assert(!kCanKsplit || kRedStage + 4 * kQStageBytes <= kOffOut, "cluster split buffers fit the ring");
    static_assert(!kCanKsplit || kRedOff + BN * 128 * 4 <= kOffOut, "a staged FP32 decode tile fits the ring");
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

// Instruction descriptor of the dense BF16 MMA (PTX ISA, instruction
// descriptor for .kind::f16): D type F32 (1) at bits [4,6), A and B type
// BF16 (1) at [7,10) and [10,13), both K-major, N >> 3 at [17,23), M >> 4 at
// [24,29).
template <int BN>
__host__ __device__ constexpr uint32_t idesc_bf16()
{
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
           (static_cast<uint32_t>(128 >> 4) << 24);
}



// Where one output tile lives: rows [prow, prow+128) of the row operand
// (valid below plim), rows [qrow, qrow+BN) of the column operand (valid
// below qlim) and its first output column (C column for the plain layout, C
// row for the swapped one).
struct TileCoord {
    int64_t prow, plim, qrow, qlim, qcol;
};

// Tile walk of a grouped GEMM.  Tiles are numbered group by group; inside
// a group the 128-row index runs fastest.  A walk only moves forward: seek()
// takes non-decreasing tile numbers, as every role's loop produces them.
// Offsets read from memory are clamped to [0, rows] and a group whose end
// lies before its start is empty, so no offset can send an access out of
// bounds.  init() reads no memory: the offsets may be written by the kernel
// this one follows, so the first read happens in seek(), which every role
// calls only after its dependency wait.
struct GroupWalk {
    const int64_t *off;
    int64_t rows;          // rows of A and C in all
    int64_t n;             // columns of C (rows of B per group)
    uint32_t groups, tilesQ, bn;
    uint32_t g, gfirst, gtiles, gmt;
    int64_t r0, r1;
    bool started;
    __device__ __forceinline__ int64_t clampr(int64_t v) const { return v < 0 ? 0 : (v > rows ? rows : v); }
    __device__ __forceinline__ void load()
    {
        r0 = clampr(off[g]);
        r1 = clampr(off[g + 1]);
        if (r1 < r0)
            r1 = r0;
        gmt = static_cast<uint32_t>((r1 - r0 + 127) / 128);
        gtiles = gmt * tilesQ;
    }
    __device__ __forceinline__ void init(const int64_t *off_, int64_t rows_, int64_t n_, uint32_t groups_,
                                         uint32_t tilesQ_, uint32_t bn_)
    {
        off = off_;
        rows = rows_;
        n = n_;
        groups = groups_;
        tilesQ = tilesQ_;
        bn = bn_;
        g = 0;
        gfirst = 0;
        gtiles = 0;
        gmt = 0;
        r0 = r1 = 0;
        started = false;
    }
    // Position the walk on tile t; false once t lies past the last group.
    __device__ __forceinline__ bool seek(uint32_t t)
    {
        if (!started) {
            started = true;
            load();
        }
        while (t - gfirst >= gtiles) {
            gfirst += gtiles;
            if (++g >= groups)
                return false;
            load();
        }
        return true;
    }
    __device__ __forceinline__ TileCoord coord(uint32_t t) const
    {
        const uint32_t l = t - gfirst, tq = l / gmt, mt = l - tq * gmt;
        TileCoord c;
        c.prow = r0 + static_cast<int64_t>(mt) * 128;
        c.plim = r1;
        c.qrow = static_cast<int64_t>(g) * n + static_cast<int64_t>(tq) * bn;
        c.qlim = static_cast<int64_t>(g) * n + n;
        c.qcol = static_cast<int64_t>(tq) * bn;
        return c;
    }
};

// Coordinates of tile t of a plain (ungrouped) GEMM.
__device__ __forceinline__ TileCoord plain_coord(const KParams &kp, uint32_t t, int bn)
{
    const uint32_t tq = t / kp.tilesP, tp = t - tq * kp.tilesP;
    TileCoord c;
    c.prow = static_cast<int64_t>(tp) * 128;
    c.plim = kp.P;
    c.qrow = static_cast<int64_t>(tq) * bn;
    c.qlim = kp.Q;
    c.qcol = c.qrow;
    return c;
}



// Work decomposition shared by the three roles.  All index arithmetic is
// 32-bit (64-bit integer division is a long software sequence on the GPU and
// sat on the critical path of every hand-off); whole-tile schedules take a
// division-free path.
struct Sched {
    uint32_t I, W, KT, tilesP;
    bool dp;
    // first K-iteration of worker g: floor(g * I / W)
    __device__ __forceinline__ uint32_t begin(uint32_t g) const { return dp ? g * KT : (g * I) / W; }
    // worker owning K-iteration i: the largest g with begin(g) <= i
    __device__ __forceinline__ uint32_t owner(uint32_t i) const { return dp ? i / KT : ((i + 1) * W - 1) / I; }
};

// Walks the K-iterations of the workers a CTA owns (blockIdx.x, +gridDim.x,
// ...) in order, tracking the tile and its K step incrementally.
struct IterCursor {
    Sched sc;
    uint32_t w, step;
    uint32_t it, end, tile, k;
    __device__ __forceinline__ IterCursor(const Sched &sc_, uint32_t first, uint32_t step_)
        : sc(sc_), w(first), step(step_), it(0), end(0), tile(0), k(0)
    {
        enter();
    }
    __device__ __forceinline__ void enter()
    {
        while (w < sc.W) {
            it = sc.begin(w);
            end = sc.begin(w + 1);
            if (it < end)
                break;
            w += step;
        }
        if (w < sc.W) {
            tile = sc.dp ? w : it / sc.KT;
            k = it - tile * sc.KT;
        }
    }
    __device__ __forceinline__ bool valid() const { return w < sc.W; }
    __device__ __forceinline__ void advance()
    {
        ++it;
        if (it >= end) {
            w += step;
            enter();
            return;
        }
        if (++k == sc.KT) {
            k = 0;
            ++tile;
        }
    }
    __device__ __forceinline__ uint32_t total() const
    {
        uint32_t n = 0;
        for (uint32_t g = w; g < sc.W; g += step)
            n += sc.begin(g + 1) - sc.begin(g);
        return n;
    }
};

// One maximal run of a worker's K-iterations inside one tile.
struct Segment {
    uint32_t tile, kb, ke, tp, tq;
};

__device__ __forceinline__ Segment segment_at(const Sched &sc, uint32_t it, uint32_t end)
{
    Segment g;
    g.tile = it / sc.KT;
    g.kb = it - g.tile * sc.KT;
    g.ke = (g.kb + (end - it) < sc.KT) ? g.kb + (end - it) : sc.KT;
    g.tq = g.tile / sc.tilesP;
    g.tp = g.tile - g.tq * sc.tilesP;
    return g;
}



// Store CW FP32 values as BF16 into C.  Non-swapped: thread's row p = C row,
// values are C[p][q0 .. q0+CW).  Swapped: thread's row p = C column, values
// are C[q0 .. q0+CW)[p].
struct OutView {
    __nv_bfloat16 *C;
    int64_t ldc, P, Q;
    int swap;
};

template <int CW>
__device__ __forceinline__ void store_bf16(const OutView o, int64_t p, int64_t q0, const float (&v)[CW])
{
    if (p >= o.P)
        return;
    if (!o.swap) {
        __nv_bfloat16 *dst = o.C + p * o.ldc + q0;
        const int64_t nvalid = o.Q - q0;
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
            if (q < o.Q)
                o.C[q * o.ldc + p] = __float2bfloat16_rn(v[j]);
        }
    }
}



// The fused activations in FP32: ReLU, SiLU x * sigmoid(x) (as x / (1 +
// e^-x) for x >= 0 and x e^x / (1 + e^x) below, so no intermediate
// overflows), GELU x * Phi(x) with Phi(x) = erfc(-x / sqrt 2) / 2 (no
// cancellation in the negative tail).  NaN passes through all three.
__device__ __forceinline__ float act_relu(float x) { return x < 0.0f ? 0.0f : x; }

__device__ __forceinline__ float act_silu(float x)
{
    if (x >= 0.0f)
        return __fdiv_rn(x, __fadd_rn(1.0f, expf(-x)));
    const float e = expf(x);
    return __fdiv_rn(__fmul_rn(x, e), __fadd_rn(1.0f, e));
}

__device__ __forceinline__ float act_gelu(float x)
{
    return __fmul_rn(__fmul_rn(0.5f, x), erfcf(__fmul_rn(x, -0.70710678118654752f)));
}

struct EpiOps {
    const uint16_t *bias, *residual;
    int act, swap;
    int64_t P, Q, ldc;
};

// act(v + b) + r on four values at a time, out of line: eight calls of one
// four-wide copy instead of 32 inlined ones (the same speed -- the time goes
// to the arithmetic on four epilogue warps, not to fetching its code -- in
// half the build time).  The four values are independent chains, and they
// travel in registers (no local arrays, no register saves around a call
// holding arrays).
struct Val4 {
    float a, b, c, d;
};

template <int ACT>
static __device__ __noinline__ Val4 ops4(Val4 v, float bias, Val4 bv, Val4 r, int has_bias, int has_res)
{
    float x[4] = {v.a, v.b, v.c, v.d};
    const float bb[4] = {bv.a, bv.b, bv.c, bv.d};
    const float rr[4] = {r.a, r.b, r.c, r.d};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float y = has_bias ? __fadd_rn(x[j], bias + bb[j]) : x[j];
        y = ACT == 1 ? act_relu(y) : (ACT == 2 ? act_silu(y) : (ACT == 3 ? act_gelu(y) : y));
        x[j] = has_res ? __fadd_rn(y, rr[j]) : y;
    }
    return Val4{x[0], x[1], x[2], x[3]};
}

// Fused operations on cw (<= 32) values of C held by one thread: v =
// act(v + bias[n]) + residual[m][n], each step rounded to FP32.  Plain
// layout: the thread holds row m = p, columns n = q0 + j (valid below Q);
// swapped: column n = p (valid below P), rows m = q0 + j (valid below Q).
// Values outside C are left alone.  All bias and residual loads are issued
// before any arithmetic (unrolled: they are few instructions); the
// arithmetic runs four values per call of ops4.
__device__ __forceinline__ void apply_epilogue_ops(float (&v)[32], int cw, const EpiOps e, int64_t p, int64_t plim,
                                                   int64_t q0)
{
    float b[32], r[32];
    float bp = 0.0f;                     // swapped layout: one bias per thread (column n = p)
    int64_t nv;
    if (!e.swap) {
        if (p >= plim)
            return;
        nv = e.Q - q0 < cw ? e.Q - q0 : cw;
        const uint16_t *res = e.residual ? e.residual + p * e.ldc + q0 : nullptr;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            b[j] = (e.bias && j < nv) ? bf16_bits_to_float(e.bias[q0 + j]) : 0.0f;
            r[j] = (res && j < nv) ? bf16_bits_to_float(res[j]) : 0.0f;
        }
    } else {
        if (p >= e.P)
            return;
        nv = e.Q - q0 < cw ? e.Q - q0 : cw;
        bp = e.bias ? bf16_bits_to_float(e.bias[p]) : 0.0f;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            b[j] = 0.0f;
            r[j] = (e.residual && j < nv) ? bf16_bits_to_float(e.residual[(q0 + j) * e.ldc + p]) : 0.0f;
        }
    }
    const int hb = e.bias != nullptr, hr = e.residual != nullptr;
#pragma unroll
    for (int g = 0; g < 32; g += 4) {
        if (g < nv) {
            const Val4 in{v[g], v[g + 1], v[g + 2], v[g + 3]};
            const Val4 bv{b[g], b[g + 1], b[g + 2], b[g + 3]};
            const Val4 rv{r[g], r[g + 1], r[g + 2], r[g + 3]};
            Val4 o;
            switch (e.act) {
            case 1: o = ops4<1>(in, bp, bv, rv, hb, hr); break;
            case 2: o = ops4<2>(in, bp, bv, rv, hb, hr); break;
            case 3: o = ops4<3>(in, bp, bv, rv, hb, hr); break;
            default: o = ops4<0>(in, bp, bv, rv, hb, hr); break;
            }
            // values past the valid count keep their (unused) input
            v[g] = g < nv ? o.a : v[g];
            v[g + 1] = g + 1 < nv ? o.b : v[g + 1];
            v[g + 2] = g + 2 < nv ? o.c : v[g + 2];
            v[g + 3] = g + 3 < nv ? o.d : v[g + 3];
        }
    }
}

struct QOut {
    uint8_t *Cq, *Cs;
    int64_t ldc;           // N
    int qfmt;
};

static __device__ __forceinline__ void quantise_store_plain(const float *vin, const QOut kp, int64_t p, int64_t q0)
{
    float v[32];
    uint32_t amax = 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        v[j] = __bfloat162float(__float2bfloat16_rn(vin[j]));
        amax = max(amax, __float_as_uint(v[j]) & 0x7FFFFFFFu);
    }
    float inv;
    const uint32_t sb = kp.qfmt == kFmtMXFP8 ? mx_block_scale<8>(amax, &inv) : mx_block_scale<2>(amax, &inv);
    uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    if (kp.qfmt == kFmtMXFP8) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const float q = sb == 0xFFu ? 0.0f : __fmul_rn(v[j], inv);
            w[j / 4] |= cvt_e4m3(q) << (8 * (j % 4));
        }
        uint4 *dst = reinterpret_cast<uint4 *>(kp.Cq + p * kp.ldc + q0);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float lo = sb == 0xFFu ? 0.0f : __fmul_rn(v[2 * j], inv);
            const float hi = sb == 0xFFu ? 0.0f : __fmul_rn(v[2 * j + 1], inv);
            w[j / 4] |= cvt_e2m1x2(hi, lo) << (8 * (j % 4));
        }
        *reinterpret_cast<uint4 *>(kp.Cq + p * (kp.ldc / 2) + q0 / 2) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    kp.Cs[p * (kp.ldc / 32) + q0 / 32] = static_cast<uint8_t>(sb);
}

// Quantised output, swapped layout: the 32 lanes of the calling warp hold
// C[m][n] for 32 consecutive n (n = p of each lane, the first a multiple of
// 32) and rows m = m0 .. m0 + nm - 1 (values vin[j], nm <= 32); for each row
// the 32 lanes form one run.  All 32 lanes must call with the same m0 and
// nm.  Unrolled over the rows so their reductions and conversions overlap;
// inlined like apply_epilogue_ops (quantised decode step 18.4 -> 16.1 us).
static __device__ __forceinline__ void quantise_store_swapped(const float *vin, int nm, const QOut kp, int64_t p,
                                                           int64_t m0, int lane)
{
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j)
        v[j] = j < nm ? __bfloat162float(__float2bfloat16_rn(vin[j])) : 0.0f;
    uint32_t amax[32];
#pragma unroll
    for (int j = 0; j < 32; ++j)
        amax[j] = __reduce_max_sync(0xffffffffu, __float_as_uint(v[j]) & 0x7FFFFFFFu);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        if (j < nm) {
            const int64_t m = m0 + j;
            float inv;
            const uint32_t sb =
                kp.qfmt == kFmtMXFP8 ? mx_block_scale<8>(amax[j], &inv) : mx_block_scale<2>(amax[j], &inv);
            const float q = sb == 0xFFu ? 0.0f : __fmul_rn(v[j], inv);
            if (kp.qfmt == kFmtMXFP8) {
                kp.Cq[m * kp.ldc + p] = static_cast<uint8_t>(cvt_e4m3(q));
            } else {
                const float hi = __shfl_down_sync(0xffffffffu, q, 1);
                if ((lane & 1) == 0)
                    kp.Cq[m * (kp.ldc / 2) + p / 2] = static_cast<uint8_t>(cvt_e2m1x2(hi, q));
            }
            if (lane == 0)
                kp.Cs[m * (kp.ldc / 32) + p / 32] = static_cast<uint8_t>(sb);
        }
    }
}

// One row of quantised output, swapped layout: the 32 lanes of the calling
// warp hold C[m][n] for 32 consecutive n (n = p, the first a multiple of 32);
// all lanes call with the same m (lanes with n past N pass valid = false and
// a zero value).  The same rule as quantise_store_swapped.
__device__ __forceinline__ void quantise_row_swapped(float vin, const QOut &kp, int64_t m, int64_t p, int lane,
                                                     bool valid)
{
    const float v = __bfloat162float(__float2bfloat16_rn(vin));
    const uint32_t amax = __reduce_max_sync(0xffffffffu, __float_as_uint(v) & 0x7FFFFFFFu);
    float inv;
    const uint32_t sb = kp.qfmt == kFmtMXFP8 ? mx_block_scale<8>(amax, &inv) : mx_block_scale<2>(amax, &inv);
    const float q = sb == 0xFFu ? 0.0f : __fmul_rn(v, inv);
    if (kp.qfmt == kFmtMXFP8) {
        if (valid)
            kp.Cq[m * kp.ldc + p] = static_cast<uint8_t>(cvt_e4m3(q));
    } else {
        const float hi = __shfl_down_sync(0xffffffffu, q, 1);
        if ((lane & 1) == 0 && valid)
            kp.Cq[m * (kp.ldc / 2) + p / 2] = static_cast<uint8_t>(cvt_e2m1x2(hi, q));
    }
    if (lane == 0)
        kp.Cs[m * (kp.ldc / 32) + p / 32] = static_cast<uint8_t>(sb);
}

template <int FMT, int BN, int KC>
__global__ void __launch_bounds__(Cfg<FMT, BN, KC>::kThreads, 1)
    mx_gemm_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmQ,
                   const __grid_constant__ CUtensorMap tmSP, const __grid_constant__ CUtensorMap tmSQ,
                   const __grid_constant__ CUtensorMap tmC, const KParams kp_in)
{
    using C_ = Cfg<FMT, BN, KC>;
    constexpr int S = C_::kStages;
    constexpr int CW = C_::kCW;
    constexpr int NM = C_::kNMma;

    // Work on a register copy of the parameters: the inline-asm memory
    // clobbers of the pipeline would otherwise force reloads from parameter
    // space after each TMA / MMA / barrier instruction.
    const KParams kp = kp_in;

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
    const uint32_t go_bar = drain_bar + 8u;       // cluster K split: every other rank's ring is free
    const uint32_t red_bar = drain_bar + 16u;     // cluster K split: the other ranks' partials are in
    volatile uint32_t *s_tmem = reinterpret_cast<volatile uint32_t *>(smem + C_::kOffMisc);
    volatile int *s_abort = reinterpret_cast<volatile int *>(smem + C_::kOffMisc + 4);
    volatile int *s_last = reinterpret_cast<volatile int *>(smem + C_::kOffMisc + 8);

    if (blockDim.x != C_::kThreads) {
        if (threadIdx.x == 0)
            atomicCAS(kp.error, 0, kErrLaunch);
        return;
    }
    // Every wait in this kernel parks the thread in the suspending try_wait
    // at once: the producer and MMA warps share SM sub-partitions, and a
    // warp spinning on test_wait would take issue slots from an MMA warp.
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const bool producer = warp == 0 || warp == 6 || (C_::kScaled && (warp == 7 || warp == 8));
    const int mma_idx = warp == 1 ? 0 : (warp >= 9 ? warp - 8 : -1);

    // Each producer fetches its own tensor map while the CTA sets up.
    if (lane == 0) {
        if (warp == 0)
            tma_prefetch_desc(&tmP);
        else if (warp == 6)
            tma_prefetch_desc(&tmQ);
        else if (warp == 7 && C_::kScaled)
            tma_prefetch_desc(&tmSP);
        else if (warp == 8 && C_::kScaled)
            tma_prefetch_desc(&tmSQ);
        else if (warp == 2)
            tma_prefetch_desc(&tmC);
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            // one arming per producer warp; with fused scales, one async
            // arrival per lane of the two scale warps; BF16 operands have
            // only the two operand producers
            mbar_init(full_bar(s), !C_::kScaled ? 2 : (kp.fused_sf ? 2 + 64 : 4));
            mbar_init(empty_bar(s), NM);        // one commit per MMA warp
        }
        for (int a = 0; a < C_::kNumAcc; ++a) {
            mbar_init(accf_bar(a), NM);
            mbar_init(acce_bar(a), 4);
        }
        mbar_init(drain_bar, NM);
        mbar_init(go_bar, kp.ksplit > 1 ? kp.ksplit - 1 : 1);
        mbar_init(red_bar, 1);
        *s_abort = 0;
        *s_last = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (C_::kScaled && BN < 128 && kp.fused_sf) {
        // rows of the column operand's scale atoms that no stage writes (see
        // the gather): zero once, by every thread, before the setup barrier
        uint32_t *z = reinterpret_cast<uint32_t *>(smem + C_::kOffSFB);
        for (int i = threadIdx.x; i < S * C_::kSFBBytes / 4; i += C_::kThreads)
            z[i] = 0u;
    }
    if (warp == 1) {
        tmem_alloc(sbase + C_::kOffMisc, C_::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    // A cluster K split signals between CTAs: every barrier must be
    // initialised before any CTA of the cluster can arrive on it.
    if (kp.ksplit > 1)
        cluster_sync_all();
    bool cl_arrived = false;          // this thread's arrival on the final cluster barrier

    const Sched sc{kp.iters, kp.workers, kp.kt, kp.tilesP, kp.dp != 0};
    const uint32_t W = sc.W;
    // Grouped plans walk their tiles through the group offsets (each role its
    // own walk, all in the same order); plain plans compute them directly.
    const bool grouped = kp.goff != nullptr;
    // Decode tiles with fused operations or quantised output, one tile per
    // CTA: on that tile the epilogue warps only stage the FP32 accumulator in
    // the drained ring, and every warp of the CTA -- the producers and MMA
    // warps are idle by then -- shares the operations and the stores (the
    // same decision in every warp, from the parameters alone).
    const bool spread = C_::kCanKsplit && kp.swap && sc.dp && W <= gridDim.x && !grouped && kp.ksplit <= 1 &&
                        (kp.has_ops || kp.qfmt >= 0);
    GroupWalk walk;
    if (grouped)
        walk.init(kp.goff, kp.P, kp.Q, kp.groups, kp.tilesQ, BN);
    auto coord_of = [&](uint32_t t) { return grouped ? walk.coord(t) : plain_coord(kp, t, BN); };
    // The CTA is set up: a programmatic dependent launch may start.
    grid_launch_dependents();

    if (producer && kp.fused_sf && warp >= 7) {
        // ------------------------------------- scale atoms gathered directly
        // Warp 7 (row operand) and warp 8 (column operand) build each stage's
        // scale atoms in shared memory from the row-major scales: atom a of a
        // 128-row block holds, for row r and K block 4a + j, the byte at
        // (r % 32) * 16 + (r / 32) * 4 + j.  Lane l moves rows l, l+32, l+64,
        // l+96 with 4-byte cp.async copies (rows past the operand and K
        // blocks past K are zero-filled) and arrives on the stage's full
        // barrier once its copies have landed.
        const bool sideP = warp == 7;
        // the column operand of a tile narrower than 128 rows has scales in
        // only its first BN rows of the atom: 32-row groups past them stay
        // zero from setup instead of being zero-filled on every stage
        constexpr int kGatherQ = BN >= 128 ? 4 : (BN + 31) / 32;
        const uint8_t *raw = sideP ? kp.rawP : kp.rawQ;
        const uint32_t bytes = sideP ? C_::kSFABytes : C_::kSFBBytes;
        const uint32_t off = sideP ? C_::kOffSFA : C_::kOffSFB;
        const int nrb = sideP ? 1 : C_::kRBQ;
        const int64_t kblocks = kp.ldS;
        // scales of an early operand: gathered ahead until the ring is full
        bool dep_pending = (kp.early & (sideP ? 1 : 2)) != 0;
        if (!dep_pending)
            grid_dependency_wait();
        uint32_t issued = 0;
        int s = 0;
        uint32_t ph = 0;
        for (IterCursor cur(sc, blockIdx.x, gridDim.x); cur.valid(); cur.advance()) {
            if (dep_pending && issued == static_cast<uint32_t>(S)) {
                grid_dependency_wait();
                dep_pending = false;
            }
            if (grouped && !walk.seek(cur.tile))
                break;
            ++issued;
            int good = 1;
            if (lane == 0)
                good = mbar_wait_parked(empty_bar(s), ph ^ 1u, s_abort, kp.limit_ns);
            good = __shfl_sync(0xffffffffu, good, 0);
            if (!good) {
                if (lane == 0)
                    record_error(kp.error, kErrProducerEmpty, s_abort);
                break;
            }
            // the tile's rows: its own 128 rows of the row operand; for the
            // column operand the 128-row blocks holding its BN rows (a swapped
            // tile narrower than 128 has only tile 0 along that side)
            const TileCoord tc = coord_of(cur.tile);
            const int64_t row0 = sideP ? tc.prow : (BN < 128 ? 0 : tc.qrow);
            const int64_t nrows = sideP ? tc.plim : tc.qlim;
            const int64_t kb0 = static_cast<int64_t>(cur.k) * C_::kAtoms * 4;
            const uint32_t dst0 = sbase + off + s * bytes + lane * 16;
            for (int rb = 0; rb < nrb; ++rb) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if (!sideP && i >= kGatherQ)
                        break;          // rows of the atom past the tile: zero since setup
                    const int64_t row = row0 + rb * 128 + i * 32 + lane;
                    const bool rv = row < nrows;
#pragma unroll
                    for (int a = 0; a < C_::kAtoms; ++a) {
                        const int64_t kb = kb0 + 4 * a;
                        const bool v = rv && kb < kblocks;
                        cp_async_4(dst0 + (rb * C_::kAtoms + a) * 512 + i * 4, v ? raw + row * kblocks + kb : raw,
                                   v ? 4u : 0u);
                    }
                }
            }
            cp_async_arrive_noinc(full_bar(s));
            if (++s == S) {
                s = 0;
                ph ^= 1u;
            }
        }
        cp_async_wait_all();
        __syncwarp();
    } else if (producer) {
        // ----------------------------------------------------- TMA producers
        // Four producer warps, one TMA operation each per stage: warp 0 the
        // MMA row-operand tile, warp 6 the column-operand tile, warps 7 and 8
        // their scale atoms.  Issuing a TMA operation occupies the issuing
        // thread for ~0.1-0.15 us, so one thread per operation keeps the
        // ring's refill off the critical path.  An operand named in
        // KParams::early fills the ring before the producer waits for the
        // prerequisite grid; everything else waits first.
        // L2 policy: in the swapped (decode) form the weights stream through
        // once and the small activation is re-read by every tile; otherwise
        // both operands are re-read across tiles.
        if (lane == 0) {
            const bool sideP = warp == 0 || warp == 7;
            const bool scales = warp >= 7;
            const uint64_t pol = sideP ? (kp.swap ? policy_evict_first() : policy_evict_normal())
                                       : (kp.swap ? policy_evict_last() : policy_evict_normal());
            const uint32_t bytes = scales ? (sideP ? C_::kSFABytes : C_::kSFBBytes)
                                          : (sideP ? C_::kABytes : C_::kBBytes);
            const uint32_t off = scales ? (sideP ? C_::kOffSFA : C_::kOffSFB) : (sideP ? C_::kOffA : C_::kOffB);
            bool dep_pending = !scales && (kp.early & (sideP ? 1 : 2)) != 0;
            if (!dep_pending)
                grid_dependency_wait();
            uint32_t armed = 0;         // stages armed so far (round-robin over the ring)
            int skipped_stage = -1;
            bool inject = warp == 0 && kp.inject == 1;
            int s = 0;
            uint32_t ph = 0;
            for (IterCursor cur(sc, blockIdx.x, gridDim.x); cur.valid(); cur.advance()) {
                if (dep_pending && armed == static_cast<uint32_t>(S)) {
                    grid_dependency_wait();
                    dep_pending = false;
                }
                if (grouped && !walk.seek(cur.tile))
                    break;
                if (!mbar_wait_parked(empty_bar(s), ph ^ 1u, s_abort, kp.limit_ns)) {
                    record_error(kp.error, kErrProducerEmpty, s_abort);
                    break;
                }
                const TileCoord tc = coord_of(cur.tile);
                const uint32_t fb = full_bar(s);
                const uint32_t dst = sbase + off + s * bytes;
                if (inject) {
                    inject = false;             // test hook: leave this stage unarmed
                    skipped_stage = s;
                } else {
                    mbar_arrive_expect_tx(fb, bytes);
                    if (warp == 0) {
                        const int32_t row = static_cast<int32_t>(tc.prow);
                        if constexpr (KC == 1)      // 2-D maps: x = byte offset along K
                            tma_load_2d(dst, &tmP, static_cast<int32_t>(cur.k * 128), row, fb, pol);
                        else                        // 3-D maps: {byte in chunk, row, 128-byte K chunk}
                            tma_load_3d(dst, &tmP, 0, row, static_cast<int32_t>(cur.k * KC), fb, pol);
                    } else if (warp == 6) {
                        const int32_t row = static_cast<int32_t>(tc.qrow);
                        if constexpr (KC == 1)
                            tma_load_2d(dst, &tmQ, static_cast<int32_t>(cur.k * 128), row, fb, pol);
                        else
                            tma_load_3d(dst, &tmQ, 0, row, static_cast<int32_t>(cur.k * KC), fb, pol);
                    } else if (warp == 7) {         // repacked scales: plain plans only
                        tma_load_3d(dst, &tmSP, 0, static_cast<int32_t>(cur.k * C_::kAtoms),
                                    static_cast<int32_t>(tc.prow / 128), fb, pol);
                    } else {
                        tma_load_3d(dst, &tmSQ, 0, static_cast<int32_t>(cur.k * C_::kAtoms),
                                    static_cast<int32_t>(tc.qrow / 128), fb, pol);
                    }
                }
                ++armed;
                if (++s == S) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            // Let every armed copy land before the CTA can exit: wait for the
            // latest armed phase of each stage (already complete on the normal
            // path, where the MMA warps consumed every stage).
            for (int st = 0; st < S; ++st) {
                const uint32_t n = armed / S + (static_cast<uint32_t>(st) < armed % S ? 1u : 0u);
                if (n == 0 || (st == skipped_stage && n == 1))
                    continue;
                const uint32_t parity = static_cast<uint32_t>((n - 1) & 1);
                int dummy_abort = 0;
                if (!mbar_wait_parked(full_bar(st), parity, &dummy_abort, kp.limit_ns))
                    atomicCAS(kp.error, 0, kErrDrain);
            }
        }
        __syncwarp();
    } else if (mma_idx >= 0) {
        // ------------------------------------------------------ MMA issuers
        // MMA warp m takes work units [m * kUnitsPerMma, (m + 1) * kUnitsPerMma)
        // of every stage -- scale atoms with their scale copies into TMEM and
        // block-scaled MMAs, or for BF16 operands whole 128-byte K chunks --
        // into its own accumulator.  Each commit releases the stage once that
        // warp's MMAs have read it; the stage is free after all NM commits.
        constexpr uint32_t kIdesc = C_::kScaled ? idesc_base<FMT, BN>() : idesc_bf16<BN>();
        const uint32_t t_sfa0 = tmem + C_::kAccCols;
        const uint32_t t_sfb0 = t_sfa0 + S * C_::kSFACols;
        const int a_begin = mma_idx * C_::kUnitsPerMma;
        grid_dependency_wait();
        int s = 0;
        uint32_t ph = 0;
        int acc = 0;
        uint32_t acc_ph = 0;
        bool ok = true;
        for (uint32_t w = blockIdx.x; w < W && ok; w += gridDim.x) {
            if (grouped && !walk.seek(w))
                break;
            uint32_t it = sc.begin(w);
            const uint32_t end = sc.begin(w + 1);
            while (it < end && ok) {
                const Segment sg = segment_at(sc, it, end);
                const uint32_t kb = sg.kb, ke = sg.ke;
                int good = 1;
                if (lane == 0)
                    good = mbar_wait_parked(acce_bar(acc), acc_ph ^ 1u, s_abort, kp.limit_ns);
                good = __shfl_sync(0xffffffffu, good, 0);
                if (!good) {
                    if (lane == 0)
                        record_error(kp.error, kErrMmaAccEmpty, s_abort);
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t t_acc = tmem + (acc * NM + mma_idx) * BN;
                for (uint32_t k = kb; k < ke; ++k) {
                    good = 1;
                    if (lane == 0)
                        good = mbar_wait_parked(full_bar(s), ph, s_abort, kp.limit_ns);
                    good = __shfl_sync(0xffffffffu, good, 0);
                    if (!good) {
                        if (lane == 0)
                            record_error(kp.error, kErrMmaFull, s_abort);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (lane == 0) {
                        if constexpr (C_::kScaled) {
                            if (kp.fused_sf)        // scale atoms written by cp.async (generic proxy)
                                fence_proxy_async_smem();
                            const uint32_t t_sfa = t_sfa0 + s * C_::kSFACols;
                            const uint32_t t_sfb = t_sfb0 + s * C_::kSFBCols;
                            const uint32_t s_sfa = sbase + C_::kOffSFA + s * C_::kSFABytes;
                            const uint32_t s_sfb = sbase + C_::kOffSFB + s * C_::kSFBBytes;
#pragma unroll
                            for (int a = a_begin; a < a_begin + C_::kUnitsPerMma; ++a)
                                tmem_cp_32x128b_x4(t_sfa + 4 * a, sdesc_rows16(s_sfa + 512 * a));
#pragma unroll
                            for (int rb = 0; rb < C_::kRBQ; ++rb)
#pragma unroll
                                for (int a = a_begin; a < a_begin + C_::kUnitsPerMma; ++a)
                                    tmem_cp_32x128b_x4(t_sfb + a * 4 * C_::kRBQ + 4 * rb,
                                                       sdesc_rows16(s_sfb + (rb * C_::kAtoms + a) * 512));
                            // MMA q of the stage (chunk q / 4, 32-byte step q % 4) reads atom
                            // q / kMmaPerAtom: MXFP8 one scale block per MMA (byte q % 4 of
                            // the chunk's atom), MXFP4 two (byte pair 2 * (q % 2)).
#pragma unroll
                            for (int q = a_begin * C_::kMmaPerUnit; q < (a_begin + C_::kUnitsPerMma) * C_::kMmaPerUnit;
                                 ++q) {
                                const int c = q / C_::kMmaPerChunk, j = q % C_::kMmaPerChunk;
                                const int atom = q / C_::kMmaPerAtom;
                                const uint64_t adesc =
                                    sdesc_sw128_kmajor(sbase + C_::kOffA + s * C_::kABytes + c * C_::kAChunk);
                                const uint64_t bdesc =
                                    sdesc_sw128_kmajor(sbase + C_::kOffB + s * C_::kBBytes + c * C_::kBChunk);
                                const uint32_t sf_id = FMT == kFmtMXFP8 ? j : 2 * (j % 2);
                                const uint32_t idesc = kIdesc | (sf_id << 4) | (sf_id << 29);
                                const uint32_t acc_flag = (k > kb || q > a_begin * C_::kMmaPerUnit) ? 1u : 0u;
                                const uint64_t koff = static_cast<uint64_t>(j * 32) >> 4;
                                if (FMT == kFmtMXFP8)
                                    mma_mxf8f6f4(t_acc, adesc + koff, bdesc + koff, idesc, t_sfa + 4 * atom,
                                                 t_sfb + atom * 4 * C_::kRBQ, acc_flag);
                                else
                                    mma_mxf4(t_acc, adesc + koff, bdesc + koff, idesc, t_sfa + 4 * atom,
                                             t_sfb + atom * 4 * C_::kRBQ, acc_flag);
                            }
                        } else {
                            // BF16: the warp's K chunks, four K = 16 MMAs each
#pragma unroll
                            for (int q = a_begin * C_::kMmaPerUnit; q < (a_begin + C_::kUnitsPerMma) * C_::kMmaPerUnit;
                                 ++q) {
                                const int c = q / C_::kMmaPerChunk, j = q % C_::kMmaPerChunk;
                                const uint64_t adesc =
                                    sdesc_sw128_kmajor(sbase + C_::kOffA + s * C_::kABytes + c * C_::kAChunk);
                                const uint64_t bdesc =
                                    sdesc_sw128_kmajor(sbase + C_::kOffB + s * C_::kBBytes + c * C_::kBChunk);
                                const uint32_t acc_flag = (k > kb || q > a_begin * C_::kMmaPerUnit) ? 1u : 0u;
                                const uint64_t koff = static_cast<uint64_t>(j * 32) >> 4;
                                mma_bf16(t_acc, adesc + koff, bdesc + koff, kIdesc, acc_flag);
                            }
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
        // Drain: every tcgen05 operation of every MMA warp has completed.
        if (lane == 0) {
            tc_commit(drain_bar);
            int dummy_abort = 0;
            if (!mbar_wait_parked(drain_bar, 0, &dummy_abort, kp.limit_ns))
                atomicCAS(kp.error, 0, kErrDrain);
        }
        __syncwarp();
    } else if (warp >= 2 && warp <= 5) {
        // ---------------------------------------------------------- epilogue
        grid_dependency_wait();
        const int quad = warp & 3;             // TMEM lanes 32*quad .. +31
        const int row = quad * 32 + lane;      // accumulator row = MMA row in tile
        const int etid = threadIdx.x - 64;     // 0..127
        int acc = 0;
        uint32_t acc_ph = 0;
        uint32_t out_chunks = 0;               // BF16 chunks staged so far (buffer = parity)
        bool stop = false;
        bool ring_out = false;                 // this segment may stage its output in ring stage 0
        bool tma_tile = false;                 // this tile's BF16 output may go out by TMA stores

        // The tile's accumulator is the sum of the NM MMA warps' accumulators.
        // Two loads per wait: each load-and-wait round trip costs ~0.2 us.
        auto load_acc = [&](uint32_t t_acc, int c, float (&v)[CW]) {
            uint32_t r0[CW], r1[CW];
#pragma unroll
            for (int m = 0; m < NM; m += 2) {
                tmem_ld_cols<CW>(t_acc + m * BN + c, r0);
                if (m + 1 < NM)
                    tmem_ld_cols<CW>(t_acc + (m + 1) * BN + c, r1);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < CW; ++j) {
                    const float x = __uint_as_float(r0[j]) + (m + 1 < NM ? __uint_as_float(r1[j]) : 0.0f);
                    v[j] = m == 0 ? x : v[j] + x;
                }
            }
        };

        // Fused operations (apply_epilogue_ops) on this thread's CW values.
        const EpiOps eo{kp.bias, kp.residual, kp.act, kp.swap, kp.P, kp.Q, kp.ldc};
        auto apply_ops = [&](float (&v)[CW], int64_t p, int64_t plim, int64_t q0) {
            float t[32];
#pragma unroll
            for (int j = 0; j < 32; ++j)
                t[j] = j < CW ? v[j] : 0.0f;
            apply_epilogue_ops(t, CW, eo, p, plim, q0);
#pragma unroll
            for (int j = 0; j < CW; ++j)
                v[j] = t[j];
        };

        // Quantised output: the BF16 result becomes the next layer's MX
        // operand (quantise_store_plain / quantise_store_swapped).
        const QOut qo{kp.Cq, kp.Cs, kp.ldc, kp.qfmt};
        auto emit_q = [&](const float (&v)[CW], int64_t p, int64_t plim, int64_t q0) {
            if (!kp.swap) {
                if (CW == 32 && p < plim && q0 < kp.Q) {
                    float t[CW];
#pragma unroll
                    for (int j = 0; j < CW; ++j)
                        t[j] = v[j];
                    quantise_store_plain(t, qo, p, q0);
                }
            } else if (p - lane < kp.P && q0 < kp.Q) {   // the warp's first n: uniform over the warp
                const int nq = static_cast<int>(kp.Q - q0 < CW ? kp.Q - q0 : CW);
                float t[CW];
#pragma unroll
                for (int j = 0; j < CW; ++j)
                    t[j] = v[j];
                quantise_store_swapped(t, nq, qo, p, q0, lane);
            }
        };

        // Convert one CW-column chunk of the tile (this thread's row) to BF16
        // and write it to C: through shared memory and a TMA store when the
        // output layout allows, else with predicated global stores; or, with
        // quantised output, as MX codes and scales.
        auto emit = [&](const float (&v)[CW], const TileCoord &tc, int64_t qcol) {
            const int64_t p = tc.prow + row;
            if (kp.qfmt >= 0) {
                emit_q(v, p, tc.plim, qcol);
                return;
            }
            if (!tma_tile || !(C_::kStaged || ring_out)) {
                const OutView o{kp.C, kp.ldc, tc.plim, kp.Q, kp.swap};
                store_bf16<CW>(o, p, qcol, v);
                return;
            }
            const int b = static_cast<int>(out_chunks & 1u);
            uint8_t *buf = C_::kStaged ? smem + C_::kOffOut + b * C_::kOutBytes
                                       : smem + C_::kOffA + b * C_::kChunkOutBytes;
            if (etid == 0)
                bulk_wait_group_read<1>();      // the store that last read this buffer is done
            named_bar_sync(1, 128);
            if (!kp.swap) {                     // [128 rows][CW] row-major, this thread's row
                uint4 *dst = reinterpret_cast<uint4 *>(buf + row * CW * 2);
#pragma unroll
                for (int j = 0; j < CW / 8; ++j) {
                    uint4 w;
                    w.x = pack_bf16x2(v[8 * j + 0], v[8 * j + 1]);
                    w.y = pack_bf16x2(v[8 * j + 2], v[8 * j + 3]);
                    w.z = pack_bf16x2(v[8 * j + 4], v[8 * j + 5]);
                    w.w = pack_bf16x2(v[8 * j + 6], v[8 * j + 7]);
                    dst[j] = w;
                }
            } else {                            // [CW rows of C][128 columns of C]
                __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(buf) + row;
#pragma unroll
                for (int j = 0; j < CW; ++j)
                    dst[j * 128] = __float2bfloat16_rn(v[j]);
            }
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            if (etid == 0) {
                if (!kp.swap)
                    tma_store_2d(&tmC, smem_u32(buf), static_cast<int32_t>(qcol), static_cast<int32_t>(tc.prow));
                else
                    tma_store_2d(&tmC, smem_u32(buf), static_cast<int32_t>(tc.prow), static_cast<int32_t>(qcol));
                bulk_commit_group();
            }
            ++out_chunks;
        };

        for (uint32_t w = blockIdx.x; w < W && !stop; w += gridDim.x) {
            if (grouped && !walk.seek(w))
                break;
            uint32_t it = sc.begin(w);
            const uint32_t end = sc.begin(w + 1);
            bool first = true;
            while (it < end) {
                const Segment sg = segment_at(sc, it, end);
                const uint32_t tile = sg.tile, kb = sg.kb, ke = sg.ke;
                const TileCoord tc = coord_of(tile);
                // the CTA's final segment: once its accumulator is complete every
                // stage has been consumed and no further loads are coming
                ring_out = (w + gridDim.x >= W) && (it + (ke - kb) >= end);
                if (grouped)        // a group's last tile may end inside the box a TMA store writes
                    ring_out = false;
                tma_tile = kp.tma_store && (!grouped || tc.prow + 128 <= tc.plim);
                int good = 1;
                if (lane == 0)
                    good = mbar_wait_parked(accf_bar(acc), acc_ph, s_abort, kp.limit_ns);
                good = __shfl_sync(0xffffffffu, good, 0);
                if (!good && lane == 0)
                    record_error(kp.error, kErrEpiAccFull, s_abort);
                // One decision for all four epilogue warps.
                if (named_bar_or(1, 128, (!good || *s_abort) ? 1 : 0)) {
                    stop = true;
                    break;
                }
                tc_fence_after();
                const uint32_t t_acc = tmem + acc * NM * BN + (static_cast<uint32_t>(quad * 32) << 16);
                const uint32_t g_first = sc.dp ? tile : sc.owner(tile * sc.KT);
                const uint32_t g_last = sc.dp ? tile : sc.owner(tile * sc.KT + sc.KT - 1);
                const int64_t p = tc.prow + row;
                bool released = false;
                if (g_first == g_last && spread) {
                    // the CTA's only tile: FP32 [BN][128] into the drained ring
                    float *stage = reinterpret_cast<float *>(smem + C_::kRedOff);
#pragma unroll
                    for (int c = 0; c < BN; c += CW) {
                        float v[CW];
                        load_acc(t_acc, c, v);
#pragma unroll
                        for (int j = 0; j < CW; ++j)
                            stage[(c + j) * 128 + row] = v[j];
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(acce_bar(acc));
                    released = true;
                } else if (g_first == g_last) {
                    // Drain the accumulator row into registers as BF16 pairs and
                    // hand the accumulator back before any store, so the next
                    // tile's MMAs overlap this tile's output traffic.
                    uint32_t packed[BN / 2];
#pragma unroll
                    for (int c = 0; c < BN; c += CW) {
                        float v[CW];
                        load_acc(t_acc, c, v);
                        if (kp.has_ops)
                            apply_ops(v, p, tc.plim, tc.qcol + c);
#pragma unroll
                        for (int j = 0; j < CW / 2; ++j)
                            packed[c / 2 + j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(acce_bar(acc));
                    released = true;
#pragma unroll
                    for (int c = 0; c < BN; c += CW) {
                        float v[CW];     // BF16 values widened back exactly
#pragma unroll
                        for (int j = 0; j < CW / 2; ++j) {
                            v[2 * j] = __uint_as_float(packed[c / 2 + j] << 16);
                            v[2 * j + 1] = __uint_as_float(packed[c / 2 + j] & 0xFFFF0000u);
                        }
                        emit(v, tc, tc.qcol + c);
                    }
                } else if (kp.ksplit > 1) {
                    // Cluster K split, reduced by scatter: one work unit per
                    // CTA, the tile's ranks in one cluster.  A rank's ring is
                    // drained once its accumulator is complete; it then arms
                    // its reduction barrier for the partials of its rows and
                    // tells the other ranks.  Each warp quarter whose rows
                    // another rank owns stages its FP32 partial in its own
                    // ring and pushes it there with one bulk copy that counts
                    // its bytes on the owner's barrier.  The owner's quarters
                    // add the others' partials to their own in rank order and
                    // write their rows.
                    const uint32_t S = static_cast<uint32_t>(kp.ksplit);
                    const uint32_t rank = w - g_first;
                    const uint32_t qpr = 4u / (S == 4u ? 4u : 2u);      // lane quarters per rank
                    const uint32_t owner = static_cast<uint32_t>(quad) / qpr;
                    // the plan puts exactly one cluster of 2 or 4 on each tile;
                    // anything else would address buffers that do not exist
                    const bool shape_ok = C_::kCanKsplit && (S == 2u || S == 4u) && g_first % S == 0 &&
                                          g_last - g_first + 1 == S;
                    if (!shape_ok) {
                        if (lane == 0)
                            record_error(kp.error, kErrReduce, s_abort);
                    } else if (owner != rank) {
                        float4 *out = reinterpret_cast<float4 *>(smem + C_::kRedOut + quad * C_::kQuadBytes);
#pragma unroll 1
                        for (int c = 0; c < BN; c += CW) {
                            float v[CW];
                            load_acc(t_acc, c, v);
#pragma unroll
                            for (int j = 0; j < CW / 4; ++j)
                                out[(c / 4 + j) * 32 + lane] =
                                    make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                        }
                        fence_proxy_async_smem();       // the copy engine reads what the lanes wrote
                        __syncwarp();
                        if (lane == 0) {
                            if (mbar_wait_cluster_bounded(go_bar, 0, s_abort, kp.limit_ns)) {
                                const uint32_t slot = rank < owner ? rank : rank - 1;
                                const uint32_t dst =
                                    sbase + C_::kRedOff + (slot * qpr + (quad - owner * qpr)) * C_::kQuadBytes;
                                bulk_copy_to_cluster(cluster_addr(dst, owner),
                                                     sbase + C_::kRedOut + quad * C_::kQuadBytes,
                                                     static_cast<uint32_t>(C_::kQuadBytes),
                                                     cluster_addr(red_bar, owner));
                            } else {
                                record_error(kp.error, kErrReduce, s_abort);
                            }
                        }
                    } else {
                        if (static_cast<uint32_t>(quad) == rank * qpr) {
                            // lane 0 arms for the incoming bytes (a copy that
                            // lands first only drives the byte count below
                            // zero until then); lanes 1.. each tell one other
                            // rank.  The go-ahead carries no data: this ring
                            // was last touched by the TMA and the MMAs, both
                            // complete, so a relaxed arrive suffices.
                            if (lane == 0)
                                mbar_arrive_expect_tx(red_bar,
                                                      static_cast<uint32_t>((S - 1) * qpr * C_::kQuadBytes));
                            else if (static_cast<uint32_t>(lane) < S)
                                mbar_arrive_remote_relaxed(go_bar, static_cast<uint32_t>(lane) - 1 < rank
                                                                       ? static_cast<uint32_t>(lane) - 1
                                                                       : static_cast<uint32_t>(lane));
                        }
                        // the CTA's other roles are done: spin rather than park
                        // (a parked wait wakes late on a remote completion)
                        int got = 1;
                        if (lane == 0)
                            got = mbar_wait_cluster_bounded(red_bar, 0, s_abort, kp.limit_ns);
                        got = __shfl_sync(0xffffffffu, got, 0);
                        if (!got && lane == 0)
                            record_error(kp.error, kErrReduce, s_abort);
                        // nothing more arrives here: the cluster may finish
                        cluster_arrive();
                        cl_arrived = true;
                        if (got) {
                            const uint32_t qj = static_cast<uint32_t>(quad) - rank * qpr;
                            // BF16 output through this quarter's [BN][32] staging
                            // block and one TMA store (the map's box)
                            uint8_t *stage = smem + C_::kRedStage + quad * C_::kQStageBytes;
                            // own partial first, then the others in rank order
                            // (a fixed order: the result does not depend on
                            // which copy lands first)
#pragma unroll 1
                            for (int c = 0; c < BN; c += CW) {
                                float v[CW];
                                load_acc(t_acc, c, v);
#pragma unroll 1
                                for (uint32_t slot = 0; slot + 1 < S; ++slot) {
                                    const float4 *src = reinterpret_cast<const float4 *>(
                                        smem + C_::kRedOff + (slot * qpr + qj) * C_::kQuadBytes);
#pragma unroll
                                    for (int j = 0; j < CW / 4; ++j) {
                                        const float4 x = src[(c / 4 + j) * 32 + lane];
                                        v[4 * j + 0] += x.x;
                                        v[4 * j + 1] += x.y;
                                        v[4 * j + 2] += x.z;
                                        v[4 * j + 3] += x.w;
                                    }
                                }
                                if (kp.has_ops)
                                    apply_ops(v, p, tc.plim, tc.qcol + c);
                                if (kp.qfmt >= 0) {
                                    emit_q(v, p, tc.plim, tc.qcol + c);
                                } else if (!tma_tile) {
                                    const OutView o{kp.C, kp.ldc, tc.plim, kp.Q, kp.swap};
                                    store_bf16<CW>(o, p, tc.qcol + c, v);
                                } else {
                                    __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(stage) + c * 32 + lane;
#pragma unroll
                                    for (int j = 0; j < CW; ++j)
                                        dst[j * 32] = __float2bfloat16_rn(v[j]);
                                }
                            }
                            if (kp.qfmt < 0 && tma_tile) {
                                fence_proxy_async_smem();
                                __syncwarp();
                                if (lane == 0) {
                                    tma_store_2d(&tmC, smem_u32(stage), static_cast<int32_t>(tc.prow + quad * 32),
                                                 static_cast<int32_t>(tc.qcol));
                                    bulk_commit_group();
                                    bulk_wait_group_read<0>();
                                }
                            }
                        }
                    }
                } else {
                    const int64_t slot = 2 * static_cast<int64_t>(w) + (first ? 0 : 1);
                    float *mine = kp.partials + (slot * 128 + row) * BN;
#pragma unroll 1
                    for (int c = 0; c < BN; c += CW) {
                        float v[CW];
                        load_acc(t_acc, c, v);
#pragma unroll
                        for (int j = 0; j < CW / 4; ++j)
                            reinterpret_cast<float4 *>(mine + c)[j] =
                                make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                    }
                    __threadfence();
                    named_bar_sync(1, 128);
                    if (etid == 0) {
                        const uint32_t nseg = g_last - g_first + 1;
                        const uint32_t old = atomicAdd(kp.counters + tile, 1u);
                        const int last = (old == nseg - 1) ? 1 : 0;
                        if (last)
                            kp.counters[tile] = 0u;
                        *s_last = last;
                    }
                    named_bar_sync(1, 128);
                    if (*s_last) {
                        __threadfence();
#pragma unroll 1
                        for (int c = 0; c < BN; c += CW) {
                            float own[CW];
                            load_acc(t_acc, c, own);
                            float v[CW];
#pragma unroll
                            for (int j = 0; j < CW; ++j)
                                v[j] = 0.0f;
                            for (uint32_t g = g_first; g <= g_last; ++g) {
                                if (g == w) {
#pragma unroll
                                    for (int j = 0; j < CW; ++j)
                                        v[j] += own[j];
                                } else {
                                    const int64_t gslot =
                                        2 * static_cast<int64_t>(g) + ((sc.begin(g) / sc.KT == tile) ? 0 : 1);
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
                            if (kp.has_ops)
                                apply_ops(v, p, tc.plim, tc.qcol + c);
                            emit(v, tc, tc.qcol + c);
                        }
                    }
                }
                if (!released) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(acce_bar(acc));
                }
                if (++acc == C_::kNumAcc) {
                    acc = 0;
                    acc_ph ^= 1u;
                }
                first = false;
                it += ke - kb;
            }
        }
        // Output stores must finish reading shared memory before the CTA
        // exits; the kernel's completion covers their writes.
        if (etid == 0)
            bulk_wait_group_read<0>();
    }

    if (spread) {
        // Every warp takes units of the staged tile: unit u is 32 consecutive
        // rows of the row operand (32 consecutive n of C, one per lane) of
        // output row m.  Residual and bias loads for all of a warp's units go
        // out first; the operations run four units per call of ops4.
        named_bar_sync(2, C_::kThreads);
        if (!*s_abort) {
            constexpr int kU = 4 * BN;
            constexpr int kW = C_::kWarps;
            constexpr int kMaxU = (kU + kW - 1) / kW;
            const TileCoord tc = plain_coord(kp, blockIdx.x, BN);
            const float *stage = reinterpret_cast<const float *>(smem + C_::kRedOff);
            float sv[kMaxU], bv[kMaxU], rv[kMaxU];
#pragma unroll
            for (int i = 0; i < kMaxU; ++i) {
                const int u = warp + i * kW;
                const int pb = u & 3, ml = u >> 2;
                const int64_t p = tc.prow + pb * 32 + lane;
                const int64_t m = tc.qcol + ml;
                const bool ok = u < kU && p < kp.P && m < kp.Q;
                sv[i] = u < kU ? stage[ml * 128 + pb * 32 + lane] : 0.0f;
                bv[i] = (ok && kp.bias) ? bf16_bits_to_float(kp.bias[p]) : 0.0f;
                rv[i] = (ok && kp.residual) ? bf16_bits_to_float(kp.residual[m * kp.ldc + p]) : 0.0f;
            }
            if (kp.has_ops) {
                const int hb = kp.bias != nullptr, hr = kp.residual != nullptr;
#pragma unroll
                for (int i = 0; i < kMaxU; i += 4) {
                    const Val4 in{sv[i], i + 1 < kMaxU ? sv[i + 1] : 0.0f, i + 2 < kMaxU ? sv[i + 2] : 0.0f,
                                  i + 3 < kMaxU ? sv[i + 3] : 0.0f};
                    const Val4 b4{bv[i], i + 1 < kMaxU ? bv[i + 1] : 0.0f, i + 2 < kMaxU ? bv[i + 2] : 0.0f,
                                  i + 3 < kMaxU ? bv[i + 3] : 0.0f};
                    const Val4 r4{rv[i], i + 1 < kMaxU ? rv[i + 1] : 0.0f, i + 2 < kMaxU ? rv[i + 2] : 0.0f,
                                  i + 3 < kMaxU ? rv[i + 3] : 0.0f};
                    Val4 o;
                    switch (kp.act) {
                    case 1: o = ops4<1>(in, 0.0f, b4, r4, hb, hr); break;
                    case 2: o = ops4<2>(in, 0.0f, b4, r4, hb, hr); break;
                    case 3: o = ops4<3>(in, 0.0f, b4, r4, hb, hr); break;
                    default: o = ops4<0>(in, 0.0f, b4, r4, hb, hr); break;
                    }
                    sv[i] = o.a;
                    if (i + 1 < kMaxU)
                        sv[i + 1] = o.b;
                    if (i + 2 < kMaxU)
                        sv[i + 2] = o.c;
                    if (i + 3 < kMaxU)
                        sv[i + 3] = o.d;
                }
            }
            const QOut qo{kp.Cq, kp.Cs, kp.ldc, kp.qfmt};
#pragma unroll
            for (int i = 0; i < kMaxU; ++i) {
                const int u = warp + i * kW;
                const int pb = u & 3, ml = u >> 2;
                const int64_t p = tc.prow + pb * 32 + lane;
                const int64_t m = tc.qcol + ml;
                // rows past P hold zeros (the loads zero-fill them): valid lanes
                // and the block's scale depend only on the warp-uniform start
                if (u < kU && m < kp.Q && tc.prow + pb * 32 < kp.P) {
                    if (kp.qfmt < 0) {
                        if (p < kp.P)
                            kp.C[m * kp.ldc + p] = __float2bfloat16_rn(sv[i]);
                    } else {
                        quantise_row_swapped(sv[i], qo, m, p, lane, p < kp.P);
                    }
                }
            }
        }
    }
    if (kp.ksplit > 1 && !cl_arrived)
        cluster_arrive();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        tmem_dealloc(tmem, C_::kTmemCols);
    // No CTA of a cluster K split leaves while another may still touch its
    // shared memory: each thread arrived when its part was done (rank 0's
    // epilogue once every partial was in), so the other ranks leave as soon
    // as rank 0 has its partials.
    if (kp.ksplit > 1)
        cluster_wait();
}


// ------------------------------------------------------------------- host

namespace {

template <int FMT, int BN, int KC>
cudaError_t set_attrs()
{
    return cudaFuncSetAttribute(mx_gemm_kernel<FMT, BN, KC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Cfg<FMT, BN, KC>::kSmemBytes);
}

template <int FMT, int BN, int KC>
cudaError_t launch_t(const GemmPlan &pl, const GemmBuffers &b, uint64_t limit_ns, int inject, int pdl,
                     cudaStream_t st)
{
    using C_ = Cfg<FMT, BN, KC>;
    const int64_t rbytes = row_bytes(FMT, pl.K);
    const bool grouped = pl.groups > 0;
    const void *Pptr = pl.swap ? b.B : b.A;
    const void *Qptr = pl.swap ? b.A : b.B;
    // rows of the two operand tensors (grouped: B holds G blocks of N rows)
    const int64_t Prows = pl.P;
    const int64_t Qrows = grouped ? pl.groups * pl.N : pl.Q;
    CUtensorMap tmP, tmQ, tmC;
    if (KC == 1) {
        if (!make_operand_map(&tmP, Pptr, Prows, rbytes, 128) || !make_operand_map(&tmQ, Qptr, Qrows, rbytes, BN))
            return cudaErrorInvalidValue;
    } else {
        if (!make_operand_map_3d(&tmP, Pptr, Prows, rbytes, 128, KC) ||
            !make_operand_map_3d(&tmQ, Qptr, Qrows, rbytes, BN, KC))
            return cudaErrorInvalidValue;
    }
    // TMA stores need 16-byte row pitch; other widths take the predicated
    // store path (the map is then a never-used placeholder over C).  With
    // quantised output C is not written and the map is a placeholder too.
    const bool quantised = b.epi.qfmt >= 0;
    const int tma_store = (pl.N % 8 == 0 && !quantised) ? 1 : 0;
    void *Cbase = quantised ? static_cast<void *>(b.epi.Cq) : b.C;
    // (a cluster K split stores each 32-row lane quarter of a tile, all its
    // BN columns, with one box)
    const bool okC = tma_store ? (pl.ksplit > 1 ? make_output_map(&tmC, Cbase, pl.M, pl.N, 32, BN)
                                  : pl.swap    ? make_output_map(&tmC, Cbase, pl.M, pl.N, 128, C_::kCW)
                                               : make_output_map(&tmC, Cbase, pl.M, pl.N, C_::kCW, 128))
                               : make_output_map(&tmC, Cbase, 1, 8, 8, 1);
    if (!okC)
        return cudaErrorInvalidValue;
    CUtensorMap tmSP, tmSQ;
    const bool fused = b.rawA != nullptr;
    const uint8_t *rawP = pl.swap ? b.rawB : b.rawA;
    const uint8_t *rawQ = pl.swap ? b.rawA : b.rawB;
    if (C_::kScaled) {
        // with fused scales the repacked maps are never read: encode them
        // over the row-major scales so they are valid
        const uint8_t *sfP = fused ? rawP : (pl.swap ? b.sfB : b.sfA);
        const uint8_t *sfQ = fused ? rawQ : (pl.swap ? b.sfA : b.sfB);
        if (!make_sf_map(&tmSP, sfP, pl.kaP, sf_row_blocks(pl.P), C_::kAtoms, 1) ||
            !make_sf_map(&tmSQ, sfQ, pl.kaQ, sf_row_blocks(pl.Q), C_::kAtoms, C_::kRBQ))
            return cudaErrorInvalidValue;
    } else {
        // BF16 operands carry no scales: placeholders that are never read
        if (!make_sf_map(&tmSP, static_cast<const uint8_t *>(Pptr), 1, 1, 1, 1) ||
            !make_sf_map(&tmSQ, static_cast<const uint8_t *>(Qptr), 1, 1, 1, 1))
            return cudaErrorInvalidValue;
    }
    KParams kp;
    kp.C = reinterpret_cast<__nv_bfloat16 *>(b.C);
    kp.partials = b.partials;
    kp.counters = b.counters;
    kp.error = b.error;
    kp.P = pl.P;
    kp.Q = pl.Q;
    kp.ldc = pl.N;
    kp.tilesP = static_cast<uint32_t>(pl.tilesP);
    kp.kt = static_cast<uint32_t>(pl.kt);
    kp.iters = static_cast<uint32_t>(pl.iters);
    kp.workers = static_cast<uint32_t>(pl.workers);
    kp.dp = pl.workers == pl.tiles ? 1 : 0;
    kp.limit_ns = limit_ns;
    kp.swap = pl.swap;
    kp.inject = inject;
    kp.tma_store = tma_store;
    kp.fused_sf = (C_::kScaled && fused) ? 1 : 0;
    kp.rawP = rawP;
    kp.rawQ = rawQ;
    kp.ldS = pl.K / 32;
    // bits of b.early are per operand (A, B); the kernel's are per side (P, Q)
    kp.early = pl.swap ? (((b.early & 1) << 1) | ((b.early >> 1) & 1)) : b.early;
    kp.bias = b.epi.bias;
    kp.residual = b.epi.residual;
    kp.act = b.epi.act;
    kp.has_ops = (b.epi.bias || b.epi.residual || b.epi.act) ? 1 : 0;
    kp.qfmt = b.epi.qfmt;
    kp.Cq = b.epi.Cq;
    kp.Cs = b.epi.Cs;
    kp.goff = grouped ? b.group_offsets : nullptr;
    kp.groups = static_cast<uint32_t>(pl.groups);
    kp.tilesQ = static_cast<uint32_t>(pl.tilesQ);
    kp.band = 0;
    kp.tail_first = 0;
    kp.tail_split = 1;
    kp.ksplit = static_cast<int>(pl.ksplit);
    if (pl.ksplit > 1 && (!C_::kCanKsplit || !pl.swap || (pl.ksplit != 2 && pl.ksplit != 4) ||
                          pl.grid != pl.workers || pl.grid % pl.ksplit != 0))
        return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(pl.grid));
    cfg.blockDim = dim3(C_::kThreads);
    cfg.dynamicSmemBytes = C_::kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    if (pl.ksplit > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = static_cast<unsigned>(pl.ksplit);
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, mx_gemm_kernel<FMT, BN, KC>, tmP, tmQ, tmSP, tmSQ, tmC, kp);
}

template <int FMT, int KC>
cudaError_t dispatch_bn(const GemmPlan &pl, const GemmBuffers &b, uint64_t limit_ns, int inject, int pdl,
                        cudaStream_t st)
{
    switch (pl.bn) {
    case 16: return launch_t<FMT, 16, KC>(pl, b, limit_ns, inject, pdl, st);
    case 32: return launch_t<FMT, 32, KC>(pl, b, limit_ns, inject, pdl, st);
    case 64: return launch_t<FMT, 64, KC>(pl, b, limit_ns, inject, pdl, st);
    case 128: return launch_t<FMT, 128, KC>(pl, b, limit_ns, inject, pdl, st);
    case 256: return launch_t<FMT, 256, KC>(pl, b, limit_ns, inject, pdl, st);
    default: return cudaErrorInvalidValue;
    }
}

template <int FMT>
cudaError_t dispatch_bn4(const GemmPlan &pl, const GemmBuffers &b, uint64_t limit_ns, int inject, int pdl,
                         cudaStream_t st)
{
    switch (pl.bn) {
    case 16: return launch_t<FMT, 16, 4>(pl, b, limit_ns, inject, pdl, st);
    case 32: return launch_t<FMT, 32, 4>(pl, b, limit_ns, inject, pdl, st);
    case 64: return launch_t<FMT, 64, 4>(pl, b, limit_ns, inject, pdl, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

}  // namespace mxg
