// api.cu -- the C ABI declared in include/mxgemm.h.
//
// Host-side responsibilities only: argument validation (before any launch),
// the workspace the handle owns, the scheduling plan, and the order of the
// two launches of the hot path (scale repack, then the GEMM) on the caller's
// stream.  Every step of the arithmetic runs in the CUDA kernels of
// repack.cu, gemm.cu and quant.cu; there is no host fallback.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>

#include "../../include/mxgemm.h"
#include "mx_internal.h"

// Events of one blocked mxgemm_run_host: entry, exit, one per uploaded band
// (at most 8 + 8) and one per block of C (at most 64).
constexpr int kHostParts = 8;
constexpr int kHostEvents = 2 + 2 * kHostParts + kHostParts * kHostParts;

struct mxgemm_ctx {
    int device = 0;
    int num_sms = 0;
    // scale workspace: repacked A scales then repacked B scales
    uint8_t *sf = nullptr;
    size_t sf_cap = 0;
    int64_t sf_offB = 0;
    // split partials and per-tile counters (counters kept zero between launches)
    float *partials = nullptr;
    size_t partials_cap = 0;
    uint32_t *counters = nullptr;
    size_t counters_cap = 0;
    int *err = nullptr;
    // device staging of mxgemm_run_host, its upload and download streams and
    // the events that order them against the GEMMs on the caller's stream
    uint8_t *stage = nullptr;
    size_t stage_cap = 0;
    cudaStream_t up = nullptr, down = nullptr;
    cudaEvent_t hev[kHostEvents] = {};
    // schedule override
    int sched = MXGEMM_SCHED_AUTO;
    int splits = 1;
    int workers = 0;
    int kchunks = 0;        // 0 = auto
    uint64_t limit_ns = 2000000000ull;
    int inject = 0;
    // shape of the last repack
    int last_fmt = -1;
    int64_t last_M = 0, last_N = 0, last_K = 0;
    // profiling: events around the repack and the GEMM of the last run
    int profiling = 0;
    cudaEvent_t ev[3] = {nullptr, nullptr, nullptr};
    int ev_valid = 0;
    // caller's promise: B and its scales are not written by the work that
    // precedes mxgemm_run on its stream (constant weights)
    int prefetch_b = 0;
};

namespace {

constexpr uint64_t kDefaultLimitNs = 2000000000ull;
constexpr int64_t kMaxDim = int64_t(1) << 24;
constexpr int64_t kMaxGroups = int64_t(1) << 16;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_shape(int fmt, int64_t M, int64_t N, int64_t K)
{
    if (fmt != MXGEMM_FMT_MXFP8_E4M3 && fmt != MXGEMM_FMT_MXFP4_E2M1)
        return MXGEMM_ERR_INVALID_ARG;
    if (M < 1 || N < 1 || K < 128 || K % 128 != 0)
        return MXGEMM_ERR_INVALID_ARG;
    if (M > kMaxDim || N > kMaxDim || K > kMaxDim)
        return MXGEMM_ERR_INVALID_ARG;
    return MXGEMM_OK;
}

int check_ptrs(std::initializer_list<const void *> ptrs)
{
    for (const void *p : ptrs)
        if (p == nullptr)
            return MXGEMM_ERR_INVALID_ARG;
    for (const void *p : ptrs)
        if (!aligned16(p))
            return MXGEMM_ERR_ALIGNMENT;
    return MXGEMM_OK;
}

// Grow a workspace buffer to at least `need` bytes.  Growing allocates
// device memory (and frees the old buffer), which a stream capture cannot
// record: while `st` is capturing, a buffer that must grow gives
// MXGEMM_ERR_CAPTURE and nothing is allocated.
template <typename T>
int grow(T **buf, size_t *cap, size_t need, bool zero, cudaStream_t st)
{
    if (need <= *cap)
        return MXGEMM_OK;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) {
        cudaGetLastError();
        return MXGEMM_ERR_CUDA;
    }
    if (cs != cudaStreamCaptureStatusNone)
        return MXGEMM_ERR_CAPTURE;
    if (*buf) {
        cudaFree(*buf);
        *buf = nullptr;
        *cap = 0;
    }
    size_t want = need + need / 4;
    if (cudaMalloc(reinterpret_cast<void **>(buf), want) != cudaSuccess) {
        cudaGetLastError();
        *buf = nullptr;
        return MXGEMM_ERR_OOM;
    }
    if (zero && cudaMemset(*buf, 0, want) != cudaSuccess)
        return MXGEMM_ERR_CUDA;
    *cap = want;
    return MXGEMM_OK;
}

int enter_device(mxgemm_handle h)
{
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess)
        return MXGEMM_ERR_CUDA;
    if (cur != h->device && cudaSetDevice(h->device) != cudaSuccess)
        return MXGEMM_ERR_CUDA;
    return MXGEMM_OK;
}

int do_repack(mxgemm_handle h, int fmt, int64_t M, int64_t N, int64_t K, const uint8_t *sa, const uint8_t *sb,
              cudaStream_t st)
{
    const int64_t ba = mxg::sf_repacked_bytes(fmt, M, K);
    const int64_t bb = mxg::sf_repacked_bytes(fmt, N, K);
    int rc = grow(&h->sf, &h->sf_cap, static_cast<size_t>(ba + bb), false, st);
    if (rc != MXGEMM_OK)
        return rc;
    h->sf_offB = ba;
    if (mxg::launch_repack(fmt, M, N, K, sa, sb, h->sf, h->sf + ba, st) != cudaSuccess)
        return MXGEMM_ERR_CUDA;
    h->last_fmt = fmt;
    h->last_M = M;
    h->last_N = N;
    h->last_K = K;
    return MXGEMM_OK;
}

// mxgemm_run converts the row-major scales inside the GEMM for one-CTA
// plans whose ring is at least four stages deep (the gather's latency hides
// behind the ring); otherwise it runs the separate repack first.
bool fuse_scales(const mxg::GemmPlan &pl) { return pl.valid && !pl.pair && pl.stages >= 4; }

// GEMM launch of plan `pl`.  With raw scales (SA, SB non-NULL) the kernel
// converts the row-major scales itself; otherwise it reads the last
// repack's workspace, which must be for this shape (BF16 operands have no
// scales).  pdl and early as mxg::launch_gemm and GemmBuffers::early.
int launch_plan(mxgemm_handle h, const mxg::GemmPlan &pl, const void *A, const void *B, void *C, cudaStream_t st,
                int pdl, int early, const uint8_t *SA, const uint8_t *SB, const mxg::Epilogue &epi,
                const int64_t *goff = nullptr)
{
    if (!pl.valid)
        return MXGEMM_ERR_INVALID_ARG;
    if (pl.fmt != mxg::kFmtBF16 && !SA &&
        (h->last_fmt != pl.fmt || h->last_M != pl.M || h->last_N != pl.N || h->last_K != pl.K))
        return MXGEMM_ERR_INVALID_ARG;
    int rc = grow(&h->partials, &h->partials_cap, static_cast<size_t>(pl.partial_bytes > 0 ? pl.partial_bytes : 16),
                  false, st);
    if (rc != MXGEMM_OK)
        return rc;
    rc = grow(&h->counters, &h->counters_cap, static_cast<size_t>(pl.counter_bytes), true, st);
    if (rc != MXGEMM_OK)
        return rc;
    mxg::GemmBuffers b;
    b.A = A;
    b.B = B;
    b.sfA = h->sf;
    b.sfB = h->sf + h->sf_offB;
    b.C = C;
    b.partials = h->partials;
    b.counters = h->counters;
    b.error = h->err;
    b.rawA = SA;
    b.rawB = SB;
    b.early = early;
    b.epi = epi;
    b.group_offsets = goff;
    const int inject = h->inject;
    h->inject = 0;
    if (mxg::launch_gemm(pl, b, h->limit_ns, inject, pdl, st) != cudaSuccess)
        return MXGEMM_ERR_CUDA;
    return MXGEMM_OK;
}

mxg::GemmPlan plan_for(mxgemm_handle h, int fmt, int64_t M, int64_t N, int64_t K, bool allow_pair = true)
{
    return mxg::make_plan(fmt, M, N, K, h->num_sms, h->sched, h->splits, h->workers, h->kchunks, allow_pair);
}

// The GEMM alone on the last repack's workspace (mxgemm_gemm).
int do_gemm(mxgemm_handle h, int fmt, int64_t M, int64_t N, int64_t K, const void *A, const void *B, void *C,
            cudaStream_t st, int pdl, int early)
{
    return launch_plan(h, plan_for(h, fmt, M, N, K), A, B, C, st, pdl, early, nullptr, nullptr, mxg::Epilogue());
}

// The hot path.  Plans on one CTA per tile convert the row-major scales
// inside the GEMM (one launch); CTA-pair plans run the scale repack, then
// the GEMM as a programmatic dependent of it.  The one-launch GEMM is itself
// a programmatic dependent of whatever precedes it: its CTAs set up while a
// previous GEMM of this library finishes, and read nothing before that GEMM
// has completed, except B and its scales under the prefetch-B promise.
// With profiling on, events bracket the launches and nothing overlaps (the
// middle event keeps the GEMM from starting before the repack ends; with
// the conversion fused it records no repack time).  A fused epilogue
// (epi) keeps the plan on one-CTA tiles, whose epilogue implements it.
// chain = false launches the GEMM without the programmatic dependency, so it
// starts only once everything before it on the stream has completed.
int repack_and_gemm(mxgemm_handle h, int fmt, int64_t M, int64_t N, int64_t K, const void *A, const uint8_t *SA,
                    const void *B, const uint8_t *SB, void *C, cudaStream_t st,
                    const mxg::Epilogue &epi = mxg::Epilogue(), bool allow_pair = true, bool chain = true)
{
    const bool prof = h->profiling != 0;
    const int pdl = (prof || !chain) ? 0 : 1;
    h->ev_valid = 0;
    const mxg::GemmPlan pl = plan_for(h, fmt, M, N, K, allow_pair);
    if (!pl.valid)
        return MXGEMM_ERR_INVALID_ARG;
    const bool fused = fuse_scales(pl);
    if (prof && cudaEventRecord(h->ev[0], st) != cudaSuccess)
        return MXGEMM_ERR_CUDA;
    int rc = MXGEMM_OK;
    if (!fused) {
        rc = do_repack(h, fmt, M, N, K, SA, SB, st);
        if (rc != MXGEMM_OK)
            return rc;
    }
    if (prof && cudaEventRecord(h->ev[1], st) != cudaSuccess)
        return MXGEMM_ERR_CUDA;
    rc = fused ? launch_plan(h, pl, A, B, C, st, pdl, h->prefetch_b ? 2 : 0, SA, SB, epi)
               : launch_plan(h, pl, A, B, C, st, pdl, 3, nullptr, nullptr, epi);
    if (rc != MXGEMM_OK)
        return rc;
    if (prof) {
        if (cudaEventRecord(h->ev[2], st) != cudaSuccess)
            return MXGEMM_ERR_CUDA;
        h->ev_valid = 1;
    }
    return MXGEMM_OK;
}

bool optional_aligned16(const void *p) { return p == nullptr || aligned16(p); }

// How mxgemm_run_host cuts a large product into blocks of C.  Over PCIe the
// copies dominate such a product (8192^3 MXFP8: 132 MB up and 128 MB down
// against a 0.45 ms GEMM), so the operands go up in row bands of A and of
// B, each block of C is computed once its two bands have landed, and goes
// down while later bands still go up.  Parts are multiples of 256 rows (the
// CTA pair's tile); a block keeps at least 2^22 elements (64 tiles of
// 256 x 256) so that its GEMM still fills the GPU; under 32 MB of copies the
// product stays one block.  MXGEMM_HOST_BLOCKS (a measurement knob): "0"
// keeps every product in one block, "PxQ" cuts products of 32 MB or more
// into P parts of M and Q of N (1 to 8 each, parts still multiples of 256).
struct HostBlocks {
    int64_t mb, nb;  // rows of a full part of M and of N
    int pm, pn;      // parts
};

HostBlocks host_blocks(int64_t M, int64_t N, size_t copy_bytes)
{
    HostBlocks b{M, N, 1, 1};
    const char *e = getenv("MXGEMM_HOST_BLOCKS");
    if (copy_bytes < (size_t(32) << 20) || (e && e[0] == '0' && e[1] == 0))
        return b;
    int pm = M >= 4096 ? 4 : (M >= 2048 ? 2 : 1);
    int pn = N >= 4096 ? 4 : (N >= 2048 ? 2 : 1);
    auto part = [](int64_t d, int p) { return ((d + p - 1) / p + 255) / 256 * 256; };
    int fm = 0, fn = 0;
    if (e && sscanf(e, "%dx%d", &fm, &fn) == 2 && fm >= 1 && fm <= kHostParts && fn >= 1 && fn <= kHostParts) {
        pm = fm;
        pn = fn;
    } else {
        while ((pm > 1 || pn > 1) && part(M, pm) * part(N, pn) < (int64_t(1) << 22)) {
            if (pm >= pn)
                pm /= 2;
            else
                pn /= 2;
        }
    }
    if (pm == 1 && pn == 1)
        return b;
    b.mb = part(M, pm);
    b.nb = part(N, pn);
    b.pm = static_cast<int>((M + b.mb - 1) / b.mb);
    b.pn = static_cast<int>((N + b.nb - 1) / b.nb);
    return b;
}

// The blocked form of mxgemm_run_host.  Three streams: the uploads on
// h->up, the GEMMs on the caller's stream, the downloads on h->down, ordered
// by events.  The bands go up as A_0, B_0, A_1, B_1, ...; each block's GEMM
// waits for the later of its two bands and runs unchained (its operands come
// from a copy, not from the kernel before it); each block goes down into its
// rows and columns of C_host once its GEMM is done.  Everything is queued
// before the first download (one into pageable memory may hold the host
// thread until it is done), and every stream is drained before returning,
// on error too, so no copy still touches the caller's buffers.
int run_host_blocked(mxgemm_handle h, int fmt, int64_t M, int64_t N, int64_t K, const uint8_t *A_host,
                     const uint8_t *SA_host, const uint8_t *B_host, const uint8_t *SB_host, uint8_t *C_host,
                     uint8_t *dA, uint8_t *dSA, uint8_t *dB, uint8_t *dSB, uint8_t *dC, const HostBlocks &hb,
                     cudaStream_t st)
{
    if (!h->up && cudaStreamCreateWithFlags(&h->up, cudaStreamNonBlocking) != cudaSuccess)
        return MXGEMM_ERR_CUDA;
    if (!h->down && cudaStreamCreateWithFlags(&h->down, cudaStreamNonBlocking) != cudaSuccess)
        return MXGEMM_ERR_CUDA;
    for (cudaEvent_t &e : h->hev)
        if (!e && cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess)
            return MXGEMM_ERR_CUDA;
    const size_t rb = static_cast<size_t>(mxg::row_bytes(fmt, K));   // bytes of an operand row
    const size_t sb = static_cast<size_t>(K / 32);                    // bytes of a row's scales
    auto part_rows = [](int64_t total, int64_t part, int i) {
        return static_cast<size_t>(total - part * i < part ? total - part * i : part);
    };
    cudaEvent_t *ev = h->hev;  // 0 entry, 1 exit, then the bands, then the blocks
    int next = 2;
    int a_ev[kHostParts] = {}, b_ev[kHostParts] = {};
    int blk[kHostParts * kHostParts][2];
    int nblk = 0, na = 0, nb = 0;
    auto drain = [&](int rc) {
        cudaStreamSynchronize(h->up);
        cudaStreamSynchronize(h->down);
        cudaStreamSynchronize(st);
        cudaGetLastError();
        return rc;
    };
    if (cudaEventRecord(ev[0], st) != cudaSuccess || cudaStreamWaitEvent(h->up, ev[0], 0) != cudaSuccess ||
        cudaStreamWaitEvent(h->down, ev[0], 0) != cudaSuccess)
        return drain(MXGEMM_ERR_CUDA);
    for (int t = 0; t < hb.pm || t < hb.pn; ++t) {
        if (t < hb.pm) {
            const size_t r0 = static_cast<size_t>(hb.mb) * t, r = part_rows(M, hb.mb, t);
            if (cudaMemcpyAsync(dA + r0 * rb, A_host + r0 * rb, r * rb, cudaMemcpyHostToDevice, h->up) !=
                    cudaSuccess ||
                cudaMemcpyAsync(dSA + r0 * sb, SA_host + r0 * sb, r * sb, cudaMemcpyHostToDevice, h->up) !=
                    cudaSuccess ||
                cudaEventRecord(ev[next], h->up) != cudaSuccess)
                return drain(MXGEMM_ERR_CUDA);
            a_ev[t] = next++;
            for (int j = 0; j < nb; ++j) {
                blk[nblk][0] = t;
                blk[nblk++][1] = j;
            }
            ++na;
        }
        if (t < hb.pn) {
            const size_t r0 = static_cast<size_t>(hb.nb) * t, r = part_rows(N, hb.nb, t);
            if (cudaMemcpyAsync(dB + r0 * rb, B_host + r0 * rb, r * rb, cudaMemcpyHostToDevice, h->up) !=
                    cudaSuccess ||
                cudaMemcpyAsync(dSB + r0 * sb, SB_host + r0 * sb, r * sb, cudaMemcpyHostToDevice, h->up) !=
                    cudaSuccess ||
                cudaEventRecord(ev[next], h->up) != cudaSuccess)
                return drain(MXGEMM_ERR_CUDA);
            b_ev[t] = next++;
            for (int i = 0; i < na; ++i) {
                blk[nblk][0] = i;
                blk[nblk++][1] = t;
            }
            ++nb;
        }
    }
    const int gemm_ev = next;
    for (int k = 0; k < nblk; ++k) {
        const int i = blk[k][0], j = blk[k][1];
        const size_t mi = part_rows(M, hb.mb, i), nj = part_rows(N, hb.nb, j);
        const size_t m0 = static_cast<size_t>(hb.mb) * i, n0 = static_cast<size_t>(hb.nb) * j;
        uint8_t *c = dC + (m0 * static_cast<size_t>(N) + mi * n0) * 2;
        if (cudaStreamWaitEvent(st, ev[a_ev[i] > b_ev[j] ? a_ev[i] : b_ev[j]], 0) != cudaSuccess)
            return drain(MXGEMM_ERR_CUDA);
        int rc = repack_and_gemm(h, fmt, static_cast<int64_t>(mi), static_cast<int64_t>(nj), K, dA + m0 * rb,
                                 dSA + m0 * sb, dB + n0 * rb, dSB + n0 * sb, c, st, mxg::Epilogue(), true, false);
        if (rc != MXGEMM_OK)
            return drain(rc);
        if (cudaEventRecord(ev[gemm_ev + k], st) != cudaSuccess)
            return drain(MXGEMM_ERR_CUDA);
    }
    for (int k = 0; k < nblk; ++k) {
        const int i = blk[k][0], j = blk[k][1];
        const size_t mi = part_rows(M, hb.mb, i), nj = part_rows(N, hb.nb, j);
        const size_t m0 = static_cast<size_t>(hb.mb) * i, n0 = static_cast<size_t>(hb.nb) * j;
        const uint8_t *c = dC + (m0 * static_cast<size_t>(N) + mi * n0) * 2;
        if (cudaStreamWaitEvent(h->down, ev[gemm_ev + k], 0) != cudaSuccess ||
            cudaMemcpy2DAsync(C_host + (m0 * static_cast<size_t>(N) + n0) * 2, static_cast<size_t>(N) * 2, c,
                              nj * 2, nj * 2, mi, cudaMemcpyDeviceToHost, h->down) != cudaSuccess)
            return drain(MXGEMM_ERR_CUDA);
    }
    if (cudaEventRecord(ev[1], h->down) != cudaSuccess || cudaStreamWaitEvent(st, ev[1], 0) != cudaSuccess)
        return drain(MXGEMM_ERR_CUDA);
    if (cudaStreamSynchronize(st) != cudaSuccess)
        return drain(MXGEMM_ERR_CUDA);
    return MXGEMM_OK;
}

void format_plan(const mxg::GemmPlan &pl, char *buf, size_t cap)
{
    static const char *names[] = {"auto", "dp", "splitk", "streamk", "ksplit", "dptail"};
    const char *scales = pl.fmt == mxg::kFmtBF16 ? "none" : ((fuse_scales(pl) || pl.groups > 0) ? "fused" : "repack");
    int n = snprintf(buf, cap,
                     "fmt=%d swap=%d pair=%d BN=%d kc=%d stages=%d tiles=%lld kt=%lld workers=%lld grid=%d sched=%s "
                     "partial_bytes=%lld scales=%s",
                     pl.fmt, pl.swap, pl.pair, pl.bn, pl.kc, pl.stages, static_cast<long long>(pl.tiles),
                     static_cast<long long>(pl.kt), static_cast<long long>(pl.workers), pl.grid,
                     names[pl.sched >= 0 && pl.sched <= 5 ? pl.sched : 0],
                     static_cast<long long>(pl.partial_bytes), scales);
    if (pl.groups > 0 && n > 0 && static_cast<size_t>(n) < cap)
        snprintf(buf + n, cap - n, " groups=%lld", static_cast<long long>(pl.groups));
    if (pl.pair && n > 0 && static_cast<size_t>(n) < cap)
        n += snprintf(buf + n, cap - n, " band=%lld", static_cast<long long>(pl.band));
    if (pl.ksplit > 1 && n > 0 && static_cast<size_t>(n) < cap)
        n += snprintf(buf + n, cap - n, " ksplit=%lld", static_cast<long long>(pl.ksplit));
    if (pl.pair && pl.tail_split > 1 && n > 0 && static_cast<size_t>(n) < cap)
        snprintf(buf + n, cap - n, " tail_first=%lld tail_split=%lld", static_cast<long long>(pl.tail_first),
                 static_cast<long long>(pl.tail_split));
}


}  // namespace

extern "C" {

const char *mxgemm_version(void) { return "0.1.0"; }

const char *mxgemm_status_string(int status)
{
    switch (status) {
    case MXGEMM_OK: return "ok";
    case MXGEMM_ERR_INVALID_ARG: return "invalid argument";
    case MXGEMM_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case MXGEMM_ERR_UNSUPPORTED_DEVICE: return "device is not sm_100 (B200)";
    case MXGEMM_ERR_OOM: return "workspace allocation failed";
    case MXGEMM_ERR_CUDA: return "CUDA call failed";
    case MXGEMM_ERR_TIMEOUT: return "a kernel gave up on a bounded wait";
    case MXGEMM_ERR_TOO_LARGE: return "problem exceeds the fixed scratch of mxgemm_run_noalloc (8 MiB of scales)";
    case MXGEMM_ERR_CAPTURE:
        return "the workspace must grow, which cannot happen during stream capture: run or reserve this shape first";
    default: return "unknown status";
    }
}

int mxgemm_create(mxgemm_handle *out)
{
    if (!out)
        return MXGEMM_ERR_INVALID_ARG;
    *out = nullptr;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return MXGEMM_ERR_UNSUPPORTED_DEVICE;
    }
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
        cudaGetLastError();
        return MXGEMM_ERR_CUDA;
    }
    if (prop.major != 10 || prop.minor != 0)
        return MXGEMM_ERR_UNSUPPORTED_DEVICE;
    if (mxg::prepare_gemm_kernels() != cudaSuccess)
        return MXGEMM_ERR_CUDA;
    mxgemm_ctx *h = new (std::nothrow) mxgemm_ctx();
    if (!h)
        return MXGEMM_ERR_OOM;
    h->device = dev;
    h->num_sms = prop.multiProcessorCount;
    if (cudaMalloc(reinterpret_cast<void **>(&h->err), 16) != cudaSuccess ||
        cudaMemset(h->err, 0, 16) != cudaSuccess) {
        cudaGetLastError();
        delete h;
        return MXGEMM_ERR_OOM;
    }
    *out = h;
    return MXGEMM_OK;
}

int mxgemm_destroy(mxgemm_handle h)
{
    if (!h)
        return MXGEMM_OK;
    int rc = enter_device(h);
    cudaDeviceSynchronize();
    cudaFree(h->sf);
    cudaFree(h->partials);
    cudaFree(h->counters);
    cudaFree(h->err);
    cudaFree(h->stage);
    for (cudaEvent_t &e : h->ev)
        if (e)
            cudaEventDestroy(e);
    for (cudaEvent_t &e : h->hev)
        if (e)
            cudaEventDestroy(e);
    if (h->up)
        cudaStreamDestroy(h->up);
    if (h->down)
        cudaStreamDestroy(h->down);
    delete h;
    return rc;
}

int mxgemm_repack(mxgemm_handle h, int fmt, int64_t M, int64_t N, int64_t K, const uint8_t *A_scales,
                  const uint8_t *B_scales, void *stream)
{
    if (!h)
        return MXGEMM_ERR_INVALID_ARG;
    int rc = check_shape(fmt, M, N, K);
    if (rc == MXGEMM_OK)
        rc = check_ptrs({A_scales, B_scales});
    if (rc == MXGEMM_OK)
        rc = enter_device(h);
    if (rc != MXGEMM_OK)
        return rc;
    return do_repack(h, fmt, M, N, K, A_scales, B_scales, static_cast<cudaStream_t>(stream));
}

int mxgemm_gemm(mxgemm_handle h, int fmt, int64_t M, int64_t N, int64_t K, const void *A, const void *B, void *C,
                void *stream)
{
    if (!h)
        return MXGEMM_ERR_INVALID_ARG;
    int rc = check_shape(fmt, M, N, K);
    if (rc == MXGEMM_OK)
        rc = check_ptrs({A, B, C});
    if (rc == MXGEMM_OK)
        rc = enter_device(h);
    if (rc != MXGEMM_OK)
        return rc;
    return do_gemm(h, fmt, M, N, K, A, B, C, static_cast<cudaStream_t>(stream), 0, 0);
}

int mxgemm_run(mxgemm_handle h, int fmt, int64_t M, int64_t N, int64_t K, const void *A, const uint8_t *A_scales,
               const void *B, const uint8_t *B_scales, void *C, void *stream)
{
    if (!h)
        return MXGEMM_ERR_INVALID_ARG;
    int rc = check_shape(fmt, M, N, K);
    if (rc == MXGEMM_OK)
        rc = check_ptrs({A, A_scales, B, B_scales, C});
    if (rc == MXGEMM_OK)
        rc = enter_device(h);
    if (rc != MXGEMM_OK)
        return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return repack_and_gemm(h, fmt, M, N, K, A, A_scales, B, B_scales, C, st);
}

int mxgemm_run_host(mxgemm_handle h, int fmt, int64_t M, int64_t N, int64_t K, const void *A_host,
                    const uint8_t *A_scales_host, const void *B_host, const uint8_t *B_scales_host, void *C_host,
                    void *stream)
{
    if (!h)
        return MXGEMM_ERR_INVALID_ARG;
    int rc = check_shape(fmt, M, N, K);
    if (rc == MXGEMM_OK && (!A_host || !A_scales_host || !B_host || !B_scales_host || !C_host))
        rc = MXGEMM_ERR_INVALID_ARG;
    if (rc == MXGEMM_OK)
        rc = enter_device(h);
    if (rc != MXGEMM_OK)
        return rc;
    auto up16 = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    const size_t rbytes = static_cast<size_t>(mxg::row_bytes(fmt, K));
    const size_t nA = static_cast<size_t>(M) * rbytes, nB = static_cast<size_t>(N) * rbytes;
    const size_t nSA = static_cast<size_t>(M) * static_cast<size_t>(K / 32);
    const size_t nSB = static_cast<size_t>(N) * static_cast<size_t>(K / 32);
    const size_t nC = static_cast<size_t>(M) * static_cast<size_t>(N) * 2;
    const size_t oA = 0, oSA = oA + up16(nA), oB = oSA + up16(nSA), oSB = oB + up16(nB), oC = oSB + up16(nSB);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    rc = grow(&h->stage, &h->stage_cap, oC + up16(nC), false, st);
    if (rc != MXGEMM_OK)
        return rc;
    uint8_t *d = h->stage;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) {
        cudaGetLastError();
        return MXGEMM_ERR_CUDA;
    }
    const HostBlocks hb = host_blocks(M, N, nA + nSA + nB + nSB + nC);
    if ((hb.pm > 1 || hb.pn > 1) && !h->profiling && cs == cudaStreamCaptureStatusNone)
        return run_host_blocked(h, fmt, M, N, K, static_cast<const uint8_t *>(A_host), A_scales_host,
                                static_cast<const uint8_t *>(B_host), B_scales_host, static_cast<uint8_t *>(C_host),
                                d + oA, d + oSA, d + oB, d + oSB, d + oC, hb, st);
    // on error, wait for the copies already queued (a capturing stream holds
    // none: its work has not run)
    auto drain = [&](int code) {
        if (cs == cudaStreamCaptureStatusNone)
            cudaStreamSynchronize(st);
        cudaGetLastError();
        return code;
    };
    if (cudaMemcpyAsync(d + oA, A_host, nA, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(d + oSA, A_scales_host, nSA, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(d + oB, B_host, nB, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(d + oSB, B_scales_host, nSB, cudaMemcpyHostToDevice, st) != cudaSuccess)
        return drain(MXGEMM_ERR_CUDA);
    rc = repack_and_gemm(h, fmt, M, N, K, d + oA, d + oSA, d + oB, d + oSB, d + oC, st);
    if (rc != MXGEMM_OK)
        return drain(rc);
    if (cudaMemcpyAsync(C_host, d + oC, nC, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return drain(MXGEMM_ERR_CUDA);
    if (cudaStreamSynchronize(st) != cudaSuccess)
        return MXGEMM_ERR_CUDA;
    return MXGEMM_OK;
}

int mxgemm_run_fused(mxgemm_handle h, int fmt, int64_t M, int64_t N, int64_t K, const void *A,
                     const uint8_t *A_scales, const void *B, const uint8_t *B_scales, const void *bias, int act,
                     const void *residual, void *C, void *stream)
{
    if (!h || act < MXGEMM_ACT_NONE || act > MXGEMM_ACT_GELU)
        return MXGEMM_ERR_INVALID_ARG;
    int rc = check_shape(fmt, M, N, K);
    if (rc == MXGEMM_OK)
        rc = check_ptrs({A, A_scales, B, B_scales, C});
    if (rc == MXGEMM_OK && !(optional_aligned16(bias) && optional_aligned16(residual)))
        rc = MXGEMM_ERR_ALIGNMENT;
    if (rc == MXGEMM_OK)
        rc = enter_device(h);
    if (rc != MXGEMM_OK)
        return rc;
    mxg::Epilogue epi;
    epi.bias = static_cast<const uint16_t *>(bias);
    epi.residual = static_cast<const uint16_t *>(residual);
    epi.act = act;
    return repack_and_gemm(h, fmt, M, N, K, A, A_scales, B, B_scales, C, static_cast<cudaStream_t>(stream), epi,
                           false);
}

int mxgemm_run_quantized(mxgemm_handle h, int fmt, int64_t M, int64_t N, int64_t K, const void *A,
                         const uint8_t *A_scales, const void *B, const uint8_t *B_scales, const void *bias, int act,
                         const void *residual, int out_fmt, void *C_codes, uint8_t *C_scales, void *stream)
{
    if (!h || act < MXGEMM_ACT_NONE || act > MXGEMM_ACT_GELU)
        return MXGEMM_ERR_INVALID_ARG;
    if (out_fmt != MXGEMM_FMT_MXFP8_E4M3 && out_fmt != MXGEMM_FMT_MXFP4_E2M1)
        return MXGEMM_ERR_INVALID_ARG;
    int rc = check_shape(fmt, M, N, K);
    if (rc == MXGEMM_OK && N % 32 != 0)
        rc = MXGEMM_ERR_INVALID_ARG;
    if (rc == MXGEMM_OK)
        rc = check_ptrs({A, A_scales, B, B_scales, C_codes, C_scales});
    if (rc == MXGEMM_OK && !(optional_aligned16(bias) && optional_aligned16(residual)))
        rc = MXGEMM_ERR_ALIGNMENT;
    if (rc == MXGEMM_OK)
        rc = enter_device(h);
    if (rc != MXGEMM_OK)
        return rc;
    mxg::Epilogue epi;
    epi.bias = static_cast<const uint16_t *>(bias);
    epi.residual = static_cast<const uint16_t *>(residual);
    epi.act = act;
    epi.qfmt = out_fmt;
    epi.Cq = static_cast<uint8_t *>(C_codes);
    epi.Cs = C_scales;
    // C itself is not written; the codes stand in for it in the launch
    return repack_and_gemm(h, fmt, M, N, K, A, A_scales, B, B_scales, C_codes, static_cast<cudaStream_t>(stream),
                           epi, false);
}

int mxgemm_quantize_bf16(int fmt, int64_t R, int64_t K, const void *X, void *Q, uint8_t *scales, void *stream)
{
    if (fmt != MXGEMM_FMT_MXFP8_E4M3 && fmt != MXGEMM_FMT_MXFP4_E2M1)
        return MXGEMM_ERR_INVALID_ARG;
    if (R < 1 || K < 32 || K % 32 != 0 || R > kMaxDim || K > kMaxDim)
        return MXGEMM_ERR_INVALID_ARG;
    if (!X || !Q || !scales)
        return MXGEMM_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(Q) || !aligned16(scales))
        return MXGEMM_ERR_ALIGNMENT;
    if (mxg::launch_quantize(fmt, R, K, nullptr, static_cast<uint8_t *>(Q), scales, static_cast<cudaStream_t>(stream),
                             static_cast<const uint16_t *>(X)) != cudaSuccess)
        return MXGEMM_ERR_CUDA;
    return MXGEMM_OK;
}

int mxgemm_run_bf16(mxgemm_handle h, int64_t M, int64_t N, int64_t K, const void *A, const void *B, void *C,
                    void *stream)
{
    if (!h)
        return MXGEMM_ERR_INVALID_ARG;
    if (M < 1 || N < 1 || K < 8 || K % 8 != 0 || M > kMaxDim || N > kMaxDim || K > kMaxDim)
        return MXGEMM_ERR_INVALID_ARG;
    int rc = check_ptrs({A, B, C});
    if (rc == MXGEMM_OK)
        rc = enter_device(h);
    if (rc != MXGEMM_OK)
        return rc;
    h->ev_valid = 0;
    const mxg::GemmPlan pl = plan_for(h, mxg::kFmtBF16, M, N, K, false);
    return launch_plan(h, pl, A, B, C, static_cast<cudaStream_t>(stream), 1, h->prefetch_b ? 2 : 0, nullptr, nullptr,
                       mxg::Epilogue());
}

int mxgemm_run_grouped(mxgemm_handle h, int fmt, int64_t G, int64_t M_total, int64_t N, int64_t K,
                       const int64_t *group_offsets, const void *A, const uint8_t *A_scales, const void *B,
                       const uint8_t *B_scales, void *C, void *stream)
{
    if (!h || G < 1 || G > kMaxGroups || M_total < 0)
        return MXGEMM_ERR_INVALID_ARG;
    const bool bf16 = fmt == MXGEMM_FMT_BF16;
    int rc = check_shape(bf16 ? MXGEMM_FMT_MXFP8_E4M3 : fmt, M_total > 0 ? M_total : 1, N, K);
    if (rc == MXGEMM_OK && G * N > kMaxDim)
        rc = MXGEMM_ERR_INVALID_ARG;
    if (rc == MXGEMM_OK)
        rc = bf16 ? check_ptrs({group_offsets, A, B, C}) : check_ptrs({group_offsets, A, A_scales, B, B_scales, C});
    if (rc == MXGEMM_OK)
        rc = enter_device(h);
    if (rc != MXGEMM_OK)
        return rc;
    h->ev_valid = 0;
    if (M_total == 0)
        return MXGEMM_OK;                 // every group is empty: nothing to compute
    const mxg::GemmPlan pl = mxg::make_grouped_plan(fmt, G, M_total, N, K, h->num_sms);
    if (!pl.valid)
        return MXGEMM_ERR_INVALID_ARG;
    return launch_plan(h, pl, A, B, C, static_cast<cudaStream_t>(stream), 1, 0, bf16 ? nullptr : A_scales,
                       bf16 ? nullptr : B_scales, mxg::Epilogue(), group_offsets);
}

int mxgemm_describe_grouped_plan(int num_sms, int fmt, int64_t G, int64_t M_total, int64_t N, int64_t K, char *buf,
                                 size_t cap)
{
    if (!buf || cap == 0 || num_sms < 2 || num_sms > 4096 || G < 1 || G > kMaxGroups || M_total < 1)
        return MXGEMM_ERR_INVALID_ARG;
    int rc = check_shape(fmt == MXGEMM_FMT_BF16 ? MXGEMM_FMT_MXFP8_E4M3 : fmt, M_total, N, K);
    if (rc != MXGEMM_OK || G * N > kMaxDim)
        return MXGEMM_ERR_INVALID_ARG;
    format_plan(mxg::make_grouped_plan(fmt, G, M_total, N, K, num_sms), buf, cap);
    return MXGEMM_OK;
}

int mxgemm_reserve(mxgemm_handle h, int fmt, int64_t M, int64_t N, int64_t K)
{
    if (!h)
        return MXGEMM_ERR_INVALID_ARG;
    int rc = check_shape(fmt, M, N, K);
    if (rc == MXGEMM_OK)
        rc = enter_device(h);
    if (rc != MXGEMM_OK)
        return rc;
    const mxg::GemmPlan pl = mxg::make_plan(fmt, M, N, K, h->num_sms, h->sched, h->splits, h->workers, h->kchunks);
    if (!pl.valid)
        return MXGEMM_ERR_INVALID_ARG;
    const size_t sf = static_cast<size_t>(mxg::sf_repacked_bytes(fmt, M, K) + mxg::sf_repacked_bytes(fmt, N, K));
    cudaStream_t st = nullptr;
    rc = grow(&h->sf, &h->sf_cap, sf, false, st);
    if (rc == MXGEMM_OK)
        rc = grow(&h->partials, &h->partials_cap,
                  static_cast<size_t>(pl.partial_bytes > 0 ? pl.partial_bytes : 16), false, st);
    if (rc == MXGEMM_OK)
        rc = grow(&h->counters, &h->counters_cap, static_cast<size_t>(pl.counter_bytes), true, st);
    return rc;
}

int mxgemm_set_profiling(mxgemm_handle h, int on)
{
    if (!h || (on != 0 && on != 1))
        return MXGEMM_ERR_INVALID_ARG;
    int rc = enter_device(h);
    if (rc != MXGEMM_OK)
        return rc;
    if (on)
        for (cudaEvent_t &e : h->ev)
            if (!e && cudaEventCreate(&e) != cudaSuccess)
                return MXGEMM_ERR_CUDA;
    h->profiling = on;
    h->ev_valid = 0;
    return MXGEMM_OK;
}

int mxgemm_set_prefetch_b(mxgemm_handle h, int on)
{
    if (!h || (on != 0 && on != 1))
        return MXGEMM_ERR_INVALID_ARG;
    h->prefetch_b = on;
    return MXGEMM_OK;
}

int mxgemm_last_timing(mxgemm_handle h, float *repack_ms, float *gemm_ms)
{
    if (!h || !repack_ms || !gemm_ms || !h->ev_valid)
        return MXGEMM_ERR_INVALID_ARG;
    int rc = enter_device(h);
    if (rc != MXGEMM_OK)
        return rc;
    if (cudaEventSynchronize(h->ev[2]) != cudaSuccess ||
        cudaEventElapsedTime(repack_ms, h->ev[0], h->ev[1]) != cudaSuccess ||
        cudaEventElapsedTime(gemm_ms, h->ev[1], h->ev[2]) != cudaSuccess)
        return MXGEMM_ERR_CUDA;
    return MXGEMM_OK;
}

int mxgemm_quantize(int fmt, int64_t R, int64_t K, const float *X, void *Q, uint8_t *scales, void *stream)
{
    if (fmt != MXGEMM_FMT_MXFP8_E4M3 && fmt != MXGEMM_FMT_MXFP4_E2M1)
        return MXGEMM_ERR_INVALID_ARG;
    if (R < 1 || K < 32 || K % 32 != 0 || R > kMaxDim || K > kMaxDim)
        return MXGEMM_ERR_INVALID_ARG;
    if (!X || !Q || !scales)
        return MXGEMM_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(Q) || !aligned16(scales))
        return MXGEMM_ERR_ALIGNMENT;
    if (mxg::launch_quantize(fmt, R, K, X, static_cast<uint8_t *>(Q), scales, static_cast<cudaStream_t>(stream)) !=
        cudaSuccess)
        return MXGEMM_ERR_CUDA;
    return MXGEMM_OK;
}

int mxgemm_set_schedule(mxgemm_handle h, int schedule, int splits, int workers)
{
    if (!h || schedule < MXGEMM_SCHED_AUTO || schedule > MXGEMM_SCHED_KSPLIT || splits < 1 || workers < 0)
        return MXGEMM_ERR_INVALID_ARG;
    h->sched = schedule;
    h->splits = splits;
    h->workers = workers;
    return MXGEMM_OK;
}

int mxgemm_set_kchunks(mxgemm_handle h, int kc)
{
    if (!h || kc < 0 || kc > 4 || kc == 3)
        return MXGEMM_ERR_INVALID_ARG;
    h->kchunks = kc;
    return MXGEMM_OK;
}

int mxgemm_describe_plan(mxgemm_handle h, int fmt, int64_t M, int64_t N, int64_t K, char *buf, size_t cap)
{
    if (!h || !buf || cap == 0)
        return MXGEMM_ERR_INVALID_ARG;
    if (fmt == MXGEMM_FMT_BF16) {           // the plan of mxgemm_run_bf16
        if (M < 1 || N < 1 || K < 8 || K % 8 != 0 || M > kMaxDim || N > kMaxDim || K > kMaxDim)
            return MXGEMM_ERR_INVALID_ARG;
        format_plan(mxg::make_plan(fmt, M, N, K, h->num_sms, h->sched, h->splits, h->workers, h->kchunks, false),
                    buf, cap);
        return MXGEMM_OK;
    }
    int rc = check_shape(fmt, M, N, K);
    if (rc != MXGEMM_OK)
        return rc;
    format_plan(mxg::make_plan(fmt, M, N, K, h->num_sms, h->sched, h->splits, h->workers, h->kchunks), buf, cap);
    return MXGEMM_OK;
}

int mxgemm_describe_plan_for(int num_sms, int fmt, int64_t M, int64_t N, int64_t K, char *buf, size_t cap)
{
    if (!buf || cap == 0 || num_sms < 2 || num_sms > 4096)
        return MXGEMM_ERR_INVALID_ARG;
    if (fmt == MXGEMM_FMT_BF16) {           // the plan of mxgemm_run_bf16
        if (M < 1 || N < 1 || K < 8 || K % 8 != 0 || M > kMaxDim || N > kMaxDim || K > kMaxDim)
            return MXGEMM_ERR_INVALID_ARG;
        format_plan(mxg::make_plan(fmt, M, N, K, num_sms, MXGEMM_SCHED_AUTO, 1, 0, 0, false), buf, cap);
        return MXGEMM_OK;
    }
    int rc = check_shape(fmt, M, N, K);
    if (rc != MXGEMM_OK)
        return rc;
    format_plan(mxg::make_plan(fmt, M, N, K, num_sms, MXGEMM_SCHED_AUTO, 1, 0, 0), buf, cap);
    return MXGEMM_OK;
}

int mxgemm_check_device_error(mxgemm_handle h, int *code)
{
    if (!h || !code)
        return MXGEMM_ERR_INVALID_ARG;
    int rc = enter_device(h);
    if (rc != MXGEMM_OK)
        return rc;
    int v = 0;
    if (cudaDeviceSynchronize() != cudaSuccess || cudaMemcpy(&v, h->err, sizeof(int), cudaMemcpyDeviceToHost) !=
                                                      cudaSuccess)
        return MXGEMM_ERR_CUDA;
    *code = v;
    if (v != 0) {
        // A CTA that gave up may have left split counters behind: clear them.
        if (cudaMemset(h->err, 0, sizeof(int)) != cudaSuccess ||
            (h->counters && cudaMemset(h->counters, 0, h->counters_cap) != cudaSuccess) ||
            cudaDeviceSynchronize() != cudaSuccess)
            return MXGEMM_ERR_CUDA;
        return MXGEMM_ERR_TIMEOUT;
    }
    return MXGEMM_OK;
}

int mxgemm_set_wait_limit(mxgemm_handle h, uint64_t ns)
{
    if (!h)
        return MXGEMM_ERR_INVALID_ARG;
    h->limit_ns = ns == 0 ? kDefaultLimitNs : ns;
    return MXGEMM_OK;
}

int mxgemm_debug_inject(mxgemm_handle h, int mode)
{
    if (!h || mode < 0 || mode > 1)
        return MXGEMM_ERR_INVALID_ARG;
    h->inject = mode;
    return MXGEMM_OK;
}

}  // extern "C"
