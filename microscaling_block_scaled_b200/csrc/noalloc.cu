// noalloc.cu -- mxgemm_run_noalloc: the repack + GEMM hot path without any
// device allocation.
//
// Who needs it: callers that cannot call cudaMalloc at the point where they
// run the GEMM -- for example code running inside a memory pool or allocator
// hook that must not re-enter the allocator, a runtime whose allocations are
// all made up front at start-up, or a process that has handed its memory
// budget to another framework.  mxgemm_run needs a handle, and a handle
// allocates its workspace (repacked scales, error word) with cudaMalloc;
// this entry point keeps that workspace in a fixed-size array compiled into
// the library instead.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds it until the process exits.  In host code its name is only a
// stand-in for the device symbol, so the device address is fetched once per
// device with cudaGetSymbolAddress and passed to the kernels.
//
// Limits and sharing:
//  * the repacked scales of A and B must fit in kNoAllocScratchBytes
//    (8 MiB); larger problems get MXGEMM_ERR_TOO_LARGE;
//  * the GEMM always runs whole output tiles (no split-K), so it needs no
//    partial sums or tile counters;
//  * every call uses the same array and leaves its contents behind; the
//    error word is cleared at the start of each call, the scale region is
//    fully rewritten by the repack.  Calls whose work overlaps on the GPU
//    (two streams, or two host threads) race on the array and give wrong
//    results: order them on one stream;
//  * the kernels' bounded waits still end a stuck launch cleanly, but this
//    entry point has no query for the error word they set.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/mxgemm.h"
#include "mx_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;   // repacked scales of A and B
constexpr size_t kNoAllocErrorBytes = 256;                 // device error word (+ padding)

// The scratch: [scales of A | scales of B | ... free ... ][error word]
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes + kNoAllocErrorBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
uint8_t *g_scratch_ptr[kMaxDevices] = {};
int g_num_sms[kMaxDevices] = {};

// Once per device (with that device current): check it is an sm_100 part,
// set the GEMM kernels' shared-memory limits and fetch the device address
// of the scratch array.
int setup_device(int dev, uint8_t **scratch, int *num_sms)
{
    if (dev < 0 || dev >= kMaxDevices)
        return MXGEMM_ERR_UNSUPPORTED_DEVICE;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
            cudaGetLastError();
            return MXGEMM_ERR_CUDA;
        }
        if (prop.major != 10 || prop.minor != 0)
            return MXGEMM_ERR_UNSUPPORTED_DEVICE;
        if (mxg::prepare_gemm_kernels() != cudaSuccess)
            return MXGEMM_ERR_CUDA;
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return MXGEMM_ERR_CUDA;
        }
        g_num_sms[dev] = prop.multiProcessorCount;
        g_scratch_ptr[dev] = static_cast<uint8_t *>(p);
    }
    *scratch = g_scratch_ptr[dev];
    *num_sms = g_num_sms[dev];
    return MXGEMM_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

int mxgemm_run_noalloc(int fmt, int64_t M, int64_t N, int64_t K, const void *A, const uint8_t *A_scales,
                       const void *B, const uint8_t *B_scales, void *C, void *stream)
{
    if (fmt != MXGEMM_FMT_MXFP8_E4M3 && fmt != MXGEMM_FMT_MXFP4_E2M1)
        return MXGEMM_ERR_INVALID_ARG;
    if (M < 1 || N < 1 || K < 128 || K % 128 != 0 || M > (int64_t(1) << 24) || N > (int64_t(1) << 24) ||
        K > (int64_t(1) << 24))
        return MXGEMM_ERR_INVALID_ARG;
    if (!A || !A_scales || !B || !B_scales || !C)
        return MXGEMM_ERR_INVALID_ARG;
    if (!aligned16(A) || !aligned16(A_scales) || !aligned16(B) || !aligned16(B_scales) || !aligned16(C))
        return MXGEMM_ERR_ALIGNMENT;
    const int64_t ba = mxg::sf_repacked_bytes(fmt, M, K);
    const int64_t bb = mxg::sf_repacked_bytes(fmt, N, K);
    if (ba + bb > static_cast<int64_t>(kNoAllocScratchBytes))
        return MXGEMM_ERR_TOO_LARGE;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return MXGEMM_ERR_UNSUPPORTED_DEVICE;
    }
    uint8_t *scratch = nullptr;
    int num_sms = 0;
    int rc = setup_device(dev, &scratch, &num_sms);
    if (rc != MXGEMM_OK)
        return rc;
    const mxg::GemmPlan pl = mxg::make_plan(fmt, M, N, K, num_sms, MXGEMM_SCHED_DP, 1, 0, 0);
    if (!pl.valid || pl.partial_bytes != 0)
        return MXGEMM_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int *err = reinterpret_cast<int *>(scratch + kNoAllocScratchBytes);
    if (cudaMemsetAsync(err, 0, sizeof(int), st) != cudaSuccess)
        return MXGEMM_ERR_CUDA;
    uint8_t *sfa = scratch;
    uint8_t *sfb = scratch + ba;
    if (mxg::launch_repack(fmt, M, N, K, A_scales, B_scales, sfa, sfb, st) != cudaSuccess)
        return MXGEMM_ERR_CUDA;
    mxg::GemmBuffers b;
    b.A = A;
    b.B = B;
    b.sfA = sfa;
    b.sfB = sfb;
    b.C = C;
    b.partials = nullptr;      // whole tiles only: never touched
    b.counters = nullptr;
    b.error = err;
    b.early = 3;               // the preceding kernel is the repack, which writes neither operand
    if (mxg::launch_gemm(pl, b, 2000000000ull, 0, 1, st) != cudaSuccess)
        return MXGEMM_ERR_CUDA;
    return MXGEMM_OK;
}

}  // extern "C"
