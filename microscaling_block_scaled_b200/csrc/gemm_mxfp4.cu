// gemm_mxfp4.cu -- instantiates the one-CTA GEMM kernel for MXFP4 (E2M1)
// operands (the kernel itself is in gemm_kernel.cuh).
#include "gemm_kernel.cuh"

namespace mxg {

namespace {

template <int KC>
int stages_kc(int bn)
{
    switch (bn) {
    case 16: return Cfg<kFmtMXFP4, 16, KC>::kStages;
    case 32: return Cfg<kFmtMXFP4, 32, KC>::kStages;
    case 64: return Cfg<kFmtMXFP4, 64, KC>::kStages;
    default: break;
    }
    if constexpr (KC != 4) {                // four chunks per stage: tiles of at most 64 columns
        if (bn == 128)
            return Cfg<kFmtMXFP4, 128, KC>::kStages;
        if (bn == 256)
            return Cfg<kFmtMXFP4, 256, KC>::kStages;
    }
    return 0;
}

}  // namespace

int stages_mxfp4(int bn, int kc)
{
    return kc == 4 ? stages_kc<4>(bn) : (kc == 1 ? stages_kc<1>(bn) : stages_kc<2>(bn));
}

cudaError_t launch_gemm_mxfp4(const GemmPlan &pl, const GemmBuffers &b, uint64_t limit_ns, int inject, int pdl,
                             cudaStream_t st)
{
    if (pl.kc == 4)
        return dispatch_bn4<kFmtMXFP4>(pl, b, limit_ns, inject, pdl, st);
    return pl.kc == 1 ? dispatch_bn<kFmtMXFP4, 1>(pl, b, limit_ns, inject, pdl, st)
                      : dispatch_bn<kFmtMXFP4, 2>(pl, b, limit_ns, inject, pdl, st);
}

cudaError_t prepare_mxfp4()
{
    cudaError_t e = cudaSuccess;
    cudaError_t (*const fns[])() = {
        set_attrs<kFmtMXFP4, 16, 1>, set_attrs<kFmtMXFP4, 32, 1>, set_attrs<kFmtMXFP4, 64, 1>, set_attrs<kFmtMXFP4, 128, 1>,
        set_attrs<kFmtMXFP4, 256, 1>, set_attrs<kFmtMXFP4, 16, 2>, set_attrs<kFmtMXFP4, 32, 2>, set_attrs<kFmtMXFP4, 64, 2>,
        set_attrs<kFmtMXFP4, 128, 2>, set_attrs<kFmtMXFP4, 256, 2>, set_attrs<kFmtMXFP4, 16, 4>, set_attrs<kFmtMXFP4, 32, 4>,
        set_attrs<kFmtMXFP4, 64, 4>};
    for (auto f : fns)
        if (e == cudaSuccess)
            e = f();
    return e;
}

}  // namespace mxg
