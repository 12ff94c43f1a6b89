// gemm_bf16.cu -- instantiates the one-CTA GEMM kernel for dense BF16
// operands (the kernel itself is in gemm_kernel.cuh).
#include "gemm_kernel.cuh"

namespace mxg {

namespace {

template <int KC>
int stages_kc(int bn)
{
    switch (bn) {
    case 16: return Cfg<kFmtBF16, 16, KC>::kStages;
    case 32: return Cfg<kFmtBF16, 32, KC>::kStages;
    case 64: return Cfg<kFmtBF16, 64, KC>::kStages;
    default: break;
    }
    if constexpr (KC != 4) {                // four chunks per stage: tiles of at most 64 columns
        if (bn == 128)
            return Cfg<kFmtBF16, 128, KC>::kStages;
        if (bn == 256)
            return Cfg<kFmtBF16, 256, KC>::kStages;
    }
    return 0;
}

}  // namespace

int stages_bf16(int bn, int kc)
{
    return kc == 4 ? stages_kc<4>(bn) : (kc == 1 ? stages_kc<1>(bn) : stages_kc<2>(bn));
}

cudaError_t launch_gemm_bf16(const GemmPlan &pl, const GemmBuffers &b, uint64_t limit_ns, int inject, int pdl,
                             cudaStream_t st)
{
    if (pl.kc == 4)
        return dispatch_bn4<kFmtBF16>(pl, b, limit_ns, inject, pdl, st);
    return pl.kc == 1 ? dispatch_bn<kFmtBF16, 1>(pl, b, limit_ns, inject, pdl, st)
                      : dispatch_bn<kFmtBF16, 2>(pl, b, limit_ns, inject, pdl, st);
}

cudaError_t prepare_bf16()
{
    cudaError_t e = cudaSuccess;
    cudaError_t (*const fns[])() = {
        set_attrs<kFmtBF16, 16, 1>, set_attrs<kFmtBF16, 32, 1>, set_attrs<kFmtBF16, 64, 1>, set_attrs<kFmtBF16, 128, 1>,
        set_attrs<kFmtBF16, 256, 1>, set_attrs<kFmtBF16, 16, 2>, set_attrs<kFmtBF16, 32, 2>, set_attrs<kFmtBF16, 64, 2>,
        set_attrs<kFmtBF16, 128, 2>, set_attrs<kFmtBF16, 256, 2>, set_attrs<kFmtBF16, 16, 4>, set_attrs<kFmtBF16, 32, 4>,
        set_attrs<kFmtBF16, 64, 4>};
    for (auto f : fns)
        if (e == cudaSuccess)
            e = f();
    return e;
}

}  // namespace mxg
