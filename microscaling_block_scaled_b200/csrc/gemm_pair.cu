// gemm_pair.cu -- instantiates the CTA-pair (cta_group::2) GEMM kernel for
// MXFP8 and MXFP4 operands (the kernel itself is in gemm_pair_kernel.cuh).
#include "gemm_pair_kernel.cuh"

namespace mxg {

int stages_pair(int fmt, int kc)
{
    return fmt == kFmtMXFP8 ? (kc == 1 ? PairCfg<0, 1>::kStages : PairCfg<0, 2>::kStages)
                            : (kc == 1 ? PairCfg<1, 1>::kStages : PairCfg<1, 2>::kStages);
}

cudaError_t launch_gemm_pair(const GemmPlan &pl, const GemmBuffers &b, uint64_t limit_ns, int inject, int pdl,
                             cudaStream_t st)
{
    if (pl.fmt == kFmtMXFP8)
        return pl.kc == 1 ? launch_pair_t<0, 1>(pl, b, limit_ns, inject, pdl, st)
                          : launch_pair_t<0, 2>(pl, b, limit_ns, inject, pdl, st);
    return pl.kc == 1 ? launch_pair_t<1, 1>(pl, b, limit_ns, inject, pdl, st)
                      : launch_pair_t<1, 2>(pl, b, limit_ns, inject, pdl, st);
}

cudaError_t prepare_pair()
{
    cudaError_t e = cudaSuccess;
#define MXG_ATTRP(F, KCV)                                                                             \
    if (e == cudaSuccess)                                                                             \
        e = cudaFuncSetAttribute(mx_gemm_pair_kernel<F, KCV>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                 PairCfg<F, KCV>::kSmemBytes);
    MXG_ATTRP(0, 1) MXG_ATTRP(0, 2) MXG_ATTRP(1, 1) MXG_ATTRP(1, 2)
#undef MXG_ATTRP
    return e;
}

}  // namespace mxg
