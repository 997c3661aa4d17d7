// qmv_inst_tcf_fp.cu -- CUDA-core qmv kernels with the weight ring for the
// block-scaled FP formats, one bf16 x row (E2M1 and E4M3 / E5M2 elements; 8 or
// 12 compute warps and a producer warp).
#include "qmv_launch.cuh"
#include "qmv_tcf.cuh"

namespace qmv {

namespace {

template <int FAM, int B>
cudaError_t tcf_fp(int ncw, const Params& p, const Launch& L) {
    if (ncw == 8) {
        static std::atomic<unsigned> cfg_{0};
        return launch_kernel(qmv_tcf_kernel<FAM, B, kTcbStages, 288>, cfg_, L, p);
    }
    if (ncw == 12) {
        static std::atomic<unsigned> cfg_{0};
        return launch_kernel(qmv_tcf_kernel<FAM, B, kTcbStages, 416>, cfg_, L, p);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_tcf_fp(int fam, int ncw, const Params& p, const Launch& L) {
    switch (fam) {
        case FAM_MXFP4: return tcf_fp<FAM_MXFP4, 4>(ncw, p, L);
        case FAM_NVFP4: return tcf_fp<FAM_NVFP4, 4>(ncw, p, L);
        case FAM_E2M1: return tcf_fp<FAM_E2M1, 4>(ncw, p, L);
        case FAM_MXFP8: return tcf_fp<FAM_MXFP8, 8>(ncw, p, L);
        case FAM_E4M3: return tcf_fp<FAM_E4M3, 8>(ncw, p, L);
        case FAM_E5M2: return tcf_fp<FAM_E5M2, 8>(ncw, p, L);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace qmv
