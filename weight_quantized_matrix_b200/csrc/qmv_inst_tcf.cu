// qmv_inst_tcf.cu -- CUDA-core affine qmv kernels with the weight ring, one
// bf16 x row (every code width; 8 or 12 compute warps and a producer warp).
#include "qmv_launch.cuh"
#include "qmv_tcf.cuh"

namespace qmv {

namespace {

template <int B>
cudaError_t tcf_b(int ncw, const Params& p, const Launch& L) {
    if (ncw == 8) {
        static std::atomic<unsigned> cfg_{0};
        return launch_kernel(qmv_tcf_kernel<FAM_AFFINE, B, kTcbStages, 288>, cfg_, L, p);
    }
    if (ncw == 12) {
        static std::atomic<unsigned> cfg_{0};
        return launch_kernel(qmv_tcf_kernel<FAM_AFFINE, B, kTcbStages, 416>, cfg_, L, p);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_tcf_affine(int bits, int ncw, const Params& p, const Launch& L) {
    switch (bits) {
        case 2: return tcf_b<2>(ncw, p, L);
        case 3: return tcf_b<3>(ncw, p, L);
        case 4: return tcf_b<4>(ncw, p, L);
        case 5: return tcf_b<5>(ncw, p, L);
        case 6: return tcf_b<6>(ncw, p, L);
        case 8: return tcf_b<8>(ncw, p, L);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace qmv
