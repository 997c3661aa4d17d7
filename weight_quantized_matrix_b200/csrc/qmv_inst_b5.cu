// qmv_inst_b5.cu -- affine 5-bit qmv kernels (all dtypes and launch shapes).
#include "qmv_launch.cuh"

namespace qmv {

cudaError_t launch_affine_b5(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L) {
#define FAM_ FAM_AFFINE
#define BITS_ 5
    QMV_DISPATCH_DTYPE()
#undef FAM_
#undef BITS_
}

}  // namespace qmv
