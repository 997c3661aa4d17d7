// qmv_inst_b4.cu -- affine 4-bit qmv kernels (all dtypes and launch shapes).
#include "qmv_launch.cuh"

namespace qmv {

cudaError_t launch_affine_b4(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L) {
#define FAM_ FAM_AFFINE
#define BITS_ 4
    QMV_DISPATCH_DTYPE()
#undef FAM_
#undef BITS_
}

}  // namespace qmv
