// qmv_inst_tc_b5.cu -- tensor-core affine 5-bit qmv kernels (all dtypes).
#include "qmv_launch.cuh"

namespace qmv {

cudaError_t launch_tc_affine_b5(int dtype, int npass, const Params& p, const Launch& L) {
#define BITS_ 5
    QMV_TC_DISPATCH_DTYPE()
#undef BITS_
}

}  // namespace qmv
