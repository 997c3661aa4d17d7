// qmv_inst_tc_b2.cu -- tensor-core affine 2-bit qmv kernels (all dtypes).
#include "qmv_launch.cuh"

namespace qmv {

cudaError_t launch_tc_affine_b2(int dtype, int npass, const Params& p, const Launch& L) {
#define BITS_ 2
    QMV_TC_DISPATCH_DTYPE()
#undef BITS_
}

}  // namespace qmv
