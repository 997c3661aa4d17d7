// qmv_inst_tc_b8.cu -- tensor-core affine 8-bit qmv kernels (all dtypes).
#include "qmv_launch.cuh"

namespace qmv {

cudaError_t launch_tc_affine_b8(int dtype, int npass, const Params& p, const Launch& L) {
#define BITS_ 8
    QMV_TC_DISPATCH_DTYPE()
#undef BITS_
}

}  // namespace qmv
