// qmv_inst_tcb_b5.cu -- tensor-core affine 5-bit qmv kernels with the bulk-copy
// weight ring (all dtypes).
#include "qmv_launch.cuh"

namespace qmv {

cudaError_t launch_tcb_affine_b5(int dtype, int npass, int spb, int ncw, const Params& p, const Launch& L) {
#define BITS_ 5
    QMV_TCB_DISPATCH_DTYPE()
#undef BITS_
}

}  // namespace qmv
