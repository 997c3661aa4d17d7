// qmv_inst_tcb_b3.cu -- tensor-core affine 3-bit qmv kernels with the bulk-copy
// weight ring (all dtypes).
#include "qmv_launch.cuh"

namespace qmv {

cudaError_t launch_tcb_affine_b3(int dtype, int npass, int spb, int ncw, const Params& p, const Launch& L) {
#define BITS_ 3
    QMV_TCB_DISPATCH_DTYPE()
#undef BITS_
}

}  // namespace qmv
