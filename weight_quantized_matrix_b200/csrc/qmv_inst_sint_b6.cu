// qmv_inst_sint_b6.cu -- symmetric signed 6-bit qmv kernels (int6 / mxint6 and the
// FP16-scale twin; all dtypes and launch shapes).
#include "qmv_launch.cuh"

namespace qmv {

cudaError_t launch_sint_b6(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L) {
#define FAM_ FAM_SINT
#define BITS_ 6
    QMV_DISPATCH_DTYPE()
#undef FAM_
#undef BITS_
}

}  // namespace qmv
