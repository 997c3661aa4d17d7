// qmv_inst_sint_b5.cu -- symmetric signed 5-bit qmv kernels (int5 / mxint5 and the
// FP16-scale twin; all dtypes and launch shapes).
#include "qmv_launch.cuh"

namespace qmv {

cudaError_t launch_sint_b5(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L) {
#define FAM_ FAM_SINT
#define BITS_ 5
    QMV_DISPATCH_DTYPE()
#undef FAM_
#undef BITS_
}

}  // namespace qmv
