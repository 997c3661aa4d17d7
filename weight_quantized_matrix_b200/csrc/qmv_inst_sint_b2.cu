// qmv_inst_sint_b2.cu -- symmetric signed 2-bit qmv kernels (int2 / mxint2 and the
// FP16-scale twin; all dtypes and launch shapes).
#include "qmv_launch.cuh"

namespace qmv {

cudaError_t launch_sint_b2(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L) {
#define FAM_ FAM_SINT
#define BITS_ 2
    QMV_DISPATCH_DTYPE()
#undef FAM_
#undef BITS_
}

}  // namespace qmv
