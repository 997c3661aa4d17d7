// qmv_inst_sint_b4.cu -- symmetric signed 4-bit qmv kernels (int4 / mxint4 and the
// FP16-scale twin; all dtypes and launch shapes).
#include "qmv_launch.cuh"

namespace qmv {

cudaError_t launch_sint_b4(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L) {
#define FAM_ FAM_SINT
#define BITS_ 4
    QMV_DISPATCH_DTYPE()
#undef FAM_
#undef BITS_
}

}  // namespace qmv
