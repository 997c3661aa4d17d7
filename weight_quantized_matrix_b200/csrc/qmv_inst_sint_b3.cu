// qmv_inst_sint_b3.cu -- symmetric signed 3-bit qmv kernels (int3 / mxint3 and the
// FP16-scale twin; all dtypes and launch shapes).
#include "qmv_launch.cuh"

namespace qmv {

cudaError_t launch_sint_b3(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L) {
#define FAM_ FAM_SINT
#define BITS_ 3
    QMV_DISPATCH_DTYPE()
#undef FAM_
#undef BITS_
}

}  // namespace qmv
