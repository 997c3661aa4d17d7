// qmv_inst_pair_b5.cu -- fused gate + up SwiGLU kernels, affine 5-bit (all
// dtypes and pair launch shapes).
#include "qmv_launch.cuh"

namespace qmv {

cudaError_t launch_affine_pair_b5(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L) {
#define BITS_ 5
    QMV_PAIR_DISPATCH_DTYPE()
#undef BITS_
}

}  // namespace qmv
