// qmv_inst_qkv_b2.cu -- Q / K / V in one call, affine 2-bit (all dtypes and
// the row-tiled shapes of large N).
#include "qmv_launch.cuh"

namespace qmv {

cudaError_t launch_affine_qkv_b2(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L) {
#define BITS_ 2
    QMV_QKV_DISPATCH_DTYPE()
#undef BITS_
}

}  // namespace qmv
