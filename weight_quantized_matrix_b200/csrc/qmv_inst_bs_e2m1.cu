// qmv_inst_bs_e2m1.cu -- E2M1-element qmv kernels with a run-time block scale (type
// E8M0 / E4M3 / FP32 / FP16, block 16 or 32; all dtypes and launch shapes).
#include "qmv_launch.cuh"

namespace qmv {

cudaError_t launch_bs_e2m1(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L) {
#define FAM_ FAM_E2M1
#define BITS_ 4
    QMV_DISPATCH_DTYPE()
#undef FAM_
#undef BITS_
}

}  // namespace qmv
