// qmv_inst_bs_e4m3.cu -- E4M3-element qmv kernels with a run-time block scale (type
// E8M0 / E4M3 / FP32 / FP16, block 16 or 32; all dtypes and launch shapes).
#include "qmv_launch.cuh"

namespace qmv {

cudaError_t launch_bs_e4m3(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L) {
#define FAM_ FAM_E4M3
#define BITS_ 8
    QMV_DISPATCH_DTYPE()
#undef FAM_
#undef BITS_
}

}  // namespace qmv
