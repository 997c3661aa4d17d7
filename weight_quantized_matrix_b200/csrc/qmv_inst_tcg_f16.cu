// qmv_inst_tcg_f16.cu -- the per-group tensor-core ring kernels for f16 x.
#include "qmv_inst_tcg.cuh"

namespace qmv {

cudaError_t launch_tcg_f16(int G, int nt, const Params& p, const Launch& L) {
    return launch_tcg_g<__half>(G, nt, p, L);
}

}  // namespace qmv
