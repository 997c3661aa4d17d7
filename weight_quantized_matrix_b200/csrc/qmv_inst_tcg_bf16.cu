// qmv_inst_tcg_bf16.cu -- the per-group tensor-core ring kernels for bf16 x,
// and the dtype dispatcher.
#include "qmv_inst_tcg.cuh"

namespace qmv {

cudaError_t launch_tcg_bf16(int G, int nt, const Params& p, const Launch& L) {
    return launch_tcg_g<__nv_bfloat16>(G, nt, p, L);
}

cudaError_t launch_tcg_affine(int dtype, int G, int nt, const Params& p, const Launch& L) {
    if (dtype == 2) return launch_tcg_bf16(G, nt, p, L);
    if (dtype == 1) return launch_tcg_f16(G, nt, p, L);
    return cudaErrorInvalidValue;
}

}  // namespace qmv
