// qmv_tc_dispatch.cu -- bits -> tensor-core kernel dispatchers.
#include "qmv_launch.cuh"

namespace qmv {

cudaError_t launch_tc_affine_b2(int, int, const Params&, const Launch&);
cudaError_t launch_tc_affine_b3(int, int, const Params&, const Launch&);
cudaError_t launch_tc_affine_b4(int, int, const Params&, const Launch&);
cudaError_t launch_tc_affine_b5(int, int, const Params&, const Launch&);
cudaError_t launch_tc_affine_b6(int, int, const Params&, const Launch&);
cudaError_t launch_tc_affine_b8(int, int, const Params&, const Launch&);

cudaError_t launch_tcb_affine_b2(int, int, int, int, const Params&, const Launch&);
cudaError_t launch_tcb_affine_b3(int, int, int, int, const Params&, const Launch&);
cudaError_t launch_tcb_affine_b4(int, int, int, int, const Params&, const Launch&);
cudaError_t launch_tcb_affine_b5(int, int, int, int, const Params&, const Launch&);
cudaError_t launch_tcb_affine_b6(int, int, int, int, const Params&, const Launch&);
cudaError_t launch_tcb_affine_b8(int, int, int, int, const Params&, const Launch&);

cudaError_t launch_tc_affine(int bits, int dtype, int npass, const Params& p, const Launch& L) {
    switch (bits) {
        case 2: return launch_tc_affine_b2(dtype, npass, p, L);
        case 3: return launch_tc_affine_b3(dtype, npass, p, L);
        case 4: return launch_tc_affine_b4(dtype, npass, p, L);
        case 5: return launch_tc_affine_b5(dtype, npass, p, L);
        case 6: return launch_tc_affine_b6(dtype, npass, p, L);
        case 8: return launch_tc_affine_b8(dtype, npass, p, L);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_tcb_affine(int bits, int dtype, int npass, int spb, int ncw, const Params& p, const Launch& L) {
    switch (bits) {
        case 2: return launch_tcb_affine_b2(dtype, npass, spb, ncw, p, L);
        case 3: return launch_tcb_affine_b3(dtype, npass, spb, ncw, p, L);
        case 4: return launch_tcb_affine_b4(dtype, npass, spb, ncw, p, L);
        case 5: return launch_tcb_affine_b5(dtype, npass, spb, ncw, p, L);
        case 6: return launch_tcb_affine_b6(dtype, npass, spb, ncw, p, L);
        case 8: return launch_tcb_affine_b8(dtype, npass, spb, ncw, p, L);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace qmv
