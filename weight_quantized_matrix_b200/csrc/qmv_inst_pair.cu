// qmv_inst_pair.cu -- bits -> the fused gate + up SwiGLU and the Q / K / V
// instantiation units.
#include "qmv_launch.cuh"

namespace qmv {

cudaError_t launch_affine_pair_b2(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_affine_pair_b3(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_affine_pair_b4(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_affine_pair_b5(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_affine_pair_b6(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_affine_pair_b8(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);

cudaError_t launch_affine_qkv_b2(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_affine_qkv_b3(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_affine_qkv_b4(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_affine_qkv_b5(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_affine_qkv_b6(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_affine_qkv_b8(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);

cudaError_t launch_affine_pair(int bits, int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L) {
    switch (bits) {
        case 2: return launch_affine_pair_b2(dtype, maxm, R, wide, p, L);
        case 3: return launch_affine_pair_b3(dtype, maxm, R, wide, p, L);
        case 4: return launch_affine_pair_b4(dtype, maxm, R, wide, p, L);
        case 5: return launch_affine_pair_b5(dtype, maxm, R, wide, p, L);
        case 6: return launch_affine_pair_b6(dtype, maxm, R, wide, p, L);
        case 8: return launch_affine_pair_b8(dtype, maxm, R, wide, p, L);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_affine_qkv(int bits, int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L) {
    switch (bits) {
        case 2: return launch_affine_qkv_b2(dtype, maxm, R, wide, p, L);
        case 3: return launch_affine_qkv_b3(dtype, maxm, R, wide, p, L);
        case 4: return launch_affine_qkv_b4(dtype, maxm, R, wide, p, L);
        case 5: return launch_affine_qkv_b5(dtype, maxm, R, wide, p, L);
        case 6: return launch_affine_qkv_b6(dtype, maxm, R, wide, p, L);
        case 8: return launch_affine_qkv_b8(dtype, maxm, R, wide, p, L);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace qmv
