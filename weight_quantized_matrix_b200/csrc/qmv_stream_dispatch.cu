// qmv_stream_dispatch.cu -- bits -> streaming-kernel dispatcher.
#include "qmv_launch.cuh"

namespace qmv {

cudaError_t launch_stream_affine_b2(int, int, int, const Params&, const Launch&);
cudaError_t launch_stream_affine_b3(int, int, int, const Params&, const Launch&);
cudaError_t launch_stream_affine_b4(int, int, int, const Params&, const Launch&);
cudaError_t launch_stream_affine_b5(int, int, int, const Params&, const Launch&);
cudaError_t launch_stream_affine_b6(int, int, int, const Params&, const Launch&);
cudaError_t launch_stream_affine_b8(int, int, int, const Params&, const Launch&);

cudaError_t launch_stream_affine(int bits, int dtype, int maxm, int R, const Params& p, const Launch& L) {
    switch (bits) {
        case 2: return launch_stream_affine_b2(dtype, maxm, R, p, L);
        case 3: return launch_stream_affine_b3(dtype, maxm, R, p, L);
        case 4: return launch_stream_affine_b4(dtype, maxm, R, p, L);
        case 5: return launch_stream_affine_b5(dtype, maxm, R, p, L);
        case 6: return launch_stream_affine_b6(dtype, maxm, R, p, L);
        case 8: return launch_stream_affine_b8(dtype, maxm, R, p, L);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace qmv
