// qmv_inst_direct_fp.cu -- the few-rows (latency) kernels, block-scaled FP formats;
// the format dispatcher.
#include "qmv_direct.cuh"
#include "qmv_launch.cuh"

namespace qmv {

namespace {

template <int FAM, int BITS, class T, int MAXM, bool WIDE>
cudaError_t direct_one(const Params& p, const Launch& L) {
    static std::atomic<unsigned> cfg{0};
    return launch_kernel(qmv_direct_kernel<FAM, BITS, T, MAXM, WIDE, 2>, cfg, L, p);
}

template <int FAM, int BITS, class T, bool WIDE>
cudaError_t direct_m(int maxm, const Params& p, const Launch& L) {
    switch (maxm) {
        case 1: return direct_one<FAM, BITS, T, 1, WIDE>(p, L);
        case 2: return direct_one<FAM, BITS, T, 2, WIDE>(p, L);
        case 4: return direct_one<FAM, BITS, T, 4, WIDE>(p, L);
        case 8: return direct_one<FAM, BITS, T, 8, WIDE>(p, L);
        default: return cudaErrorInvalidValue;
    }
}

template <int FAM, int BITS, class T>
cudaError_t direct_t(int maxm, bool wide, const Params& p, const Launch& L) {
    constexpr bool CW = Fmt<FAM, BITS>::kBits % 4 == 0;    // units of 16 / 32 bytes
    if (CW && wide) return direct_m<FAM, BITS, T, CW>(maxm, p, L);
    return direct_m<FAM, BITS, T, false>(maxm, p, L);
}

template <int FAM, int BITS>
cudaError_t direct_fb(int dtype, int maxm, bool wide, const Params& p, const Launch& L) {
    switch (dtype) {
        case 0: return direct_t<FAM, BITS, float>(maxm, wide, p, L);
        case 1: return direct_t<FAM, BITS, __half>(maxm, wide, p, L);
        case 2: return direct_t<FAM, BITS, __nv_bfloat16>(maxm, wide, p, L);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_direct_fp(int fam, int dtype, int maxm, bool wide, const Params& p, const Launch& L) {
    switch (fam) {
        case FAM_MXFP4: return direct_fb<FAM_MXFP4, 4>(dtype, maxm, wide, p, L);
        case FAM_NVFP4: return direct_fb<FAM_NVFP4, 4>(dtype, maxm, wide, p, L);
        case FAM_MXFP8: return direct_fb<FAM_MXFP8, 8>(dtype, maxm, wide, p, L);
        case FAM_E2M1: return direct_fb<FAM_E2M1, 4>(dtype, maxm, wide, p, L);
        case FAM_E4M3: return direct_fb<FAM_E4M3, 8>(dtype, maxm, wide, p, L);
        case FAM_E5M2: return direct_fb<FAM_E5M2, 8>(dtype, maxm, wide, p, L);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_direct_affine(int bits, int dtype, int maxm, bool wide, const Params& p, const Launch& L);
cudaError_t launch_direct_sint(int bits, int dtype, int maxm, bool wide, const Params& p, const Launch& L);

cudaError_t launch_direct(int fam, int bits, int dtype, int maxm, bool wide, const Params& p, const Launch& L) {
    return fam == FAM_AFFINE ? launch_direct_affine(bits, dtype, maxm, wide, p, L)
         : fam == FAM_SINT   ? launch_direct_sint(bits, dtype, maxm, wide, p, L)
                             : launch_direct_fp(fam, dtype, maxm, wide, p, L);
}

}  // namespace qmv
