// qmv_inst_fp.cu -- block-scaled FP qmv kernels (MXFP4, NVFP4, MXFP8-E4M3), the
// dispatcher of every block-scaled family, and every dequantization check
// kernel.
#include "qmv_launch.cuh"

namespace qmv {

static cudaError_t launch_mxfp4(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L) {
#define FAM_ FAM_MXFP4
#define BITS_ 4
    QMV_DISPATCH_DTYPE()
#undef FAM_
#undef BITS_
}
static cudaError_t launch_nvfp4(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L) {
#define FAM_ FAM_NVFP4
#define BITS_ 4
    QMV_DISPATCH_DTYPE()
#undef FAM_
#undef BITS_
}
static cudaError_t launch_mxfp8(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L) {
#define FAM_ FAM_MXFP8
#define BITS_ 8
    QMV_DISPATCH_DTYPE()
#undef FAM_
#undef BITS_
}

cudaError_t launch_fp(int fam, int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L) {
    switch (fam) {
        case FAM_MXFP4: return launch_mxfp4(dtype, maxm, R, wide, p, L);
        case FAM_NVFP4: return launch_nvfp4(dtype, maxm, R, wide, p, L);
        case FAM_MXFP8: return launch_mxfp8(dtype, maxm, R, wide, p, L);
        case FAM_E2M1: return launch_bs_e2m1(dtype, maxm, R, wide, p, L);
        case FAM_E4M3: return launch_bs_e4m3(dtype, maxm, R, wide, p, L);
        case FAM_E5M2: return launch_bs_e5m2(dtype, maxm, R, wide, p, L);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_sint(int bits, int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L) {
    switch (bits) {
        case 2: return launch_sint_b2(dtype, maxm, R, wide, p, L);
        case 3: return launch_sint_b3(dtype, maxm, R, wide, p, L);
        case 4: return launch_sint_b4(dtype, maxm, R, wide, p, L);
        case 5: return launch_sint_b5(dtype, maxm, R, wide, p, L);
        case 6: return launch_sint_b6(dtype, maxm, R, wide, p, L);
        case 8: return launch_sint_b8(dtype, maxm, R, wide, p, L);
        default: return cudaErrorInvalidValue;
    }
}

template <int FAM, int BITS, class T>
static cudaError_t dq(const uint8_t* w, const void* s, const void* b, const float* g, float* out, int N,
                      int K, int G, long long w_row, cudaStream_t st, int skind = 0) {
    long long units = (long long)N * (K / 32);
    if (K % 32) units += (long long)N * 16;         // the 16-code tails
    const int threads = 256;
    long long blocks = (units + threads - 1) / threads;
    if (blocks > 148LL * 64) blocks = 148LL * 64;
    if (blocks < 1) blocks = 1;
    dequant_kernel<FAM, BITS, T><<<(unsigned)blocks, threads, 0, st>>>(w, s, b, g, out, N, K, G, w_row, skind);
    return cudaGetLastError();
}

cudaError_t launch_dequant(int fam, int bits, int dtype, const uint8_t* w, const void* scales,
                           const void* biases, const float* gscale, float* out, int N, int K, int G,
                           long long w_row, cudaStream_t s, int skind) {
#define QMV_DQ_T(FAM_, BITS_)                                                                       \
    switch (dtype) {                                                                                \
        case 0: return dq<FAM_, BITS_, float>(w, scales, biases, gscale, out, N, K, G, w_row, s);        \
        case 1: return dq<FAM_, BITS_, __half>(w, scales, biases, gscale, out, N, K, G, w_row, s);       \
        case 2: return dq<FAM_, BITS_, __nv_bfloat16>(w, scales, biases, gscale, out, N, K, G, w_row, s);\
        default: return cudaErrorInvalidValue;                                                      \
    }
    if (fam == FAM_AFFINE) {
        switch (bits) {
            case 2: QMV_DQ_T(FAM_AFFINE, 2)
            case 3: QMV_DQ_T(FAM_AFFINE, 3)
            case 4: QMV_DQ_T(FAM_AFFINE, 4)
            case 5: QMV_DQ_T(FAM_AFFINE, 5)
            case 6: QMV_DQ_T(FAM_AFFINE, 6)
            case 8: QMV_DQ_T(FAM_AFFINE, 8)
            default: return cudaErrorInvalidValue;
        }
    }
    if (fam == FAM_SINT) {
        switch (bits) {
            case 2: return dq<FAM_SINT, 2, float>(w, scales, nullptr, nullptr, out, N, K, G, w_row, s, skind);
            case 3: return dq<FAM_SINT, 3, float>(w, scales, nullptr, nullptr, out, N, K, G, w_row, s, skind);
            case 4: return dq<FAM_SINT, 4, float>(w, scales, nullptr, nullptr, out, N, K, G, w_row, s, skind);
            case 5: return dq<FAM_SINT, 5, float>(w, scales, nullptr, nullptr, out, N, K, G, w_row, s, skind);
            case 6: return dq<FAM_SINT, 6, float>(w, scales, nullptr, nullptr, out, N, K, G, w_row, s, skind);
            case 8: return dq<FAM_SINT, 8, float>(w, scales, nullptr, nullptr, out, N, K, G, w_row, s, skind);
            default: return cudaErrorInvalidValue;
        }
    }
    if (fam == FAM_E2M1) return dq<FAM_E2M1, 4, float>(w, scales, nullptr, nullptr, out, N, K, G, w_row, s, skind);
    if (fam == FAM_E4M3) return dq<FAM_E4M3, 8, float>(w, scales, nullptr, nullptr, out, N, K, G, w_row, s, skind);
    if (fam == FAM_E5M2) return dq<FAM_E5M2, 8, float>(w, scales, nullptr, nullptr, out, N, K, G, w_row, s, skind);
    if (fam == FAM_MXFP4) return dq<FAM_MXFP4, 4, float>(w, scales, nullptr, nullptr, out, N, K, 32, w_row, s);
    if (fam == FAM_NVFP4) return dq<FAM_NVFP4, 4, float>(w, scales, nullptr, gscale, out, N, K, 16, w_row, s);
    if (fam == FAM_MXFP8) return dq<FAM_MXFP8, 8, float>(w, scales, nullptr, nullptr, out, N, K, 32, w_row, s);
    return cudaErrorInvalidValue;
#undef QMV_DQ_T
}

}  // namespace qmv
