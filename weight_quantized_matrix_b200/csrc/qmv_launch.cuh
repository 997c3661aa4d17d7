// qmv_launch.cuh -- host-side launch helpers shared by the instantiation units
// and the C ABI.  Each instantiation unit (qmv_inst_*.cu) compiles one family
// of kernels and exposes one dispatcher declared here.
#pragma once

#include <atomic>
#include <cuda_runtime.h>
#include "qmv_device.cuh"
#include "qmv_tc.cuh"
#include "qmv_tcb.cuh"

namespace qmv {

// Launch shape chosen by the picker (qmv_api.cu).
struct Launch {
    dim3 grid, block;
    size_t smem;
    cudaStream_t stream;
    bool pdl;        // programmatic dependent launch
};

// Largest dynamic shared memory any kernel here asks for; set once per
// (kernel, device) before the first launch.
constexpr int kMaxSmem = 227 * 1024;

template <class Kern>
inline cudaError_t launch_kernel(Kern kern, std::atomic<unsigned>& configured, const Launch& L,
                                 const Params& p) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned bit = 1u << (dev & 31);
    if (!(configured.load(std::memory_order_acquire) & bit)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit, std::memory_order_acq_rel);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = L.grid;
    cfg.blockDim = L.block;
    cfg.dynamicSmemBytes = L.smem;
    cfg.stream = L.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = L.pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

// dtype: 0 f32, 1 f16, 2 bf16.  Returns cudaErrorInvalidValue for a
// (maxm, R, wide) combination that is not instantiated.
cudaError_t launch_affine_b2(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_affine_b3(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_affine_b4(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_affine_b5(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_affine_b6(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_affine_b8(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_fp(int fam, int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
// Run-time-scaled FP elements (qmv_inst_bs_*.cu) and the signed integers
// (qmv_inst_sint_b*.cu); launch_fp dispatches the former, launch_sint the latter.
cudaError_t launch_bs_e2m1(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_bs_e4m3(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_bs_e5m2(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_sint_b2(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_sint_b3(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_sint_b4(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_sint_b5(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_sint_b6(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_sint_b8(int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
cudaError_t launch_sint(int bits, int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);

// Tensor-core kernels (qmv_tc_kernel): npass in {1, 2, 4}.
cudaError_t launch_tc_affine(int bits, int dtype, int npass, const Params& p, const Launch& L);
// Tensor-core kernels with the bulk-copy weight ring (qmv_tcb_kernel):
// (npass, spb) in {(1,1), (1,2), (1,4), (1,8), (2,1), (4,1)}; ncw = consumer
// warps per block in {8, 12} (plus the producer warp).
cudaError_t launch_tcb_affine(int bits, int dtype, int npass, int spb, int ncw, const Params& p, const Launch& L);
constexpr int kTcbStages = 4;
// CUDA-core kernels with the weight ring, one bf16 x row (qmv_tcf_kernel):
// ncw = compute warps per block in {8, 12} (plus the producer warp).
cudaError_t launch_tcf_affine(int bits, int ncw, const Params& p, const Launch& L);
// Per-group tensor-core ring kernels (qmv_tcg.cuh): 4-bit codes, dtype 1 (f16)
// or 2 (bf16), G in {32, 64, 128}, nt n-tiles of 8 x rows in {1, 2, 4}
// (qmv_inst_tcg_{f16,bf16}.cu); p.wk * p.wr consumer warps, at most 16.
cudaError_t launch_tcg_affine(int dtype, int G, int nt, const Params& p, const Launch& L);
cudaError_t launch_tcg_f16(int G, int nt, const Params& p, const Launch& L);
cudaError_t launch_tcg_bf16(int G, int nt, const Params& p, const Launch& L);
// The same ring for the block-scaled FP families (qmv_inst_tcf_fp.cu): fam one
// of FAM_MXFP4 / NVFP4 / E2M1 / MXFP8 / E4M3 / E5M2.
cudaError_t launch_tcf_fp(int fam, int ncw, const Params& p, const Launch& L);



// Few-rows latency kernels (qmv_direct_kernel): maxm in {1, 2, 4, 8}; wide =
// 16-byte unit loads (4- and 8-bit codes, 16-byte aligned rows).
cudaError_t launch_direct(int fam, int bits, int dtype, int maxm, bool wide, const Params& p, const Launch& L);

// qvm (qmv_qvm.cu): x [M, K] times W stored [K, N]; workspace may be null.
size_t qvm_workspace_bytes(int M, int N);
cudaError_t launch_qvm_affine(int bits, int dtype, const void* x, const void* w, const void* scales,
                              const void* biases, void* y, void* workspace, int M, int N, int K, int G,
                              cudaStream_t st);

// FP quantizer (qmv_quantize_fp.cu): mode 0 MXFP4, 1 NVFP4, 2 MXFP8-E4M3; vec =
// 16-byte loads of w and vector stores of the codes (aligned buffers).
cudaError_t launch_quantize_fp(int mode, int dtype, const void* w, void* wq, void* scales, const float* gscale,
                               int N, int K, bool vec, cudaStream_t st);

// Affine quantizer (qmv_quantize.cu): w [N, K] in dtype -> packed codes,
// scales, biases; vec = 16-byte loads of w (aligned rows).
cudaError_t launch_quantize_affine(int bits, int dtype, const void* w, void* wq, void* scales, void* biases,
                                   int N, int K, int G, int vec, cudaStream_t st);

// skind: the block-scale type of FAM_E2M1 / FAM_E4M3 / FAM_E5M2 / FAM_SINT.
cudaError_t launch_dequant(int fam, int bits, int dtype, const uint8_t* w, const void* scales,
                           const void* biases, const float* gscale, float* out, int N, int K, int G,
                           long long w_row, cudaStream_t s, int skind = 0);

// Fused gate + up with SwiGLU (qmv_kernel<..., PAIR = true>, affine): R in
// {2, 4} wide (4 only for maxm <= 2), R = 2 narrow.  Returns
// cudaErrorInvalidValue for a shape that is not instantiated.
cudaError_t launch_affine_pair(int bits, int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
inline bool pair_shape_instantiated(int maxm, int R, bool wide) {
    if (!wide) return R == 2 && (maxm == 1 || maxm == 2 || maxm == 4 || maxm == 8);
    if (maxm == 1 || maxm == 2) return R == 2 || R == 4;
    return (maxm == 4 || maxm == 8) && R == 2;
}

// Tensor-memory (tcgen05) kernels (qmv_umma.cuh), bf16 x: mld = the power of
// two >= M (1..64); the grid is (S, clusters), cluster (S, 1, 1).
struct UmmaParams;
cudaError_t launch_umma_affine(int bits, int mld, const Params& p, const UmmaParams& u, const Launch& L);
// Clusters of the tensor-memory kernel that fit on the device at once.
cudaError_t umma_max_clusters(int bits, const UmmaParams& u, size_t smem, int* out);

// Q / K / V in one call (qmv_kernel<..., RMODE_QKV>, affine): the shapes the
// row-tiled picker takes for large N (R = 4 wide at maxm <= 2, R = 2 wide
// above; R = 1 on the 4-byte path).
cudaError_t launch_affine_qkv(int bits, int dtype, int maxm, int R, bool wide, const Params& p, const Launch& L);
inline bool qkv_shape_instantiated(int maxm, int R, bool wide) {
    if (!wide) return R == 1 && (maxm == 1 || maxm == 2 || maxm == 4 || maxm == 8);
    return (maxm <= 2 && R == 4) || ((maxm == 4 || maxm == 8) && R == 2);
}

// Which (maxm, R, wide) shapes exist.
inline bool shape_instantiated(int maxm, int R, bool wide) {
    if (!wide) return R == 1 && (maxm == 1 || maxm == 2 || maxm == 4 || maxm == 8);
    if (maxm == 1 || maxm == 2) return R == 1 || R == 2 || R == 4;
    if (maxm == 4 || maxm == 8) return R == 1 || R == 2;
    return false;
}

}  // namespace qmv

// Dispatch body shared by the instantiation units: FAM/BITS fixed, switch on
// dtype and shape.
#define QMV_SHAPE(T_, MAXM_, R_, WIDE_)                                                      \
    if (maxm == MAXM_ && R == R_ && wide == WIDE_) {                                         \
        static std::atomic<unsigned> cfg_{0};                                                \
        return launch_kernel(qmv_kernel<FAM_, BITS_, T_, MAXM_, R_, WIDE_>, cfg_, L, p);     \
    }
#define QMV_ALL_SHAPES(T_)                                                                   \
    QMV_SHAPE(T_, 1, 1, true) QMV_SHAPE(T_, 1, 2, true) QMV_SHAPE(T_, 1, 4, true)            \
    QMV_SHAPE(T_, 2, 1, true) QMV_SHAPE(T_, 2, 2, true) QMV_SHAPE(T_, 2, 4, true)            \
    QMV_SHAPE(T_, 4, 1, true) QMV_SHAPE(T_, 4, 2, true)                                      \
    QMV_SHAPE(T_, 8, 1, true) QMV_SHAPE(T_, 8, 2, true)                                      \
    QMV_SHAPE(T_, 1, 1, false) QMV_SHAPE(T_, 2, 1, false) QMV_SHAPE(T_, 4, 1, false)         \
    QMV_SHAPE(T_, 8, 1, false)
#define QMV_PAIR_SHAPE(T_, MAXM_, R_, WIDE_)                                                 \
    if (maxm == MAXM_ && R == R_ && wide == WIDE_) {                                         \
        static std::atomic<unsigned> cfg_{0};                                                \
        return launch_kernel(qmv_kernel<FAM_AFFINE, BITS_, T_, MAXM_, R_, WIDE_, RMODE_PAIR>, cfg_, L, p); \
    }
#define QMV_PAIR_SHAPES(T_)                                                                  \
    QMV_PAIR_SHAPE(T_, 1, 2, true) QMV_PAIR_SHAPE(T_, 1, 4, true)                            \
    QMV_PAIR_SHAPE(T_, 2, 2, true) QMV_PAIR_SHAPE(T_, 2, 4, true)                            \
    QMV_PAIR_SHAPE(T_, 4, 2, true) QMV_PAIR_SHAPE(T_, 8, 2, true)                            \
    QMV_PAIR_SHAPE(T_, 1, 2, false) QMV_PAIR_SHAPE(T_, 2, 2, false)                          \
    QMV_PAIR_SHAPE(T_, 4, 2, false) QMV_PAIR_SHAPE(T_, 8, 2, false)
#define QMV_PAIR_DISPATCH_DTYPE()                                                            \
    switch (dtype) {                                                                         \
        case 0: { QMV_PAIR_SHAPES(float) break; }                                            \
        case 1: { QMV_PAIR_SHAPES(__half) break; }                                           \
        case 2: { QMV_PAIR_SHAPES(__nv_bfloat16) break; }                                    \
        default: break;                                                                      \
    }                                                                                        \
    return cudaErrorInvalidValue;
#define QMV_QKV_SHAPE(T_, MAXM_, R_, WIDE_)                                                  \
    if (maxm == MAXM_ && R == R_ && wide == WIDE_) {                                         \
        static std::atomic<unsigned> cfg_{0};                                                \
        return launch_kernel(qmv_kernel<FAM_AFFINE, BITS_, T_, MAXM_, R_, WIDE_, RMODE_QKV>, cfg_, L, p); \
    }
#define QMV_QKV_SHAPES(T_)                                                                   \
    QMV_QKV_SHAPE(T_, 1, 4, true) QMV_QKV_SHAPE(T_, 2, 4, true)                              \
    QMV_QKV_SHAPE(T_, 4, 2, true) QMV_QKV_SHAPE(T_, 8, 2, true)                              \
    QMV_QKV_SHAPE(T_, 1, 1, false) QMV_QKV_SHAPE(T_, 2, 1, false)                            \
    QMV_QKV_SHAPE(T_, 4, 1, false) QMV_QKV_SHAPE(T_, 8, 1, false)
#define QMV_QKV_DISPATCH_DTYPE()                                                             \
    switch (dtype) {                                                                         \
        case 0: { QMV_QKV_SHAPES(float) break; }                                             \
        case 1: { QMV_QKV_SHAPES(__half) break; }                                            \
        case 2: { QMV_QKV_SHAPES(__nv_bfloat16) break; }                                     \
        default: break;                                                                      \
    }                                                                                        \
    return cudaErrorInvalidValue;
#define QMV_TC_SHAPE(T_, NPASS_)                                                             \
    if (npass == NPASS_) {                                                                   \
        static std::atomic<unsigned> cfg_{0};                                                \
        return launch_kernel(qmv_tc_kernel<BITS_, T_, NPASS_, QMV_TC_PD(BITS_)>, cfg_, L, p); \
    }
#define QMV_TCB_SHAPE(T_, NPASS_, SPB_)                                                      \
    if (npass == NPASS_ && spb == SPB_) {                                                    \
        if (ncw == 8) {                                                                      \
            static std::atomic<unsigned> cfg_{0};                                            \
            return launch_kernel(qmv_tcb_kernel<BITS_, T_, NPASS_, SPB_, kTcbStages, 288>, cfg_, L, p); \
        }                                                                                    \
        if (ncw == 12) {                                                                     \
            static std::atomic<unsigned> cfg_{0};                                            \
            return launch_kernel(qmv_tcb_kernel<BITS_, T_, NPASS_, SPB_, kTcbStages, 416>, cfg_, L, p); \
        }                                                                                    \
    }
#define QMV_TCB_SHAPES(T_)                                                                   \
    QMV_TCB_SHAPE(T_, 1, 1) QMV_TCB_SHAPE(T_, 1, 2) QMV_TCB_SHAPE(T_, 1, 4)                 \
    QMV_TCB_SHAPE(T_, 1, 8) QMV_TCB_SHAPE(T_, 2, 1) QMV_TCB_SHAPE(T_, 4, 1)
#define QMV_TCB_DISPATCH_DTYPE()                                                             \
    switch (dtype) {                                                                         \
        case 0: { QMV_TCB_SHAPES(float) break; }                                             \
        case 1: { QMV_TCB_SHAPES(__half) break; }                                            \
        case 2: { QMV_TCB_SHAPES(__nv_bfloat16) break; }                                     \
        default: break;                                                                      \
    }                                                                                        \
    return cudaErrorInvalidValue;
#define QMV_TC_PD(B_) (((B_) == 5 || (B_) == 6) ? 2 : 4)
#define QMV_TC_DISPATCH_DTYPE()                                                              \
    switch (dtype) {                                                                         \
        case 0: { QMV_TC_SHAPE(float, 1) QMV_TC_SHAPE(float, 2) QMV_TC_SHAPE(float, 4) break; }                 \
        case 1: { QMV_TC_SHAPE(__half, 1) QMV_TC_SHAPE(__half, 2) QMV_TC_SHAPE(__half, 4) break; }              \
        case 2: { QMV_TC_SHAPE(__nv_bfloat16, 1) QMV_TC_SHAPE(__nv_bfloat16, 2) QMV_TC_SHAPE(__nv_bfloat16, 4) break; } \
        default: break;                                                                      \
    }                                                                                        \
    return cudaErrorInvalidValue;
#define QMV_DISPATCH_DTYPE()                                                                 \
    switch (dtype) {                                                                         \
        case 0: { QMV_ALL_SHAPES(float) break; }                                             \
        case 1: { QMV_ALL_SHAPES(__half) break; }                                            \
        case 2: { QMV_ALL_SHAPES(__nv_bfloat16) break; }                                     \
        default: break;                                                                      \
    }                                                                                        \
    return cudaErrorInvalidValue;
