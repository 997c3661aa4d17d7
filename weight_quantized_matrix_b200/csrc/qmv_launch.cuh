// qmv_launch.cuh -- host-side launch helpers shared by the instantiation units
// and the C ABI.  Each instantiation unit (qmv_inst_*.cu) compiles one family
// of kernels and exposes one dispatcher declared here.
#pragma once

#include <atomic>
#include <cuda_runtime.h>
#include "qmv_device.cuh"

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

// Persistent streaming kernels: L.grid.x is an upper bound (enough blocks for
// every row block); it is capped to the number of blocks that are resident at
// once (occupancy x SMs), so the blocks stay resident and stage x once.
template <class Kern>
inline cudaError_t launch_stream_kernel(Kern kern, std::atomic<unsigned>& configured, Launch L,
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
    int per_sm = 0, sms = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, (int)L.block.x, L.smem);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const unsigned cap = (unsigned)per_sm * (unsigned)sms;
    if (L.grid.x > cap) L.grid.x = cap;
    return launch_kernel(kern, configured, L, p);
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

// Streaming kernels (qmv_stream_kernel, S = kStreamStages ring stages).
constexpr int kStreamStages = 4;
cudaError_t launch_stream_affine(int bits, int dtype, int maxm, int R, const Params& p, const Launch& L);
cudaError_t launch_stream_fp(int fam, int dtype, int maxm, int R, const Params& p, const Launch& L);
inline bool stream_instantiated(int maxm, int R) {
    if (maxm == 1 || maxm == 2) return R == 2 || R == 4;
    if (maxm == 4 || maxm == 8) return R == 1 || R == 2;
    return false;
}

cudaError_t launch_dequant(int fam, int bits, int dtype, const uint8_t* w, const void* scales,
                           const void* biases, const float* gscale, float* out, int N, int K, int G,
                           long long w_row, cudaStream_t s);

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
#define QMV_STREAM_SHAPE(T_, MAXM_, R_)                                                      \
    if (maxm == MAXM_ && R == R_) {                                                          \
        static std::atomic<unsigned> cfg_{0};                                                \
        return launch_stream_kernel(qmv_stream_kernel<FAM_, BITS_, T_, MAXM_, R_, kStreamStages>, cfg_, L, p); \
    }
#define QMV_STREAM_ALL(T_)                                                                   \
    QMV_STREAM_SHAPE(T_, 1, 2) QMV_STREAM_SHAPE(T_, 1, 4) QMV_STREAM_SHAPE(T_, 2, 2)          \
    QMV_STREAM_SHAPE(T_, 2, 4) QMV_STREAM_SHAPE(T_, 4, 1) QMV_STREAM_SHAPE(T_, 4, 2)          \
    QMV_STREAM_SHAPE(T_, 8, 1) QMV_STREAM_SHAPE(T_, 8, 2)
#define QMV_STREAM_DISPATCH_DTYPE()                                                          \
    switch (dtype) {                                                                         \
        case 0: { QMV_STREAM_ALL(float) break; }                                             \
        case 1: { QMV_STREAM_ALL(__half) break; }                                            \
        case 2: { QMV_STREAM_ALL(__nv_bfloat16) break; }                                     \
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
