// qmv_quantize.cu -- affine quantizer on the GPU: w [N, K] in the element type
// T -> packed codes, scales and biases in the layout the qmv kernels read.
//
// The pages list affine quantize kernels for every width (wh-iron kernel-op
// coverage audit, "quantized (affine_quantize / affine_dequantize)" row) but
// do not state their arithmetic.  The reading implemented here is the
// plainest one consistent with w = scale * q + bias (MLX quantized_nax.h,
// dequantize): per group of G consecutive weights of a row,
//     bias  = min(w),  scale = (max(w) - min(w)) / (2^B - 1),
// both rounded to T (to nearest, ties to even), and
//     q = rint((w - bias_T) / scale_T)  clamped to [0, 2^B - 1]
// (q = 0 when scale_T is 0), every step one fp32 IEEE operation.  Codes are
// packed LSB first: with a group starting on a pack boundary (G a multiple of
// 32), code k of the group occupies bits [k B, k B + B) of the group's byte
// stream read as little-endian words, for every width.
//
// One thread per (row, group): a first pass over the group's G values finds
// min and max, a second computes and packs the codes, 32-bit words at a time.
// Memory-bound: G * sizeof(T) bytes in, G * B / 8 + 2 sizeof(T) bytes out.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "qmv_device.cuh"

namespace qmv {

namespace {

// T -> fp32 (exact) and fp32 -> T (to nearest, ties to even), as values.
template <class T> struct QT;
template <> struct QT<float> {
    static __device__ __forceinline__ float rt(float v) { return v; }
};
template <> struct QT<__half> {
    static __device__ __forceinline__ float rt(float v) { return __half2float(__float2half_rn(v)); }
};
template <> struct QT<__nv_bfloat16> {
    static __device__ __forceinline__ float rt(float v) { return __bfloat162float(__float2bfloat16_rn(v)); }
};

// The 16 bytes at element k of a group as 16 / sizeof(T) fp32 values.
template <class T>
__device__ __forceinline__ void load16(const T* src, int k, float* o) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + k));
    if constexpr (sizeof(T) == 4) {
        o[0] = __uint_as_float(v.x); o[1] = __uint_as_float(v.y); o[2] = __uint_as_float(v.z); o[3] = __uint_as_float(v.w);
    } else {
        widen8<T>(v, o);
    }
}

template <int B, class T, int G>
__global__ void __launch_bounds__(256) quantize_affine_kernel(const T* __restrict__ w, uint32_t* __restrict__ wq,
                                                              T* __restrict__ scales, T* __restrict__ biases,
                                                              long long ngroups, int K, long long row_words,
                                                              int vec) {
    constexpr int E = 16 / (int)sizeof(T);          // elements per 16-byte load
    constexpr int QMAX = (1 << B) - 1;
    const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= ngroups) return;
    const int KG = K / G;
    const long long n = gid / KG;
    const int gj = (int)(gid - n * KG);
    const T* src = w + n * K + (long long)gj * G;

    // ---- pass 1: min and max (exact) ----------------------------------------
    float lo = DT<T>::ld(src, 0), hi = lo;
    if (vec) {
#pragma unroll 4
        for (int k = 0; k < G; k += E) {
            float v[E];
            load16<T>(src, k, v);
#pragma unroll
            for (int e = 0; e < E; ++e) {
                if (v[e] < lo) lo = v[e];       // strict comparisons, in order: the first of
                if (v[e] > hi) hi = v[e];       // equal values (+0 / -0) is kept
            }
        }
    } else {
        for (int k = 1; k < G; ++k) {
            const float v = DT<T>::ld(src, k);
            if (v < lo) lo = v;
            if (v > hi) hi = v;
        }
    }
    const float scale = __fdiv_rn(__fsub_rn(hi, lo), (float)QMAX);
    const long long gi = n * KG + gj;
    DT<T>::st(scales, gi, scale);
    DT<T>::st(biases, gi, lo);
    const float sT = QT<T>::rt(scale), bT = QT<T>::rt(lo);

    // ---- pass 2: codes, packed LSB first into 32-bit words ------------------
    uint32_t* dst = wq + n * row_words + (long long)gj * (G * B / 32);
    uint64_t acc = 0;
    int nb = 0, wi = 0;
    auto put = [&](float v) {
        uint32_t q = 0;
        if (sT != 0.0f) {
            const float r = rintf(__fdiv_rn(__fsub_rn(v, bT), sT));
            q = r <= 0.0f ? 0u : r >= (float)QMAX ? (uint32_t)QMAX : (uint32_t)r;
        }
        acc |= (uint64_t)q << nb;
        nb += B;
        if (nb >= 32) {
            dst[wi++] = (uint32_t)acc;
            acc >>= 32;
            nb -= 32;
        }
    };
    if (vec) {
#pragma unroll 4
        for (int k = 0; k < G; k += E) {
            float v[E];
            load16<T>(src, k, v);
#pragma unroll
            for (int e = 0; e < E; ++e) put(v[e]);
        }
    } else {
        for (int k = 0; k < G; ++k) put(DT<T>::ld(src, k));
    }
}

template <int B, class T>
cudaError_t quantize_bt(const void* w, void* wq, void* s, void* b, int N, int K, int G, int vec, cudaStream_t st) {
    const long long ngroups = (long long)N * (K / G);
    const long long row_words = (long long)K * B / 32;
    const unsigned grid = (unsigned)((ngroups + 255) / 256);
    auto* wp = static_cast<const T*>(w);
    auto* qp = static_cast<uint32_t*>(wq);
    auto* sp = static_cast<T*>(s);
    auto* bp = static_cast<T*>(b);
    switch (G) {
        case 32: quantize_affine_kernel<B, T, 32><<<grid, 256, 0, st>>>(wp, qp, sp, bp, ngroups, K, row_words, vec); break;
        case 64: quantize_affine_kernel<B, T, 64><<<grid, 256, 0, st>>>(wp, qp, sp, bp, ngroups, K, row_words, vec); break;
        case 128: quantize_affine_kernel<B, T, 128><<<grid, 256, 0, st>>>(wp, qp, sp, bp, ngroups, K, row_words, vec); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

template <int B>
cudaError_t quantize_b(int dtype, const void* w, void* wq, void* s, void* b, int N, int K, int G, int vec,
                       cudaStream_t st) {
    switch (dtype) {
        case 0: return quantize_bt<B, float>(w, wq, s, b, N, K, G, vec, st);
        case 1: return quantize_bt<B, __half>(w, wq, s, b, N, K, G, vec, st);
        case 2: return quantize_bt<B, __nv_bfloat16>(w, wq, s, b, N, K, G, vec, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_quantize_affine(int bits, int dtype, const void* w, void* wq, void* scales, void* biases,
                                   int N, int K, int G, int vec, cudaStream_t st) {
    switch (bits) {
        case 2: return quantize_b<2>(dtype, w, wq, scales, biases, N, K, G, vec, st);
        case 3: return quantize_b<3>(dtype, w, wq, scales, biases, N, K, G, vec, st);
        case 4: return quantize_b<4>(dtype, w, wq, scales, biases, N, K, G, vec, st);
        case 5: return quantize_b<5>(dtype, w, wq, scales, biases, N, K, G, vec, st);
        case 6: return quantize_b<6>(dtype, w, wq, scales, biases, N, K, G, vec, st);
        case 8: return quantize_b<8>(dtype, w, wq, scales, biases, N, K, G, vec, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace qmv
