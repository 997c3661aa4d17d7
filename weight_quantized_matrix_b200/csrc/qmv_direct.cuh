// qmv_direct.cuh -- the qmv kernel for few output rows (N <= 64), built for
// latency: in a chain of dependent calls (each output feeding the next x) a
// call's time is the critical path from "previous kernel done" to "y stored".
//
// One block per output row n; its lanes take the row's 32-code units (unit u
// = lane, lane + blockDim, ...).  Everything that does not depend on x runs
// BEFORE the grid-dependency wait, overlapped with the previous kernel: the
// packed codes and scales of the lane's first units are loaded and dequantized
// to fp32 weights in registers
//   affine:  w = fmaf(scale, q, bias)   (the dequantized value, one rounding)
//   MXFP4/8: w = element * E8M0 scale   (exact)
//   NVFP4:   w = element * E4M3 scale   (exact; the FP32 global scale is
//            applied once to the row's sum)
//   E2M1 / E4M3 / E5M2 with a typed block scale: w = element * scale
//   signed int: the affine form on offset-binary codes, bias = -2^(b-1) * scale
// With K % 32 == 16 (blocks of 16) lanes 0..15 also take the row's last 16
// codes after the wait.
// After the wait only x is read: y[m, n] = sum_k x[m, k] * w[n, k], fp32
// products and sums (warp butterfly, then one shared-memory step across
// warps), rounded once to the output dtype.  Units past the first UPRE per
// lane (K > UPRE * 32 * blockDim) are loaded and dequantized after the wait.
#pragma once

#include "qmv_device.cuh"

namespace qmv {

// The 32 dequantized weights of unit u of row n (fp32; NVFP4 without the
// global scale).  wv: the unit's B words.
template <int FAM, int B, class T>
__device__ __forceinline__ void direct_dequant(const Params& p, const uint32_t (&wv)[B], long long srow, int u,
                                               uint32_t kf32, float (&o)[32]) {
    const long long k0 = (long long)u * 32;
    if constexpr (affine_like<FAM>()) {
        const long long gi = srow + k0 / p.G;
        float s, b;
        uint32_t wx[B];
#pragma unroll
        for (int q = 0; q < B; ++q) wx[q] = FAM == FAM_SINT ? wv[q] ^ sint_sign_mask<B>(q) : wv[q];
        if constexpr (FAM == FAM_SINT) {
            s = block_scale(p.scales, gi, p.skind);
            b = -s * (float)(1 << (B - 1));
        } else {
            s = DT<T>::ld(p.scales, gi);
            b = DT<T>::ld(p.biases, gi);
        }
#define QMV_DD4(QQ)                                                                                            \
    {                                                                                                          \
        const float2 d0 = magic_pair_ored(field_magic<B, 4 * QQ>(wx, kf32), field_magic<B, 4 * QQ + 1>(wx, kf32)); \
        const float2 d1 =                                                                                      \
            magic_pair_ored(field_magic<B, 4 * QQ + 2>(wx, kf32), field_magic<B, 4 * QQ + 3>(wx, kf32));       \
        const float c[4] = {d0.x, d0.y, d1.x, d1.y};                                                           \
        _Pragma("unroll") for (int e = 0; e < 4; ++e) {                                                        \
            const float q_ = __fmul_rn(c[e], __uint_as_float((127u - field_p(B, 4 * QQ + e)) << 23));         \
            o[4 * QQ + e] = fmaf(s, q_, b);                                                                    \
        }                                                                                                      \
    }
        QMV_DD4(0) QMV_DD4(1) QMV_DD4(2) QMV_DD4(3) QMV_DD4(4) QMV_DD4(5) QMV_DD4(6) QMV_DD4(7)
#undef QMV_DD4
    } else if constexpr (FAM == FAM_E2M1 || FAM == FAM_E4M3 || FAM == FAM_E5M2) {
        const float s0 = block_scale(p.scales, srow + k0 / p.G, p.skind);
        const float s1 = p.G == 16 ? block_scale(p.scales, srow + k0 / p.G + 1, p.skind) : s0;
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
            const float2 e = B == 4 ? half2_bits_to_float2(cvt_e2m1x2(wv[j / 8] >> (4 * (j % 8))))
                                    : half2_bits_to_float2(cvt_fp8x2<FAM>(wv[j / 4] >> (8 * (j % 4))));
            o[j] = __fmul_rn(e.x, j < 16 ? s0 : s1);
            o[j + 1] = __fmul_rn(e.y, j < 16 ? s0 : s1);
        }
    } else if constexpr (B == 4) {
        const uint8_t* s8 = reinterpret_cast<const uint8_t*>(p.scales) + srow;
        float s0, s1;
        if constexpr (FAM == FAM_NVFP4) {
            s0 = e4m3_value(__ldg(s8 + k0 / 16));
            s1 = e4m3_value(__ldg(s8 + k0 / 16 + 1));
        } else {
            s0 = s1 = e8m0_value(__ldg(s8 + k0 / 32));
        }
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
            const float2 e = half2_bits_to_float2(cvt_e2m1x2(wv[j / 8] >> (4 * (j % 8))));
            o[j] = __fmul_rn(e.x, j < 16 ? s0 : s1);
            o[j + 1] = __fmul_rn(e.y, j < 16 ? s0 : s1);
        }
    } else {
        const uint8_t* s8 = reinterpret_cast<const uint8_t*>(p.scales) + srow;
        const float s = e8m0_value(__ldg(s8 + k0 / 32));
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
            const float2 e = half2_bits_to_float2(cvt_fp8x2<FAM>(wv[j / 4] >> (8 * (j % 4))));
            o[j] = __fmul_rn(e.x, s);
            o[j + 1] = __fmul_rn(e.y, s);
        }
    }
}

// Load the B words of unit u of a row (16-byte loads when WIDE).
template <int B, bool WIDE>
__device__ __forceinline__ void direct_load(const uint8_t* row, int u, uint32_t (&wv)[B]) {
    const uint8_t* src = row + (long long)u * 4 * B;
    if constexpr (WIDE && B % 4 == 0) {
#pragma unroll
        for (int q = 0; q < B / 4; ++q) {
            const uint4 t = __ldg(reinterpret_cast<const uint4*>(src) + q);
            wv[4 * q] = t.x; wv[4 * q + 1] = t.y; wv[4 * q + 2] = t.z; wv[4 * q + 3] = t.w;
        }
    } else {
#pragma unroll
        for (int q = 0; q < B; ++q) wv[q] = __ldg(reinterpret_cast<const uint32_t*>(src) + q);
    }
}

// sum over the 32 x values of unit u of every x row, times the unit's weights.
template <class T, int MAXM>
__device__ __forceinline__ void direct_fma(const Params& p, const T* X, int u, const float (&w)[32],
                                           float (&acc)[MAXM]) {
#pragma unroll
    for (int m = 0; m < MAXM; ++m) {
        if (m >= p.M) break;
        const T* xr = X + (long long)m * p.K + (long long)u * 32;
        float v[32];
        if constexpr (sizeof(T) == 2) {
            if (p.x_vec) {
#pragma unroll
                for (int q = 0; q < 4; ++q) widen8<T>(__ldg(reinterpret_cast<const uint4*>(xr) + q), v + 8 * q);
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = DT<T>::ld(xr, j);
            }
        } else {
            if (p.x_vec) {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 f = __ldg(reinterpret_cast<const float4*>(xr) + q);
                    v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
                }
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = DT<T>::ld(xr, j);
            }
        }
        float2 a = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < 32; j += 2) a = fma2(make_float2(v[j], v[j + 1]), make_float2(w[j], w[j + 1]), a);
        acc[m] += a.x + a.y;
    }
}

// Block: blockDim = 32 * warps (<= 256) lanes over the row's K / 32 units;
// grid (N, 1, batch).  Dynamic shared memory: 8 * MAXM floats.
template <int FAM, int BITS, class T, int MAXM, bool WIDE, int UPRE>
__global__ void __launch_bounds__(256) qmv_direct_kernel(const Params p) {
    constexpr int B = Fmt<FAM, BITS>::kBits;
    extern __shared__ float4 smem4[];
    float* red = reinterpret_cast<float*>(smem4);      // [8 warps][MAXM]
    const int n = blockIdx.x, bz = blockIdx.z;
    const int units = p.K / 32;
    const int nthr = blockDim.x;
    // gather: entry bz's weights are matrix ids[bz] (read before the grid
    // wait: gather launches without programmatic dependent launch); an id
    // outside the stack gives NaN outputs
    int be = bz;
    if (p.ids) {
        be = __ldg(p.ids + bz);
        if (be < 0 || be >= p.n_experts) {
            if ((int)threadIdx.x < p.M)
                DT<T>::st(reinterpret_cast<T*>(p.y) + bz * p.y_bs, (long long)threadIdx.x * p.N + n,
                          __int_as_float(0x7FC00000));
            return;
        }
    }
    const uint8_t* row = p.w + be * p.w_bs + (long long)n * p.w_row;
    const long long srow = be * p.s_bs + (long long)n * (p.K / p.G);
    const uint32_t kf32 = p.kf32;

    // the next kernel in the stream may launch and start fetching its own
    // weights now; it still waits for this grid to complete before reading y
    grid_launch_dependents();

    // ---- before the wait: this lane's first units, dequantized -------------
    float w[UPRE][32];
#pragma unroll
    for (int i = 0; i < UPRE; ++i) {
        const int u = threadIdx.x + i * nthr;
        if (u < units) {
            uint32_t wv[B];
            direct_load<B, WIDE>(row, u, wv);
            direct_dequant<FAM, B, T>(p, wv, srow, u, kf32, w[i]);
        }
    }
    grid_wait();

    // ---- after the wait: x, products, sums ---------------------------------
    const T* X = reinterpret_cast<const T*>(p.x) + bz * p.x_bs;
    float acc[MAXM];
#pragma unroll
    for (int m = 0; m < MAXM; ++m) acc[m] = 0.f;
#pragma unroll
    for (int i = 0; i < UPRE; ++i) {
        const int u = threadIdx.x + i * nthr;
        if (u < units) direct_fma<T, MAXM>(p, X, u, w[i], acc);
    }
    for (int u = threadIdx.x + UPRE * nthr; u < units; u += nthr) {
        uint32_t wv[B];
        float wu[32];
        direct_load<B, WIDE>(row, u, wv);
        direct_dequant<FAM, B, T>(p, wv, srow, u, kf32, wu);
        direct_fma<T, MAXM>(p, X, u, wu, acc);
    }
    if constexpr (half_units<FAM>()) {
        // K % 32 == 16: the row's last 16 codes, one per lane of warp 0
        if ((p.K & 31) && threadIdx.x < 16) {
            const long long k = (long long)p.K - 16 + threadIdx.x;
            float e;
            if constexpr (B == 4) e = e2m1_value(__ldg(row + (k >> 1)) >> (4 * (int)(k & 1)));
            else e = fp8_value<FAM>(__ldg(row + k));
            const long long si = srow + k / p.G;
            const float sv = FAM == FAM_NVFP4 ? e4m3_value(__ldg(reinterpret_cast<const uint8_t*>(p.scales) + si))
                                              : block_scale(p.scales, si, p.skind);
            const float ws = __fmul_rn(e, sv);
#pragma unroll
            for (int m = 0; m < MAXM; ++m)
                if (m < p.M) acc[m] = fmaf(DT<T>::ld(X, (long long)m * p.K + k), ws, acc[m]);
        }
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int m = 0; m < MAXM; ++m) {
#pragma unroll
        for (int o = 16; o; o >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], o);
        if (lane == 0) red[warp * MAXM + m] = acc[m];
    }
    __syncthreads();
    if (threadIdx.x < p.M) {
        const int m = threadIdx.x;
        float v = 0.f;
        for (int k = 0; k < (nthr >> 5); ++k) v += red[k * MAXM + m];
        if constexpr (FAM == FAM_NVFP4) v = v * __ldg(p.gscale + be);
        DT<T>::st(reinterpret_cast<T*>(p.y) + bz * p.y_bs, (long long)m * p.N + n, v);
    }
}

}  // namespace qmv
