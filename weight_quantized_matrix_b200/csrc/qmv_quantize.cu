// qmv_quantize.cu -- affine quantizer on the GPU: w [N, K] in the element type
// T -> packed codes, scales and biases in the layout the qmv kernels read.
//
// The pages list affine quantize kernels for every width (wh-iron kernel-op
// coverage audit, "quantized (affine_quantize / affine_dequantize)" row) but
// do not state their arithmetic.  The reading implemented here is the
// plainest one consistent with w = scale * q + bias (MLX quantized_nax.h,
// dequantize), whose inverse is the quotient (w - bias) / scale: per group of
// G consecutive weights of a row,
//     bias  = min(w),  scale = (max(w) - min(w)) / (2^B - 1),
// both rounded to T (to nearest, ties to even), and
//     q = rint((w - bias_T) / scale_T)  clamped to [0, 2^B - 1]
// with the difference and the quotient each one fp32 IEEE operation (q = 0
// when scale_T is 0 or the quotient is NaN).  min and max keep, of +0 and -0,
// the first met in element order (what strict in-order comparisons give);
// weights are finite.  Codes are packed LSB first: with a group starting on a
// pack boundary (G a multiple of 32), code k of the group occupies bits
// [k B, k B + B) of the group's byte stream read as little-endian words, for
// every width.
//
// The division per weight is exact but slow; the kernels get the same codes
// from one reciprocal per group.  With inv = 1 / scale_T rounded to fp32 and t
// the fp32 product (w - bias_T) * inv, t lies within 2.0001 * 2^-24 |Q| of the
// exact quotient Q (two roundings, while inv and t are normal) and the
// correctly rounded quotient d within 2^-24 |Q|, so |t - d| <= 3.0001 * 2^-24
// |Q|.  When t is
// farther than that from every half-integer, t and d round (and clamp) to the
// same code.  The kernels test the clamped t against the conservative margin
// (2^B - 1) * 2^-21 and decide a weight that is closer exactly (near_code):
// with h the half-integer next to t, the residual diff - h * scale_T from one
// FMA has the sign (and zeroness) of the exact residual, since the FMA rounds
// the exact value once.  Zero means the quotient IS h, which rounds to the
// even neighbour; a residual larger than scale_T * 2^(B-23) puts the quotient
// more than half an ulp of h away, on the side its sign gives, so its
// correctly rounded value rounds the same way; anything closer, a scale
// outside [2^-100, 2^100] (where the residual could underflow) or a
// reciprocal that is not a normal number takes the IEEE division.  Exact
// half-integer quotients are common with bf16 / f16 weights (few mantissa
// bits), so the FMA test keeps them off the division.  The codes are those of
// the division, bit for bit.
//
// Two forms: quantize_affine_tiles (aligned buffers: a warp double-buffers 32
// groups at a time through shared memory for coalesced loads and stores) and
// quantize_affine_kernel (one thread per (row, group), any alignment).  Both
// make a first pass over a group's G values for min and max and a second that
// computes and packs the codes, 32-bit words at a time.  Memory-bound:
// G * sizeof(T) bytes in, G * B / 8 + 2 sizeof(T) bytes out per group.
#include <algorithm>

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

// Codes of v[0..E): (v - bias_T) * inv clamped to [0, QMAX], then rounded to
// the nearest integer, ties to even, by adding 2^23: an fp32 in [2^23, 2^24)
// has unit spacing, so the sum is 2^23 plus the rounded value and its low bits
// are the code.  Two values per packed fp32x2 op.  Returns the mask of the
// values whose clamped product lies within QMAX * 2^-21 of a half-integer,
// where it might round differently from the quotient (the caller decides
// those with near_code), and leaves the clamped products in c.
template <int QMAX, int E>
__device__ __forceinline__ uint32_t quantize_codes(const float* v, float bT, float inv, uint32_t* q, float* c) {
    static_assert(E % 2 == 0 && E <= 32, "pairs");
    constexpr float EDGE = 0.5f - (float)QMAX * 4.76837158203125e-07f;      // 0.5 - QMAX * 2^-21
    uint32_t near = 0;
#pragma unroll
    for (int e = 0; e < E; e += 2) {
        const float2 d = mul2(add2(make_float2(v[e], v[e + 1]), make_float2(-bT, -bT)), make_float2(inv, inv));
        const float2 cc = make_float2(fminf(fmaxf(d.x, 0.0f), (float)QMAX), fminf(fmaxf(d.y, 0.0f), (float)QMAX));
        const float2 r = add2(cc, make_float2(8388608.0f, 8388608.0f));
        q[e] = __float_as_uint(r.x) & (uint32_t)QMAX;
        q[e + 1] = __float_as_uint(r.y) & (uint32_t)QMAX;
        c[e] = cc.x;
        c[e + 1] = cc.y;
        // cc minus its rounded value (both exact): in [-0.5, 0.5]
        const float2 f = add2(cc, add2(make_float2(-r.x, -r.y), make_float2(8388608.0f, 8388608.0f)));
        near |= (fabsf(f.x) >= EDGE ? 1u : 0u) << e;
        near |= (fabsf(f.y) >= EDGE ? 1u : 0u) << (e + 1);
    }
    return near;
}

// The code by the defining division: rint(fl(fl(v - bias_T) / scale_T)),
// clamped; 0 for a zero scale or a NaN quotient.
template <int QMAX>
__device__ __forceinline__ uint32_t exact_code(float v, float bT, float sT) {
    if (sT == 0.0f) return 0u;
    const float r = rintf(__fdiv_rn(__fsub_rn(v, bT), sT));
    return !(r > 0.0f) ? 0u : r >= (float)QMAX ? (uint32_t)QMAX : (uint32_t)r;
}

// The code of a weight whose product t (unclamped: a clamped product is never
// near a half-integer) lies near the half-integer h = floor(t) + 1/2, decided
// by the sign of the exact residual diff - h * sT (see the header).
template <int QMAX>
__device__ __forceinline__ uint32_t near_code(float v, float bT, float sT, float t) {
    constexpr float ULP_MAX = (float)(QMAX + 1) * 1.1920928955078125e-07f;  // 2^(B-23) >= ulp(h)
    if (sT >= 7.888609052210118e-31f && sT <= 1.2676506002282294e+30f) {   // 2^-100 .. 2^100
        const float diff = __fsub_rn(v, bT);
        const float k = floorf(t);
        const float e = fmaf(-(k + 0.5f), sT, diff);
        const uint32_t ki = (uint32_t)k;
        if (e == 0.0f) return (ki & 1u) ? ki + 1u : ki;                    // the quotient is h: even
        if (fabsf(e) > sT * ULP_MAX) return e > 0.0f ? ki + 1u : ki;
    }
    return exact_code<QMAX>(v, bT, sT);
}

// Whether the reciprocal fast path applies to a group: a zero scale (every
// code 0, which the product with inv = 0 gives), or a normal reciprocal.
__device__ __forceinline__ bool reciprocal_ok(float sT, float inv) {
    return sT == 0.0f || (inv >= 2.350988701644575e-38f && inv <= 4.253529586511731e+37f);   // 2^-125, 2^125
}

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
    const float inv = sT != 0.0f ? __fdiv_rn(1.0f, sT) : 0.0f;
    const bool fast = reciprocal_ok(sT, inv);

    // ---- pass 2: codes, packed LSB first into 32-bit words ------------------
    uint32_t* dst = wq + n * row_words + (long long)gj * (G * B / 32);
    uint64_t acc = 0;
    int nb = 0, wi = 0;
    auto put = [&](float v) {
        const float two[2] = {v, v};
        uint32_t qq[2];
        float cc[2];
        const uint32_t near = quantize_codes<QMAX, 2>(two, bT, inv, qq, cc);
        const uint32_t q = !fast ? exact_code<QMAX>(v, bT, sT) : near ? near_code<QMAX>(v, bT, sT, cc[0]) : qq[0];
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

// Coalesced form (16-byte aligned w, w_packed and rows).  A warp (one per
// block) takes 32 consecutive groups per tile -- a contiguous span of 32 * G
// elements, rows being contiguous -- and double-buffers the spans in shared
// memory: 16-byte asynchronous copies of the next tile are in flight while the
// current one is quantized.  Each group's row in shared memory is padded by 16
// bytes (an odd number of 16-byte chunks), so lane l reading group l 16 bytes
// at a time hits 8 different bank groups per phase.  Lane l then quantizes
// group l: min / max by min / max instructions (packed for 16-bit types) with
// the sign of a zero result taken from the first zero in element order, which
// is what in-order strict comparisons keep; codes with quantize_code, packed
// 32 codes (B words) at a time at compile-time bit offsets into a padded
// shared-memory row, and the warp copies the tile's contiguous code words out
// with consecutive 4-byte stores.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_prev() { asm volatile("cp.async.wait_group 1;\n" ::: "memory"); }

// Running min and max of a 16-byte chunk of T values.
template <class T> struct MinMax;
template <> struct MinMax<float> {
    float lo, hi;
    __device__ __forceinline__ void init(const uint4& u) { lo = hi = __uint_as_float(u.x); }
    __device__ __forceinline__ void add(const uint4& u) {
        const float v[4] = {__uint_as_float(u.x), __uint_as_float(u.y), __uint_as_float(u.z), __uint_as_float(u.w)};
#pragma unroll
        for (int e = 0; e < 4; ++e) { lo = fminf(lo, v[e]); hi = fmaxf(hi, v[e]); }
    }
    __device__ __forceinline__ float min() const { return lo; }
    __device__ __forceinline__ float max() const { return hi; }
};
template <class H2> struct MinMax16 {
    H2 lo, hi;
    __device__ __forceinline__ void init(const uint4& u) { lo = hi = *reinterpret_cast<const H2*>(&u.x); }
    __device__ __forceinline__ void add(const uint4& u) {
        const H2* h = reinterpret_cast<const H2*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) { lo = __hmin2(lo, h[e]); hi = __hmax2(hi, h[e]); }
    }
};
template <> struct MinMax<__nv_bfloat16> : MinMax16<__nv_bfloat162> {
    __device__ __forceinline__ float min() const { return fminf(__low2float(lo), __high2float(lo)); }
    __device__ __forceinline__ float max() const { return fmaxf(__low2float(hi), __high2float(hi)); }
};
template <> struct MinMax<__half> : MinMax16<__half2> {
    __device__ __forceinline__ float min() const { return fminf(__low2float(lo), __high2float(lo)); }
    __device__ __forceinline__ float max() const { return fmaxf(__low2float(hi), __high2float(hi)); }
};

template <class T>
__device__ __forceinline__ void widen16(const uint4& u, float* v) {
    if constexpr (sizeof(T) == 4) {
        v[0] = __uint_as_float(u.x); v[1] = __uint_as_float(u.y); v[2] = __uint_as_float(u.z); v[3] = __uint_as_float(u.w);
    } else {
        widen8<T>(u, v);
    }
}

// The first value of a group (n chunks of 16 bytes) that compares equal to 0.
template <class T>
__device__ __noinline__ float first_zero(const uint4* my, int n) {
    constexpr int E = 16 / (int)sizeof(T);
    for (int c = 0; c < n; ++c) {
        float v[E];
        widen16<T>(my[c], v);
        for (int e = 0; e < E; ++e)
            if (v[e] == 0.0f) return v[e];
    }
    return 0.0f;
}

template <int B, class T, int G>
struct TileShape {
    static constexpr int ES = (int)sizeof(T);
    static constexpr int E = 16 / ES;                 // elements per 16-byte chunk
    static constexpr int CPG = G * ES / 16;           // chunks per group (even)
    static constexpr int IN_STRIDE = CPG + 1;         // chunks per padded group row (odd)
    static constexpr int WPG = G * B / 32;            // code words per group
    static constexpr int OUT_STRIDE = WPG | 1;        // words per padded group row (odd)
    static constexpr int BUF = 32 * IN_STRIDE;        // chunks per input buffer
    static constexpr int OUT = (32 * OUT_STRIDE + 3) / 4;
    static constexpr size_t SMEM = (size_t)(2 * BUF + OUT) * 16;
};

template <int B, class T, int G>
__global__ void __launch_bounds__(32) quantize_affine_tiles(const T* __restrict__ w, uint32_t* __restrict__ wq,
                                                            T* __restrict__ scales, T* __restrict__ biases,
                                                            long long ngroups) {
    using S = TileShape<B, T, G>;
    constexpr int E = S::E, CPG = S::CPG, WPG = S::WPG;
    constexpr int QMAX = (1 << B) - 1;
    extern __shared__ uint4 smq[];
    const int lane = threadIdx.x;
    uint32_t* out = reinterpret_cast<uint32_t*>(smq + 2 * S::BUF);
    const long long ntiles = (ngroups + 31) / 32;

    auto issue = [&](long long tile, uint4* buf) {
        const long long g0 = tile * 32;
        const int n = (int)min(32LL, ngroups - g0) * CPG;
        const uint4* src = reinterpret_cast<const uint4*>(w + g0 * G);
        for (int c = lane; c < n; c += 32) cp_async16(buf + (c / CPG) * S::IN_STRIDE + c % CPG, src + c);
    };

    long long tile = blockIdx.x;
    if (tile < ntiles) issue(tile, smq);
    cp_async_commit();
    for (int it = 0; tile < ntiles; ++it, tile += gridDim.x) {
        const long long next = tile + gridDim.x;
        if (next < ntiles) issue(next, smq + ((it + 1) & 1) * S::BUF);
        cp_async_commit();
        cp_async_wait_prev();
        __syncwarp();
        const long long g0 = tile * 32;
        const int ng = (int)min(32LL, ngroups - g0);
        if (lane < ng) {
            const uint4* my = smq + (it & 1) * S::BUF + lane * S::IN_STRIDE;
            MinMax<T> mm;
            mm.init(my[0]);
#pragma unroll 8
            for (int c = 0; c < CPG; ++c) mm.add(my[c]);
            float lo = mm.min(), hi = mm.max();
            if (lo == 0.0f) lo = first_zero<T>(my, CPG);
            if (hi == 0.0f) hi = first_zero<T>(my, CPG);
            const float scale = __fdiv_rn(__fsub_rn(hi, lo), (float)QMAX);
            const long long gi = g0 + lane;
            DT<T>::st(scales, gi, scale);
            DT<T>::st(biases, gi, lo);
            const float sT = QT<T>::rt(scale), bT = QT<T>::rt(lo);
            const float inv = sT != 0.0f ? __fdiv_rn(1.0f, sT) : 0.0f;
            const bool fast = reciprocal_ok(sT, inv);
            uint32_t* mo = out + lane * S::OUT_STRIDE;
#pragma unroll 1
            for (int blk = 0; blk < G / 32; ++blk) {
                uint32_t W[B];
#pragma unroll
                for (int i = 0; i < B; ++i) W[i] = 0;
#pragma unroll
                for (int cc = 0; cc < 32 / E; ++cc) {
                    float v[E];
                    widen16<T>(my[blk * (32 / E) + cc], v);
                    uint32_t q[E];
                    float cv[E];
                    uint32_t near = quantize_codes<QMAX, E>(v, bT, inv, q, cv);
                    if (!fast) {
                        // (fully unrolled: a run-time index would move v[] and
                        // q[] to local memory for the whole loop)
#pragma unroll
                        for (int e = 0; e < E; ++e) q[e] = exact_code<QMAX>(v[e], bT, sT);
                    } else {
                        while (near) {                       // the few values near a half-integer
                            const int e = __ffs(near) - 1;
                            near &= near - 1u;
                            float ve = v[0], ce = cv[0];
#pragma unroll
                            for (int j = 1; j < E; ++j)
                                if (j == e) { ve = v[j]; ce = cv[j]; }
                            const uint32_t qe = near_code<QMAX>(ve, bT, sT, ce);
#pragma unroll
                            for (int j = 0; j < E; ++j)
                                if (j == e) q[j] = qe;
                        }
                    }
#pragma unroll
                    for (int e = 0; e < E; ++e) {
                        const int p = (cc * E + e) * B, wi = p >> 5, sh = p & 31;
                        W[wi] |= q[e] << sh;
                        if (sh + B > 32) W[wi + 1] |= q[e] >> (32 - sh);
                    }
                }
#pragma unroll
                for (int i = 0; i < B; ++i) mo[blk * B + i] = W[i];
            }
        }
        __syncwarp();
        uint32_t* dst = wq + g0 * WPG;
        for (int i = lane; i < ng * WPG; i += 32) dst[i] = out[(i / WPG) * S::OUT_STRIDE + i % WPG];
        __syncwarp();
    }
}

template <int B, class T, int G>
cudaError_t quantize_tiles(const void* w, void* wq, void* s, void* b, long long ngroups, cudaStream_t st) {
    using S = TileShape<B, T, G>;
    static int blocks_per_sm = 0;
    if (!blocks_per_sm) {
        cudaError_t e = cudaFuncSetAttribute(quantize_affine_tiles<B, T, G>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S::SMEM);
        if (e == cudaSuccess)
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks_per_sm, quantize_affine_tiles<B, T, G>, 32,
                                                              S::SMEM);
        if (e != cudaSuccess) return e;
        if (blocks_per_sm < 1) return cudaErrorInvalidConfiguration;
    }
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long ntiles = (ngroups + 31) / 32;
    const long long grid = std::min<long long>(ntiles, (long long)sms * blocks_per_sm);
    quantize_affine_tiles<B, T, G><<<(unsigned)grid, 32, S::SMEM, st>>>(
        static_cast<const T*>(w), static_cast<uint32_t*>(wq), static_cast<T*>(s), static_cast<T*>(b), ngroups);
    return cudaGetLastError();
}

template <int B, class T>
cudaError_t quantize_bt(const void* w, void* wq, void* s, void* b, int N, int K, int G, int vec, cudaStream_t st) {
    if (vec == 2) {                                  // w and w_packed 16-byte aligned: coalesced tiles
        const long long ngroups = (long long)N * (K / G);
        switch (G) {
            case 32: return quantize_tiles<B, T, 32>(w, wq, s, b, ngroups, st);
            case 64: return quantize_tiles<B, T, 64>(w, wq, s, b, ngroups, st);
            case 128: return quantize_tiles<B, T, 128>(w, wq, s, b, ngroups, st);
            default: return cudaErrorInvalidValue;
        }
    }
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
