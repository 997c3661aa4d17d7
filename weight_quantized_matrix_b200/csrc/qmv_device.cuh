// qmv_device.cuh -- device code of the weight-quantized matrix-vector product
// for sm_100a: per-format decoders, the warp-per-row-block qmv kernel and the
// dequantization check kernel.
//
// Formats (see include/qmv.h for the page citations):
//   affine  2/3/4/5/6/8-bit codes, LSB-first bit stream per row (MLX
//           quantized_nax.h, get_pack_factor / get_bytes_per_pack, qdot),
//           w = scale * q + bias per group of G codes;
//   MXFP4 / NVFP4 / MXFP8: E2M1 or E4M3 elements with E8M0 (per 32) or E4M3
//           (per 16, times an FP32 global) block scales (wh-iron audit, Track 1);
//   the rest of the audit's Track 1 table: E2M1 / E4M3 / E5M2 elements with a
//           block scale whose type (E8M0, E4M3, FP32 or FP16) and block (16 or
//           32) are run-time parameters (FAM_E2M1 / FAM_E4M3 / FAM_E5M2), and
//           the symmetric signed integers int2..int8 / mxint2..mxint8
//           (FAM_SINT): two's-complement codes in the affine bit stream, read
//           through the affine machinery after flipping every field's sign bit
//           (offset binary, field + 2^(b-1)) with bias = -2^(b-1) * scale.
//
// Work decomposition (B200-first, not the pages' Metal layout):
//   * The K axis of a row is cut into CHUNKS of C codes (C a multiple of 32).
//     A chunk is U "units" of 32 codes; a unit of b-bit codes is exactly b
//     32-bit words, so every unit has the same bit layout.  The wide path loads
//     a chunk with 16-byte vector loads (C chosen so a chunk is a whole number
//     of 16-byte vectors); the narrow path uses 4-byte loads and C = 32.
//   * A block has wr x wk warps.  Warp (wr, wk) owns R consecutive rows; its 32
//     lanes together with the other wk warps ("k-threads", kt = 32*wk + lane)
//     take the chunks of those rows round-robin, so small N still spreads one
//     row over up to 256 threads (split-K inside the block), and large N keeps
//     wk = 1 with R rows sharing every x load.
//   * x is staged per block in shared memory, widened to fp32 and PRE-SCALED
//     per code position: a code whose field sits at bit p of the word it is
//     masked from is used unshifted (value c * 2^p), so its x is stored as
//     x * 2^-p (exact: a power-of-two scale).  This is the x pre-scaling of
//     MLX's load_vector, re-derived for 32-bit words.  The integer field is
//     turned into a float without an int->float conversion: OR-ing it into the
//     mantissa of 2^23 and subtracting 2^23 is exact for fields below bit 23.
//   * Affine groups: each lane keeps fp32 partials sum(x~ * c 2^p) per
//     segment (the part of a group inside one chunk), then adds
//     scale * partial + bias * sum(x), where sum(x) of the segment is formed in
//     the staging pass from x values widened to fp32 one by one (the precision
//     fix of the MLX pull request).
//   * Products and partial sums use Blackwell's packed fp32x2 FMA/ADD.
//   * Reduction: lane partials -> warp butterfly shuffle -> (wk > 1) shared
//     memory across the k-warps -> one rounding to the output dtype.
//   * Rows past N in the last block read the last valid row and are not stored
//     (the row-tail rule of the MLX fast_rows kernels).
//   * The kernel waits on the previous grid (griddepcontrol.wait) before it
//     reads x, so it may be launched with programmatic dependent launch; the
//     first weight chunk is fetched before that wait, and dependents are let
//     launch right after it (they too wait before reading this grid's y).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <string.h>

namespace qmv {

enum Family {
    FAM_AFFINE = 0, FAM_MXFP4 = 1, FAM_NVFP4 = 2, FAM_MXFP8 = 3,
    FAM_E2M1 = 4, FAM_E4M3 = 5, FAM_E5M2 = 6,     // block and scale type at run time
    FAM_SINT = 7                                  // symmetric signed integers
};
// Block-scale storage of the run-time-scaled families (Params::skind).
enum ScaleKind { SK_E8M0 = 0, SK_E4M3 = 1, SK_F32 = 2, SK_F16 = 3 };

// Families read through the affine machinery (codes in the LSB-first bit
// stream, fp32 sum(x) per unit, scale * partial + bias * sum(x)).
template <int FAM> __host__ __device__ constexpr bool affine_like() { return FAM == FAM_AFFINE || FAM == FAM_SINT; }
// Families with one scale per 16 codes possible: a 32-code unit keeps two
// partial sums, one per half.
template <int FAM> __host__ __device__ constexpr bool half_units() {
    return FAM == FAM_NVFP4 || FAM == FAM_E2M1 || FAM == FAM_E4M3 || FAM == FAM_E5M2;
}

struct Params {
    const void* x;          // [batch?][M][K] dtype
    const uint8_t* w;       // [batch][N][row bytes]
    const void* scales;     // [batch][N][K/G] (dtype for affine, u8 for FP)
    const void* biases;     // [batch][N][K/G] dtype (affine)
    const float* gscale;    // NVFP4: [batch] floats
    void* y;                // [batch][M][N] dtype
    int M, N, K, G;         // G: group (affine) or block (FP) size
    int wk, wr;             // warps along K, warps along rows
    int tile_iters;         // x tile = 32*wk*tile_iters chunks
    int x_vec;              // 1: x rows are 16-byte aligned (vector staging loads)
    long long x_bs;         // x batch stride in elements (0 = shared x)
    long long w_bs;         // w batch stride in bytes
    long long s_bs;         // scales/biases batch stride in elements
    long long y_bs;         // y batch stride in elements
    long long w_row;        // bytes per packed row
    int sps;                // bulk-ring kernel: super-blocks per ring stage
    int pitch;              // bulk-ring kernel: bytes per ring row
    unsigned* fault;        // bulk-ring kernel: device fault word (bounded waits that expired)
    int sring;              // bulk-ring kernel: 1 = scales / biases travel in the ring (tensor copies)
    int soff, boff;         // bulk-ring kernel: byte offsets of the scale / bias tiles in a ring stage
    int sbw;                // bulk-ring kernel: bytes per row of those tiles
    CUtensorMap smap, bmap; // bulk-ring kernel: scales / biases as [batch][N][K/G] tensors
    CUtensorMap wmap;       // bulk-ring kernel: packed rows as [batch][N][row bytes / 8] u64
    // Exponent patterns OR-ed into decoded fields, passed in so that kernels
    // hold them in registers: then mask-and-OR is one three-input logic op
    // (with both operands immediate it would take two).
    unsigned kf32;          // 0x4B000000: fp32 2^23
    unsigned kbf16;         // 0x43004300: bf16 pair {128, 128}
    // Gather (expert-indexed batches): batch entry z multiplies by weight
    // matrix ids[z] of the stack (x and y stay entry z's); null: matrix z.
    // Only the CUDA-core row-tiled and the few-rows kernels read it.
    const int* ids;
    int n_experts;
    // Fused gate + up with SwiGLU (pair kernels only): w / scales / biases
    // are the gate matrix, w2 / scales2 / biases2 the up matrix; output row n
    // is silu(clamp(gate_n)) * clamp(up_n) * route_w[m] (see swiglu_act).
    const uint8_t* w2;
    const void* scales2;
    const void* biases2;
    const float* route_w;   // [M] per x row, or null for 1
    float act_clamp;        // clamp value; inactive at or below 1e-6
    // Q / K / V in one call (RMODE_QKV kernels): output rows [0, n1) read
    // w / scales / biases, [n1, n2) w2 / scales2 / biases2, [n2, N) w3 /
    // scales3 / biases3; y is [M, N] with the three parts side by side.
    const uint8_t* w3;
    const void* scales3;
    const void* biases3;
    int n1, n2;
    // RMSNorm of x fused in (row-tiled kernel): non-null gamma [K] (dtype)
    // scales x staged for the products by gamma[k] / sqrt(mean(x[m]^2) + eps).
    const void* gamma;
    float eps;
    // Block-scale type of FAM_E2M1 / FAM_E4M3 / FAM_E5M2 / FAM_SINT (ScaleKind).
    int skind;
    // Weight-ring kernels, tests only (qmv_test_skip_last_copy): nonzero makes
    // block (0, 0)'s producer skip its final stage, so the bounded waits on it
    // run out.
    int test_skip;
};

// Row mapping of the row-tiled kernel: plain, the interleaved gate / up
// pair (SwiGLU), or the three Q / K / V matrices.
enum RowMode { RMODE_PLAIN = 0, RMODE_PAIR = 1, RMODE_QKV = 2 };

// ---------------------------------------------------------------- dtypes ---
template <class T> struct DT;
template <> struct DT<float> {
    static __device__ __forceinline__ float ld(const void* p, long long i) {
        return __ldg(reinterpret_cast<const float*>(p) + i);
    }
    static __device__ __forceinline__ void st(void* p, long long i, float v) {
        reinterpret_cast<float*>(p)[i] = v;
    }
};
template <> struct DT<__half> {
    static __device__ __forceinline__ float ld(const void* p, long long i) {
        return __half2float(reinterpret_cast<const __half*>(p)[i]);
    }
    static __device__ __forceinline__ void st(void* p, long long i, float v) {
        reinterpret_cast<__half*>(p)[i] = __float2half_rn(v);
    }
};
template <> struct DT<__nv_bfloat16> {
    static __device__ __forceinline__ float ld(const void* p, long long i) {
        return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
    }
    static __device__ __forceinline__ void st(void* p, long long i, float v) {
        reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
    }
};

// Widen 8 consecutive dtype elements loaded as one 16-byte vector.
template <class T> __device__ __forceinline__ void widen8(const uint4& v, float* o);
template <> __device__ __forceinline__ void widen8<__half>(const uint4& v, float* o) {
    const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) { float2 f = __half22float2(h[i]); o[2 * i] = f.x; o[2 * i + 1] = f.y; }
}
template <> __device__ __forceinline__ void widen8<__nv_bfloat16>(const uint4& v, float* o) {
    const uint32_t* u = reinterpret_cast<const uint32_t*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        o[2 * i] = __uint_as_float(u[i] << 16);
        o[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
    }
}

// ------------------------------------------------------- packed fp32 math --
// Blackwell fp32x2 instructions through the compiler's builtins (so constant
// operands stay in registers or immediates instead of being re-materialised
// around inline asm): two independent IEEE fp32 operations per issue slot,
// round to nearest even.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }

// ------------------------------------------------- grid dependency control --
__device__ __forceinline__ void grid_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// -------------------------------------------------- affine field extraction --
// Field j (0..31) of a 32-code unit of B-bit codes held in B 32-bit words
// (little-endian, LSB-first stream): starts at bit o = B*j of the unit.
//   * r + B <= 23       : mask in place, value c * 2^r          (p = r)
//   * 23 < r + B <= 32  : mask the word shifted right by 9     (p = r - 9)
//   * r + B > 32        : funnel-shift the word pair to bit 0  (p = 0)
// In every case the masked field lies below bit 23, so OR-ing it into the
// mantissa of 2^23 and subtracting 2^23 yields c * 2^p exactly.
__host__ __device__ constexpr int field_p(int B, int j) {
    return ((B * j) % 32 + B > 32) ? 0
         : ((B * j) % 32 + B <= 23) ? (B * j) % 32
         : (B * j) % 32 - 9;
}

template <int B, int J>
__device__ __forceinline__ uint32_t field_bits(const uint32_t* w) {
    constexpr int o = B * J, wi = o / 32, r = o % 32;
    constexpr uint32_t m = (1u << B) - 1u;
    if constexpr (r + B > 32) {
        return __funnelshift_r(w[wi], w[wi + 1], r) & m;
    } else if constexpr (r + B <= 23) {
        return w[wi] & (m << r);
    } else {
        return (w[wi] >> 9) & (m << (r - 9));
    }
}

// (a & MASK) | c as one three-input logic op.
template <uint32_t MASK>
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "n"(MASK), "r"(c));
    return d;
}

// field_bits OR-ed with kf32 (the fp32 pattern of 2^23) in the same op.
template <int B, int J>
__device__ __forceinline__ uint32_t field_magic(const uint32_t* w, uint32_t kf32) {
    constexpr int o = B * J, wi = o / 32, r = o % 32;
    constexpr uint32_t m = (1u << B) - 1u;
    if constexpr (r + B > 32) {
        return and_or<m>(__funnelshift_r(w[wi], w[wi + 1], r), kf32);
    } else if constexpr (r + B <= 23) {
        return and_or<(m << r)>(w[wi], kf32);
    } else {
        return and_or<(m << (r - 9))>(w[wi] >> 9, kf32);
    }
}

// {a, b}: fields already OR-ed into 2^23 -> their values as exact floats.
__device__ __forceinline__ float2 magic_pair_ored(uint32_t a, uint32_t b) {
    return add2(make_float2(__uint_as_float(a), __uint_as_float(b)), make_float2(-8388608.0f, -8388608.0f));
}

__device__ __forceinline__ float2 magic_pair(uint32_t a, uint32_t b) {
    // {a, b} fields (< 2^23) -> {a, b} as exact floats
    return add2(make_float2(__uint_as_float(a | 0x4B000000u), __uint_as_float(b | 0x4B000000u)),
                make_float2(-8388608.0f, -8388608.0f));
}

// ------------------------------------------------------- FP element decode --
// E2M1 nibble -> float: the 3 magnitude bits placed at fp32 bits 22..24 form
// a number equal to the E2M1 magnitude times 2^-126 (the subnormal code lands
// on an fp32 subnormal of the same ratio); the sign goes to bit 31.  One exact
// multiply by 2^126 restores the value (wh-iron audit: bit-pattern decode
// followed by an exact power-of-two multiply).
__device__ __forceinline__ uint32_t e2m1_pattern(uint32_t nib) {
    return ((nib & 7u) << 22) | ((nib & 8u) << 28);
}
__device__ __forceinline__ float e2m1_value(uint32_t nib) {
    return __uint_as_float(e2m1_pattern(nib)) * 0x1p126f;
}
// E4M3 byte -> float: exponent+mantissa bits at fp32 bits 20..26, times 2^120;
// S.1111.111 is NaN.
__device__ __forceinline__ float e4m3_value(uint32_t c) {
    c &= 0xFFu;
    float v = __uint_as_float(((c & 0x7Fu) << 20) | ((c & 0x80u) << 24)) * 0x1p120f;
    return ((c & 0x7Fu) == 0x7Fu) ? __uint_as_float(0x7FC00000u) : v;
}
// E8M0 byte -> 2^(e-127); e = 0 is the fp32 subnormal 2^-127; 0xFF is NaN.
__device__ __forceinline__ float e8m0_value(uint32_t e) {
    e &= 0xFFu;
    return e == 0xFFu ? __uint_as_float(0x7FC00000u)
         : e == 0u ? __uint_as_float(0x00400000u) : __uint_as_float(e << 23);
}

// E5M2 byte -> float: exponent+mantissa bits at fp32 bits 21..27 form the
// value times 2^-112 (subnormals included), restored by one exact multiply;
// exponent field 31 is infinity (mantissa 0) or NaN.
__device__ __forceinline__ float e5m2_value(uint32_t c) {
    c &= 0xFFu;
    const float v = __uint_as_float(((c & 0x7Fu) << 21) | ((c & 0x80u) << 24)) * 0x1p112f;
    return ((c & 0x7Cu) == 0x7Cu)
               ? __uint_as_float((c & 3u) ? 0x7FC00000u : (((c & 0x80u) << 24) | 0x7F800000u))
               : v;
}
// 8-bit element of a family (E5M2 for FAM_E5M2, E4M3 otherwise).
template <int FAM> __device__ __forceinline__ float fp8_value(uint32_t c) {
    if constexpr (FAM == FAM_E5M2) return e5m2_value(c);
    else return e4m3_value(c);
}
// Hardware element decode for the inner loops: two E2M1 codes (one byte, low
// nibble first) or two E4M3 / E5M2 codes (two bytes, low byte first) -> f16x2
// (low half first).  Exact: every value of these element types is a binary16
// value (E4M3 NaN and E5M2 infinities / NaN included); widening to fp32 is
// exact too.  The bit-pattern decoders above serve the check kernel.
__device__ __forceinline__ uint32_t cvt_e2m1x2(uint32_t v) {
    uint32_t d;
    asm("{.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;}" : "=r"(d) : "r"(v));
    return d;
}
template <int FAM>
__device__ __forceinline__ uint32_t cvt_fp8x2(uint32_t v) {
    uint32_t d;
    if constexpr (FAM == FAM_E5M2)
        asm("{.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e5m2x2 %0, t;}" : "=r"(d) : "r"(v));
    else
        asm("{.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;}" : "=r"(d) : "r"(v));
    return d;
}
__device__ __forceinline__ float2 half2_bits_to_float2(uint32_t h) {
    __half2 v;
    memcpy(&v, &h, 4);
    return __half22float2(v);
}

// Block scale i of a run-time-typed scale array.
__device__ __forceinline__ float block_scale(const void* s, long long i, int kind) {
    switch (kind) {
        case SK_E8M0: return e8m0_value(__ldg(reinterpret_cast<const uint8_t*>(s) + i));
        case SK_E4M3: return e4m3_value(__ldg(reinterpret_cast<const uint8_t*>(s) + i));
        case SK_F32: return __ldg(reinterpret_cast<const float*>(s) + i);
        default: return __half2float(__ldg(reinterpret_cast<const __half*>(s) + i));
    }
}
// Signed-int codes: the bits of word wi of a B-word unit that are a field's
// top (sign) bit.  XOR-ing them maps a two's-complement field q to the offset
// binary q + 2^(B-1), a plain unsigned code.
template <int B> __host__ __device__ constexpr uint32_t sint_sign_mask(int wi) {
    uint32_t m = 0;
    for (int j = 0; j < 32; ++j) {
        const int b = B * j + B - 1;
        if (b / 32 == wi) m |= 1u << (b % 32);
    }
    return m;
}

// ----------------------------------------------------------- format traits --
template <int FAM, int BITS> struct Fmt {
    static constexpr int kBits = affine_like<FAM>() ? BITS : ((FAM == FAM_MXFP8 || FAM == FAM_E4M3 || FAM == FAM_E5M2) ? 8 : 4);
    static constexpr int kUnitWords = kBits;                 // words per 32 codes
    // Units per chunk on the wide path: the smallest whole number of units
    // whose byte size is a multiple of 16 (and at least 32 bytes for 2/4-bit).
    static constexpr int kWideUnits =
        kBits == 2 ? 4 : kBits == 3 ? 4 : kBits == 4 ? 2 : kBits == 5 ? 4 : kBits == 6 ? 2 : 1;
};

// ------------------------------------------------------- shared pieces -----
// x staging: one work item = (m, chunk, unit) = 32 consecutive x values of
// row m; writes the fp32 (pre-scaled for affine) values to
// xs[((m*TI + i)*(C/4) + u*8 + q)*KT + kt] and, for affine, the unit's
// sum(x) -- accumulated from values widened to fp32 one by one -- to
// sx[((m*TI + i)*U + u)*KT + kt], where chunk cc of the tile is owned by
// k-thread cc % KT at iteration cc / KT.
template <int FAM, int B, class T, int MAXM, int U>
__device__ __forceinline__ void stage_x(const Params& p, const char* Xb, float4* xs, float* sx, int t0,
                                        int tcn, int KT, int TI, const float* rnorm = nullptr) {
    constexpr int C = 32 * U;
    constexpr bool AFF = affine_like<FAM>();
    const int items = MAXM * tcn * U;
    for (int it = threadIdx.x; it < items; it += blockDim.x) {
        const int u = it % U;
        const int cc = (it / U) % tcn;
        const int m = it / (U * tcn);
        const int i = cc / KT, ktt = cc % KT;
        float v[32];
        if (m < p.M) {
            const long long k0 = (long long)(t0 + cc) * C + u * 32;
            const T* xr = reinterpret_cast<const T*>(Xb) + (long long)m * p.K + k0;
            if constexpr (sizeof(T) == 2) {
                if (p.x_vec) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 vv = __ldg(reinterpret_cast<const uint4*>(xr) + q);
                        widen8<T>(vv, v + 8 * q);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = DT<T>::ld(xr, j);
                }
            } else {
                if (p.x_vec) {
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        float4 f = __ldg(reinterpret_cast<const float4*>(xr) + q);
                        v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = DT<T>::ld(xr, j);
                }
            }
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0.f;
        }
        if (rnorm && m < p.M) {
            // RMSNorm: x * r_m * gamma[k], in fp32 (kept unrounded)
            const long long k0 = (long long)(t0 + cc) * C + u * 32;
            const float r = rnorm[m];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __fmul_rn(__fmul_rn(v[j], r), DT<T>::ld(p.gamma, k0 + j));
        }
        if constexpr (AFF) {
            float s = 0.f;                      // sum(x), widened per element
#pragma unroll
            for (int j = 0; j < 32; ++j) s += v[j];
            sx[(((size_t)m * TI + i) * U + u) * KT + ktt] = s;
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __fmul_rn(v[j], __uint_as_float((127u - field_p(B, j)) << 23));
        }
        float4* dst = xs + (((size_t)m * TI + i) * (C / 4) + u * 8) * KT + ktt;
#pragma unroll
        for (int q = 0; q < 8; ++q)
            dst[(size_t)q * KT] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
}

// Per-unit scales of chunk c for R rows (affine: scale + bias of the unit's
// group; MX: one block scale; NV: two block scales per unit).  PAIR: row r is
// virtual row rowc[r] of the interleaved gate / up pair (odd rows: up).
template <int FAM, int B, class T, int R, int U, int RMODE = RMODE_PLAIN>
__device__ __forceinline__ void load_scales(const Params& p, const int (&rowc)[R], int c, long long sb,
                                            float (&sc)[R][U][2], float (&bi)[R][U]) {
    constexpr int C = 32 * U;
    const int G = p.G;
    const long long KG = p.K / G;
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const long long k0 = (long long)c * C + u * 32;
            long long row = rowc[r];
            const void* sp = p.scales;
            const void* bp = p.biases;
            if constexpr (RMODE == RMODE_PAIR) {
                if (row & 1) { sp = p.scales2; bp = p.biases2; }
                row >>= 1;
            } else if constexpr (RMODE == RMODE_QKV) {
                if (row >= p.n2) { sp = p.scales3; bp = p.biases3; row -= p.n2; }
                else if (row >= p.n1) { sp = p.scales2; bp = p.biases2; row -= p.n1; }
            }
            const long long rb = row * KG;
            if constexpr (FAM == FAM_AFFINE) {
                const long long gi = sb + rb + k0 / G;
                sc[r][u][0] = DT<T>::ld(sp, gi);
                bi[r][u] = DT<T>::ld(bp, gi);
            } else if constexpr (FAM == FAM_SINT) {
                // offset-binary codes: w = s * (q' - 2^(B-1)) = s * q' + bias
                const float sv = block_scale(p.scales, sb + rb + k0 / G, p.skind);
                sc[r][u][0] = sv;
                sc[r][u][1] = 0.f;
                bi[r][u] = -sv * (float)(1 << (B - 1));
            } else if constexpr (FAM == FAM_E2M1 || FAM == FAM_E4M3 || FAM == FAM_E5M2) {
                const long long si = sb + rb + k0 / G;
                sc[r][u][0] = block_scale(p.scales, si, p.skind);
                sc[r][u][1] = G == 16 ? block_scale(p.scales, si + 1, p.skind) : sc[r][u][0];
                bi[r][u] = 0.f;
            } else if constexpr (FAM == FAM_NVFP4) {
                const uint8_t* s8 = reinterpret_cast<const uint8_t*>(p.scales) + sb + rb + k0 / 16;
                sc[r][u][0] = e4m3_value(__ldg(s8));
                sc[r][u][1] = e4m3_value(__ldg(s8 + 1));
                bi[r][u] = 0.f;
            } else {
                const uint8_t* s8 = reinterpret_cast<const uint8_t*>(p.scales) + sb + rb + k0 / 32;
                sc[r][u][0] = e8m0_value(__ldg(s8));
                sc[r][u][1] = 0.f;
                bi[r][u] = 0.f;
            }
        }
}

// Dot products of one chunk (U units of 32 codes) for R rows and MAXM x rows.
//   wv    chunk words of each row (registers)
//   xb    &xs[(i*(C/4))*KT + kt]; x row m, unit u, step q at xb[m*xm + (u*8+q)*KT]
//   sxb   &sx[(i*U)*KT + kt];     x row m, unit u        at sxb[m*sxm + u*KT]
template <int FAM, int B, int MAXM, int R, int U>
__device__ __forceinline__ void compute_chunk(const uint32_t (&wv)[R][B * U], const float (&sc)[R][U][2],
                                              const float (&bi)[R][U], const float4* xb, size_t xm,
                                              const float* sxb, size_t sxm, int KT, float (&acc)[R][MAXM],
                                              uint32_t kf32) {
    constexpr int UW = B;
    constexpr bool AFF = affine_like<FAM>();
#pragma unroll
    for (int u = 0; u < U; ++u) {
        float2 part[R][MAXM][2];                  // NV: one per 16-code block
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int m = 0; m < MAXM; ++m) { part[r][m][0] = make_float2(0.f, 0.f); part[r][m][1] = make_float2(0.f, 0.f); }
#pragma unroll
        for (int q = 0; q < 8; ++q) {              // 4 codes per step
            float4 xv[MAXM];
#pragma unroll
            for (int m = 0; m < MAXM; ++m) xv[m] = xb[(size_t)m * xm + (size_t)(u * 8 + q) * KT];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const uint32_t* wu = &wv[r][u * UW];
                float2 d0, d1;                     // codes 4q..4q+3 as two float pairs
                if constexpr (AFF) {
                    uint32_t f0, f1, f2, f3;
                    switch (q) {
#define QMV_F4(QQ) case QQ: f0 = field_magic<B, 4 * QQ>(wu, kf32); f1 = field_magic<B, 4 * QQ + 1>(wu, kf32); \
                   f2 = field_magic<B, 4 * QQ + 2>(wu, kf32); f3 = field_magic<B, 4 * QQ + 3>(wu, kf32); break;
                        QMV_F4(0) QMV_F4(1) QMV_F4(2) QMV_F4(3) QMV_F4(4) QMV_F4(5) QMV_F4(6) QMV_F4(7)
#undef QMV_F4
                        default: f0 = f1 = f2 = f3 = kf32;
                    }
                    d0 = magic_pair_ored(f0, f1);
                    d1 = magic_pair_ored(f2, f3);
                } else if constexpr (B == 4) {
                    const uint32_t wd = wu[q >> 1] >> (16 * (q & 1));
                    d0 = half2_bits_to_float2(cvt_e2m1x2(wd));
                    d1 = half2_bits_to_float2(cvt_e2m1x2(wd >> 8));
                } else {
                    const uint32_t wd = wu[q];
                    d0 = half2_bits_to_float2(cvt_fp8x2<FAM>(wd));
                    d1 = half2_bits_to_float2(cvt_fp8x2<FAM>(wd >> 16));
                }
                const int h = half_units<FAM>() ? (q >> 2) : 0;    // 16-code half of the unit
#pragma unroll
                for (int m = 0; m < MAXM; ++m) {
                    float2 a = part[r][m][h];
                    a = fma2(make_float2(xv[m].x, xv[m].y), d0, a);
                    a = fma2(make_float2(xv[m].z, xv[m].w), d1, a);
                    part[r][m][h] = a;
                }
            }
        }
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int m = 0; m < MAXM; ++m) {
                if constexpr (AFF) {
                    const float s = sxb[(size_t)m * sxm + (size_t)u * KT];
                    const float pr = part[r][m][0].x + part[r][m][0].y;
                    acc[r][m] = fmaf(sc[r][u][0], pr, fmaf(bi[r][u], s, acc[r][m]));
                } else if constexpr (half_units<FAM>()) {
                    acc[r][m] = fmaf(sc[r][u][0], part[r][m][0].x + part[r][m][0].y, acc[r][m]);
                    acc[r][m] = fmaf(sc[r][u][1], part[r][m][1].x + part[r][m][1].y, acc[r][m]);
                } else {
                    acc[r][m] = fmaf(sc[r][u][0], part[r][m][0].x + part[r][m][0].y, acc[r][m]);
                }
            }
    }
}

// SwiGLU of one output (DS4 moe.metal, the routed-expert activation): with a
// clamp c above 1e-6 the gate is limited to <= c and up to [-c, c]; then
// silu(g) * u = g / (1 + exp(-g)) * u, in fp32.  The caller multiplies by the
// route weight.
__device__ __forceinline__ float swiglu_act(float g, float u, float c) {
    if (c > 1.0e-6f) {
        g = fminf(g, c);
        u = fminf(fmaxf(u, -c), c);
    }
    return __fdiv_rn(g, 1.0f + expf(-g)) * u;
}

template <int R, int MAXM>
__device__ __forceinline__ void warp_allreduce(float (&acc)[R][MAXM]) {
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < MAXM; ++m) {
            float v = acc[r][m];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
            acc[r][m] = v;
        }
}

// ------------------------------------------------ kernel 1: narrow / general --
// Shared memory layout (floats):
//   xs : [MAXM][tile_iters][C/4][KT] float4   pre-scaled x of the tile
//   sx : [MAXM][tile_iters][U][KT]            affine: sum(x) per unit
//   red: [wk][wr*R*MAXM]                       cross-warp partials
// KT = 32*wk.  Chunk c of the tile belongs to k-thread c % KT, iteration c / KT.
//
// PAIR (affine only, R even): the fused gate + up projection with SwiGLU.
// The rows are the 2N virtual rows of the interleaved pair (virtual row 2n =
// gate row n, 2n + 1 = up row n), so each warp holds both sums of its R / 2
// outputs and writes y[m, n] = swiglu_act(gate, up) * route_w[m].
template <int FAM, int BITS, class T, int MAXM, int R, bool WIDE, int RMODE = RMODE_PLAIN>
__global__ void __launch_bounds__(256) qmv_kernel(const Params p) {
    constexpr bool PAIR = RMODE == RMODE_PAIR;
    static_assert(!PAIR || (FAM == FAM_AFFINE && R % 2 == 0), "pair rows come in twos");
    static_assert(RMODE != RMODE_QKV || FAM == FAM_AFFINE, "Q / K / V are affine");
    using F = Fmt<FAM, BITS>;
    constexpr int B = F::kBits;
    constexpr int U = WIDE ? F::kWideUnits : 1;
    constexpr int C = 32 * U;
    constexpr int CW = B * U;
    constexpr bool AFF = affine_like<FAM>();

    extern __shared__ float4 smem4[];
    const int KT = 32 * p.wk;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wkid = warp % p.wk, wrid = warp / p.wk;
    const int kt = wkid * 32 + lane;
    const int bz = blockIdx.z;
    const int row0 = (blockIdx.x * p.wr + wrid) * R;
    // gather: entry bz's weights are matrix ids[bz]; an id outside the stack
    // has no weights, and this block's outputs of the entry become NaN
    // (gather launches without programmatic dependent launch, so the ids
    // written by the previous kernel are complete)
    int be = bz;
    if (p.ids) {
        be = __ldg(p.ids + bz);
        if (be < 0 || be >= p.n_experts) {
            T* Yn = reinterpret_cast<T*>(p.y) + bz * p.y_bs;
            const int rows = p.wr * R, r0 = blockIdx.x * rows;
            for (int i = threadIdx.x; i < rows * p.M; i += blockDim.x) {
                const int n = r0 + i / p.M, m = i % p.M;
                if (n < p.N) DT<T>::st(Yn, (long long)m * p.N + n, __int_as_float(0x7FC00000));
            }
            return;
        }
    }
    const int NC = p.K / C;
    const int TI = p.tile_iters;
    const int TC = KT * TI;

    float4* xs = smem4;
    float* sx = reinterpret_cast<float*>(xs + (size_t)MAXM * TI * (C / 4) * KT);
    float* red = sx + (AFF ? (size_t)MAXM * TI * U * KT : 0);

    const uint8_t* W = p.w + be * p.w_bs;
    const char* Xb = reinterpret_cast<const char*>(p.x) + bz * p.x_bs * (long long)sizeof(T);
    const long long sb = be * p.s_bs;

    const int NV = PAIR ? 2 * p.N : p.N;           // rows of the (virtual) matrix
    int rowc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) rowc[r] = min(row0 + r, NV - 1);

    float acc[R][MAXM];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < MAXM; ++m) acc[r][m] = 0.f;

    uint32_t wv[R][CW];
    float sc[R][U][2], bi[R][U];
    auto load_chunk = [&](int c) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const uint8_t* base = W;
            long long prow = rowc[r];
            if constexpr (PAIR) {
                base = (prow & 1) ? p.w2 : W;
                prow >>= 1;
            } else if constexpr (RMODE == RMODE_QKV) {
                if (prow >= p.n2) { base = p.w3; prow -= p.n2; }
                else if (prow >= p.n1) { base = p.w2; prow -= p.n1; }
            }
            const uint8_t* src = base + prow * p.w_row + (long long)c * (C * B / 8);
            if constexpr (WIDE) {
#pragma unroll
                for (int q = 0; q < CW / 4; ++q) {
                    uint4 t = __ldg(reinterpret_cast<const uint4*>(src) + q);
                    wv[r][4 * q] = t.x; wv[r][4 * q + 1] = t.y; wv[r][4 * q + 2] = t.z; wv[r][4 * q + 3] = t.w;
                }
            } else {
#pragma unroll
                for (int q = 0; q < CW; ++q) wv[r][q] = __ldg(reinterpret_cast<const uint32_t*>(src) + q);
            }
            if constexpr (FAM == FAM_SINT) {
#pragma unroll
                for (int q = 0; q < CW; ++q) wv[r][q] ^= sint_sign_mask<B>(q % B);
            }
        }
        load_scales<FAM, B, T, R, U, RMODE>(p, rowc, c, sb, sc, bi);
    };

    const uint32_t kf32 = p.kf32;
    // The first chunk's weights (packed codes, scales, biases) are loaded
    // before waiting on the previous kernel in the stream: weights are not
    // produced by it (a precondition of the C ABI), x and y may be.
    bool have = kt < min(TC, NC);
    if (have) load_chunk(kt);
    // let the next kernel in the stream start its own weight fetch now; it
    // still waits for this grid to complete before it reads x
    grid_launch_dependents();
    grid_wait();

    // RMSNorm: r_m = 1 / sqrt(mean_k x[m,k]^2 + eps) for every x row, by the
    // whole block (fp32 sums of squares, warp shuffles, then one shared pass)
    float* rnorm = nullptr;
    if (p.gamma) {
        float* part = red + (size_t)p.wk * p.wr * R * MAXM;      // [warps][MAXM], then r[MAXM]
        const int nw = blockDim.x >> 5;
#pragma unroll
        for (int m = 0; m < MAXM; ++m) {
            float q = 0.f;
            if (m < p.M) {
                const T* xr = reinterpret_cast<const T*>(Xb) + (long long)m * p.K;
                for (int k = threadIdx.x; k < p.K; k += blockDim.x) {
                    const float v = DT<T>::ld(xr, k);
                    q = fmaf(v, v, q);
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xFFFFFFFFu, q, o);
            if (lane == 0) part[warp * MAXM + m] = q;
        }
        __syncthreads();
        if (threadIdx.x < MAXM) {
            float q = 0.f;
            for (int w = 0; w < nw; ++w) q += part[w * MAXM + threadIdx.x];
            part[nw * MAXM + threadIdx.x] = 1.0f / sqrtf(q / (float)p.K + p.eps);
        }
        __syncthreads();
        rnorm = part + nw * MAXM;
    }

    for (int t0 = 0; t0 < NC; t0 += TC) {
        const int tcn = min(TC, NC - t0);          // chunks in this tile
        __syncthreads();
        // the tile's first chunk of weights is independent of x: issue it
        // before staging x so both latencies overlap
        if (t0 > 0) {
            have = kt < tcn;
            if (have) load_chunk(t0 + kt);
        }
        stage_x<FAM, B, T, MAXM, U>(p, Xb, xs, sx, t0, tcn, KT, TI, rnorm);
        __syncthreads();
        for (int i = 0; have;) {
            compute_chunk<FAM, B, MAXM, R, U>(wv, sc, bi, xs + (size_t)i * (C / 4) * KT + kt,
                                              (size_t)TI * (C / 4) * KT, sx + (size_t)i * U * KT + kt,
                                              (size_t)TI * U * KT, KT, acc, kf32);
            ++i;
            const int cc = i * KT + kt;
            have = i < TI && cc < tcn;
            if (have) load_chunk(t0 + cc);
        }
    }

    if constexpr (half_units<FAM>()) {
        // K % 32 == 16 (blocks of 16): the row's last 16 codes lie outside
        // the 32-code units; the first k-warp's lanes 0..15 take one each
        if ((p.K & 31) && wkid == 0 && lane < 16) {
            const long long k = (long long)p.K - 16 + lane;
            const T* Xt = reinterpret_cast<const T*>(Xb);
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const uint8_t* rp = W + (long long)rowc[r] * p.w_row;
                float e;
                if constexpr (B == 4) e = e2m1_value(__ldg(rp + (k >> 1)) >> (4 * (int)(k & 1)));
                else e = fp8_value<FAM>(__ldg(rp + k));
                const long long si = sb + (long long)rowc[r] * (p.K / p.G) + k / p.G;
                const float sv = FAM == FAM_NVFP4 ? e4m3_value(__ldg(reinterpret_cast<const uint8_t*>(p.scales) + si))
                                                  : block_scale(p.scales, si, p.skind);
                const float ws = __fmul_rn(e, sv);
#pragma unroll
                for (int m = 0; m < MAXM; ++m)
                    if (m < p.M) acc[r][m] = fmaf(DT<T>::ld(Xt, (long long)m * p.K + k), ws, acc[r][m]);
            }
        }
    }
    warp_allreduce<R, MAXM>(acc);
    float gs = 1.f;
    if constexpr (FAM == FAM_NVFP4) gs = __ldg(p.gscale + be);
    T* Y = reinterpret_cast<T*>(p.y) + bz * p.y_bs;
    const int RM = R * MAXM;
    if constexpr (PAIR) {
        // output n = virtual rows (2n, 2n + 1); row0 is even
        const float c = p.act_clamp;
        if (p.wk == 1) {
#pragma unroll
            for (int j = 0; j < R / 2; ++j)
#pragma unroll
                for (int m = 0; m < MAXM; ++m)
                    if (lane == j * MAXM + m && row0 + 2 * j < NV && m < p.M) {
                        const float rw = p.route_w ? __ldg(p.route_w + m) : 1.0f;
                        DT<T>::st(Y, (long long)m * p.N + (row0 >> 1) + j,
                                  swiglu_act(acc[2 * j][m], acc[2 * j + 1][m], c) * rw);
                    }
        } else {
            if (lane == 0) {
#pragma unroll
                for (int r = 0; r < R; ++r)
#pragma unroll
                    for (int m = 0; m < MAXM; ++m) red[(wkid * p.wr + wrid) * RM + r * MAXM + m] = acc[r][m];
            }
            __syncthreads();
            const int tot = p.wr * RM;
            const int outs = p.wr * (R / 2) * MAXM;
            for (int t = threadIdx.x; t < outs; t += blockDim.x) {
                const int wr_ = t / ((R / 2) * MAXM), jm = t % ((R / 2) * MAXM), j = jm / MAXM, m = jm % MAXM;
                const int ig = wr_ * RM + (2 * j) * MAXM + m, iu = ig + MAXM;
                float g = 0.f, u = 0.f;
                for (int k = 0; k < p.wk; ++k) { g += red[k * tot + ig]; u += red[k * tot + iu]; }
                const int row = (blockIdx.x * p.wr + wr_) * R + 2 * j;
                if (row < NV && m < p.M) {
                    const float rw = p.route_w ? __ldg(p.route_w + m) : 1.0f;
                    DT<T>::st(Y, (long long)m * p.N + (row >> 1), swiglu_act(g, u, c) * rw);
                }
            }
        }
        return;
    }
    if (p.wk == 1) {
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int m = 0; m < MAXM; ++m)
                if (lane == r * MAXM + m && row0 + r < p.N && m < p.M)
                    DT<T>::st(Y, (long long)m * p.N + row0 + r, acc[r][m] * gs);
    } else {
        if (lane == 0) {
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int m = 0; m < MAXM; ++m) red[(wkid * p.wr + wrid) * RM + r * MAXM + m] = acc[r][m];
        }
        __syncthreads();
        const int tot = p.wr * RM;
        for (int t = threadIdx.x; t < tot; t += blockDim.x) {
            float v = 0.f;
            for (int k = 0; k < p.wk; ++k) v += red[k * tot + t];
            const int wr_ = t / RM, rm = t % RM, r = rm / MAXM, m = rm % MAXM;
            const int row = (blockIdx.x * p.wr + wr_) * R + r;
            if (row < p.N && m < p.M) DT<T>::st(Y, (long long)m * p.N + row, v * gs);
        }
    }
}

// ------------------------------------------------- dequantization check ----
// One thread per 32-code unit of one row; writes 32 fp32 weights.
//   affine: fmaf(scale, c, bias) with c = (c * 2^p) * 2^-p (exact)
//   signed int: the same on the offset-binary codes with bias = -2^(b-1) *
//           scale, i.e. the one rounding of scale * q
//   MX:     elem * e8m0 (exact in fp32)
//   NV:     (elem * e4m3) * global (the first product exact, one rounding)
//   E2M1 / E4M3 / E5M2 with a typed block scale: elem * scale, one rounding
// With K % 32 == 16 (blocks of 16) the last 16 codes of each row follow, one
// thread each.
template <int FAM, int B>
__device__ __forceinline__ float fp_elem_at(const uint32_t* wv, int j) {
    if constexpr (B == 4) return e2m1_value(wv[j / 8] >> (4 * (j % 8)));
    else return fp8_value<FAM>(wv[j / 4] >> (8 * (j % 4)));
}

template <int FAM>
__device__ __forceinline__ float fp_scale_at(const void* scales, const float* gscale, long long si, int skind) {
    const uint8_t* s8 = reinterpret_cast<const uint8_t*>(scales);
    if constexpr (FAM == FAM_NVFP4) return e4m3_value(__ldg(s8 + si));
    else if constexpr (FAM == FAM_MXFP4 || FAM == FAM_MXFP8) return e8m0_value(__ldg(s8 + si));
    else return block_scale(scales, si, skind);
}

template <int FAM, int BITS, class T>
__global__ void __launch_bounds__(256) dequant_kernel(const uint8_t* __restrict__ w,
                                                      const void* scales, const void* biases,
                                                      const float* gscale, float* __restrict__ out,
                                                      int N, int K, int G, long long w_row, int skind) {
    using F = Fmt<FAM, BITS>;
    constexpr int B = F::kBits;
    const long long units = (long long)N * (K / 32);
    grid_wait();
    for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < units;
         t += (long long)gridDim.x * blockDim.x) {
        const long long n = t / (K / 32);
        const int u = (int)(t % (K / 32));
        const uint32_t* src = reinterpret_cast<const uint32_t*>(w + n * w_row + (long long)u * 4 * B);
        uint32_t wv[B];
#pragma unroll
        for (int q = 0; q < B; ++q) wv[q] = __ldg(src + q);
        float o[32];
        const long long k0 = (long long)u * 32;
        if constexpr (affine_like<FAM>()) {
            const long long gi = n * (K / G) + k0 / G;
            float s, b;
            if constexpr (FAM == FAM_SINT) {
#pragma unroll
                for (int q = 0; q < B; ++q) wv[q] ^= sint_sign_mask<B>(q);
                s = block_scale(scales, gi, skind);
                b = -s * (float)(1 << (B - 1));
            } else {
                s = DT<T>::ld(scales, gi);
                b = DT<T>::ld(biases, gi);
            }
#define QMV_D4(QQ) { float2 d0 = magic_pair(field_bits<B, 4 * QQ>(wv), field_bits<B, 4 * QQ + 1>(wv)); \
                     float2 d1 = magic_pair(field_bits<B, 4 * QQ + 2>(wv), field_bits<B, 4 * QQ + 3>(wv)); \
                     float c[4] = {d0.x, d0.y, d1.x, d1.y}; \
                     _Pragma("unroll") for (int e = 0; e < 4; ++e) { \
                         const float q_ = __fmul_rn(c[e], __uint_as_float((127u - field_p(B, 4 * QQ + e)) << 23)); \
                         o[4 * QQ + e] = fmaf(s, q_, b); } }
            QMV_D4(0) QMV_D4(1) QMV_D4(2) QMV_D4(3) QMV_D4(4) QMV_D4(5) QMV_D4(6) QMV_D4(7)
#undef QMV_D4
        } else {
            const long long sr = n * (K / G);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float v = __fmul_rn(fp_elem_at<FAM, B>(wv, j), fp_scale_at<FAM>(scales, gscale, sr + (k0 + j) / G, skind));
                o[j] = FAM == FAM_NVFP4 ? __fmul_rn(v, __ldg(gscale)) : v;
            }
        }
        float4* dst = reinterpret_cast<float4*>(out + n * (long long)K + k0);
#pragma unroll
        for (int q = 0; q < 8; ++q) dst[q] = make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
    }
    if constexpr (half_units<FAM>()) {
        if (K & 31) {
            const long long tails = (long long)N * 16;
            for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < tails;
                 t += (long long)gridDim.x * blockDim.x) {
                const long long n = t / 16, k = (long long)K - 16 + (t % 16);
                const uint8_t* rp = w + n * w_row;
                float e;
                if constexpr (B == 4) e = e2m1_value(__ldg(rp + (k >> 1)) >> (4 * (int)(k & 1)));
                else e = fp8_value<FAM>(__ldg(rp + k));
                const float v = __fmul_rn(e, fp_scale_at<FAM>(scales, gscale, n * (K / G) + k / G, skind));
                out[n * (long long)K + k] = FAM == FAM_NVFP4 ? __fmul_rn(v, __ldg(gscale)) : v;
            }
        }
    }
}

}  // namespace qmv
