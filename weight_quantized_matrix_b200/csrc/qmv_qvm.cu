// qmv_qvm.cu -- qvm: x [M, K] times an affine weight matrix stored [K, N].
//
// MLX "quantized_nax.h" (mlx 1.0.0 source page), qouter: the outer-product
// accumulate result[j] += x * (scale * q_j + bias) over a row of packed codes;
// the wh-iron kernel-op coverage audit's qvm family ("x.W with W [K, N]",
// qvm_int4_fast with 8 columns per threadgroup).  Row k of w_packed packs the N
// codes of the output columns exactly like a qmv row (LSB-first packs), and
// scales / biases are [K, N / G], grouped along N:
//     y[m, n] = sum_k x[m, k] * (scale[k, n/G] * q[k, n] + bias[k, n/G]).
//
// B200 design (HBM-bound; CUDA cores, no tensor cores):
//  * A unit is 32 consecutive codes of a row (B 32-bit words), which always
//    lies inside one group (G is a multiple of 32).  Lane l of a warp owns unit
//    l of a 1024-column tile; a row's tile is one contiguous 128 * B byte span,
//    read with the widest aligned vector loads.
//  * The 8 warps of a block take interleaved rows of the block's K range.  Each
//    warp streams its rows through its own ring of 8 row slots in shared
//    memory: every lane copies its own unit with cp.async (no registers held
//    while the copy is in flight, about 64 KB in flight per SM) and reads back
//    only its own bytes, so no barrier is needed.  Per row a lane forms
//    x * scale once; the bias term is a running x * bias per lane (the unit
//    shares one bias).
//    Codes are decoded in place by OR-ing the masked field into the mantissa of
//    2^23 (value c * 2^p exactly, p a compile-time offset), and accumulated as
//    (x * scale * 2^-p) * (c * 2^p) with packed fp32x2 FMA on the code pair
//    (j, j + 16).  fp32 accumulation throughout.
//  * The 8 warps' partial sums are added in shared memory.  When K is split
//    over several blocks (blocks are few otherwise: one per 1024 columns), each
//    block adds its partials into an fp32 workspace with global atomic adds,
//    then counts itself in on a per-tile counter; the last block to arrive
//    rounds the tile to the element type, writes y and returns the workspace
//    and the counter to zero.  No block waits on another.  The summation order
//    over the K split therefore varies from run to run (results differ only by
//    fp32 rounding).  Without a workspace the whole K range stays in one block.
//  * x rows are processed MC (1 or 2) at a time; for M > 2 the row chunks are
//    the fastest-varying block index, so the chunks of a tile run together and
//    share its weights through L2.
#include <algorithm>
#include <atomic>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "qmv_device.cuh"

namespace qmv {

namespace {

constexpr int kQvmWarps = 8;
constexpr int kQvmDepth = 8;               // row slots per warp ring
constexpr int kQvmRedStride = 33;           // floats per lane row of the reduction buffer

struct QvmParams {
    const void* x;
    const uint8_t* w;
    const void* scales;
    const void* biases;
    void* y;
    float* ws;          // [M, N] fp32, all zero between calls (nullptr: ksplit == 1)
    unsigned* cnt;      // [ntiles * mchunks] arrival counters, zero between calls
    long long row_bytes;
    int M, N, K, NG, units, ntiles, mchunks, ksplit, rows, gshift;
};

// The B words of unit u of a packed row, with the widest aligned loads.
template <int B>
__device__ __forceinline__ void load_unit(const uint8_t* p, uint32_t* w) {
    if constexpr (B == 4) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (B == 8) {
        const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
        const uint4 b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    } else if constexpr (B == 2 || B == 6) {
#pragma unroll
        for (int i = 0; i < B / 2; ++i) {
            const uint2 v = __ldg(reinterpret_cast<const uint2*>(p) + i);
            w[2 * i] = v.x; w[2 * i + 1] = v.y;
        }
    } else {
#pragma unroll
        for (int i = 0; i < B; ++i) w[i] = __ldg(reinterpret_cast<const uint32_t*>(p) + i);
    }
}

// 2^-p as an fp32 constant.
__host__ __device__ constexpr uint32_t pow2_neg_bits(int p) { return (uint32_t)(127 - p) << 23; }

// One lane's unit copied global -> shared with cp.async (no registers held
// while in flight), in chunks of CS bytes (the widest the unit's alignment
// allows), stored chunk-major (chunk c of lane l at (c * 32 + l) * CS) so that
// reading it back is conflict-free.
template <int B>
struct UnitCopy {
    static constexpr int CS = (B == 4 || B == 8) ? 16 : (B == 2 || B == 6) ? 8 : 4;
    static constexpr int NCH = 4 * B / CS;
    static constexpr int SLOT = 32 * 4 * B;             // bytes of one row slot (a warp's units)

    static __device__ __forceinline__ void issue(uint32_t slot, const uint8_t* src, int lane) {
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const uint32_t dst = slot + (uint32_t)((c * 32 + lane) * CS);
            if constexpr (CS == 16)
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src + c * CS) : "memory");
            else
                asm volatile("cp.async.ca.shared.global [%0], [%1], %2;\n" ::"r"(dst), "l"(src + c * CS), "n"(CS)
                             : "memory");
        }
    }
    static __device__ __forceinline__ void read(const char* slot, int lane, uint32_t* w) {
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const char* q = slot + (c * 32 + lane) * CS;
            if constexpr (CS == 16) {
                const uint4 v = *reinterpret_cast<const uint4*>(q);
                w[4 * c] = v.x; w[4 * c + 1] = v.y; w[4 * c + 2] = v.z; w[4 * c + 3] = v.w;
            } else if constexpr (CS == 8) {
                const uint2 v = *reinterpret_cast<const uint2*>(q);
                w[2 * c] = v.x; w[2 * c + 1] = v.y;
            } else {
                w[c] = *reinterpret_cast<const uint32_t*>(q);
            }
        }
    }
};

// Raw element bits kept in a register until use: converting right after the
// load would stall the warp on the load's latency at issue time.
template <class T> struct Raw;
template <> struct Raw<float> {
    using type = float;
    static __device__ __forceinline__ type ld(const void* p, long long i) {
        return __ldg(reinterpret_cast<const float*>(p) + i);
    }
    static __device__ __forceinline__ float f(type v) { return v; }
};
template <> struct Raw<__half> {
    using type = unsigned short;
    static __device__ __forceinline__ type ld(const void* p, long long i) {
        return __ldg(reinterpret_cast<const unsigned short*>(p) + i);
    }
    static __device__ __forceinline__ float f(type v) { return __half2float(__ushort_as_half(v)); }
};
template <> struct Raw<__nv_bfloat16> {
    using type = unsigned short;
    static __device__ __forceinline__ type ld(const void* p, long long i) {
        return __ldg(reinterpret_cast<const unsigned short*>(p) + i);
    }
    static __device__ __forceinline__ float f(type v) { return __uint_as_float((uint32_t)v << 16); }
};

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

// acc[m][j] += (x_m * scale) * code j (pairs j, j + 16); bsum[m] += x_m * bias.
template <int B, int MC>
__device__ __forceinline__ void qvm_row(const uint32_t* wd, float s, float b, const float* x,
                                        float2 (&acc)[MC][16], float (&bsum)[MC]) {
    const uint32_t kf32 = 0x4B000000u;      // fp32 2^23
    float xs[MC];
#pragma unroll
    for (int m = 0; m < MC; ++m) {
        bsum[m] = fmaf(x[m], b, bsum[m]);
        xs[m] = __fmul_rn(x[m], s);
    }
#define QVM_PAIR(J)                                                                                     \
    {                                                                                                   \
        const float2 f_ = magic_pair_ored(field_magic<B, (J)>(wd, kf32), field_magic<B, (J) + 16>(wd, kf32)); \
        _Pragma("unroll") for (int m = 0; m < MC; ++m) {                                                \
            const float2 sx_ = make_float2(__fmul_rn(xs[m], __uint_as_float(pow2_neg_bits(field_p(B, (J))))), \
                                           __fmul_rn(xs[m], __uint_as_float(pow2_neg_bits(field_p(B, (J) + 16))))); \
            acc[m][(J)] = fma2(sx_, f_, acc[m][(J)]);                                                   \
        }                                                                                               \
    }
    QVM_PAIR(0) QVM_PAIR(1) QVM_PAIR(2) QVM_PAIR(3) QVM_PAIR(4) QVM_PAIR(5) QVM_PAIR(6) QVM_PAIR(7)
    QVM_PAIR(8) QVM_PAIR(9) QVM_PAIR(10) QVM_PAIR(11) QVM_PAIR(12) QVM_PAIR(13) QVM_PAIR(14) QVM_PAIR(15)
#undef QVM_PAIR
}

template <int B, class T, int MC>
__global__ void __launch_bounds__(kQvmWarps * 32) qvm_affine_kernel(const __grid_constant__ QvmParams p) {
    extern __shared__ __align__(16) float qvm_smem[];   // weight rings, then the reduction buffer
    float* qvm_red = qvm_smem;              // [warps][MC][32 * kQvmRedStride]
    __shared__ int s_last;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int bid = blockIdx.x;
    const int mc = bid % p.mchunks;
    bid /= p.mchunks;
    const int tile = bid % p.ntiles;
    const int ks = bid / p.ntiles;
    const int m0 = mc * MC;
    const int mn = min(MC, p.M - m0);
    const int u = tile * 32 + lane;
    const int uc = min(u, p.units - 1);     // idle lanes past N read a valid unit, results dropped
    const int g = (uc * 32) >> p.gshift;
    const int k0 = ks * p.rows, k1 = min(p.K, k0 + p.rows);
    const uint8_t* wu = p.w + (long long)uc * (4 * B);

    float2 acc[MC][16];
    float bsum[MC];
#pragma unroll
    for (int m = 0; m < MC; ++m) {
        bsum[m] = 0.0f;
#pragma unroll
        for (int j = 0; j < 16; ++j) acc[m][j] = make_float2(0.0f, 0.0f);
    }
    // Rows of this warp: k0 + warp + 8 i, i < n.  A ring of kQvmDepth row slots
    // per warp: row i + kQvmDepth is copied into row i's slot once row i has
    // been computed; its scale, bias and x values wait in registers as raw
    // element bits (converted at use).
    using UC = UnitCopy<B>;
    const int kw = k0 + warp;
    const int n = kw < k1 ? (k1 - kw + kQvmWarps - 1) / kQvmWarps : 0;
    char* ring = reinterpret_cast<char*>(qvm_smem) + warp * (kQvmDepth * UC::SLOT);
    const uint32_t ring_s = (uint32_t)__cvta_generic_to_shared(ring);
    using R = Raw<T>;
    typename R::type sr[kQvmDepth], br[kQvmDepth], xr[kQvmDepth][MC];
    auto fetch = [&](int d, int i) {             // row i into slot d (i < n)
        const int k = kw + i * kQvmWarps;
        UC::issue(ring_s + d * UC::SLOT, wu + (long long)k * p.row_bytes, lane);
        sr[d] = R::ld(p.scales, (long long)k * p.NG + g);
        br[d] = R::ld(p.biases, (long long)k * p.NG + g);
#pragma unroll
        for (int m = 0; m < MC; ++m) xr[d][m] = R::ld(p.x, (long long)(m0 + (m < mn ? m : 0)) * p.K + k);
    };
#pragma unroll
    for (int d = 0; d < kQvmDepth; ++d) {
        if (d < n) fetch(d, d);
        cp_async_commit();
    }
    for (int i0 = 0; i0 < n; i0 += kQvmDepth) {
#pragma unroll
        for (int d = 0; d < kQvmDepth; ++d) {
            const int i = i0 + d;
            if (i >= n) break;
            cp_async_wait<kQvmDepth - 1>();          // row i's copies (group i) have landed
            uint32_t wd[B];
            UC::read(ring + d * UC::SLOT, lane, wd);
            const float s_ = R::f(sr[d]), b_ = R::f(br[d]);
            float x_[MC];
#pragma unroll
            for (int m = 0; m < MC; ++m) x_[m] = m < mn ? R::f(xr[d][m]) : 0.0f;
            qvm_row<B, MC>(wd, s_, b_, x_, acc, bsum);
            // the slot is refilled only after the row's words have been used,
            // so the read above has completed before the copy can land
            if (i + kQvmDepth < n) fetch(d, i + kQvmDepth);
            cp_async_commit();
        }
    }
    cp_async_wait<0>();
    __syncthreads();                             // every warp is done with its ring

    // ---- the block's 8 warps: add in shared memory -------------------------
    constexpr int PLANE = 32 * kQvmRedStride;
#pragma unroll
    for (int m = 0; m < MC; ++m) {
        float* row = qvm_red + (warp * MC + m) * PLANE + lane * kQvmRedStride;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            row[j] = acc[m][j].x + bsum[m];
            row[j + 16] = acc[m][j].y + bsum[m];
        }
    }
    __syncthreads();
    const int ncols = min(1024, (p.units - tile * 32) * 32);     // valid columns of this tile
    const long long col0 = (long long)tile * 1024;
    const bool split = p.ksplit > 1;
    for (int i = threadIdx.x; i < MC * 1024; i += kQvmWarps * 32) {
        const int m = i >> 10, c = i & 1023;
        if (m >= mn || c >= ncols) continue;
        const int off = m * PLANE + (c >> 5) * kQvmRedStride + (c & 31);
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < kQvmWarps; ++w) v += qvm_red[w * MC * PLANE + off];
        const long long yi = (long long)(m0 + m) * p.N + col0 + c;
        if (split) atomicAdd(p.ws + yi, v);
        else DT<T>::st(p.y, yi, v);
    }
    if (!split) return;

    // ---- K split: the last block of this tile writes y ---------------------
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned prev = atomicAdd(p.cnt + (tile * p.mchunks + mc), 1u);
        s_last = prev == (unsigned)(p.ksplit - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int i = threadIdx.x; i < MC * 1024; i += kQvmWarps * 32) {
        const int m = i >> 10, c = i & 1023;
        if (m >= mn || c >= ncols) continue;
        const long long yi = (long long)(m0 + m) * p.N + col0 + c;
        DT<T>::st(p.y, yi, __ldcg(p.ws + yi));
        p.ws[yi] = 0.0f;
    }
    if (threadIdx.x == 0) p.cnt[tile * p.mchunks + mc] = 0u;
}

template <int B, class T, int MC>
cudaError_t launch_qvm_t(QvmParams p, bool have_ws, cudaStream_t st) {
    auto kern = qvm_affine_kernel<B, T, MC>;
    const size_t smem = std::max((size_t)kQvmWarps * MC * 32 * kQvmRedStride * sizeof(float),
                                 (size_t)kQvmWarps * kQvmDepth * UnitCopy<B>::SLOT);
    static std::atomic<unsigned> configured{0};
    static std::atomic<int> bps_cache{0};
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const unsigned bit = 1u << (dev & 31);
    if (!(configured.load(std::memory_order_acquire) & bit)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        int bps = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, kern, kQvmWarps * 32, smem);
        if (e != cudaSuccess) return e;
        bps_cache.store(std::max(1, bps), std::memory_order_relaxed);
        configured.fetch_or(bit, std::memory_order_acq_rel);
    }
    const int bps = bps_cache.load(std::memory_order_relaxed);
    // K split: one wave of resident blocks (the most splits whose blocks all
    // fit at once), at least 32 rows (4 per warp) a block.
    const long long base = (long long)p.ntiles * p.mchunks;
    int ksplit = 1;
    if (have_ws && p.K > 0) {
        const long long want = ((long long)sms * bps) / base;
        const long long most = std::max(1, (p.K + 31) / 32);
        ksplit = (int)std::max(1LL, std::min(want, most));
    }
    p.rows = (p.K + ksplit - 1) / ksplit;
    p.ksplit = p.rows > 0 ? (p.K + p.rows - 1) / p.rows : 1;
    if (p.ksplit <= 1) p.ws = nullptr, p.cnt = nullptr;
    const long long grid = base * p.ksplit;
    if (grid > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
    kern<<<(unsigned)grid, kQvmWarps * 32, smem, st>>>(p);
    return cudaGetLastError();
}

template <int B, class T>
cudaError_t launch_qvm_bt(const QvmParams& p, bool have_ws, cudaStream_t st) {
    return p.M == 1 ? launch_qvm_t<B, T, 1>(p, have_ws, st) : launch_qvm_t<B, T, 2>(p, have_ws, st);
}

template <int B>
cudaError_t launch_qvm_b(int dtype, const QvmParams& p, bool have_ws, cudaStream_t st) {
    switch (dtype) {
        case 0: return launch_qvm_bt<B, float>(p, have_ws, st);
        case 1: return launch_qvm_bt<B, __half>(p, have_ws, st);
        case 2: return launch_qvm_bt<B, __nv_bfloat16>(p, have_ws, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

size_t qvm_workspace_bytes(int M, int N) {
    const size_t acc = ((size_t)M * N * sizeof(float) + 255) / 256 * 256;
    const size_t tiles = ((size_t)N / 32 + 31) / 32;
    return acc + ((size_t)M * tiles * sizeof(unsigned) + 255) / 256 * 256;
}

cudaError_t launch_qvm_affine(int bits, int dtype, const void* x, const void* w, const void* scales,
                              const void* biases, void* y, void* workspace, int M, int N, int K, int G,
                              cudaStream_t st) {
    QvmParams p = {};
    p.x = x; p.w = static_cast<const uint8_t*>(w); p.scales = scales; p.biases = biases; p.y = y;
    p.M = M; p.N = N; p.K = K; p.NG = N / G;
    p.units = N / 32;
    p.ntiles = (p.units + 31) / 32;
    p.mchunks = M == 1 ? 1 : (M + 1) / 2;
    p.row_bytes = (long long)N * bits / 8;
    p.gshift = G == 32 ? 5 : G == 64 ? 6 : 7;
    const bool have_ws = workspace != nullptr;
    if (have_ws) {
        p.ws = static_cast<float*>(workspace);
        p.cnt = reinterpret_cast<unsigned*>(static_cast<char*>(workspace) +
                                            ((size_t)M * N * sizeof(float) + 255) / 256 * 256);
    }
    switch (bits) {
        case 2: return launch_qvm_b<2>(dtype, p, have_ws, st);
        case 3: return launch_qvm_b<3>(dtype, p, have_ws, st);
        case 4: return launch_qvm_b<4>(dtype, p, have_ws, st);
        case 5: return launch_qvm_b<5>(dtype, p, have_ws, st);
        case 6: return launch_qvm_b<6>(dtype, p, have_ws, st);
        case 8: return launch_qvm_b<8>(dtype, p, have_ws, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace qmv
