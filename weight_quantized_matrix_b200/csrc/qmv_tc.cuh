// qmv_tc.cuh -- affine qmv on the tensor cores (mma.sync m16n8k16, bf16 in,
// fp32 accumulate), the path for sizes where the weight decode, not HBM, would
// bind the CUDA cores.
//
// Mapping (one warp = one 16-row tile of W; K may be split over the block's
// k-warps, each taking every wk-th super-block):
//   * A (16 x 16) is W: thread (g = lane/4, t = lane%4) decodes rows g and g+8
//     from its own "unit" of packed bytes (16 bytes for 2/4/8-bit codes, 32
//     codes for 3/5/6-bit).  The quad's four units form a SUPER-BLOCK of the
//     row; a k16 step takes two code pairs of each thread's unit.  A code pair
//     becomes one bf16x2 register with a single masked OR (qmv_tc_plan.cuh):
//     {128 + c_lo 2^s_lo, 128 + c_hi 2^s_hi}, and one bf16x2 subtraction
//     removes both 128 offsets exactly ({c_lo 2^s_lo, c_hi 2^s_hi}).  (Left in
//     and taken out of the fp32 sum as 128 * sum(x~), the offsets made the
//     accumulator carry terms about 128 / c times the codes' own: with x all
//     positive and a symmetric zero point that cancellation cost about
//     2.6e-5 * sum|x * w| at 2 bits, above the f32 bar.)
//   * B (16 x 8) is x, with its 8 columns used as SLOTS (super-block in the
//     batch, segment, x row): the B value of k-slot k in slot column c is x~[k]
//     when code k belongs to that super-block and segment, else 0 (inactive
//     lanes read a zero row).  A segment is min(group, super-block) codes, so
//     every D column is the partial dot product of one x row over one
//     (super-block, group) pair, and the exact fp32 epilogue applies that
//     group's scale and bias:   Y += scale * D + bias * sum x.
//     Filling all 8 columns with several super-blocks ("batch") runs the
//     epilogue once per batch; more slots than 8 use several MMAs per step.
//   * x is staged per block per K tile in shared memory, permuted into
//     fragment order and split into bf16 planes that add up to x exactly (one
//     plane for bf16 x, two for f16, three for f32); sum(x) per segment is
//     formed from values widened to fp32 one by one.
//   * Weights are prefetched PD super-blocks ahead in registers; scales are
//     loaded at the start of a batch for its epilogue.
//   * Results: per-thread slot partials -> shared memory -> sum over slots of
//     the same x row and over k-warps -> one rounding to the output dtype.
#pragma once

#include <utility>

#include "qmv_device.cuh"
#include "qmv_tc_plan.cuh"

namespace qmv {

template <class T> struct TcSplit { static constexpr int n = 1; };
template <> struct TcSplit<__half> { static constexpr int n = 2; };
template <> struct TcSplit<float> { static constexpr int n = 3; };

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// {a.lo - b.lo, a.hi - b.hi} on bf16x2 (round to nearest; exact here).
__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Pair p of a unit as bf16x2 {128 + low field * 2^slo, 128 + high field *
// 2^shi}: one masked OR, offsets kept (an empty high half is 128 + 0; an
// empty pair is 0).  For kernels that take the offsets out of their own fp32
// sums.
template <int B, int p>
__device__ __forceinline__ uint32_t tc_pair_offset(const uint32_t (&w)[TcGeom<B>::NW], uint32_t kbf16) {
    constexpr TcPlanData P = tc_make_plan<B, false>();
    if constexpr (P.lo[p] < 0) {
        return 0u;
    } else {
        constexpr int NW = TcGeom<B>::NW, fb = TcGeom<B>::FB;
        constexpr int sh = P.sh[p], a = sh / 32, r = sh % 32;
        uint32_t v;
        if constexpr (r == 0) {
            v = w[a];
        } else if constexpr (a + 1 < NW && r + 16 + P.shi[p] + fb > 32) {
            v = __funnelshift_r(w[a], w[a + 1], r);
        } else if constexpr (a + 1 < NW && P.hi[p] < 0 && r + P.slo[p] + fb > 32) {
            v = __funnelshift_r(w[a], w[a + 1], r);
        } else {
            v = w[a] >> r;
        }
        constexpr uint32_t fm = (1u << fb) - 1u;
        constexpr uint32_t m = (fm << P.slo[p]) | (P.hi[p] >= 0 ? (fm << (16 + P.shi[p])) : 0u);
        return and_or<m>(v, kbf16);      // kbf16 = 0x43004300, held in a register
    }
}

// Pair p of a unit as bf16x2 {low field * 2^slo, high field * 2^shi}: the
// masked OR gives {128 + c_lo 2^slo, 128 + c_hi 2^shi} (fields below bit 7 of
// the bf16 mantissa), and one bf16x2 subtraction of {128, 128} removes the
// offsets exactly, so every product the MMA accumulates is an exact code
// times x~ (an empty high half is 0; an empty pair is 0).
template <int B, int p>
__device__ __forceinline__ uint32_t tc_pair(const uint32_t (&w)[TcGeom<B>::NW], uint32_t kbf16) {
    constexpr TcPlanData P = tc_make_plan<B, false>();
    if constexpr (P.lo[p] < 0) {
        return 0u;
    } else {
        return bf16x2_sub(tc_pair_offset<B, p>(w, kbf16), kbf16);
    }
}

// fp32 -> bf16 bits, round to nearest even (exact for the split planes).
__device__ __forceinline__ uint32_t bf16_bits(float v) {
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// The k16 steps of one super-block for one tile, two steps per B load.
template <int B, int NPASS, int NSPLIT, int... S2>
__device__ __forceinline__ void tc_steps(std::integer_sequence<int, S2...>, const uint32_t (&wg)[TcGeom<B>::NW],
                                         const uint32_t (&wh)[TcGeom<B>::NW], float (&D)[NPASS][4],
                                         const uint32_t* __restrict__ xb, const int (&xoff)[NPASS], int plane,
                                         uint32_t kbf16) {
    (
        [&] {
            constexpr int s = 2 * S2;
            const uint32_t a0 = tc_pair<B, 2 * s>(wg, kbf16), a2 = tc_pair<B, 2 * s + 1>(wg, kbf16);
            const uint32_t a1 = tc_pair<B, 2 * s>(wh, kbf16), a3 = tc_pair<B, 2 * s + 1>(wh, kbf16);
            const uint32_t c0 = tc_pair<B, 2 * s + 2>(wg, kbf16), c2 = tc_pair<B, 2 * s + 3>(wg, kbf16);
            const uint32_t c1 = tc_pair<B, 2 * s + 2>(wh, kbf16), c3 = tc_pair<B, 2 * s + 3>(wh, kbf16);
#pragma unroll
            for (int pp = 0; pp < NPASS; ++pp)
#pragma unroll
                for (int sp = 0; sp < NSPLIT; ++sp) {
                    const uint4 b = *reinterpret_cast<const uint4*>(xb + xoff[pp] + sp * plane + 2 * s);
                    mma_bf16_16816(D[pp], a0, a1, a2, a3, b.x, b.y);
                    mma_bf16_16816(D[pp], c0, c1, c2, c3, b.z, b.w);
                }
        }(),
        ...);
}

// As tc_steps, with the two k-steps of each B load accumulated into separate
// registers (D, E): two independent MMA dependency chains instead of one.
template <int B, int NPASS, int NSPLIT, int... S2>
__device__ __forceinline__ void tc_steps2(std::integer_sequence<int, S2...>, const uint32_t (&wg)[TcGeom<B>::NW],
                                          const uint32_t (&wh)[TcGeom<B>::NW], float (&D)[NPASS][4],
                                          float (&E)[NPASS][4], const uint32_t* __restrict__ xb,
                                          const int (&xoff)[NPASS], int plane, uint32_t kbf16) {
    (
        [&] {
            constexpr int s = 2 * S2;
            const uint32_t a0 = tc_pair<B, 2 * s>(wg, kbf16), a2 = tc_pair<B, 2 * s + 1>(wg, kbf16);
            const uint32_t a1 = tc_pair<B, 2 * s>(wh, kbf16), a3 = tc_pair<B, 2 * s + 1>(wh, kbf16);
            const uint32_t c0 = tc_pair<B, 2 * s + 2>(wg, kbf16), c2 = tc_pair<B, 2 * s + 3>(wg, kbf16);
            const uint32_t c1 = tc_pair<B, 2 * s + 2>(wh, kbf16), c3 = tc_pair<B, 2 * s + 3>(wh, kbf16);
#pragma unroll
            for (int pp = 0; pp < NPASS; ++pp)
#pragma unroll
                for (int sp = 0; sp < NSPLIT; ++sp) {
                    const uint4 b = *reinterpret_cast<const uint4*>(xb + xoff[pp] + sp * plane + 2 * s);
                    mma_bf16_16816(D[pp], a0, a1, a2, a3, b.x, b.y);
                    mma_bf16_16816(E[pp], c0, c1, c2, c3, b.z, b.w);
                }
        }(),
        ...);
}

// Shared memory:
//   xs  : [NSPLIT][M+1][xrow] u32 (bf16 pairs; row M is zero); xrow = TU*NP + 4
//   sx  : [M][TSB*NGS] float   sum(x) per segment of the tile
//   sxt : [M][TSB*NGS] float   sum(x~) per segment (fragment-ordered values)
//   us  : [M][TU][2] float     per-unit sums, combined into sx / sxt
//   red : [wk*wr][16][8*NPASS] float
template <int B, class T, int NPASS, int PD>
__global__ void __launch_bounds__(256) qmv_tc_kernel(const Params p) {
    using Gm = TcGeom<B>;
    constexpr TcPlanData P = tc_make_plan<B, false>();
    constexpr int NP = P.np, NSTEP = NP / 2;
    constexpr int NW = Gm::NW, UB = Gm::UNIT_BYTES, UC = Gm::UNIT_CODES, SB = Gm::SB;
    constexpr int NSPLIT = TcSplit<T>::n;

    extern __shared__ float4 smem4[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int wk = p.wk, wr = p.wr;
    const int wkid = warp % wk, wrid = warp / wk;
    const int bz = blockIdx.z;
    const int M = p.M;
    const int row0 = (blockIdx.x * wr + wrid) * 16;
    const int NSBK = p.K / SB;
    const int TSB = p.tile_iters;
    const int TU = TSB * 4;
    const int segsz = min(p.G, SB);
    const int NGS = SB / segsz;
    const int G = p.G;
    const long long KG = p.K / G;
    const int xrow = TU * NP + 4;                 // u32 per x row of the tile
    const int plane = (M + 1) * xrow;             // u32 per split plane (row M: zeros)
    const int NSEG = TSB * NGS;

    uint32_t* xs = reinterpret_cast<uint32_t*>(smem4);
    float* sx = reinterpret_cast<float*>(xs + (size_t)NSPLIT * plane);
    float* sxt = sx + (size_t)M * NSEG;
    float* us = sxt + (size_t)M * NSEG;
    float* red = us + (size_t)M * TU * 2;

    const uint8_t* W = p.w + bz * p.w_bs;
    const T* X = reinterpret_cast<const T*>(p.x) + bz * p.x_bs;
    const long long sb0 = bz * p.s_bs;
    const int rg = min(row0 + g, p.N - 1), rh = min(row0 + g + 8, p.N - 1);
    const uint8_t* Wg = W + (long long)rg * p.w_row + t * UB;
    const uint8_t* Wh = W + (long long)rh * p.w_row + t * UB;
    const T* scg = reinterpret_cast<const T*>(p.scales) + sb0 + (long long)rg * KG;
    const T* sch = reinterpret_cast<const T*>(p.scales) + sb0 + (long long)rh * KG;
    const T* big = reinterpret_cast<const T*>(p.biases) + sb0 + (long long)rg * KG;
    const T* bih = reinterpret_cast<const T*>(p.biases) + sb0 + (long long)rh * KG;

    // Slot geometry: column j of pass pp = 8 pp + c holds slot j = (sbi*NGS + gs)*M + m,
    // sbi = super-block within the batch.  SPB super-blocks per batch.
    const int per_sb = NGS * M;                   // slots one super-block needs
    const int SPB = max(1, (8 * NPASS) / per_sb);
    const int nslots = SPB * per_sb;
    const int gmul = G < SB ? __ffs(SB / G) - 1 : 0;
    const int gdiv = G > SB ? __ffs(G / SB) - 1 : 0;
    const int useg = (t * UC) / segsz;            // segment of this thread's unit
    // B column of this lane in each pass: super-block slot it serves (-1: none) and x row
    int bsbi[NPASS], brow[NPASS];
#pragma unroll
    for (int pp = 0; pp < NPASS; ++pp) {
        const int j = 8 * pp + g;
        const int m = j % M, q = j / M, gs = q % NGS, sbi = q / NGS;
        bsbi[pp] = (j < nslots && gs == useg) ? sbi : -1;
        brow[pp] = m;
    }
    // D slots of this lane: (row g / g+8, column 8 pp + 2t + c)
    int dsbi[NPASS][2], dgs[NPASS][2], dm[NPASS][2];
#pragma unroll
    for (int pp = 0; pp < NPASS; ++pp)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int j = 8 * pp + 2 * t + c;
            const int q = j / M;
            dm[pp][c] = j % M;
            dgs[pp][c] = q % NGS;
            dsbi[pp][c] = j < nslots ? q / NGS : -1;
        }

    float D[NPASS][4], Y[NPASS][4];
#pragma unroll
    for (int pp = 0; pp < NPASS; ++pp)
#pragma unroll
        for (int e = 0; e < 4; ++e) { D[pp][e] = 0.f; Y[pp][e] = 0.f; }

    auto loadW = [&](uint32_t (&wg)[NW], uint32_t (&wh)[NW], int sb) {
        const long long off = (long long)sb * 4 * UB;
        if constexpr (UB == 16) {
            const uint4 a = __ldg(reinterpret_cast<const uint4*>(Wg + off));
            const uint4 b = __ldg(reinterpret_cast<const uint4*>(Wh + off));
            wg[0] = a.x; wg[1] = a.y; wg[2] = a.z; wg[3] = a.w;
            wh[0] = b.x; wh[1] = b.y; wh[2] = b.z; wh[3] = b.w;
        } else {
#pragma unroll
            for (int q = 0; q < NW; ++q) {
                wg[q] = __ldg(reinterpret_cast<const uint32_t*>(Wg + off) + q);
                wh[q] = __ldg(reinterpret_cast<const uint32_t*>(Wh + off) + q);
            }
        }
    };

    const uint32_t kbf16 = p.kbf16;
    uint32_t wring[PD][2][NW];
    float sc[NPASS][4], bi[NPASS][4];

    // The first super-blocks' weights are loaded before waiting on the
    // previous kernel in the stream: weights are not produced by it (a
    // precondition of the C ABI), x and y may be.
#pragma unroll
    for (int q = 0; q < PD; ++q)
        if (wkid + q * wk < min(TSB, NSBK)) loadW(wring[q][0], wring[q][1], wkid + q * wk);
    grid_launch_dependents();        // the next kernel may start fetching its weights
    grid_wait();

    for (int t0 = 0; t0 < NSBK; t0 += TSB) {
        const int tn = min(TSB, NSBK - t0);
        const int first = t0 + wkid, end = t0 + tn;
        __syncthreads();
        // weights of the tile's first super-blocks do not depend on x: issue
        // them before staging x
        if (t0 > 0) {
#pragma unroll
            for (int q = 0; q < PD; ++q)
                if (first + q * wk < end) loadW(wring[q][0], wring[q][1], first + q * wk);
        }

        // ---- stage x: fragment-ordered bf16 planes + per-unit sums ------------
        {
            for (int i = threadIdx.x; i < xrow; i += blockDim.x)
#pragma unroll
                for (int sp = 0; sp < NSPLIT; ++sp) xs[(size_t)sp * plane + (size_t)M * xrow + i] = 0u;
            const int items = M * tn * 4;
            for (int it = threadIdx.x; it < items; it += blockDim.x) {
                const int m = it / (tn * 4), u = it - m * (tn * 4);
                const long long k0 = (long long)t0 * SB + (long long)u * UC;
                const T* xr = X + (long long)m * p.K + k0;
                float xv[UC];
                if constexpr (sizeof(T) == 2 && UC % 8 == 0) {
                    if (p.x_vec) {
#pragma unroll
                        for (int q = 0; q < UC / 8; ++q) widen8<T>(__ldg(reinterpret_cast<const uint4*>(xr) + q), xv + 8 * q);
                    } else {
#pragma unroll
                        for (int c = 0; c < UC; ++c) xv[c] = DT<T>::ld(xr, c);
                    }
                } else if constexpr (sizeof(T) == 4 && UC % 4 == 0) {
                    if (p.x_vec) {
#pragma unroll
                        for (int q = 0; q < UC / 4; ++q) {
                            const float4 f = __ldg(reinterpret_cast<const float4*>(xr) + q);
                            xv[4 * q] = f.x; xv[4 * q + 1] = f.y; xv[4 * q + 2] = f.z; xv[4 * q + 3] = f.w;
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < UC; ++c) xv[c] = DT<T>::ld(xr, c);
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < UC; ++c) xv[c] = DT<T>::ld(xr, c);
                }
                float usum = 0.f;                      // sum(x), widened element by element
#pragma unroll
                for (int c = 0; c < UC; ++c) usum += xv[c];
                float tsum = 0.f;                      // sum of the fragment values x~
                uint32_t* dst = xs + (size_t)m * xrow + (size_t)u * NP;
#pragma unroll
                for (int q = 0; q < NP; ++q) {
                    float lo = 0.f, hi = 0.f;
                    if (P.lo[q] >= 0)
                        lo = __fmul_rn(xv[tc_field_code<B>(P.lo[q])],
                                       __uint_as_float((uint32_t)(127 + tc_field_wexp<B>(P.lo[q]) - P.slo[q]) << 23));
                    if (P.hi[q] >= 0)
                        hi = __fmul_rn(xv[tc_field_code<B>(P.hi[q])],
                                       __uint_as_float((uint32_t)(127 + tc_field_wexp<B>(P.hi[q]) - P.shi[q]) << 23));
                    tsum += lo + hi;
#pragma unroll
                    for (int sp = 0; sp < NSPLIT; ++sp) {
                        const uint32_t bl = bf16_bits(lo), bh = bf16_bits(hi);
                        dst[(size_t)sp * plane + q] = bl | (bh << 16);
                        lo = lo - __uint_as_float(bl << 16);     // exact remainders
                        hi = hi - __uint_as_float(bh << 16);
                    }
                }
                us[((size_t)m * TU + u) * 2] = usum;
                us[((size_t)m * TU + u) * 2 + 1] = tsum;
            }
            __syncthreads();
            const int upseg = segsz / UC;
            const int nseg = tn * NGS;
            for (int it = threadIdx.x; it < M * nseg; it += blockDim.x) {
                const int m = it / nseg, sg = it - m * nseg;
                const float* ur = us + ((size_t)m * TU + (size_t)sg * upseg) * 2;
                float a = 0.f, b = 0.f;
                for (int q = 0; q < upseg; ++q) { a += ur[2 * q]; b += ur[2 * q + 1]; }
                sx[(size_t)m * NSEG + sg] = a;
                sxt[(size_t)m * NSEG + sg] = b;
            }
        }
        __syncthreads();

        // ---- main loop over this k-warp's super-blocks of the tile ----------
        int sb = first;
        int bi_ = 0;                                // super-block index within the batch
        while (sb < end) {
#pragma unroll
            for (int q = 0; q < PD; ++q) {
                if (sb < end) {
                    if (bi_ == 0) {
                        // new batch: scales / biases of its slots (used at batch end)
#pragma unroll
                        for (int pp = 0; pp < NPASS; ++pp)
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int c = e & 1;
                                const int sbs = sb + dsbi[pp][c] * wk;
                                sc[pp][e] = 0.f; bi[pp][e] = 0.f;
                                if (dsbi[pp][c] >= 0 && sbs < end) {
                                    const int grp = ((sbs << gmul) >> gdiv) + dgs[pp][c];
                                    sc[pp][e] = DT<T>::ld((e >> 1) ? sch : scg, grp);
                                    bi[pp][e] = DT<T>::ld((e >> 1) ? bih : big, grp);
                                }
                            }
                    }
                    int xoff[NPASS];
#pragma unroll
                    for (int pp = 0; pp < NPASS; ++pp)
                        xoff[pp] = (bsbi[pp] == bi_ ? brow[pp] : M) * xrow + ((sb - t0) * 4 + t) * NP;
                    tc_steps<B, NPASS, NSPLIT>(std::make_integer_sequence<int, NSTEP / 2>{}, wring[q][0], wring[q][1],
                                               D, xs, xoff, plane, kbf16);
                    if (sb + PD * wk < end) loadW(wring[q][0], wring[q][1], sb + PD * wk);
                    if (bi_ == SPB - 1 || sb + wk >= end) {
                        // epilogue of the batch: each slot's (super-block, group)
                        const int sb_first = sb - bi_ * wk;
#pragma unroll
                        for (int pp = 0; pp < NPASS; ++pp)
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int c = e & 1;
                                float a = 0.f;
                                if (dsbi[pp][c] >= 0 && dsbi[pp][c] <= bi_) {
                                    const int sl = (sb_first + dsbi[pp][c] * wk - t0) * NGS + dgs[pp][c];
                                    a = sx[(size_t)dm[pp][c] * NSEG + sl];
                                }
                                Y[pp][e] = fmaf(sc[pp][e], D[pp][e], fmaf(bi[pp][e], a, Y[pp][e]));
                                D[pp][e] = 0.f;
                            }
                        bi_ = 0;
                    } else {
                        ++bi_;
                    }
                    sb += wk;
                }
            }
        }
    }

    // ---- reduce over slots of the same x row and over k-warps, store ---------
    float* myred = red + (size_t)(wrid * wk + wkid) * 16 * 8 * NPASS;
#pragma unroll
    for (int pp = 0; pp < NPASS; ++pp)
#pragma unroll
        for (int e = 0; e < 4; ++e)
            myred[(g + 8 * (e >> 1)) * 8 * NPASS + 8 * pp + 2 * t + (e & 1)] = Y[pp][e];
    __syncthreads();
    T* Yo = reinterpret_cast<T*>(p.y) + bz * p.y_bs;
    const int tot = wr * 16 * M;
    for (int i = threadIdx.x; i < tot; i += blockDim.x) {
        const int w_ = i / (16 * M), rm = i % (16 * M), r = rm / M, m = rm % M;
        const int row = (blockIdx.x * wr + w_) * 16 + r;
        float v = 0.f;
        for (int k = 0; k < wk; ++k) {
            const float* rr = red + (size_t)(w_ * wk + k) * 16 * 8 * NPASS + r * 8 * NPASS;
            for (int j = m; j < nslots; j += M) v += rr[j];
        }
        if (row < p.N) DT<T>::st(Yo, (long long)m * p.N + row, v);
    }
}

}  // namespace qmv
