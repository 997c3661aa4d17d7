// qmv_tcf.cuh -- affine qmv for one bf16 x row on the CUDA cores, with the
// weights streaming through the same shared-memory ring as qmv_tcb.cuh (one
// producer warp issuing tensor copies, full / empty barriers, bounded waits).
//
// Why: with one x row an m16n8k16 MMA uses one of its eight columns, and on
// B200 the warp-level MMAs of that kernel, issued in order between the decode
// instructions, cost more time than the decode itself (measured by removing
// them).  Here each code costs half a masked OR (a code PAIR is decoded with
// one masked OR into bf16x2 {128 + c_lo 2^s_lo, 128 + c_hi 2^s_hi}, exactly as
// for the tensor cores, qmv_tc_plan.cuh) plus one mixed-precision FMA
// (fma.rn.f32.bf16: bf16 x bf16 product, exact, added to an fp32 accumulator
// with one rounding) against the fragment-ordered x~ = x * 2^-s (exact for bf16
// x).  The 128 offsets are removed per unit in fp32, and the unit's group
// scale and bias applied:
//     y += scale * (sum_unit - 128 * sum(x~_unit)) + bias * sum(x_unit).
// (The tensor-core kernels subtract the offsets before accumulating, one more
// instruction per pair, because their f16 / f32 outputs are held to the fp32
// bar; this kernel serves bf16 x and y only, where the offset's fp32
// cancellation stays inside the output's 1-ulp bar, and it is issue-bound.)
//
// Lanes: a warp owns a 16-row tile; lane = (r4 = lane / 8, u8 = lane % 8)
// takes rows r4, r4 + 4, r4 + 8, r4 + 12 and unit u8 of a STEP of two
// super-blocks (8 units of 16 bytes for 2/4/8-bit codes): the 8 lanes of one
// shared-memory phase read 128 consecutive bytes of one ring row, and their x~
// units sit 80 bytes apart (unit stride NP + 4 words), so neither load has
// bank conflicts.  Warp (wrid, wkid) takes the steps wkid, wkid + wk, ... of
// every stage; a stage holds a multiple of 2 * wk super-blocks.
//
// The block-scaled FP formats (FAM != FAM_AFFINE; E2M1 codes B = 4, E4M3 /
// E5M2 codes B = 8) stream through the same ring and lane layout: a 16-byte
// unit holds 32 E2M1 or 16 8-bit codes, decoded two at a time by the hardware
// conversion to f16x2 and widened to fp32 (exact), against x staged as plain
// fp32 rows of UC + 4 floats per unit (the pad keeps the 8 lanes of a
// shared-memory phase on distinct banks); the unit's one or two block scales
// (blocks of 16 or 32 codes, any scale type) travel in the ring as one more
// tensor-copy tile per stage (p.sring; else from global memory), and NVFP4's
// global scale multiplies the stored row sum.
#pragma once

#include "qmv_tcb.cuh"

namespace qmv {

// d = a * b + c, a and b the low (HI = false) or high halves of two bf16x2
// registers, c and d fp32; the product is exact, one rounding.
template <bool HI>
__device__ __forceinline__ float fma_bf16_f32(uint32_t a, uint32_t b, float c) {
    float d;
    if constexpr (HI) {
        asm("{.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
            "fma.rn.f32.bf16 %0, ah, bh, %3;}"
            : "=f"(d) : "r"(a), "r"(b), "f"(c));
    } else {
        asm("{.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
            "fma.rn.f32.bf16 %0, al, bl, %3;}"
            : "=f"(d) : "r"(a), "r"(b), "f"(c));
    }
    return d;
}

// Pairs q of one unit against its x~ pairs: two accumulators (low, high halves).
template <int B, int... Q>
__device__ __forceinline__ void tcf_unit(std::integer_sequence<int, Q...>, const uint32_t (&w)[TcGeom<B>::NW],
                                         const uint32_t* xq, uint32_t kbf16, float& lo, float& hi) {
    ((lo = fma_bf16_f32<false>(tc_pair_offset<B, Q>(w, kbf16), xq[Q], lo),
      hi = fma_bf16_f32<true>(tc_pair_offset<B, Q>(w, kbf16), xq[Q], hi)),
     ...);
}

// Shared memory (bytes, in order):
//   bars  128            full[STAGES], empty[STAGES], row-block completion
//                        counters rdone[STAGES + 1] at byte 96
//   ring  STAGES stages (128-byte aligned): ROWS packed rows (pitch bytes
//         each), then (p.sring) the scale tile at p.soff and the bias tile at
//         p.boff, ROWS x p.sbw bytes each
//   xs    TU * (NP + 4) u32     x~ pairs of the tile's units (bf16x2, plan order);
//                               FP: TU * (UC + 4) fp32 x values
//   us    TU * 2 floats         {sum(x), sum(x~)} per unit (affine only)
//   red   (STAGES + 1) * NCW * 16 floats   per-warp row sums, by row block
// MAXT = 32 * (NCW + 1): NCW = wk * wr in {8, 12} compute warps + the producer.
// FP unit: the sums of x * element over the unit's halves (p1 only for 32
// E2M1 codes), with the unit's codes w (16 bytes) and its x values xf (UC
// fp32 values, held in registers for the lane's 4 rows).
template <int FAM, int B>
__device__ __forceinline__ void fpr_unit(const uint32_t (&w)[4], const float (&xf)[B == 4 ? 32 : 16], float2& p0,
                                         float2& p1) {
    if constexpr (B == 4) {
        // 32 E2M1 codes: codes 0..15 (words 0, 1) into p0, 16..31 into p1
#pragma unroll
        for (int wi = 0; wi < 4; ++wi)
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const float2 e = half2_bits_to_float2(cvt_e2m1x2(w[wi] >> (8 * b)));
                const float2 xv = make_float2(xf[8 * wi + 2 * b], xf[8 * wi + 2 * b + 1]);
                if (wi < 2) p0 = fma2(xv, e, p0);
                else p1 = fma2(xv, e, p1);
            }
    } else {
        // 16 8-bit codes, one block
#pragma unroll
        for (int wi = 0; wi < 4; ++wi)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float2 e = half2_bits_to_float2(cvt_fp8x2<FAM>(w[wi] >> (16 * h)));
                const float2 xv = make_float2(xf[4 * wi + 2 * h], xf[4 * wi + 2 * h + 1]);
                p0 = fma2(xv, e, p0);
            }
    }
}

// Block scale of an FP family at element index i of a ring scale tile row.
template <int FAM>
__device__ __forceinline__ float fpr_ring_scale(const unsigned char* row, int i, int skind) {
    if constexpr (FAM == FAM_NVFP4) return e4m3_value(row[i]);
    else if constexpr (FAM == FAM_MXFP4 || FAM == FAM_MXFP8) return e8m0_value(row[i]);
    else {
        switch (skind) {
            case SK_E8M0: return e8m0_value(row[i]);
            case SK_E4M3: return e4m3_value(row[i]);
            case SK_F32: return reinterpret_cast<const float*>(row)[i];
            default: return __half2float(reinterpret_cast<const __half*>(row)[i]);
        }
    }
}

// Block scale of an FP family at element index i of the scale array.
template <int FAM>
__device__ __forceinline__ float fpr_scale(const Params& p, long long i) {
    if constexpr (FAM == FAM_NVFP4) return e4m3_value(__ldg(reinterpret_cast<const uint8_t*>(p.scales) + i));
    else if constexpr (FAM == FAM_MXFP4 || FAM == FAM_MXFP8) return e8m0_value(__ldg(reinterpret_cast<const uint8_t*>(p.scales) + i));
    else return block_scale(p.scales, i, p.skind);
}

template <int FAM, int B, int STAGES, int MAXT>
__global__ void __launch_bounds__(MAXT, 1) qmv_tcf_kernel(const __grid_constant__ Params p) {
    using T = __nv_bfloat16;
    using Gm = TcGeom<B>;
    constexpr bool AFF = FAM == FAM_AFFINE;
    constexpr TcPlanData P = tc_make_plan<B, false>();
    constexpr int NW = Gm::NW, UB = Gm::UNIT_BYTES, UC = Gm::UNIT_CODES, SB = Gm::SB;
    // x words per unit in shared memory: bf16 pairs in plan order (affine) or
    // fp32 values (FP), plus a 4-word pad
    constexpr int NP = P.np, NPS = AFF ? NP + 4 : UC + 4;
    static_assert(AFF || ((B == 4 || B == 8) && UB == 16), "FP units are 16 bytes");
    static_assert(2 * STAGES * 8 <= 96 && 4 * (STAGES + 1) <= 32, "barrier area");

    extern __shared__ float4 smem4[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(smem4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wk = p.wk, wr = p.wr, NCW = wk * wr;
    const int ROWS = 16 * wr;
    const int nrb = (p.N + ROWS - 1) / ROWS;
    const int NSBK = p.K / SB;
    const int S = p.sps;
    const int pitch = p.pitch;
    const int sbw = p.sbw;
    const bool sring = p.sring != 0;
    const int stage_bytes = ROWS * pitch + (sring ? (AFF ? 2 : 1) * ROWS * sbw : 0);   // FP: no bias tile
    const int TSB = p.tile_iters;
    const int TU = TSB * 4;
    const int G = p.G;
    const int segsz = AFF ? min(G, SB) : SB;
    const long long KG = p.K / G;
    const int bz = blockIdx.z;
    const int gmul = G < SB ? __ffs(SB / G) - 1 : 0;
    const int gdiv = G > SB ? __ffs(G / SB) - 1 : 0;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    unsigned* rdone = reinterpret_cast<unsigned*>(smem + 96);
    unsigned char* ring = smem + 128 + ((128u - (smem_addr(smem) & 127u)) & 127u);
    uint32_t* xs = reinterpret_cast<uint32_t*>(ring + (size_t)STAGES * stage_bytes);
    float2* us = reinterpret_cast<float2*>(xs + (size_t)TU * NPS);       // affine only
    float* red = AFF ? reinterpret_cast<float*>(us + TU) : reinterpret_cast<float*>(us);
    const uint32_t bar0 = smem_addr(bars);
    auto full = [&](int s) { return bar0 + 8u * (uint32_t)s; };
    auto empty = [&](int s) { return bar0 + 8u * (uint32_t)(STAGES + s); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), (uint32_t)NCW);
        }
        for (int s = 0; s <= STAGES; ++s) rdone[s] = 0u;
        mbar_init_fence();
    }
    __syncthreads();

    const long long sb0 = bz * p.s_bs;
    const int nks = (NSBK + S - 1) / S;
    if (warp == NCW) {                               // the producer warp
        grid_launch_dependents();
        const uint32_t ring0 = smem_addr(ring);
        const uint32_t stage_tx = (uint32_t)ROWS * ((uint32_t)pitch + (sring ? (AFF ? 2u : 1u) * (uint32_t)sbw : 0u));
        int it = 0;
        bool ok = true;
        for (int rb = blockIdx.x; rb < nrb && ok; rb += gridDim.x) {
            for (int ks = 0; ks < nks; ++ks) {
                const int slot = it % STAGES, f = it / STAGES;
                if (f > 0 && !mbar_wait(empty(slot), (uint32_t)((f - 1) & 1))) { ok = false; break; }
                const uint32_t st0 = ring0 + (uint32_t)(slot * stage_bytes);
                // test hook (qmv_test_skip_last_copy): block (0, 0)'s final stage
                // gets neither its expected-bytes arrival nor its copies, so the
                // bounded waits on it run out (codes 1 and 4); no copy is left
                // in flight
                const bool skip = p.test_skip && blockIdx.x == 0 && blockIdx.z == 0 &&
                                  rb + (int)gridDim.x >= nrb && ks == nks - 1;
                if (lane == 0 && !skip) {
                    mbar_arrive_expect_tx(full(slot), stage_tx);
                    tensor_copy_3d(st0, &p.wmap, (ks * S * 4 * UB) / 8, rb * ROWS, bz, full(slot));
                    if (sring) {
                        const int g0 = ((ks * S) << gmul) >> gdiv;
                        tensor_copy_3d(st0 + (uint32_t)p.soff, &p.smap, g0, rb * ROWS, bz, full(slot));
                        if (AFF) tensor_copy_3d(st0 + (uint32_t)p.boff, &p.bmap, g0, rb * ROWS, bz, full(slot));
                    }
                }
                __syncwarp();
                ++it;
            }
        }
        unsigned code = ok ? 0u : 2u;
        for (int s = 0; s < STAGES && s < it; ++s) {
            const int last = (it - 1 - s) / STAGES;
            if (!mbar_wait(full(s), (uint32_t)(last & 1))) code |= 4u;
        }
        if (code && lane == 0) atomicOr(p.fault, code);
        return;
    }
    grid_wait();

    const int nthr = NCW * 32;
    const int r4 = lane >> 3, u8 = lane & 7;
    const int half = u8 >> 2, t = u8 & 3;          // super-block of the step, unit in it
    const int useg = AFF ? (t * UC) / segsz : 0;    // scale group of the unit within its super-block
    const int wkid = warp % wk, wrid = warp / wk;
    const T* X = reinterpret_cast<const T*>(p.x) + bz * p.x_bs;
    const uint32_t kbf16 = p.kbf16;
    T* Yo = reinterpret_cast<T*>(p.y) + bz * p.y_bs;
    int it = 0;
    bool ok = true;
    bool x_whole = false;

    int rbi = 0;                                     // row blocks done by this block
    for (int rb = blockIdx.x; rb < nrb; rb += gridDim.x) {
        const int trow = wrid * 16;                 // the warp's tile within the row block
        float Y[4] = {0.f, 0.f, 0.f, 0.f};
        long long srow[4];                           // scale row offsets (scales outside the ring)
#pragma unroll
        for (int i = 0; i < 4; ++i) srow[i] = sb0 + (long long)min(rb * ROWS + trow + r4 + 4 * i, p.N - 1) * KG;

        for (int t0 = 0; t0 < NSBK; t0 += TSB) {
            const int tn = min(TSB, NSBK - t0);
            if (!x_whole) {
                // ---- stage x: x~ pairs in plan order + per-unit sums -------------
                consumer_sync(nthr);
                for (int u = threadIdx.x; u < tn * 4; u += nthr) {
                    const long long k0 = (long long)t0 * SB + (long long)u * UC;
                    const T* xr = X + k0;
                    float xv[UC];
                    if constexpr (UC % 8 == 0) {
                        if (p.x_vec) {
#pragma unroll
                            for (int q = 0; q < UC / 8; ++q)
                                widen8<T>(__ldg(reinterpret_cast<const uint4*>(xr) + q), xv + 8 * q);
                        } else {
#pragma unroll
                            for (int c = 0; c < UC; ++c) xv[c] = DT<T>::ld(xr, c);
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < UC; ++c) xv[c] = DT<T>::ld(xr, c);
                    }
                    if constexpr (!AFF) {
                        float4* dst = reinterpret_cast<float4*>(xs + (size_t)u * NPS);
#pragma unroll
                        for (int c = 0; c < UC / 4; ++c)
                            dst[c] = make_float4(xv[4 * c], xv[4 * c + 1], xv[4 * c + 2], xv[4 * c + 3]);
                        continue;
                    }
                    float usum = 0.f, tsum = 0.f;
#pragma unroll
                    for (int c = 0; c < UC; ++c) usum += xv[c];
                    uint32_t* dst = xs + (size_t)u * NPS;
#pragma unroll
                    for (int q = 0; q < NP; ++q) {
                        float lo = 0.f, hi = 0.f;
                        if (P.lo[q] >= 0)
                            lo = __fmul_rn(xv[tc_field_code<B>(P.lo[q])],
                                           __uint_as_float((uint32_t)(127 + tc_field_wexp<B>(P.lo[q]) - P.slo[q]) << 23));
                        if (P.hi[q] >= 0)
                            hi = __fmul_rn(xv[tc_field_code<B>(P.hi[q])],
                                           __uint_as_float((uint32_t)(127 + tc_field_wexp<B>(P.hi[q]) - P.shi[q]) << 23));
                        const uint32_t bl = bf16_bits(lo), bh = bf16_bits(hi);
                        tsum += __uint_as_float(bl << 16) + __uint_as_float(bh << 16);
                        dst[q] = bl | (bh << 16);
                    }
                    us[u] = make_float2(usum, tsum);
                }
                consumer_sync(nthr);
                x_whole = (TSB >= NSBK);
            }

            const int end = t0 + tn;
            for (int ks = t0 / S; ks * S < end; ++ks) {
                const int slot = it % STAGES, f = it / STAGES;
                if (ok && !mbar_wait(full(slot), (uint32_t)(f & 1))) {
                    ok = false;
                    if (lane == 0) atomicOr(p.fault, 1u);
                }
                const int sbase = ks * S;
                const int send = min(end, sbase + S);
                if (ok) {
                    const unsigned char* stg = ring + (size_t)slot * stage_bytes;
                    const unsigned char* rows0 = stg + (size_t)(trow + r4) * pitch;
                    const unsigned char* srow0 = stg + p.soff + (size_t)(trow + r4) * sbw;
                    const unsigned char* brow0 = stg + p.boff + (size_t)(trow + r4) * sbw;
                    const int nsteps = (send - sbase + 1) >> 1;
                    // one step: unit u8 of super-blocks (2j, 2j+1) of the stage, 4 rows;
                    // RING: scales and biases from the stage's tiles, else global memory
                    auto step = [&](auto ring_c, int j) {
                        constexpr bool RING = decltype(ring_c)::value;
                        const int sbl = 2 * j + half;            // super-block within the stage
                        const int sb = sbase + sbl;
                        const bool valid = sb < send;
                        const int ut = valid ? (sb - t0) * 4 + t : 0;   // unit within the x tile
                        if constexpr (!AFF) {
                            float xf[UC];                 // the unit's x, once for the 4 rows
                            {
                                const float4* xp = reinterpret_cast<const float4*>(xs + (size_t)ut * NPS);
#pragma unroll
                                for (int c = 0; c < UC / 4; ++c) {
                                    const float4 v = xp[c];
                                    xf[4 * c] = v.x; xf[4 * c + 1] = v.y; xf[4 * c + 2] = v.z; xf[4 * c + 3] = v.w;
                                }
                            }
                            const unsigned char* src0 = rows0 + (8 * j + u8) * UB;
                            const long long k0 = (long long)sb * SB + t * UC;           // the unit's first code
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const uint4 a = *reinterpret_cast<const uint4*>(src0 + (size_t)(4 * i) * pitch);
                                const uint32_t w[4] = {a.x, a.y, a.z, a.w};
                                float2 p0 = make_float2(0.f, 0.f), p1 = make_float2(0.f, 0.f);
                                fpr_unit<FAM, B>(w, xf, p0, p1);
                                float s0, s1;
                                if constexpr (RING) {
                                    // the unit's scale(s) in this stage's tile
                                    const unsigned char* sr = srow0 + (size_t)(4 * i) * sbw;
                                    const int sidx = (sbl * SB + t * UC) / G;
                                    s0 = fpr_ring_scale<FAM>(sr, sidx, p.skind);
                                    s1 = (B == 4 && G == 16) ? fpr_ring_scale<FAM>(sr, sidx + 1, p.skind) : s0;
                                } else {
                                    const long long si = valid ? srow[i] + k0 / G : srow[i];
                                    s0 = fpr_scale<FAM>(p, si);
                                    s1 = (B == 4 && G == 16) ? fpr_scale<FAM>(p, si + 1) : s0;
                                }
                                float yn = fmaf(s0, p0.x + p0.y, Y[i]);
                                if constexpr (B == 4) yn = fmaf(s1, p1.x + p1.y, yn);
                                Y[i] = valid ? yn : Y[i];
                            }
                            return;
                        }
                        uint32_t xq[NP];
#pragma unroll
                        for (int q = 0; q < NP / 4; ++q) {
                            const uint4 v = reinterpret_cast<const uint4*>(xs + (size_t)ut * NPS)[q];
                            xq[4 * q] = v.x; xq[4 * q + 1] = v.y; xq[4 * q + 2] = v.z; xq[4 * q + 3] = v.w;
                        }
                        const float2 su = us[ut];
                        const unsigned char* src0 = rows0 + (8 * j + u8) * UB;
                        const int gl = ((sbl << gmul) >> gdiv) + useg;          // group within the stage's tile
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            uint32_t w[NW];
                            const unsigned char* src = src0 + (size_t)(4 * i) * pitch;
                            if constexpr (UB == 16) {
                                const uint4 a = *reinterpret_cast<const uint4*>(src);
                                w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
                            } else {
#pragma unroll
                                for (int q = 0; q < NW; ++q) w[q] = reinterpret_cast<const uint32_t*>(src)[q];
                            }
                            float lo = 0.f, hi = 0.f;
                            tcf_unit<B>(std::make_integer_sequence<int, NP>{}, w, xq, kbf16, lo, hi);
                            float sc, bi;
                            if constexpr (RING) {
                                sc = ring_scale<T>(srow0 + (size_t)(4 * i) * sbw, gl);
                                bi = ring_scale<T>(brow0 + (size_t)(4 * i) * sbw, gl);
                            } else {
                                const long long gg = valid ? (((long long)sb << gmul) >> gdiv) + useg : 0;
                                sc = DT<T>::ld(p.scales, srow[i] + gg);
                                bi = DT<T>::ld(p.biases, srow[i] + gg);
                            }
                            const float yn = fmaf(sc, fmaf(-128.f, su.y, lo + hi), fmaf(bi, su.x, Y[i]));
                            Y[i] = valid ? yn : Y[i];
                        }
                    };
                    if (sring) {
                        for (int j = wkid; j < nsteps; j += wk) step(std::true_type{}, j);
                    } else {
                        for (int j = wkid; j < nsteps; j += wk) step(std::false_type{}, j);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty(slot));
                ++it;
            }
        }

        // ---- reduce over the 8 unit lanes; the last warp done with the row
        // block sums over its k-warps and stores (no block-wide barrier).
        // Buffer rbi % (STAGES + 1): a warp cannot get STAGES + 1 row blocks
        // ahead of another, each row block having at least one ring stage.
        {
            const int buf = rbi % (STAGES + 1), round = rbi / (STAGES + 1);
            float* rred = red + (size_t)buf * NCW * 16;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float v = Y[i];
                v += __shfl_xor_sync(0xFFFFFFFFu, v, 1);
                v += __shfl_xor_sync(0xFFFFFFFFu, v, 2);
                v += __shfl_xor_sync(0xFFFFFFFFu, v, 4);
                if (u8 == 0) rred[warp * 16 + r4 + 4 * i] = v;
            }
            __syncwarp();
            unsigned last = 0u;
            if (lane == 0) {
                const unsigned before = arrive_count(&rdone[buf]);
                last = before + 1u == (unsigned)((round + 1) * NCW) ? 1u : 0u;
            }
            last = __shfl_sync(0xFFFFFFFFu, last, 0);
            if (last) {
                __syncwarp();                  // lane 0's acquire, for every lane
                for (int i = lane; i < ROWS; i += 32) {
                    const int w_ = i >> 4, r = i & 15;
                    float v = 0.f;
                    for (int k = 0; k < wk; ++k) v += rred[(w_ * wk + k) * 16 + r];
                    const int row = rb * ROWS + i;
                    if constexpr (FAM == FAM_NVFP4) v *= __ldg(p.gscale + bz);
                    if (row < p.N) DT<T>::st(Yo, row, v);
                }
            }
        }
        ++rbi;
    }

}

}  // namespace qmv
