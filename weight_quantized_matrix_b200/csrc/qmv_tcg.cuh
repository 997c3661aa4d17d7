// qmv_tcg.cuh -- tensor-core affine qmv for several x rows with one exact fp32
// epilogue per scale group: 4-bit codes, bf16 or f16 x, M up to 8 * NT rows.
//
// Lane layout.  The four lanes of a quad (t = lane % 4) split every group of G
// codes of a row into four contiguous quarters of G/4 codes (G/8 bytes); lane
// (g = lane / 4, t) holds quarter t of rows g and g + 8 of its warp's 16-row
// tile.  One k16 step of the m16n8k16 MMA takes four codes of each quarter, so
// every step lies inside one group: the D columns are the x rows themselves,
// D is the group's partial dot product, and the epilogue adds
// scale * D + bias * sum(x) per group in fp32 (no slot columns, no zero
// padding of B).
//
// Decode.  A 32-bit word of a quarter holds 8 codes n0..n7 (LSB first).  For
// i = 0..3, (word >> 4i) masked to bits 0..3 and 16..19 and OR-ed with the
// bf16 pair {128, 128} (f16: {1024, 1024}) is {128 + n_i, 128 + n_(i+4)}; one
// packed subtraction of the same pair leaves {n_i, n_(i+4)} exactly.  Step
// 2w + h of a group uses pairs 2h (A columns 2t, 2t + 1) and 2h + 1 (A
// columns 2t + 8, 2t + 9) of word w.
//
// x.  The B fragment of lane (g, t) in step 2w + h is {x[k0 + 2h], x[k0 + 2h +
// 4]}, {x[k0 + 2h + 1], x[k0 + 2h + 5]} for x row g of the n-tile, k0 the first
// code of word w of quarter t: a permutation of 16-bit values (two byte
// permutes per fragment), staged once per x tile in shared memory in lane
// order, so a step's fragments are one conflict-free 8-byte load.  sum(x) per
// (group, x row) is formed from the values widened to fp32 one by one, each
// quarter in order, the four quarters added in a fixed tree.
//
// Weights.  Rows stream through a shared-memory ring: a stage is 8 groups of
// ROWS = 16 * wr rows -- the packed codes as G / 32 boxes of 128 bytes a row
// with the 128-byte swizzle (16-byte chunk c of row r stored at chunk
// c ^ (r % 8): the 8 rows a load instruction touches hit 8 different chunks),
// then the scale and bias tiles, 8 groups (16 bytes) a row.  One producer
// warp issues the tensor copies under mbarrier flow control; consumer warp
// (wrid, wkid) takes row tile wrid and the groups wkid, wkid + wk, ... of each
// stage.  Rows past N and groups past K are zero-filled by the copies.
// Every wait is bounded as in the other ring kernels (fault codes 1, 2, 4).
#pragma once

#include <type_traits>

#include "qmv_tcb.cuh"

namespace qmv {

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t f16x2_sub(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Pair I (0..3) of a word of eight 4-bit codes: {n_I, n_(I+4)} as bf16x2 or
// f16x2, exact.  k2 holds the offset pair ({128, 128} or {1024, 1024}).
template <class T, int I>
__device__ __forceinline__ uint32_t tcg_pair(uint32_t word, uint32_t k2) {
    const uint32_t v = I == 0 ? word : word >> (4 * I);
    const uint32_t o = and_or<0x000F000Fu>(v, k2);
    if constexpr (std::is_same<T, __half>::value) return f16x2_sub(o, k2);
    else return bf16x2_sub(o, k2);
}

template <class T>
__device__ __forceinline__ void tcg_mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint2 b) {
    if constexpr (std::is_same<T, __half>::value) mma_f16_16816(d, a0, a1, a2, a3, b.x, b.y);
    else mma_bf16_16816(d, a0, a1, a2, a3, b.x, b.y);
}

// 16-bit element -> fp32, exact.
template <class T> __device__ __forceinline__ float tcg_widen(uint32_t bits16);
template <> __device__ __forceinline__ float tcg_widen<__nv_bfloat16>(uint32_t bits16) {
    return __uint_as_float(bits16 << 16);
}
template <> __device__ __forceinline__ float tcg_widen<__half>(uint32_t bits16) {
    return __half2float(__ushort_as_half((unsigned short)bits16));
}

// Shared memory (bytes from a 1024-aligned base; the host adds the slack):
//   0      full[NST], empty[NST] barriers (8 bytes each, NST <= 8)
//   1024   ring: NST stages of SBY bytes (a multiple of 1024): G / 32 code
//          boxes of ROWS x 128 bytes, the scale tile and the bias tile
//          (ROWS x 16 bytes each)
//   then   xs   the x tile's B fragments: (XT * 8 * G / 16) steps x NT n-tiles
//               x 32 lanes x 8 bytes
//          sx   sum(x) per (group of the x tile, x row): XT * 8 x 8 * NT floats
//          red  (wk * wr) x 16 x 8 * NT floats
// Params: sps = NST ring stages, pitch = SBY, tile_iters = XT ring stages per
// x tile (the whole K when it fits), wk * wr consumer warps (at most
// kTcgMaxWarps) and one producer warp.
constexpr int kTcgMaxWarps = 16;

template <class T, int G, int NT>
__global__ void __launch_bounds__(32 * (kTcgMaxWarps + 1), 1) qmv_tcg_kernel(const __grid_constant__ Params p) {
    static_assert(G == 32 || G == 64 || G == 128, "group size");
    static_assert(sizeof(T) == 2, "16-bit x");
    constexpr int NWD = G / 32;          // 32-bit words per quarter (8 codes each)
    constexpr int QB = 4 * NWD;          // bytes per quarter
    constexpr int GST = G / 16;          // k16 steps per group
    constexpr int SPS = 8;               // groups per ring stage
    constexpr int SKB = SPS * G / 2;     // code bytes per row per stage
    constexpr int NBOX = SKB / 128;      // 128-byte boxes per row per stage
    constexpr int NC = 8 * NT;           // x rows the n-tiles cover

    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wk = p.wk, wr = p.wr, ncw = wk * wr;
    const int M = p.M;
    const int ROWS = 16 * wr;
    const int nrb = (p.N + ROWS - 1) / ROWS;
    const int KG = p.K / G;
    const int nks = (KG + SPS - 1) / SPS;
    const int NST = p.sps;
    const int SBY = p.pitch;
    const int XT = p.tile_iters;
    const int bz = blockIdx.z;

    unsigned char* ring = smem + 1024;
    uint2* xs = reinterpret_cast<uint2*>(ring + (size_t)NST * SBY);
    float* sx = reinterpret_cast<float*>(xs + (size_t)XT * SPS * GST * NT * 32);
    float* red = sx + (size_t)XT * SPS * NC;
    const uint32_t bar0 = smem_addr(smem);
    auto full = [&](int s) { return bar0 + 8u * (uint32_t)s; };
    auto empty = [&](int s) { return bar0 + 8u * (uint32_t)(NST + s); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), (uint32_t)ncw);
        }
        mbar_init_fence();
    }
    __syncthreads();

    // ---- producer warp: streams weights only, so it starts at once ---------
    if (warp == ncw) {
        grid_launch_dependents();    // the next kernel may start fetching its weights
        const uint32_t ring0 = smem_addr(ring);
        const uint32_t stage_tx = (uint32_t)ROWS * (uint32_t)(SKB + 32);
        int it = 0;
        bool ok = true;
        for (int rb = blockIdx.x; rb < nrb && ok; rb += gridDim.x) {
            for (int ks = 0; ks < nks; ++ks) {
                const int slot = it % NST, f = it / NST;
                if (f > 0 && !mbar_wait(empty(slot), (uint32_t)((f - 1) & 1))) { ok = false; break; }
                const uint32_t st0 = ring0 + (uint32_t)(slot * SBY);
                // test hook (qmv_test_skip_last_copy): block (0, 0)'s final stage
                // gets neither its expected-bytes arrival nor its copies
                const bool skip = p.test_skip && blockIdx.x == 0 && blockIdx.z == 0 &&
                                  rb + (int)gridDim.x >= nrb && ks == nks - 1;
                if (lane == 0 && !skip) {
                    mbar_arrive_expect_tx(full(slot), stage_tx);
#pragma unroll
                    for (int b = 0; b < NBOX; ++b)
                        tensor_copy_3d(st0 + (uint32_t)(b * ROWS * 128), &p.wmap, (ks * SKB + b * 128) / 8,
                                       rb * ROWS, bz, full(slot));
                    const uint32_t tiles = st0 + (uint32_t)(NBOX * ROWS * 128);
                    tensor_copy_3d(tiles, &p.smap, ks * SPS, rb * ROWS, bz, full(slot));
                    tensor_copy_3d(tiles + (uint32_t)(ROWS * 16), &p.bmap, ks * SPS, rb * ROWS, bz, full(slot));
                }
                __syncwarp();
                ++it;
            }
        }
        unsigned code = ok ? 0u : 2u;
        // wait for the copies this warp issued: the last fill of each slot
        for (int s = 0; s < NST && s < it; ++s) {
            const int last = (it - 1 - s) / NST;
            if (!mbar_wait(full(s), (uint32_t)(last & 1))) code |= 4u;
        }
        if (code && lane == 0) atomicOr(p.fault, code);
        return;
    }

    // ---- consumer warps: x and y may belong to the previous kernel ---------
    grid_wait();
    const int nthr = ncw * 32;
    const int g = lane >> 2, t = lane & 3;
    const int wkid = warp % wk, wrid = warp / wk;
    const unsigned short* X = reinterpret_cast<const unsigned short*>(p.x) + bz * p.x_bs;
    T* Yo = reinterpret_cast<T*>(p.y) + bz * p.y_bs;
    const uint32_t k2 = std::is_same<T, __half>::value ? 0x64006400u : 0x43004300u;
    const int KX = XT * SPS * G;                 // codes per x tile
    const int ntile = (p.K + KX - 1) / KX;
    const int ngt = XT * SPS;                    // groups per x tile
    bool staged = false;
    int it = 0;
    bool ok = true;

    // this lane's ring row (row g of its tile; row g + 8 is 8 * 128 bytes on,
    // with the same swizzle phase)
    const int rg = wrid * 16 + g;

    for (int rb = blockIdx.x; rb < nrb; rb += gridDim.x) {
        float Y[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) Y[nt][e] = 0.f;

        for (int xt = 0; xt < ntile; ++xt) {
            const int kt0 = xt * KX;
            if (!(ntile == 1 && staged)) {
                // ---- stage the x tile: B fragments in lane order, sum(x) ----
                consumer_sync(nthr);            // the previous tile is no longer read
                const int items = NC * ngt * 4;
                // XI items a thread per round, their loads issued first (one
                // round trip to L2 for up to XI * NWD 16-byte loads in flight)
                constexpr int XI = NWD >= 4 ? 2 : 4;
                for (int base = 0; base < items; base += XI * nthr) {
                    uint4 v[XI][NWD];
#pragma unroll
                    for (int j = 0; j < XI; ++j) {
                        const int i = base + j * nthr + (int)threadIdx.x;
                        const int tq = i & 3, q = i >> 2;
                        const int gi = q % ngt, m = q / ngt;
                        const int k0 = kt0 + gi * G + tq * (G / 4);
                        const unsigned short* xr = X + (long long)m * p.K;
#pragma unroll
                        for (int w = 0; w < NWD; ++w) {
                            v[j][w] = make_uint4(0u, 0u, 0u, 0u);
                            const int k = k0 + 8 * w;
                            if (i < items && m < M && k < p.K) {
                                if (p.x_vec) {
                                    v[j][w] = __ldg(reinterpret_cast<const uint4*>(xr + k));
                                } else {
                                    uint32_t e[8];
#pragma unroll
                                    for (int c = 0; c < 8; ++c) e[c] = xr[k + c];
                                    v[j][w] = make_uint4(e[0] | (e[1] << 16), e[2] | (e[3] << 16),
                                                         e[4] | (e[5] << 16), e[6] | (e[7] << 16));
                                }
                            }
                        }
                    }
#pragma unroll
                    for (int j = 0; j < XI; ++j) {
                        const int i = base + j * nthr + (int)threadIdx.x;
                        const bool act = i < items;
                        const int tq = i & 3, q = i >> 2;
                        const int gi = q % ngt, m = q / ngt;
                        float s = 0.f;
                        if (act) {
                            uint2* dst = xs + ((size_t)gi * GST * NT + (m >> 3)) * 32 + (m & 7) * 4 + tq;
#pragma unroll
                            for (int w = 0; w < NWD; ++w) {
                                const uint4 u4 = v[j][w];
                                dst[(size_t)(2 * w) * NT * 32] =
                                    make_uint2(__byte_perm(u4.x, u4.z, 0x5410), __byte_perm(u4.x, u4.z, 0x7632));
                                dst[(size_t)(2 * w + 1) * NT * 32] =
                                    make_uint2(__byte_perm(u4.y, u4.w, 0x5410), __byte_perm(u4.y, u4.w, 0x7632));
                                const uint32_t u[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
                                for (int c = 0; c < 4; ++c) {
                                    s += tcg_widen<T>(u[c] & 0xFFFFu);
                                    s += tcg_widen<T>(u[c] >> 16);
                                }
                            }
                        }
                        // the quad's quarters in a fixed tree: (q0 + q1) + (q2 + q3)
                        s += __shfl_xor_sync(0xFFFFFFFFu, s, 1);
                        s += __shfl_xor_sync(0xFFFFFFFFu, s, 2);
                        if (act && tq == 0) sx[(size_t)gi * NC + m] = s;
                    }
                }
                consumer_sync(nthr);
                staged = true;
            }

            // ---- the tile's ring stages -------------------------------------
            const int ksend = min(nks, (xt + 1) * XT);
            for (int ks = xt * XT; ks < ksend; ++ks) {
                const int slot = it % NST, f = it / NST;
                if (ok && !mbar_wait(full(slot), (uint32_t)(f & 1))) {
                    ok = false;
                    if (lane == 0) atomicOr(p.fault, 1u);
                }
                if (ok) {
                    const unsigned char* st = ring + (size_t)slot * SBY;
                    const unsigned char* stile = st + NBOX * ROWS * 128 + rg * 16;
                    const unsigned char* btile = stile + ROWS * 16;
                    const int gb = (ks - xt * XT) * SPS;      // the stage's first group in the x tile
                    // NGP groups at a time (independent load / decode / MMA
                    // chains the scheduler interleaves), then the rest one by one
                    auto run_groups = [&](auto ngc, int gl0) {
                        constexpr int NG = decltype(ngc)::value;
                        uint32_t wg[NG][NWD], wh[NG][NWD];
#pragma unroll
                        for (int j = 0; j < NG; ++j) {
                            const int gl = gl0 + j * wk;
                            // quarter t of group gl, rows g and g + 8 (swizzled chunk)
                            const int bo = gl * (G / 2) + t * QB;
                            const int pc = ((((bo & 127) >> 4) ^ (rg & 7)) << 4) | (bo & 15);
                            const unsigned char* pg = st + (bo >> 7) * ROWS * 128 + rg * 128 + pc;
                            const unsigned char* ph = pg + 8 * 128;
                            if constexpr (NWD == 4) {
                                const uint4 a = *reinterpret_cast<const uint4*>(pg);
                                const uint4 b = *reinterpret_cast<const uint4*>(ph);
                                wg[j][0] = a.x; wg[j][1] = a.y; wg[j][2] = a.z; wg[j][3] = a.w;
                                wh[j][0] = b.x; wh[j][1] = b.y; wh[j][2] = b.z; wh[j][3] = b.w;
                            } else if constexpr (NWD == 2) {
                                const uint2 a = *reinterpret_cast<const uint2*>(pg);
                                const uint2 b = *reinterpret_cast<const uint2*>(ph);
                                wg[j][0] = a.x; wg[j][1] = a.y;
                                wh[j][0] = b.x; wh[j][1] = b.y;
                            } else {
                                wg[j][0] = *reinterpret_cast<const uint32_t*>(pg);
                                wh[j][0] = *reinterpret_cast<const uint32_t*>(ph);
                            }
                        }
#pragma unroll
                        for (int j = 0; j < NG; ++j) {
                            const int gl = gl0 + j * wk;
                            const uint2* xf = xs + (size_t)(gb + gl) * GST * NT * 32 + lane;
                            float D[NT][4];
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                                for (int e = 0; e < 4; ++e) D[nt][e] = 0.f;
#pragma unroll
                            for (int w = 0; w < NWD; ++w) {
                                {   // step 2w: pairs 0 and 1
                                    const uint32_t a0 = tcg_pair<T, 0>(wg[j][w], k2), a2 = tcg_pair<T, 1>(wg[j][w], k2);
                                    const uint32_t a1 = tcg_pair<T, 0>(wh[j][w], k2), a3 = tcg_pair<T, 1>(wh[j][w], k2);
#pragma unroll
                                    for (int nt = 0; nt < NT; ++nt)
                                        tcg_mma<T>(D[nt], a0, a1, a2, a3, xf[(size_t)((2 * w) * NT + nt) * 32]);
                                }
                                {   // step 2w + 1: pairs 2 and 3
                                    const uint32_t a0 = tcg_pair<T, 2>(wg[j][w], k2), a2 = tcg_pair<T, 3>(wg[j][w], k2);
                                    const uint32_t a1 = tcg_pair<T, 2>(wh[j][w], k2), a3 = tcg_pair<T, 3>(wh[j][w], k2);
#pragma unroll
                                    for (int nt = 0; nt < NT; ++nt)
                                        tcg_mma<T>(D[nt], a0, a1, a2, a3, xf[(size_t)((2 * w + 1) * NT + nt) * 32]);
                                }
                            }
                            // epilogue: scale * D + bias * sum(x), rows g / g + 8, x rows 2t, 2t + 1
                            const float sg = ring_scale<T>(stile, gl), sh = ring_scale<T>(stile + 8 * 16, gl);
                            const float bg = ring_scale<T>(btile, gl), bh = ring_scale<T>(btile + 8 * 16, gl);
                            const float* sxg = sx + (size_t)(gb + gl) * NC + 2 * t;
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt) {
                                const float2 xv = *reinterpret_cast<const float2*>(sxg + nt * 8);
                                Y[nt][0] = fmaf(sg, D[nt][0], fmaf(bg, xv.x, Y[nt][0]));
                                Y[nt][1] = fmaf(sg, D[nt][1], fmaf(bg, xv.y, Y[nt][1]));
                                Y[nt][2] = fmaf(sh, D[nt][2], fmaf(bh, xv.x, Y[nt][2]));
                                Y[nt][3] = fmaf(sh, D[nt][3], fmaf(bh, xv.y, Y[nt][3]));
                            }
                        }
                    };
                    constexpr int NGP = NT <= 2 ? 2 : 1;
                    const int gend = min(SPS, KG - ks * SPS);      // groups of this stage inside K
                    int gl = wkid;
                    if constexpr (NGP > 1) {
                        for (; gl + (NGP - 1) * wk < gend; gl += NGP * wk)
                            run_groups(std::integral_constant<int, NGP>{}, gl);
                    }
                    for (; gl < gend; gl += wk) run_groups(std::integral_constant<int, 1>{}, gl);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty(slot));
                ++it;
            }
        }

        // ---- reduce over k-warps (fixed order), store ------------------------
        float* myred = red + (size_t)warp * 16 * NC;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) myred[(g + 8 * (e >> 1)) * NC + nt * 8 + 2 * t + (e & 1)] = Y[nt][e];
        consumer_sync(nthr);
        const int tot = wr * 16 * M;
        for (int i = threadIdx.x; i < tot; i += nthr) {
            const int w_ = i / (16 * M), rm = i - w_ * (16 * M), m = rm >> 4, r = rm & 15;
            const int row = rb * ROWS + w_ * 16 + r;
            float v = 0.f;
            for (int k = 0; k < wk; ++k) v += red[((size_t)(w_ * wk + k) * 16 + r) * NC + m];
            if (row < p.N) DT<T>::st(Yo, (long long)m * p.N + row, v);
        }
        consumer_sync(nthr);
    }
}

}  // namespace qmv
